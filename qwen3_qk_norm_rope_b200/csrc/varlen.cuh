// varlen.cuh - batches of sequences packed on one token axis (the batching of serving
// engines: "LLM Internals - Assembling a large model from scratch", the comparison with
// inference engines, where the tokens of many requests form one batch and attention is
// computed per request, and the review question on vLLM: flattened tokens plus batching
// metadata).
//
// Sequence b owns tokens cu[b] .. cu[b+1]-1 of q/k/v [N, H, d]; with a cache it has ctx[b]
// cached keys before them.  The prefill attention kernel runs over work items (a pair of
// query tiles of one sequence and one KV head), so the device turns the metadata into an
// item list first.  The host never reads the lengths: they stay on the device, and every
// launch is sized from host bounds (N, B and the key capacity).
//
// varlen_setup_kernel, one CTA:
//   1. validates each sequence (0 <= cu[b] <= cu[b+1] <= N, ctx >= 0, keys within what the
//      block table addresses, the running sum of keys within key_cap); an invalid sequence
//      is recorded in the status word and treated as empty;
//   2. seq[b] = {qoff, T, start, koff}: first token, new tokens, cached keys, and the first
//      row of the sequence's keys on the key axis the attention reads (without a cache the
//      keys are the tokens themselves, koff = qoff; with a paged cache the keys are read in
//      the sequence's own pages and koff is the running sum of ctx + T, kept for the key_cap
//      check);
//   3. the entry list: sequence b has np_b = ceil(T_b / 2P) pairs of query tiles (P token
//      positions per 128-row tile), and its pair p reads about c_b + (p + 1) 2P keys (its
//      cached ones and the new ones up to the pair's diagonal).  Entries go by that count,
//      largest first, ties by sequence: the heaviest items lead and the lightest fill the
//      tail, as in the uniform kernel's order.  For fresh prompts that is pair index first;
//      with long cached prefixes the prefix dominates the count, so the items of one
//      sequence come together and the CTAs that take them at the same time share its keys
//      and values in L2 (a batch's prefixes can exceed L2, and an order that visits every
//      sequence at each pair index reads each prefix from DRAM once per pair).
//      Entry e of sequence b (found by binary search over the running sum of np in b
//      order) counts, over every sequence, the entries with a larger key count or an equal
//      one and a smaller b: that is its position.  O(B) per entry, spread over the CTA;
//      the pair counts and cached lengths sit in shared memory for up to kVarlenSmemSeqs
//      sequences.  No sort is needed.
//   4. n_items = Hkv x entries; item i is entry i / Hkv for KV head i % Hkv.
#pragma once
#include "common.cuh"

namespace q3 {

constexpr int kSiteVarlenMeta = 70;  // a sequence's metadata failed validation
constexpr int kVarlenThreads = 1024;
constexpr int kVarlenSmemSeqs = 2048;  // pair counts and cached lengths kept in shared memory (16 KB)

struct VarlenParams {
  const int* cu;    // [B + 1] token offsets
  const int* ctx;   // [B] cached keys per sequence, or nullptr (none)
  int4* seq;        // [B] out: {qoff, T, start, koff}
  int4* ent;        // [2 * max_entries] out: {qoff, T, start, koff}, {pair, b, 0, 0}
  int* n_items;     // [1] out
  int* np;          // scratch [B]: pairs of each sequence
  int* sbase;       // scratch [B]: its first entry in sequence order
  long long key_cap;  // with a cache: the bound on the sum of every sequence's keys; 0 without
  int B, N, two_p, Hkv, max_entries;
  int max_keys;       // keys one sequence may address (cache: max_blocks * page_size)
};

// Exclusive prefix sum over the CTA of one value per thread (s: kVarlenThreads entries).
template <typename T>
__device__ __forceinline__ T cta_exclusive_scan(T v, T* s, T& total) {
  const int tid = threadIdx.x;
  s[tid] = v;
  __syncthreads();
  for (int off = 1; off < kVarlenThreads; off <<= 1) {
    const T add = tid >= off ? s[tid - off] : T(0);
    __syncthreads();
    s[tid] += add;
    __syncthreads();
  }
  total = s[kVarlenThreads - 1];
  const T incl = s[tid];
  __syncthreads();
  return incl - v;
}

__global__ void __launch_bounds__(kVarlenThreads, 1) varlen_setup_kernel(const __grid_constant__ VarlenParams p) {
  __shared__ long long s_scan[kVarlenThreads];
  __shared__ int s_np[kVarlenSmemSeqs], s_ctx[kVarlenSmemSeqs];
  const int tid = threadIdx.x;
  const bool in_smem = p.B <= kVarlenSmemSeqs;

  // 1-2. validate, then key offsets by a running sum over the sequences (each thread owns a
  //      contiguous run of them, so the order of koff is the order of b).
  const int per = (p.B + kVarlenThreads - 1) / kVarlenThreads;
  const int b0 = min(p.B, tid * per), b1 = min(p.B, b0 + per);
  long long mine = 0;
  for (int b = b0; b < b1; ++b) {
    const int lo = p.cu[b], hi = p.cu[b + 1];
    const int c = p.ctx != nullptr ? p.ctx[b] : 0;
    const bool ok = lo >= 0 && hi >= lo && hi <= p.N && c >= 0 && static_cast<long long>(c) + (hi - lo) <= p.max_keys;
    if (ok && p.key_cap > 0) mine += static_cast<long long>(c) + (hi - lo);
  }
  long long total_keys;
  long long koff = cta_exclusive_scan(mine, s_scan, total_keys);
  (void)total_keys;
  long long n_mine = 0;  // entries of this thread's sequences
  for (int b = b0; b < b1; ++b) {
    int lo = p.cu[b], hi = p.cu[b + 1];
    int c = p.ctx != nullptr ? p.ctx[b] : 0;
    bool ok = lo >= 0 && hi >= lo && hi <= p.N && c >= 0 && static_cast<long long>(c) + (hi - lo) <= p.max_keys;
    const long long keys = ok ? static_cast<long long>(c) + (hi - lo) : 0;
    long long kb = lo;
    if (p.key_cap > 0) {
      kb = koff;
      koff += keys;
      if (ok && kb + keys > p.key_cap) ok = false;  // more keys than the caller's bound
    }
    if (!ok) {  // treated as empty; koff keeps its running value, so koff stays nondecreasing
      record_error(QWEN3_ERR_INVALID_ARG, kSiteVarlenMeta);
      lo = max(0, min(lo, p.N));
      hi = lo;
      c = 0;
      kb = p.key_cap > 0 ? min(kb, p.key_cap) : lo;  // within [0, key_cap]: fits an int
    }
    const int T = hi - lo;
    p.seq[b] = make_int4(lo, T, c, static_cast<int>(kb));
    const int np = (T + p.two_p - 1) / p.two_p;
    p.np[b] = np;
    if (in_smem) {
      s_np[b] = np;
      s_ctx[b] = c;
    }
    n_mine += np;
  }
  // 3a. each sequence's first entry in sequence order
  long long total;
  long long e0 = cta_exclusive_scan(n_mine, s_scan, total);
  for (int b = b0; b < b1; ++b) {
    p.sbase[b] = static_cast<int>(min(e0, static_cast<long long>(p.max_entries)));
    e0 += p.np[b];
  }
  __syncthreads();

  // 3b. entries: entry e of sequence b (the last b whose first entry is <= e: sequences with
  //     no pairs share the first entry of the next one) is pair p = e - sbase[b], reading
  //     about kc = c_b + (p + 1) 2P keys; its position counts the entries with more keys,
  //     and those with as many keys in a sequence before b.
  const int* const NP = in_smem ? s_np : p.np;
  const int n_ent = static_cast<int>(min(total, static_cast<long long>(p.max_entries)));
  for (int e = tid; e < n_ent; e += kVarlenThreads) {
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.sbase[mid] <= e) {
        lo = mid;
      } else {
        hi = mid - 1;
      }
    }
    const int b = lo;
    const int pair = e - p.sbase[b];
    const int4 sq = p.seq[b];
    const long long kc = sq.z + static_cast<long long>(pair + 1) * p.two_p;
    long long pos = 0;
    for (int o = 0; o < p.B; ++o) {
      const int npo = NP[o];
      const long long k = kc - (in_smem ? s_ctx[o] : p.seq[o].z);  // pairs of o with more keys: (q + 1) 2P > k
      const long long first = k < 0 ? 0 : min(static_cast<long long>(npo), k / p.two_p);
      pos += npo - first;
      if (o < b && k >= p.two_p && k % p.two_p == 0 && k / p.two_p <= npo) ++pos;  // as many keys, earlier b
    }
    if (pos < p.max_entries) {
      p.ent[2 * pos] = sq;
      p.ent[2 * pos + 1] = make_int4(pair, b, 0, 0);
    }
  }
  if (tid == 0) *p.n_items = n_ent * p.Hkv;
}

// Keys and values of every sequence (its ctx cached keys and its new ones) out of the pages
// into the gathered layout [Hkv, key_cap, d]: sequence b's key j goes to row koff_b + j.
// One thread per 16-byte chunk, 16 per head vector.  The sequence of a row is found by
// binary search over koff.  Rows no sequence uses are zeroed: the last sequence's final key
// tile reaches into them, and masked keys still meet their values in P.V (as 0 x value).
struct VarlenGatherParams {
  const uint4* k_pages;  // [num_pages, Hkv, page, d] as 16-byte chunks
  const uint4* v_pages;
  const int* block_table;  // [B, max_blocks]
  const int4* seq;         // [B] {qoff, T, start, koff}
  uint4* k_out;            // [Hkv, key_cap, d]
  uint4* v_out;
  long long key_cap;
  int B, Hkv, max_blocks, log2_page, num_pages;
};

__global__ void __launch_bounds__(256) varlen_gather_kernel(const __grid_constant__ VarlenGatherParams p) {
  const long long total = p.key_cap * p.Hkv * 16;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int c = static_cast<int>(i & 15);
    const long long v = i >> 4;  // row * Hkv + h
    const int h = static_cast<int>(v % p.Hkv);
    const long long r = v / p.Hkv;
    // last sequence whose koff <= r (koff is nondecreasing in b; empty sequences share it)
    int lo = 0, hi = p.B - 1, b = -1;
    while (lo <= hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(&p.seq[mid].w) <= r) {
        b = mid;
        lo = mid + 1;
      } else {
        hi = mid - 1;
      }
    }
    const long long dst = (static_cast<long long>(h) * p.key_cap + r) * 16 + c;
    const int4 s = b >= 0 ? p.seq[b] : make_int4(0, 0, 0, 0);
    const long long j = r - s.w;
    if (b < 0 || j >= static_cast<long long>(s.z) + s.y) {  // a row no sequence uses
      p.k_out[dst] = make_uint4(0u, 0u, 0u, 0u);
      p.v_out[dst] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const int blk = static_cast<int>(j >> p.log2_page);
    const int page = blk < p.max_blocks ? p.block_table[static_cast<long long>(b) * p.max_blocks + blk] : -1;
    if (page < 0 || page >= p.num_pages) {
      if (c == 0 && h == 0) record_error(QWEN3_ERR_INVALID_ARG, kSitePagedTable);
      p.k_out[dst] = make_uint4(0u, 0u, 0u, 0u);
      p.v_out[dst] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const long long src =
        ((static_cast<long long>(page) * p.Hkv + h) << p.log2_page | (j & ((1 << p.log2_page) - 1))) * 16 + c;
    p.k_out[dst] = p.k_pages[src];
    p.v_out[dst] = p.v_pages[src];
  }
}

}  // namespace q3
