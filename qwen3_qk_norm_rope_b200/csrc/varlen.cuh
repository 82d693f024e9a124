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
//      block table addresses, gathered keys within the workspace); an invalid sequence is
//      recorded in the status word and treated as empty;
//   2. seq[b] = {qoff, T, start, koff}: first token, new tokens, cached keys, and the first
//      row of the sequence's keys in the gathered key layout (a running sum of ctx + T;
//      without a cache the keys are the tokens themselves, koff = qoff);
//   3. the entry list: sequence b has np_b = ceil(T_b / 2P) pairs of query tiles (P token
//      positions per 128-row tile).  Entries are ordered by pair index, highest first, so
//      the heaviest items go first (for fresh prompts an item's work grows with its pair
//      index), and within one pair index by np_b descending: at pair index L the sequences
//      with np_b > L are exactly the first count_L of that order.  A sequence's rank in it
//      is (number of sequences with more pairs) + (a tie counter), and order[rank] = b.
//      Entry e then lies at the pair index L with base_L <= e < base_L + count_L (a binary
//      search over base) and belongs to sequence order[e - base_L].  No sort is needed,
//      only a level histogram and two scans, and every loop is spread over the CTA.
//   4. n_items = Hkv x entries; item i is entry i / Hkv for KV head i % Hkv.
// The three level arrays live in shared memory when they fit in 36 KB (up to 3071 pair
// indices; with the 8 KB scan buffer the CTA stays within the default 48 KB), else in the
// workspace.
#pragma once
#include "common.cuh"

namespace q3 {

constexpr int kSiteVarlenMeta = 70;  // a sequence's metadata failed validation
constexpr int kVarlenThreads = 1024;
constexpr int kVarlenSmemLevels = 3072;  // level entries kept in shared memory: 3 arrays, 36 KB

struct VarlenParams {
  const int* cu;    // [B + 1] token offsets
  const int* ctx;   // [B] cached keys per sequence, or nullptr (none)
  int4* seq;        // [B] out: {qoff, T, start, koff}
  int4* ent;        // [2 * max_entries] out: {qoff, T, start, koff}, {pair, b, 0, 0}
  int* n_items;     // [1] out
  int* lvl;         // scratch [3 * (n_lvl + 1)]: histogram, tie counters, then count_L / base_L
  int* order;       // scratch [B]: the sequence at each rank
  int lvl_in_smem;  // the level arrays are in dynamic shared memory instead of lvl
  long long key_cap;  // key rows of the gathered layout (cache), 0 without a cache
  int B, N, two_p, Hkv, n_lvl, max_entries;
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
  extern __shared__ int s_levels[];
  const int tid = threadIdx.x;
  int* const L3 = p.lvl_in_smem ? s_levels : p.lvl;
  int* hist = L3;                    // [n_lvl + 1]: sequences with np_b = v
  int* tie = L3 + (p.n_lvl + 1);     // [n_lvl + 1]: ranks handed out among equal np_b
  int* lvl = L3 + 2 * (p.n_lvl + 1); // [n_lvl + 1]: count_L, then base_L
  for (int i = tid; i < 3 * (p.n_lvl + 1); i += kVarlenThreads) L3[i] = 0;

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
  __syncthreads();  // the level scratch is cleared before the histogram below
  for (int b = b0; b < b1; ++b) {
    int lo = p.cu[b], hi = p.cu[b + 1];
    int c = p.ctx != nullptr ? p.ctx[b] : 0;
    bool ok = lo >= 0 && hi >= lo && hi <= p.N && c >= 0 && static_cast<long long>(c) + (hi - lo) <= p.max_keys;
    const long long keys = ok ? static_cast<long long>(c) + (hi - lo) : 0;
    long long kb = lo;
    if (p.key_cap > 0) {
      kb = koff;
      koff += keys;
      if (ok && kb + keys > p.key_cap) ok = false;  // more keys than the workspace holds
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
    if (np > 0) atomicAdd(&hist[min(np, p.n_lvl)], 1);
  }
  __syncthreads();

  // 3. count_L = #{b : np_b > L} = sum of hist[v] over v > L (a suffix sum), then
  //    base_L = sum of count_L' over L' > L (another); both as CTA scans over level runs.
  const int lper = (p.n_lvl + 1 + kVarlenThreads - 1) / kVarlenThreads;
  const int l0 = min(p.n_lvl + 1, tid * lper), l1 = min(p.n_lvl + 1, l0 + lper);
  {
    // Suffix sums: the levels above a thread's run are the runs of the higher threads,
    // whose sum is the total minus this thread's inclusive prefix.
    long long run = 0;
    for (int v = l0; v < l1; ++v) run += hist[v];
    long long tot;
    const long long before = cta_exclusive_scan(run, s_scan, tot);
    long long after = tot - before - run;  // sequences counted at levels above this thread's run
    for (int v = l1 - 1; v >= l0; --v) {
      lvl[v] = static_cast<int>(after);  // count_v = #{np > v}
      after += hist[v];
    }
  }
  __syncthreads();
  int total_entries;
  {
    long long run = 0;
    for (int v = l0; v < l1; ++v) run += lvl[v];
    long long tot;
    const long long before = cta_exclusive_scan(run, s_scan, tot);
    long long after = tot - before - run;
    __syncthreads();
    for (int v = l1 - 1; v >= l0; --v) {
      const int cnt = lvl[v];
      lvl[v] = static_cast<int>(after);  // base_v: entries of all higher pair indices
      after += cnt;
    }
    total_entries = static_cast<int>(tot);
  }
  __syncthreads();

  // 4. ranks.  base_{L-1} - base_L = count_L, so the number of sequences with more pairs
  //    than this one is base_{np_b - 1} - base_{np_b}.
  for (int b = b0; b < b1; ++b) {
    const int np = min((p.seq[b].y + p.two_p - 1) / p.two_p, p.n_lvl);
    if (np == 0) continue;
    const int rank = (lvl[np - 1] - lvl[np]) + atomicAdd(&tie[np], 1);
    p.order[rank] = b;
  }
  __syncthreads();
  // 5. entries, one per thread and step: pair index L = the smallest with base_L <= e
  //    (base_L does not increase with L), sequence order[e - base_L].
  const int n_ent = min(total_entries, p.max_entries);
  for (int e = tid; e < n_ent; e += kVarlenThreads) {
    int lo = 0, hi = p.n_lvl - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (lvl[mid] <= e) {
        hi = mid;
      } else {
        lo = mid + 1;
      }
    }
    const int b = p.order[e - lvl[lo]];
    p.ent[2 * e] = p.seq[b];
    p.ent[2 * e + 1] = make_int4(lo, b, 0, 0);
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
