// prefill.cuh - causal GQA flash attention for sm_100a over the normed, rotated queries and
// keys that the QK-Norm+RoPE prologue kernel leaves in the workspace (or the KV cache).
//
// What it computes: for every query row, softmax over keys j <= i of (q'.k'_j)/sqrt(d),
// times v_j, where q' and k' are the QK-Normed and rotated vectors and query head h reads
// KV head h/G ("Assembling a large model from scratch", Attention.forward: scores, tril
// mask, fp32 softmax, repeat_interleave of KV heads; "Hand-Writing a Vision-Language Model,
// Part 1", order of operations).  The online (running-max) logsumexp that lets the key
// axis be tiled is the technique named for the fused cross-entropy in "Qwen3 Architecture
// Layer-by-Layer", Liger fused linear cross-entropy.
//
// Work decomposition.  A query tile is 128 MMA rows: P = 128/G consecutive positions x the
// G query heads of one KV group, so every K/V tile feeds all heads that share it.  A work
// item is a pair of adjacent query tiles (A = 2i, B = 2i+1) of one (batch row, KV head):
// both read the same K/V tiles, so each K/V tile is loaded once per pair and feeds 256
// rows.  CTAs are persistent (one per SM) and take items in heaviest-first order.
//
// Ten warps:
//   warp 0      TMA producer: the item's two Q' tiles (the prologue kernel wrote Q' in the
//               tiles' row order, so a tile is one 2-D box pair), then K'/V tiles (128 keys
//               x 128 dims, two 128B-swizzled boxes each) into a 2-stage ring; owns the TMEM
//               allocation.  Q'_X of the next item is loaded as soon as the last S_X MMA of
//               the current item has read the buffer, so it is resident before it is needed.
//   warp 1      MMA issuer (one thread).  Per key tile j it issues PV_A(j-1), S_A(j),
//               PV_B(j-1), S_B(j), so the tensor core works on one tile while the softmax
//               warpgroup of the other tile runs.
//   warps 2-5   softmax warpgroup of tile A, one thread per row (TMEM lane quadrant =
//   warps 6-9   warp % 4); softmax warpgroup of tile B.  Per key tile: tcgen05.ld of its S row,
//               causal mask, exp2 online softmax with a lazy rescale (O is rescaled only
//               when the running max grows by more than 2^8), bf16 P written back into TMEM
//               over its own S columns; finally O/l and the LSE.
// TMEM (512 columns): S_A [0,128) with P_A at [0,64), O_A [128,256), S_B [256,384) with
// P_B at [256,320), O_B [384,512).  PV reads P from TMEM (the TS form of tcgen05.mma).
// Ordering: one thread issues every MMA and they complete in issue order, so the commit
// that signals S_X(j) also covers PV_X(j-1): once a softmax thread sees S_X(j) it may
// overwrite P_X and rescale O_X without a further wait.
// Every wait is bounded (see mbar_wait); on a timeout every role stops, copies and MMAs in
// flight are drained, TMEM is freed and the error is left in the status word.
#pragma once
#include "common.cuh"

namespace q3 {

struct PrefillParams {
  const float* q_norm_w;  // the gains: only their max |g| is used here (the logit bound)
  const float* k_norm_w;
  float* lse;      // [B, Hq, T] or nullptr
  int B, T, Hq, Hkv, log2G, P, n_qt, n_pairs, n_items;
  int start;   // cached keys before the first query row: query t is key index start + t
  int window;  // sliding window W: query key index i sees keys i-W < j <= i; 0 = all
  float eps, scale_log2;
  float rope_scale;  // attention_scaling that scaled q' and k' (enters the logit bound squared)
  WaitCfg wait;
  int fault;
  int force_rmax;  // nonzero: the running-max softmax whatever the logit bound (a test hook)
  // Varlen batches (the kVar instance): the entry list {qoff, T, start, koff}, {pair, b}
  // and its item count, both written on the device; B is then the sequence count, T the
  // packed token count N, and `out` [N, Hq, d] takes the rows of tiles that end past their
  // sequence (a tiled store of those would write into the next sequence's rows).
  const int4* vl_ent;
  const int* vl_n_items;
  uint4* out;
  // Key-axis split (the kSplit instance): every (pair, batch row, KV head) is n_split items,
  // split s taking the s-th of n_split contiguous runs of the pair's key tiles.  Each item
  // leaves its rows' O/l (fp32) and LSE as partials, [B*T, Hq, n_split, d] and
  // [B*T, Hq, n_split], for prefill_split_combine_kernel.
  int n_split;
  float* part_o;
  float* part_lse;
  // dual != 0 (only with ring3): an item is two runs of one pair, 2s for tile A and 2s + 1
  // for tile B, and both tiles are the pair's single query tile (one Q' buffer, read by both
  // S MMAs), so the CTA's two softmax groups overlap on it.
  int dual;
  // ring3 != 0 (the kSplit instance, when every pair has a single query tile: T * G <= 128):
  // a K/V ring of three stages instead of two, for more bytes in flight per CTA.
  int ring3;
  // kv_early != 0: the keys and values before `start` that tmK and tmV cover were written
  // before the kernel ahead of this one began (a contiguous cache), so the producer may load
  // them before waiting for that kernel.
  int kv_early;
  // Keys and values read in place from page pools (block_table != nullptr): tmK and tmV are
  // 2-D maps over the pools as rows of d, [num_pages * Hkv * page, d], with boxes of
  // min(page, 128) rows, and key j of batch row (or sequence) r lies in page
  // block_table[r, j >> log2_page] at row j & (page - 1).
  const int* block_table;
  int max_blocks, log2_page, num_pages;
};

constexpr uint32_t kPfTile = 32768;  // 128 rows x 128 bf16
constexpr uint32_t kPfBox = 16384;   // 128 rows x 64 bf16: one 128B-swizzled TMA box
constexpr uint32_t kPfQ = 0;         // Q'_A, Q'_B
constexpr uint32_t kPfK = 2 * kPfTile;  // 2 stages
constexpr uint32_t kPfV = 4 * kPfTile;  // 2 stages
constexpr uint32_t kPfBar = 6 * kPfTile;
// Output staging, one 128-row x 64-dim box (16 KB, 128B-swizzled) per softmax group: the
// epilogue writes half of O/l there and one thread stores it to `out` with a tiled bulk copy.
constexpr uint32_t kPfStage = kPfBar + 1024;
// barrier block (byte offsets from kPfBar); [X] = tile A (0) or B (1), [s] = ring stage (up to 3)
constexpr uint32_t kBKFull = 0, kBKEmpty = 24, kBVFull = 48, kBVEmpty = 72, kBSFull = 96, kBPReady = 112,
                   kBOFull = 128, kBQFull = 144, kBQEmpty = 160,  // [X]: an item's last S_X MMA has read Q'_X
                   kBDone = 176,
                   kBTail = 184,  // a paged V tile past the keys' end has landed (zeroed after)
                   kBTmemSlot = 192, kBAbort = 196,
                   kBRed = 200;  // 2 groups x 4 warps x (max|g_q|, max|g_k|): 64 bytes
constexpr uint32_t kPrefillSmemBytes = kPfStage + 2 * kPfBox + 1024;  // + slack to align the base to 1024

// K/V ring stage s.  Stages 0 and 1 sit in the K and V regions.  A third stage, used when
// every item has a single query tile (ring3), takes Q'_B's buffer for K and the output
// staging for V: such items load Q' into buffer A only, and a split's epilogue writes its
// partials straight from tensor memory.
__device__ __forceinline__ uint32_t k_stage(uint32_t sb, int s) {
  return s < 2 ? sb + kPfK + s * kPfTile : sb + kPfQ + kPfTile;
}
__device__ __forceinline__ uint32_t v_stage(uint32_t sb, int s) {
  return s < 2 ? sb + kPfV + s * kPfTile : sb + kPfStage;
}
// Stage and phase bit of the t-th K/V load in a ring of R (2 or 3) stages.
__device__ __forceinline__ void ring_pos(uint32_t t, int R, int& s, uint32_t& ph) {
  if (R == 2) {
    s = static_cast<int>(t & 1);
    ph = (t >> 1) & 1;
  } else {
    s = static_cast<int>(t % 3u);
    ph = (t / 3u) & 1;
  }
}
constexpr int kPrefillThreads = 320;
constexpr uint32_t kTmPOff = 0;  // P within S: chunk c of P lands on S columns already read
constexpr float kLn2 = 0.693147180559945309f;

__device__ __forceinline__ uint32_t tm_s(int X) { return X == 0 ? 0u : 256u; }
__device__ __forceinline__ uint32_t tm_o(int X) { return X == 0 ? 128u : 384u; }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// D[tmem] (+)= A[tmem] * B[smem desc]: the TS form, A (here P) read from tensor memory.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct TileInfo {
  int t0, nkv;  // first query row; key tiles it reads from the item's first (0 = past T)
};

// The sequence an item belongs to: its first token on the query axis, its new tokens, its
// cached keys before them, and its first key row.  One batch row of a uniform batch is
// {0, T, start, 0} (its rows are addressed through the batch coordinate instead).
struct ItemSeq {
  int qoff, T, start, koff;
};

// First key tile of a pair item: 0, or with a sliding window the tile holding the first key
// that tile A's first row may see (tile B's rows start later, so they mask one tile at most).
template <bool kWin>
__device__ __forceinline__ int item_lo(const PrefillParams& p, const ItemSeq& sq, int pair) {
  if constexpr (!kWin) return 0;
  return max(0, sq.start + 2 * pair * p.P - p.window + 1) >> 7;
}

__device__ __forceinline__ TileInfo tile_info(const PrefillParams& p, const ItemSeq& sq, int qt, int lo) {
  TileInfo ti;
  ti.t0 = qt * p.P;
  ti.nkv = (ti.t0 < sq.T) ? (sq.start + min(ti.t0 + p.P, sq.T) - 1) / 128 + 1 - lo : 0;
  return ti;
}

// The key tiles an item reads: from tile lo[X] on, nX[X] of them for its query tile X (0
// when the item has no tile X).  A split item takes its own run of the pair's tiles: split
// s of n covers tiles [s*N/n, (s+1)*N/n) of the N the pair reads, and tile X reads the part
// of that run below its own tile count.  A dual item (one query tile per pair) takes run s
// of n/2 and gives its first half to tile A and the rest to tile B, which holds the same
// query rows.
template <bool kWin, bool kSplit>
__device__ __forceinline__ void item_tiles(const PrefillParams& p, const ItemSeq& sq, int pair, int split,
                                           int (&lo)[2], int (&nX)[2]) {
  const int l0 = item_lo<kWin>(p, sq, pair);
  nX[0] = tile_info(p, sq, 2 * pair, l0).nkv;
  nX[1] = tile_info(p, sq, 2 * pair + 1, l0).nkv;
  lo[0] = lo[1] = l0;
  if constexpr (kSplit) {
    if (p.dual) {
      const int runs = p.n_split / 2, N = nX[0];
      const int j0 = static_cast<int>(static_cast<long long>(split) * N / runs);
      const int j1 = static_cast<int>(static_cast<long long>(split + 1) * N / runs);
      const int m = (j1 - j0 + 1) / 2;
      lo[0] = l0 + j0;
      nX[0] = m;
      lo[1] = l0 + j0 + m;
      nX[1] = j1 - j0 - m;
    } else {
      const int n = max(nX[0], nX[1]);
      const int j0 = static_cast<int>(static_cast<long long>(split) * n / p.n_split);
      const int j1 = static_cast<int>(static_cast<long long>(split + 1) * n / p.n_split);
      nX[0] = max(0, min(nX[0], j1) - j0);
      nX[1] = max(0, min(nX[1], j1) - j0);
      lo[0] = lo[1] = l0 + j0;
    }
  }
}

// A dual item's K/V loads interleave its tiles: A0, B0, A1, B1, ..., and A's last when it
// has one more.  The u-th load's query tile X and step j.
__device__ __forceinline__ void dual_load(int u, int nB, int& X, int& j) {
  X = u < 2 * nB ? (u & 1) : 0;
  j = u < 2 * nB ? (u >> 1) : u - nB;
}

// Item this CTA takes in round k: snake order (left to right in even rounds, right to left
// in odd ones) over the heaviest-first numbering, so the heaviest and lightest items of
// consecutive rounds land on the same CTA.
__device__ __forceinline__ int round_item(int k) {
  return (k & 1) ? k * static_cast<int>(gridDim.x) + static_cast<int>(gridDim.x - 1 - blockIdx.x)
                 : k * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
}

// Work item -> (pair, batch row, KV head); items are numbered heaviest pair first.
__device__ __forceinline__ void item_coords(const PrefillParams& p, int item, int& pair, int& b, int& hkv) {
  const int BH = p.B * p.Hkv;
  pair = p.n_pairs - 1 - item / BH;
  const int bh = item % BH;
  b = bh / p.Hkv;
  hkv = bh % p.Hkv;
}

// Items of a launch: from the parameters, or for a varlen batch from the device's entry list.
template <bool kVar>
__device__ __forceinline__ int item_count(const PrefillParams& p) {
  if constexpr (kVar) return __ldcg(p.vl_n_items);
  return p.n_items;
}

// Work item -> (pair, batch coordinate, KV head, sequence).  A varlen item reads its entry
// (two independent 16-byte loads); its batch coordinate is 0 (the packed axis is one row).
template <bool kVar, bool kSplit = false>
__device__ __forceinline__ void item_fetch(const PrefillParams& p, int item, int& pair, int& b, int& hkv,
                                           ItemSeq& sq, int& split, int* seq_index = nullptr) {
  split = 0;
  if constexpr (kSplit) {
    // the items of one pair are adjacent: the heaviest-first order of pairs stays
    const int per = p.dual ? p.n_split / 2 : p.n_split;
    split = item % per;
    item_coords(p, item / per, pair, b, hkv);
    sq = ItemSeq{0, p.T, p.start, 0};
    return;
  }
  if constexpr (kVar) {
    const int e = item / p.Hkv;
    hkv = item - e * p.Hkv;
    const int4 a = __ldcg(p.vl_ent + 2 * e);
    const int4 c = __ldcg(p.vl_ent + 2 * e + 1);
    sq = ItemSeq{a.x, a.y, a.z, a.w};
    pair = c.x;
    b = 0;
    if (seq_index != nullptr) *seq_index = c.y;
  } else {
    item_coords(p, item, pair, b, hkv);
    sq = ItemSeq{0, p.T, p.start, 0};
  }
}

// Paged-cache loads.  They run in the producer warp only, and their code shares the
// instruction cache with the softmax warps' hot loop: unrolled at each of their three call
// sites they cost the prefill a third of its speed in instruction fetch stalls, so the
// copies are issued by one out-of-line function.
//
// The block-table entries of the boxes of a 128-key tile, for the boxes that start before
// the row's key count nk (boxes of R = min(page, 128) rows, each inside one page): only the
// loads, into registers, so the producer issues them a tile ahead of their use.  Entries
// past the table are -1.  Returns the box count.
__device__ __forceinline__ int paged_tile_fetch(const PrefillParams& p, const int* table_row, int key0, int nk,
                                                int (&pg)[8]) {
  const int R = min(1 << p.log2_page, 128);
  const int nsub = min(128 / R, (nk - key0 + R - 1) / R);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int blk = (key0 + i * R) >> p.log2_page;
    pg[i] = (i < nsub && blk < p.max_blocks) ? __ldg(table_row + blk) : -1;
  }
  return nsub;
}

// The loads of one 128-key tile (two 64-dim halves) into `dst`, signalled on `bar`: one box
// per entry g0..g7 below nsub, none for an out-of-range page (recorded as an invalid
// argument).  The barrier's expected bytes are set after the copies are issued, as the sum
// of what they carry; its phase cannot complete before that arrival.
__device__ __noinline__ void paged_tile_issue(const PrefillParams& p, uint32_t dst, const CUtensorMap* map,
                                              uint32_t bar, int nsub, int key0, int hkv, int g0, int g1, int g2,
                                              int g3, int g4, int g5, int g6, int g7) {
  const int R = min(1 << p.log2_page, 128);
  const int pg[8] = {g0, g1, g2, g3, g4, g5, g6, g7};
  uint32_t bytes = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i >= nsub) break;
    if (pg[i] < 0 || pg[i] >= p.num_pages) {
      record_error(QWEN3_ERR_INVALID_ARG, kSitePagedTable);
      continue;
    }
    const int row = ((pg[i] * p.Hkv + hkv) << p.log2_page) | ((key0 + i * R) & ((1 << p.log2_page) - 1));
    tma_load_2d(dst + i * R * 128, map, bar, 0, row);
    tma_load_2d(dst + kPfBox + i * R * 128, map, bar, 64, row);
    bytes += static_cast<uint32_t>(R) * 256u;
  }
  mbar_arrive_expect_tx(bar, bytes);
}

// kWin: a sliding window is set (p.window > 0); the full-causal instance carries none of its
// masks or bookkeeping.  kVar: a varlen batch (items from the device's entry list).  kSplit:
// a key-axis split (a uniform batch, no window), whose items write partials.
template <bool kWin, bool kVar, bool kSplit = false>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    fmha_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                        const __grid_constant__ PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sb - raw);
  const uint32_t bar = sb + kPfBar;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kPfBar + kBAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + kPfBar + kBTmemSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A split's combine kernel, launched next, may be scheduled now: it waits for this grid.
  if constexpr (kSplit) griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < 3; ++s) {
      mbar_init(bar + kBKFull + 8 * s, 1);
      mbar_init(bar + kBKEmpty + 8 * s, 1);
      mbar_init(bar + kBVFull + 8 * s, 1);
      mbar_init(bar + kBVEmpty + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar + kBSFull + 8 * s, 1);
      mbar_init(bar + kBPReady + 8 * s, 128);
      mbar_init(bar + kBOFull + 8 * s, 1);
      mbar_init(bar + kBQFull + 8 * s, 1);
      mbar_init(bar + kBQEmpty + 8 * s, 1);
    }
    mbar_init(bar + kBDone, 1);
    mbar_init(bar + kBTail, 1);
    *abort_flag = 0;
    mbar_init_fence();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      int k_last[3] = {-1, -1, -1}, v_last[3] = {-1, -1, -1}, q_last[2] = {-1, -1};
      const int R = kSplit && p.ring3 != 0 ? 3 : 2;  // K/V ring stages
      const int n_items = item_count<kVar>(p);
      // The first item's first K/V tiles of a contiguous cache that lie wholly before the new
      // keys were written by earlier calls, not by the prologue: they are loaded into the
      // empty ring before waiting for the prologue, so their latency overlaps it.
      int pre = 0;
      if constexpr (!kVar) {
        const int item0 = round_item(0);
        if (p.kv_early != 0 && p.block_table == nullptr && item0 < n_items) {
          int pair, b, hkv, split, lo[2], nX[2];
          ItemSeq sq;
          item_fetch<false, kSplit>(p, item0, pair, b, hkv, sq, split);
          item_tiles<kWin, kSplit>(p, sq, pair, split, lo, nX);
          const bool dual = kSplit && p.dual != 0;
          const int n = dual ? nX[0] + nX[1] : max(nX[0], nX[1]);
          for (; pre < min(n, R); ++pre) {
            int X = 0, j = pre;
            if (dual) dual_load(pre, nX[1], X, j);
            const int key0 = ((X != 0 ? lo[1] : lo[0]) + j) * 128;
            if (key0 + 128 > sq.start) break;  // keys from here on may come from the prologue
            const uint32_t sKs = k_stage(sb, pre), sVs = v_stage(sb, pre);
            if (!(p.fault != 0 && pre == 0)) {
              mbar_arrive_expect_tx(bar + kBKFull + 8 * pre, kPfTile);
              tma_load_4d(sKs, &tmK, bar + kBKFull + 8 * pre, 0, sq.koff + key0, hkv, b);
              tma_load_4d(sKs + kPfBox, &tmK, bar + kBKFull + 8 * pre, 64, sq.koff + key0, hkv, b);
              k_last[pre] = pre;
            }
            mbar_arrive_expect_tx(bar + kBVFull + 8 * pre, kPfTile);
            tma_load_4d(sVs, &tmV, bar + kBVFull + 8 * pre, 0, sq.koff + key0, hkv, b);
            tma_load_4d(sVs + kPfBox, &tmV, bar + kBVFull + 8 * pre, 64, sq.koff + key0, hkv, b);
            v_last[pre] = pre;
          }
        }
      }
      griddep_wait();  // Q', K' (and a cache's V) come from the prologue kernel before this one
      uint32_t it = 0, q_use[2] = {0, 0}, tail_use = 0;
      bool ok = true;
      for (int k = 0, item = round_item(0); item < n_items && ok; item = round_item(++k)) {
        int pair, b, hkv, split, lo[2], nX[2], seq = 0;
        ItemSeq sq;
        item_fetch<kVar, kSplit>(p, item, pair, b, hkv, sq, split, &seq);
        item_tiles<kWin, kSplit>(p, sq, pair, split, lo, nX);
        const bool dual = kSplit && p.dual != 0;
        // a paged cache: the row's block table (a varlen sequence's own row) and key count
        const int* table_row =
            p.block_table != nullptr ? p.block_table + static_cast<long long>(kVar ? seq : b) * p.max_blocks : nullptr;
        const int nk = sq.start + sq.T;
        // K/V loads: one per step, shared by both tiles, or one per tile of a dual item
        const int n = dual ? nX[0] + nX[1] : max(nX[0], nX[1]);
        // first key of the u-th load
        auto load_key = [&](int u) {
          int X = 0, j = u;
          if (dual) dual_load(u, nX[1], X, j);
          return ((X != 0 ? lo[1] : lo[0]) + j) * 128;
        };
        // the first tile's block-table entries; each later tile's are fetched one tile ahead
        int pg_next[8] = {-1, -1, -1, -1, -1, -1, -1, -1}, nsub_next = 0;
        if (table_row != nullptr && n > 0) nsub_next = paged_tile_fetch(p, table_row, load_key(0), nk, pg_next);
        for (int X = 0; X < 2 && ok; ++X) {
          if (nX[X] == 0 || (dual && X == 1)) continue;  // a dual item's tiles share buffer A
          // buffer X is free once the previous item's last S_X MMA has completed
          if (q_use[X] >= 1 &&
              !mbar_wait(bar + kBQEmpty + 8 * X, (q_use[X] - 1) & 1, p.wait, abort_flag, kSitePrefillQEmpty)) {
            ok = false;
            break;
          }
          // the tile's first row of Q' [b, hkv, T*G, d] (a varlen batch: [0, hkv, N*G, d])
          const int row0 = (sq.qoff << p.log2G) + (2 * pair + X) * 128;
          mbar_arrive_expect_tx(bar + kBQFull + 8 * X, kPfTile);
          tma_load_4d(sb + kPfQ + X * kPfTile, &tmQ, bar + kBQFull + 8 * X, 0, row0, hkv, b);
          tma_load_4d(sb + kPfQ + X * kPfTile + kPfBox, &tmQ, bar + kBQFull + 8 * X, 64, row0, hkv, b);
          q_last[X] = static_cast<int>(q_use[X]++);
        }
        for (int j = 0; j < n && ok; ++j, ++it) {
          if (k == 0 && j < pre) continue;  // loaded before the prologue's results were awaited
          int st;
          uint32_t ph;
          ring_pos(it, R, st, ph);
          const uint32_t sKs = k_stage(sb, st), sVs = v_stage(sb, st);
          if (it >= static_cast<uint32_t>(R) &&
              !mbar_wait(bar + kBKEmpty + 8 * st, ph ^ 1, p.wait, abort_flag, kSitePrefillKEmpty)) {
            ok = false;
            break;
          }
          const int key0 = load_key(j);
          if (table_row == nullptr) {
            if (!(p.fault != 0 && it == 0)) {
              mbar_arrive_expect_tx(bar + kBKFull + 8 * st, kPfTile);
              tma_load_4d(sKs, &tmK, bar + kBKFull + 8 * st, 0, sq.koff + key0, hkv, b);
              tma_load_4d(sKs + kPfBox, &tmK, bar + kBKFull + 8 * st, 64, sq.koff + key0, hkv, b);
              k_last[st] = static_cast<int>(it);
            }
            if (it >= static_cast<uint32_t>(R) &&
                !mbar_wait(bar + kBVEmpty + 8 * st, ph ^ 1, p.wait, abort_flag, kSitePrefillVEmpty)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar + kBVFull + 8 * st, kPfTile);
            tma_load_4d(sVs, &tmV, bar + kBVFull + 8 * st, 0, sq.koff + key0, hkv, b);
            tma_load_4d(sVs + kPfBox, &tmV, bar + kBVFull + 8 * st, 64, sq.koff + key0, hkv, b);
            v_last[st] = static_cast<int>(it);
          } else {
            // In place from the pages: one box per page (or per 128 rows of a larger page),
            // none for the part of the tile past the keys' end.  The bytes the barrier waits
            // for are those of the boxes issued.
            int pg[8];
            const int nsub = nsub_next;
#pragma unroll
            for (int i = 0; i < 8; ++i) pg[i] = pg_next[i];
            if (j + 1 < n) nsub_next = paged_tile_fetch(p, table_row, load_key(j + 1), nk, pg_next);
            if (!(p.fault != 0 && it == 0)) {
              paged_tile_issue(p, sKs, &tmK, bar + kBKFull + 8 * st, nsub, key0, hkv, pg[0], pg[1],
                               pg[2], pg[3], pg[4], pg[5], pg[6], pg[7]);
              k_last[st] = static_cast<int>(it);
            }
            if (it >= static_cast<uint32_t>(R) &&
                !mbar_wait(bar + kBVEmpty + 8 * st, ph ^ 1, p.wait, abort_flag, kSitePrefillVEmpty)) {
              ok = false;
              break;
            }
            if (key0 + 128 <= nk) {
              paged_tile_issue(p, sVs, &tmV, bar + kBVFull + 8 * st, nsub, key0, hkv, pg[0], pg[1],
                               pg[2], pg[3], pg[4], pg[5], pg[6], pg[7]);
            } else {
              // The tile runs past the keys' end: its rows from there on hold whatever the page
              // (or an earlier use of this buffer) left, NaN included, and P = 0 there would
              // still carry NaN into P.V.  Load on the private barrier, zero those rows, then
              // release the tile to the MMA issuer.
              paged_tile_issue(p, sVs, &tmV, bar + kBTail, nsub, key0, hkv, pg[0], pg[1], pg[2],
                               pg[3], pg[4], pg[5], pg[6], pg[7]);
              if (!mbar_wait(bar + kBTail, tail_use & 1, p.wait, abort_flag, kSitePrefillVFull)) {
                // the copies still land in this CTA's shared memory: wait for them regardless
                mbar_wait(bar + kBTail, tail_use & 1, p.wait, nullptr, kSitePrefillDrain);
                ok = false;
                break;
              }
              ++tail_use;
#pragma unroll 1
              for (int r = nk - key0; r < 128; ++r)
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                  st_shared_v4(sVs + r * 128 + c * 16, 0u, 0u, 0u, 0u);
                  st_shared_v4(sVs + kPfBox + r * 128 + c * 16, 0u, 0u, 0u, 0u);
                }
              fence_proxy_async_smem();
              mbar_arrive(bar + kBVFull + 8 * st);
            }
            v_last[st] = static_cast<int>(it);
          }
        }
      }
      // Every issued copy must land before this CTA's shared memory is released.
      for (int s = 0; s < 2; ++s)
        if (q_last[s] >= 0) mbar_wait(bar + kBQFull + 8 * s, q_last[s] & 1, p.wait, nullptr, kSitePrefillDrain);
      for (int s = 0; s < R; ++s) {
        int st;
        uint32_t ph;
        if (k_last[s] >= 0) {
          ring_pos(static_cast<uint32_t>(k_last[s]), R, st, ph);
          mbar_wait(bar + kBKFull + 8 * s, ph, p.wait, nullptr, kSitePrefillDrain);
        }
        if (v_last[s] >= 0) {
          ring_pos(static_cast<uint32_t>(v_last[s]), R, st, ph);
          mbar_wait(bar + kBVFull + 8 * s, ph, p.wait, nullptr, kSitePrefillDrain);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdQK = idesc_bf16(128, 128, false);  // B = K rows, K-major
      constexpr uint32_t kIdPV = idesc_bf16(128, 128, true);   // B = V, dims contiguous (MN-major)
      uint32_t it = 0, q_cnt[2] = {0, 0}, p_cnt[2] = {0, 0};
      bool ok = true;
      const int R = kSplit && p.ring3 != 0 ? 3 : 2;  // K/V ring stages
      const int n_items = item_count<kVar>(p);
      for (int k = 0, item = round_item(0); item < n_items && ok; item = round_item(++k)) {
        int pair, b, hkv, split, lo[2], nX[2];
        ItemSeq sq;
        item_fetch<kVar, kSplit>(p, item, pair, b, hkv, sq, split);
        item_tiles<kWin, kSplit>(p, sq, pair, split, lo, nX);
        const bool dual = kSplit && p.dual != 0;
        const int n = max(nX[0], nX[1]);
        if ((kVar || kSplit) && n == 0) continue;  // an item with no tile (the producer skips it too)
        for (int X = 0; X < (dual ? 1 : 2) && ok; ++X)
          if (nX[X] > 0) {
            ok = mbar_wait(bar + kBQFull + 8 * X, q_cnt[X] & 1, p.wait, abort_flag, kSitePrefillQFull);
            ++q_cnt[X];
          }
        if (!ok) break;
        if (dual) {
          // A dual item: each tile has its own K/V loads, taken in the producer's order, and
          // both read Q' buffer A.  Step j issues PV_X(j-1) then S_X(j), for X = A, B.
          const int nB = nX[1];
          for (int j = 0; j <= n && ok; ++j) {
            for (int X = 0; X < 2 && ok; ++X) {
              int st;
              uint32_t ph;
              if (j >= 1 && j - 1 < nX[X]) {
                ring_pos(it + (j - 1 < nB ? 2 * (j - 1) + X : nB + j - 1), R, st, ph);
                ok = mbar_wait(bar + kBVFull + 8 * st, ph, p.wait, abort_flag, kSitePrefillVFull) &&
                     mbar_wait(bar + kBPReady + 8 * X, p_cnt[X] & 1, p.wait, abort_flag, kSitePrefillPReady);
                ++p_cnt[X];
                if (!ok) break;
                tc_fence_after();
                const uint32_t sVs = v_stage(sb, st);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                  tc_mma_ts(tmem + tm_o(X), tmem + tm_s(X) + kTmPOff + kk * 8,
                            smem_desc_sw128(sVs + kk * 2048, kPfBox, 1024), kIdPV, (j > 1 || kk > 0) ? 1u : 0u);
                if (j == nX[X]) tc_commit(bar + kBOFull + 8 * X);
                tc_commit(bar + kBVEmpty + 8 * st);
              }
              if (j < nX[X]) {
                ring_pos(it + (j < nB ? 2 * j + X : nB + j), R, st, ph);
                ok = mbar_wait(bar + kBKFull + 8 * st, ph, p.wait, abort_flag, kSitePrefillKFull);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sKs = k_stage(sb, st);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                  const uint32_t koff = (kk >> 2) * kPfBox + (kk & 3) * 32;
                  tc_mma_ss(tmem + tm_s(X), smem_desc_sw128(sb + kPfQ + koff, 16, 1024),
                            smem_desc_sw128(sKs + koff, 16, 1024), kIdQK, kk > 0 ? 1u : 0u);
                }
                tc_commit(bar + kBSFull + 8 * X);
                // the item's last S MMA (B's, or A's when A has one tile more) frees buffer A
                if (j == nX[X] - 1 && (X == 1) == (nB == nX[0])) tc_commit(bar + kBQEmpty);
                tc_commit(bar + kBKEmpty + 8 * st);
              }
            }
          }
          it += nX[0] + nX[1];
          continue;
        }
        // j = 0: S_A(0), S_B(0)
        int sc;
        uint32_t pc;
        ring_pos(it, R, sc, pc);
        ok = mbar_wait(bar + kBKFull + 8 * sc, pc, p.wait, abort_flag, kSitePrefillKFull);
        if (!ok) break;
        tc_fence_after();
        for (int X = 0; X < 2; ++X)
          if (nX[X] > 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t koff = (kk >> 2) * kPfBox + (kk & 3) * 32;
              tc_mma_ss(tmem + tm_s(X), smem_desc_sw128(sb + kPfQ + X * kPfTile + koff, 16, 1024),
                        smem_desc_sw128(k_stage(sb, sc) + koff, 16, 1024), kIdQK, kk > 0 ? 1u : 0u);
            }
            tc_commit(bar + kBSFull + 8 * X);
            if (nX[X] == 1) tc_commit(bar + kBQEmpty + 8 * X);  // the item's last S_X
          }
        tc_commit(bar + kBKEmpty + 8 * sc);
        // j >= 1: PV_X(j-1) then S_X(j), for X = A, B
        for (int j = 1; j <= n && ok; ++j) {
          const int sp = sc;  // stage and phase of tile j-1
          const uint32_t pv = pc;
          if (j < n) {
            ring_pos(it + j, R, sc, pc);
            ok = mbar_wait(bar + kBKFull + 8 * sc, pc, p.wait, abort_flag, kSitePrefillKFull);
            if (!ok) break;
          }
          ok = mbar_wait(bar + kBVFull + 8 * sp, pv, p.wait, abort_flag, kSitePrefillVFull);
          if (!ok) break;
          for (int X = 0; X < 2; ++X) {
            if (j - 1 < nX[X]) {
              ok = mbar_wait(bar + kBPReady + 8 * X, p_cnt[X] & 1, p.wait, abort_flag, kSitePrefillPReady);
              ++p_cnt[X];
              if (!ok) break;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                tc_mma_ts(tmem + tm_o(X), tmem + tm_s(X) + kTmPOff + kk * 8,
                          smem_desc_sw128(v_stage(sb, sp) + kk * 2048, kPfBox, 1024), kIdPV,
                          (j > 1 || kk > 0) ? 1u : 0u);
              if (j == nX[X]) tc_commit(bar + kBOFull + 8 * X);
            }
            if (j < nX[X]) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk >> 2) * kPfBox + (kk & 3) * 32;
                tc_mma_ss(tmem + tm_s(X), smem_desc_sw128(sb + kPfQ + X * kPfTile + koff, 16, 1024),
                          smem_desc_sw128(k_stage(sb, sc) + koff, 16, 1024), kIdQK, kk > 0 ? 1u : 0u);
              }
              tc_commit(bar + kBSFull + 8 * X);
              if (j == nX[X] - 1) tc_commit(bar + kBQEmpty + 8 * X);  // the item's last S_X
            }
          }
          if (!ok) break;
          tc_commit(bar + kBVEmpty + 8 * sp);
          if (j < n) tc_commit(bar + kBKEmpty + 8 * sc);
        }
        it += n;
      }
      // Drain: every MMA issued above has completed once this arrives.
      tc_commit(bar + kBDone);
      mbar_wait(bar + kBDone, 0, p.wait, nullptr, kSitePrefillDrain);
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    const int X = (warp - 2) >> 2;     // 0: tile A, 1: tile B
    const int wq = warp & 3;           // TMEM lane quadrant this warp may access
    const int row = wq * 32 + lane;    // query-tile row owned by this thread
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + tm_s(X), tO = tmem + lane_off + tm_o(X);
    const float sl2 = p.scale_log2;
    const int G = 1 << p.log2G;
    // Reference for the exponentials.  QK-Norm bounds every logit: by Cauchy-Schwarz on the
    // normalised, rotated (norm-preserving) vectors, |q'.k'|/sqrt(d) <= sqrt(d) max|g_q|
    // max|g_k| (times 1 + 2^-7 for their bf16 rounding).  With that bound bnd (in log2
    // units) at most 60, p = 2^(s*scale*log2(e) - bnd) lies in [2^-120, 1] for every key, so
    // a fixed reference needs no row max, no rescale and can neither overflow nor go
    // subnormal; l and O stay bounded by the key count.  Larger gains take the running-max
    // path (and so does every launch while the host's test hook forces it).  The choice is
    // uniform per CTA.
    float bnd;
    {
      float gq = fabsf(p.q_norm_w[row]), gk = fabsf(p.k_norm_w[row]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        gq = fmaxf(gq, __shfl_xor_sync(0xffffffffu, gq, o));
        gk = fmaxf(gk, __shfl_xor_sync(0xffffffffu, gk, o));
      }
      volatile float* red = reinterpret_cast<volatile float*>(sgen + kPfBar + kBRed) + X * 8;
      if (lane == 0) {
        red[2 * wq] = gq;
        red[2 * wq + 1] = gk;
      }
      asm volatile("bar.sync %0, 128;" ::"r"(1 + X) : "memory");
      gq = fmaxf(fmaxf(red[0], red[2]), fmaxf(red[4], red[6]));
      gk = fmaxf(fmaxf(red[1], red[3]), fmaxf(red[5], red[7]));
      bnd = gq * gk * p.rope_scale * p.rope_scale * (11.3137085f * (1.0f + 0.0078125f) * 1.44269504f);
    }
    const bool fast = bnd <= 60.0f && p.force_rmax == 0;
    uint32_t s_cnt = 0, o_cnt = 0;
    bool ok = true;
    // The tensor core may start the next item (its Q' tiles arrive by TMA) while this
    // group stores the current item's outputs.  O_X stays safe: the next item's first PV_X
    // waits for a P that is only written after this epilogue.
    const int n_items = item_count<kVar>(p);
    for (int k = 0, item = round_item(0); item < n_items && ok; item = round_item(++k)) {
      int pair, b, hkv, split, lo[2], nX[2];
      ItemSeq sq;
      item_fetch<kVar, kSplit>(p, item, pair, b, hkv, sq, split);
      item_tiles<kWin, kSplit>(p, sq, pair, split, lo, nX);
      const bool dual = kSplit && p.dual != 0;
      if (dual) split = 2 * split + X;  // this tile's run: the index of its partials
      TileInfo ti;
      ti.t0 = (dual ? 2 * pair : 2 * pair + X) * p.P;
      ti.nkv = nX[X];
      if (ti.nkv == 0) {
        // This item has no tile X.  A split's run may hold no key a tile's rows see: its
        // partials are still written, as no contribution (LSE -inf), for the combine.
        if constexpr (kSplit) {
          const int t_row = ti.t0 + (row >> p.log2G);
          if (t_row < sq.T)
            p.part_lse[((static_cast<long long>(b) * p.T + t_row) * p.Hq + hkv * G + (row & (G - 1))) * p.n_split +
                       split] = -INFINITY;
        }
        continue;
      }
      const int t0 = ti.t0;
      const int lo_x = (kSplit && X != 0) ? lo[1] : lo[0];  // the tiles differ only in a dual item

      const int t_row = t0 + (row >> p.log2G);
      const int lim = sq.start + min(t_row, sq.T - 1);  // last key index this row may see
      const int wfirst = kWin ? lim - p.window + 1 : 0;  // first one, with a window
      float m = fast ? bnd : -INFINITY, l = 0.f;
      for (int j = 0; j < ti.nkv; ++j) {
        ok = mbar_wait(bar + kBSFull + 8 * X, s_cnt & 1, p.wait, abort_flag, kSitePrefillSFull);
        ++s_cnt;
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const int kv0 = (lo_x + j) * 128;
        // some key of this tile lies past some row's limit, or before some row's window
        const bool diag = kv0 + 127 > sq.start + t0 || (kWin && kv0 < sq.start + t0 + p.P - p.window);
        if (fast) {
          // One pass in four 32-column chunks, the next chunk's TMEM load in flight while the
          // current one is processed.  bf16 P goes to S columns [0,64): chunk c of P
          // overwrites only columns [16c,16c+16), which chunks 0..c have already read.
          const uint64_t sl2x2 = f2pack(sl2, sl2), negb2 = f2pack(-bnd, -bnd);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
          uint32_t cur[32];
          tmem_ld32(tS, cur);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t nxt[32];
            if (c < 3) tmem_ld32_nowait(tS + 32 * (c + 1), nxt);
            if (diag) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int key = kv0 + 32 * c + i;
                cur[i] = (key <= lim && (!kWin || key >= wfirst)) ? cur[i] : 0xff800000u;  // -inf
              }
            }
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float x0, x1;
              f2unpack(ffma2(f2pack(__uint_as_float(cur[2 * i]), __uint_as_float(cur[2 * i + 1])), sl2x2, negb2), x0,
                       x1);
              const float p0 = ex2(x0), p1 = ex2(x1);
              acc[i & 3] = fadd2(acc[i & 3], f2pack(p0, p1));
              pk[i] = pack_bf16x2(p0, p1);
            }
            tmem_st16_nowait(tS + kTmPOff + 16 * c, pk);
            if (c < 3) {
              tmem_wait_ld_dep(nxt);
#pragma unroll
              for (int i = 0; i < 32; ++i) cur[i] = nxt[i];
            }
          }
          float a0, a1, b0, b1, c0, c1, d0, d1;
          f2unpack(acc[0], a0, a1);
          f2unpack(acc[1], b0, b1);
          f2unpack(acc[2], c0, c1);
          f2unpack(acc[3], d0, d1);
          tmem_wait_st();
          l += ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
        } else {
        // Running-max path.  Pass 1: the row max over all 128 keys (two TMEM loads).  Pass 2
        // re-reads S in 32-column chunks, so only one chunk is live while its exponentials
        // are formed.
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t sr[64];
          tmem_ld64(tS + 64 * hh, sr);
          if (diag) {
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int key = kv0 + 64 * hh + c;
              sr[c] = (key <= lim && (!kWin || key >= wfirst)) ? sr[c] : 0xff800000u;  // -inf
            }
          }
#pragma unroll
          for (int c = 0; c < 64; c += 2)
            mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
        }
        const float mt = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
        float m_new = m;
        bool resc = false;
        if (mt > m + 8.0f) {  // lazy rescale: keep a stale max while p stays <= 2^8
          m_new = mt;
          resc = (j > 0);
        }
        // Pass 2: p = 2^(s*scale*log2(e) - m) on pairs; bf16 pairs go straight to P's TMEM
        // columns.  P occupies S columns [0,64): chunk c of P (columns [16c,16c+16)) only
        // overwrites S columns that chunks 0..c have already read.
        // a row whose keys so far all lie outside its window has no max yet: p = 0 for it
        const float mref = ((kWin || kSplit) && m_new == -INFINITY) ? 0.0f : m_new;
        const uint64_t sl2x2 = f2pack(sl2, sl2), negm2 = f2pack(-mref, -mref);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t sr[32];
          tmem_ld32(tS + 32 * c, sr);
          if (diag) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int key = kv0 + 32 * c + i;
              sr[i] = (key <= lim && (!kWin || key >= wfirst)) ? sr[i] : 0xff800000u;
            }
          }
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1;
            f2unpack(ffma2(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), sl2x2, negm2), x0,
                     x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            acc[i & 3] = fadd2(acc[i & 3], f2pack(p0, p1));  // fp32 row sum; P.V uses bf16 p
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st16_nowait(tS + kTmPOff + 16 * c, pk);
        }
        float sum;
        {
          float a0, a1, b0, b1, c0, c1, d0, d1;
          f2unpack(acc[0], a0, a1);
          f2unpack(acc[1], b0, b1);
          f2unpack(acc[2], c0, c1);
          f2unpack(acc[3], d0, d1);
          sum = ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
        }
        if (__any_sync(0xffffffffu, resc)) {
          // PV_X(j-1) has completed: the commit that signalled S_X(j) covers it.
          const float alpha = resc ? ex2(m - m_new) : 1.0f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tO + c * 32, r);
          }
          l *= alpha;
        }
        tmem_wait_st();
        l += sum;
        m = m_new;
        }
        tc_fence_before();
        mbar_arrive(bar + kBPReady + 8 * X);
      }
      if (ok) ok = mbar_wait(bar + kBOFull + 8 * X, o_cnt & 1, p.wait, abort_flag, kSitePrefillOFull);
      ++o_cnt;
      // Every warp of the group gets here, from a finished or an abandoned key loop, and the
      // four agree before the epilogue's group barriers: all go on or all stop.
      ok = group_all(1 + X, ok);
      if (!ok) break;
      tc_fence_after();
      const int h = hkv * G + (row & (G - 1));
      const bool valid = t_row < sq.T;
      if constexpr (kSplit) {
        // This run of keys' O/l (fp32) and its LSE, for the combine kernel.  A row that saw no
        // key of the run (l = 0) leaves O = 0 and LSE = -inf, which the combine weighs by 0.
        const float inv_lp = l > 0.f ? 1.0f / l : 0.f;
        const long long slot = ((static_cast<long long>(b) * p.T + t_row) * p.Hq + h) * p.n_split + split;
        float4* dst = reinterpret_cast<float4*>(p.part_o + slot * kD);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          if (valid) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              dst[c * 8 + u] = make_float4(__uint_as_float(r[4 * u]) * inv_lp, __uint_as_float(r[4 * u + 1]) * inv_lp,
                                           __uint_as_float(r[4 * u + 2]) * inv_lp,
                                           __uint_as_float(r[4 * u + 3]) * inv_lp);
          }
        }
        if (valid) p.part_lse[slot] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
        continue;
      }
      const float inv_l = 1.0f / l;
      // O/l in two 64-dim halves through this group's staging box.  Row r of the tile is row r
      // of the box [P positions][G heads][64 dims], so one tiled store writes the half to
      // out[b, t0 .. t0+P-1, hkv*G .. hkv*G+G-1, half*64 ..]; rows past T are clipped by the
      // copy (a varlen batch: out[qoff + t0 ..], with rows past the sequence stored below).
      // The storing thread waits until the previous store has read the buffer.
      const uint32_t stg = sb + kPfStage + X * kPfBox;
      const bool storer = row == 0;
      if (kVar && t0 + p.P > sq.T) {
        // A varlen tile that ends past its sequence: the rows after it on the packed axis
        // belong to the next sequence, so each thread stores its own row, if it has one,
        // straight from TMEM (eight 16-byte stores per 64 dims).
        uint4* dst = p.out + (static_cast<long long>(sq.qoff + t_row) * p.Hq + h) * (kD / 8);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          if (valid) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              dst[c * 4 + u] =
                  make_uint4(pack_bf16x2(__uint_as_float(r[8 * u + 0]) * inv_l, __uint_as_float(r[8 * u + 1]) * inv_l),
                             pack_bf16x2(__uint_as_float(r[8 * u + 2]) * inv_l, __uint_as_float(r[8 * u + 3]) * inv_l),
                             pack_bf16x2(__uint_as_float(r[8 * u + 4]) * inv_l, __uint_as_float(r[8 * u + 5]) * inv_l),
                             pack_bf16x2(__uint_as_float(r[8 * u + 6]) * inv_l, __uint_as_float(r[8 * u + 7]) * inv_l));
          }
        }
      } else {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        if (storer) bulk_wait_read_all();
        asm volatile("bar.sync %0, 128;" ::"r"(1 + X) : "memory");
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + half * 64 + c * 32, r);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            st_shared_v4(stg + sw128_offset(row, c * 4 + u),
                         pack_bf16x2(__uint_as_float(r[8 * u + 0]) * inv_l, __uint_as_float(r[8 * u + 1]) * inv_l),
                         pack_bf16x2(__uint_as_float(r[8 * u + 2]) * inv_l, __uint_as_float(r[8 * u + 3]) * inv_l),
                         pack_bf16x2(__uint_as_float(r[8 * u + 4]) * inv_l, __uint_as_float(r[8 * u + 5]) * inv_l),
                         pack_bf16x2(__uint_as_float(r[8 * u + 6]) * inv_l, __uint_as_float(r[8 * u + 7]) * inv_l));
        }
        fence_proxy_async_smem();
        asm volatile("bar.sync %0, 128;" ::"r"(1 + X) : "memory");
        if (storer) {
          tma_store_4d(&tmO, stg, half * 64, hkv * G, sq.qoff + t0, b);
          bulk_commit_group();
        }
      }
      }
      if (p.lse != nullptr && valid)
        p.lse[(static_cast<long long>(b) * p.Hq + h) * p.T + sq.qoff + t_row] = (m + log2f(l)) * kLn2;
    }
    if (row == 0) bulk_wait_all();  // this group's output stores have completed
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge of the key-split partials of a prefill: per (row of the token axis, query head),
// lse = log sum_s exp(lse_s) and out = sum_s exp(lse_s - lse) O_s (the online logsumexp of
// "Qwen3 Architecture Layer-by-Layer", Liger fused linear cross-entropy, across runs of
// keys).  One block of four warps per (token, head): every warp reads the row's LSEs (lane s
// holds run s, n_split <= 32) for the max and the weights, and warp g merges runs 8g..8g+7,
// lane i owning output dims 4i..4i+3; the four partial sums meet in shared memory.  All of a
// lane's loads are independent, so a block waits for about one round trip to L2, where the
// attention kernel just left the partials.  A programmatic dependent launch: its blocks may
// be scheduled while that kernel runs and wait (griddep_wait) before their first read.
struct SplitCombineParams {
  const float* part_o;    // [B*T, Hq, n_split, d]
  const float* part_lse;  // [B*T, Hq, n_split]
  uint2* out;             // [B*T, Hq, d] bf16
  float* lse;             // [B, Hq, T] or nullptr
  int B, T, Hq, n_split;
};
constexpr int kCombineWarps = 4;  // runs per warp: 32 / kCombineWarps

__global__ void __launch_bounds__(kCombineWarps * 32) prefill_split_combine_kernel(
    const __grid_constant__ SplitCombineParams p) {
  constexpr int kPer = 32 / kCombineWarps;
  __shared__ float4 part[kCombineWarps][32];
  griddep_wait();
  const long long row = blockIdx.x;  // (b*T + t)*Hq + h
  const int g = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = p.n_split;
  const float mine = lane < n ? p.part_lse[row * n + lane] : -INFINITY;
  const float4* po = reinterpret_cast<const float4*>(p.part_o + row * n * kD) + lane;
  float4 o[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int s = g * kPer + i;
    o[i] = s < n ? po[s * (kD / 4)] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float M = mine;
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
  const float kLog2e = 1.44269504088896341f;
  // a run with no key this row sees has LSE -inf: weight 0, and its O is never used
  const float w = (mine == -INFINITY || M == -INFINITY) ? 0.f : ex2((mine - M) * kLog2e);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    // an unused run's row may hold anything, NaN included: selected away, not multiplied by 0
    const float ws = __shfl_sync(0xffffffffu, w, g * kPer + i);
    const bool use = ws != 0.f;
    acc.x += use ? ws * o[i].x : 0.f;
    acc.y += use ? ws * o[i].y : 0.f;
    acc.z += use ? ws * o[i].z : 0.f;
    acc.w += use ? ws * o[i].w : 0.f;
  }
  part[g][lane] = acc;
  __syncthreads();
  if (g != 0) return;
  const float z = warp_sum(w);
#pragma unroll
  for (int j = 1; j < kCombineWarps; ++j) {
    const float4 a = part[j][lane];
    acc.x += a.x;
    acc.y += a.y;
    acc.z += a.z;
    acc.w += a.w;
  }
  const float inv = z > 0.f ? 1.0f / z : 0.f;
  p.out[row * (kD / 4) + lane] = make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
  if (p.lse != nullptr && lane == 0) {
    const long long bt = row / p.Hq;
    const int h = static_cast<int>(row - bt * p.Hq);
    const long long b = bt / p.T, t = bt - b * p.T;
    p.lse[(b * p.Hq + h) * p.T + t] = M + logf(z);
  }
}

}  // namespace q3
