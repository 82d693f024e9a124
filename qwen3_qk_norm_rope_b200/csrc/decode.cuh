// decode.cuh - one new token per sequence over a bf16 KV cache: split-KV attention with
// the Q prologue fused in, and the logsumexp combine of the splits.
//
// What it computes: the new token of sequence n sits at position L = cache_lens[n]; its
// normalised, rotated query attends to keys 0..L of its KV head, slot L holding the new
// token's key (appended beforehand by qk_norm_rope_kernel in write-at-pos mode)
// ("Assembling a large model from scratch", KVCache.update, Transformer.forward with
// start = cache.length, and the tril(diagonal=S-T) mask with T = 1).
//
// Split kernel: one CTA per (split of `split` keys, KV head, sequence); CTAs past a
// sequence's end exit at once, so the host never needs the lengths.  It is a programmatic
// dependent launch after the append: only the chunk holding slot L waits for the append's
// results (griddepcontrol.wait); the rest of the cache was written by earlier calls.  Warp 4
// streams 64-key chunks of K and V (two 64x64 128B-swizzled TMA boxes each, or per page for
// smaller pages) into a 3-stage ring.  Warps 0-3 each take 16 keys of every chunk: S = q'K^T and O += P V as mma.sync m16n8k16 (rows =
// the G <= 16 query heads of the group), an exp2 online softmax in registers, then the four
// warps merge their (max, sum, O) and write the split's normalised O and its LSE.
// The work per key is 4*G*d flops against 4*d bytes, so this path is bound by HBM
// bandwidth; legacy mma.sync is ample for the arithmetic.
//
// Combine kernel: per (sequence, query head), lse = log sum_s exp(lse_s) and
// out = sum_s exp(lse_s - lse) O_s.
#pragma once
#include "common.cuh"

namespace q3 {

struct DecodeParams {
  const uint32_t* q;  // [N, Hq, d] bf16 pairs (raw)
  const float* q_norm_w;
  const int* cache_lens;  // [N]
  float* part_o;          // [N, Hq, n_split_max, d]
  float* part_lse;        // [N, Hq, n_split_max]
  int N, Hq, Hkv, log2G, Lmax, split, n_split_max;
  int window;        // sliding window W: the query sees keys L-W < j <= L; 0 = all
  // Paged cache (block_table != nullptr): the tensor maps cover the page pools as rows of d,
  // [num_pages * Hkv * page, d], with boxes of min(page, 64) rows; key j of sequence n is in
  // page block_table[n, j / page] at offset j % page.  page = 1 << log2_page, >= 16.
  const int* block_table;
  int max_blocks, log2_page, num_pages;
  float eps, scale_log2;
  float rope_scale;  // attention_scaling on cos and sin
  WaitCfg wait;
  RopeTable rope;
};

constexpr int kDcStages = 3;
constexpr uint32_t kDcBox = 8192;             // 64 keys x 64 dims bf16
constexpr uint32_t kDcChunk = 2 * kDcBox;     // 64 keys x 128 dims
constexpr uint32_t kDcStage = 2 * kDcChunk;   // K chunk + V chunk
constexpr uint32_t kDcQ = kDcStages * kDcStage;  // q' [16][128] bf16 = 4096 B
constexpr uint32_t kDcBar = kDcQ + 4096;
constexpr uint32_t kDcBFull = 0, kDcBEmpty = 32, kDcBAbort = 64;
constexpr uint32_t kDcTab = kDcBar + 128;  // a paged split's page indices: <= 1024 / 16 of them
constexpr uint32_t kDecodeSmemBytes = kDcTab + 256 + 1024;
constexpr int kDecodeThreads = 160;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2d(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// A chunk of K (or V) in shared memory: key r's two 64-dim halves are the 128-byte lines
// 2r and 2r+1, as one TMA box {64 dims, 2 halves, keys} writes them, 128B-swizzled (the
// 16-byte piece c of line l sits at piece c ^ (l mod 8)).
__device__ __forceinline__ uint32_t dc_line_offset(uint32_t row, uint32_t half, uint32_t piece) {
  const uint32_t l = 2u * row + half;
  return l * 128u + ((piece ^ (l & 7u)) << 4);
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(m), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// kLines: the chunk layout of pages under 64 keys, where one TMA box per page brings both
// 64-dim halves of its keys (key r's halves are the 128-byte lines 2r and 2r+1), half as
// many boxes as one per half.  Otherwise each half is its own 64-key plane, one box each:
// its ldmatrix reads are free of bank conflicts, which the interleaved lines are not.
template <bool kLines>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ DecodeParams p) {
  const int s_idx = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int L = p.cache_lens[n];
  if (L < 0 || L >= p.Lmax) {
    if (s_idx == 0 && h == 0 && threadIdx.x == 0) record_error(QWEN3_ERR_INVALID_ARG, kSiteDecodeLen);
    return;
  }
  const int tok0 = s_idx * p.split;
  const int ntok = min(p.split, L + 1 - tok0);  // keys of this split (slot L = new token)
  if (ntok <= 0) return;
  const int wlo = p.window > 0 ? max(0, L - p.window + 1) : 0;  // first visible key
  if (tok0 + ntok <= wlo) return;  // the whole split lies before the window
  const int nchunk = (ntok + 63) >> 6;
  const int cbeg = max(0, wlo - tok0) >> 6;  // chunks wholly before the window are skipped
  const int G = 1 << p.log2G;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sb - raw);
  const uint32_t sQ = sb + kDcQ, bar = sb + kDcBar;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kDcBar + kDcBAbort);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDcStages; ++s) {
      mbar_init(bar + kDcBFull + 8 * s, 1);
      mbar_init(bar + kDcBEmpty + 8 * s, 128);
    }
    *abort_flag = 0;
    mbar_init_fence();
    fence_proxy_async_smem();
  }
  __syncthreads();

  const long long row0 = (static_cast<long long>(n) * p.Hkv + h) * p.Lmax + tok0;
  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    // A paged split first stages its page indices in shared memory, one coalesced load by
    // the warp, so the chunk loop never waits on the block table.
    int* s_tab = reinterpret_cast<int*>(sgen + kDcTab);
    const int blk0 = tok0 >> p.log2_page;
    if (p.block_table != nullptr) {
      const int nblk = min(((tok0 + ntok - 1) >> p.log2_page) - blk0 + 1, 64);
      for (int i = lane; i < nblk; i += 32)
        s_tab[i] = blk0 + i < p.max_blocks ? p.block_table[static_cast<long long>(n) * p.max_blocks + blk0 + i] : -1;
      __syncwarp();
    }
    if (lane == 0) {
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      int last[kDcStages] = {-1, -1, -1};
      for (int c = cbeg; c < nchunk; ++c) {
        const int u = c - cbeg;  // ring use
        const int st = u % kDcStages;
        const uint32_t ph = (u / kDcStages) & 1;
        if (u >= kDcStages && !mbar_wait(bar + kDcBEmpty + 8 * st, ph ^ 1, p.wait, abort_flag, kSiteDecodeEmpty))
          break;
        // slot L, the new token's key and value, comes from the append kernel before this one
        if (tok0 + c * 64 + 63 >= L) griddep_wait();
        const uint32_t dst = sb + st * kDcStage;
        const uint32_t fb = bar + kDcBFull + 8 * st;
        if (p.block_table == nullptr) {
          const int r = static_cast<int>(row0 + c * 64);
          mbar_arrive_expect_tx(fb, kDcStage);
          tma_load_2d(dst, &tmK, fb, 0, r);
          tma_load_2d(dst + kDcBox, &tmK, fb, 64, r);
          tma_load_2d(dst + kDcChunk, &tmV, fb, 0, r);
          tma_load_2d(dst + kDcChunk + kDcBox, &tmV, fb, 64, r);
        } else {
          // Boxes of br keys, each inside one page; boxes wholly past key L are not loaded
          // (the consumers mask those keys and zero their V rows).
          const int br = min(1 << p.log2_page, 64);
          int rows[4], nb = 0;
          for (int r0 = 0; r0 < 64 && nb < 4; r0 += br) {
            const int key = tok0 + c * 64 + r0;
            if (key > L) break;
            const int page = s_tab[(key >> p.log2_page) - blk0];
            if (page < 0 || page >= p.num_pages) {
              record_error(QWEN3_ERR_INVALID_ARG, kSitePagedTable);
              rows[nb++] = -1;
              continue;
            }
            rows[nb++] = ((page * p.Hkv + h) << p.log2_page) + (key & ((1 << p.log2_page) - 1));
          }
          uint32_t bytes = 0;
          for (int i = 0; i < nb; ++i)
            if (rows[i] >= 0) bytes += 4u * br * 128u;
          mbar_arrive_expect_tx(fb, bytes);
          for (int i = 0; i < nb; ++i) {
            if (rows[i] < 0) continue;
            if constexpr (kLines) {
              const uint32_t off = static_cast<uint32_t>(i * br) * 256u;  // br keys of both halves
              tma_load_3d(dst + off, &tmK, fb, 0, 0, rows[i]);
              tma_load_3d(dst + kDcChunk + off, &tmV, fb, 0, 0, rows[i]);
            } else {
              const uint32_t off = static_cast<uint32_t>(i * br) * 128u;
              tma_load_2d(dst + off, &tmK, fb, 0, rows[i]);
              tma_load_2d(dst + kDcBox + off, &tmK, fb, 64, rows[i]);
              tma_load_2d(dst + kDcChunk + off, &tmV, fb, 0, rows[i]);
              tma_load_2d(dst + kDcChunk + kDcBox + off, &tmV, fb, 64, rows[i]);
            }
          }
        }
        last[st] = u;
      }
      for (int s = 0; s < kDcStages; ++s)
        if (last[s] >= 0)
          mbar_wait(bar + kDcBFull + 8 * s, (last[s] / kDcStages) & 1, p.wait, nullptr, kSiteDecodeFull);
    }
    return;
  }

  // -------------------------------------------------------------------- q prologue
  {
    const float2 ga = reinterpret_cast<const float2*>(p.q_norm_w)[lane];
    const float2 gb = reinterpret_cast<const float2*>(p.q_norm_w)[32 + lane];
    float s0, c0, s1, c1;
    rope_sincos(L, p.rope.hi[2 * lane], p.rope.lo[2 * lane], s0, c0);
    rope_sincos(L, p.rope.hi[2 * lane + 1], p.rope.lo[2 * lane + 1], s1, c1);
    s0 *= p.rope_scale;
    c0 *= p.rope_scale;
    s1 *= p.rope_scale;
    c1 *= p.rope_scale;
    for (int g = warp; g < 16; g += 4) {
      uint32_t wa = 0u, wb = 0u;
      if (g < G) {
        const uint32_t* qs = p.q + (static_cast<long long>(n) * p.Hq + h * G + g) * (kD / 2);
        const uint32_t ua = qs[lane], ub = qs[32 + lane];
        float2 ya, yb;
        norm_rope_pairs(make_float2(bf16lo(ua), bf16hi(ua)), make_float2(bf16lo(ub), bf16hi(ub)), ga, gb, s0, c0,
                        s1, c1, p.eps, ya, yb);
        wa = pack_bf16x2(ya.x, ya.y);
        wb = pack_bf16x2(yb.x, yb.y);
      }
      st_shared_u32(sQ + g * 256 + lane * 4, wa);
      st_shared_u32(sQ + g * 256 + 128 + lane * 4, wb);
    }
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");

  // A fragments of q' for the 8 k-steps (rows = heads; rows >= G are zero).
  uint32_t qa[8][4];
  {
    const int r0 = lane >> 2, cq = (lane & 3) * 4;  // byte offset of the pair within 16 dims
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t base = sQ + kk * 32 + cq;
      asm volatile("ld.shared.b32 %0, [%1];" : "=r"(qa[kk][0]) : "r"(base + r0 * 256));
      asm volatile("ld.shared.b32 %0, [%1];" : "=r"(qa[kk][1]) : "r"(base + (r0 + 8) * 256));
      asm volatile("ld.shared.b32 %0, [%1];" : "=r"(qa[kk][2]) : "r"(base + r0 * 256 + 16));
      asm volatile("ld.shared.b32 %0, [%1];" : "=r"(qa[kk][3]) : "r"(base + (r0 + 8) * 256 + 16));
    }
  }

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows lane/4 and lane/4+8
  const float sl2 = p.scale_log2;
  const int tw = warp * 16;  // this warp's keys inside every chunk
  bool ok = true;
  for (int c = cbeg; c < nchunk; ++c) {
    const int st = (c - cbeg) % kDcStages;
    ok = mbar_wait(bar + kDcBFull + 8 * st, ((c - cbeg) / kDcStages) & 1, p.wait, abort_flag, kSiteDecodeFull);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const uint32_t sKc = sb + st * kDcStage, sVc = sKc + kDcChunk;
    const int valid = ntok - c * 64 - tw;          // keys of this warp's 16 that exist
    const int below = wlo - (tok0 + c * 64 + tw);  // keys of this warp's 16 before the window
    if (valid > 0 && below < 16) {
      if (valid < 16) {
        // Slots past the sequence hold stale cache contents: zero their V rows so that
        // P = 0 never meets a non-finite value in P.V.
        for (int t = valid + (lane >> 3); t < 16; t += 4) {
          const uint32_t rowoff = static_cast<uint32_t>(tw + t) * (kLines ? 256u : 128u) + (lane & 7) * 16u;
          st_shared_v4(sVc + rowoff, 0u, 0u, 0u, 0u);
          st_shared_v4(sVc + (kLines ? 128u : kDcBox) + rowoff, 0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }
      // ---- S = q' K^T for 16 keys: two n8 blocks
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sbk[4] = {0.f, 0.f, 0.f, 0.f};
      const int mi = lane >> 3, mr = lane & 7;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t tok = tw + ((mi >> 1) << 3) + mr;
        const uint32_t chunk = ((kk & 3) << 1) + (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sKc + (kLines ? dc_line_offset(tok, kk >> 2, chunk) : (kk >> 2) * kDcBox + sw128_offset(tok, chunk)),
                b0, b1, b2, b3);
        mma_bf16_16816(sa, qa[kk], b0, b1);
        mma_bf16_16816(sbk, qa[kk], b2, b3);
      }
      // ---- mask, online softmax (rows = heads)
      const int kc = 2 * (lane & 3);
      float x[8] = {sa[0], sa[1], sa[2], sa[3], sbk[0], sbk[1], sbk[2], sbk[3]};
      // x[0..1]: row r0, keys kc,kc+1; x[2..3]: row r0+8 same keys; x[4..7]: keys 8+kc.. likewise
      if (valid < 16) {
        if (kc >= valid) x[0] = x[2] = -INFINITY;
        if (kc + 1 >= valid) x[1] = x[3] = -INFINITY;
        if (8 + kc >= valid) x[4] = x[6] = -INFINITY;
        if (9 + kc >= valid) x[5] = x[7] = -INFINITY;
      }
      if (below > 0) {  // keys before the window (at least one of the 16 is inside it)
        if (kc < below) x[0] = x[2] = -INFINITY;
        if (kc + 1 < below) x[1] = x[3] = -INFINITY;
        if (8 + kc < below) x[4] = x[6] = -INFINITY;
        if (9 + kc < below) x[5] = x[7] = -INFINITY;
      }
      float mx0 = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[4], x[5]));
      float mx1 = fmaxf(fmaxf(x[2], x[3]), fmaxf(x[6], x[7]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0 * sl2), mn1 = fmaxf(m1, mx1 * sl2);
      const float al0 = ex2d(m0 - mn0), al1 = ex2d(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      float pr[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) pr[i] = ex2d(fmaf(x[i], sl2, -((i & 2) ? mn1 : mn0)));
      uint32_t pa[4];
      pa[0] = pack_bf16x2(pr[0], pr[1]);
      pa[1] = pack_bf16x2(pr[2], pr[3]);
      pa[2] = pack_bf16x2(pr[4], pr[5]);
      pa[3] = pack_bf16x2(pr[6], pr[7]);
      l0 = l0 * al0 + ((pr[0] + pr[1]) + (pr[4] + pr[5]));
      l1 = l1 * al1 + ((pr[2] + pr[3]) + (pr[6] + pr[7]));
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        o[i][0] *= al0;
        o[i][1] *= al0;
        o[i][2] *= al1;
        o[i][3] *= al1;
      }
      // ---- O += P V: 16 n8 blocks of dims, V fragments by transposing ldmatrix
#pragma unroll
      for (int nb2 = 0; nb2 < 8; ++nb2) {
        const uint32_t tok = tw + ((mi & 1) << 3) + mr;
        const uint32_t chunk = ((nb2 & 3) << 1) + (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(
            sVc + (kLines ? dc_line_offset(tok, nb2 >> 2, chunk) : (nb2 >> 2) * kDcBox + sw128_offset(tok, chunk)), b0,
            b1, b2, b3);
        mma_bf16_16816(o[2 * nb2], pa, b0, b1);
        mma_bf16_16816(o[2 * nb2 + 1], pa, b2, b3);
      }
      if (valid < 16) fence_proxy_async_smem();  // generic zero-writes before the next TMA refill
    }
    mbar_arrive(bar + kDcBEmpty + 8 * st);
  }

  // -------------------------------------------------------------------- merge the 4 warps
  asm volatile("bar.sync 1, 128;" ::: "memory");  // every warp is done with the stage buffers
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  float* so = reinterpret_cast<float*>(sgen);                       // [4][16][128] fp32 (32 KB)
  float* sml = reinterpret_cast<float*>(sgen + 4 * 16 * 128 * 4);  // [4][16][2]
  const int r0 = lane >> 2;
  if ((lane & 3) == 0) {
    sml[(warp * 16 + r0) * 2 + 0] = m0;
    sml[(warp * 16 + r0) * 2 + 1] = l0;
    sml[(warp * 16 + r0 + 8) * 2 + 0] = m1;
    sml[(warp * 16 + r0 + 8) * 2 + 1] = l1;
  }
#pragma unroll
  for (int nb = 0; nb < 16; ++nb) {
    const int col = nb * 8 + 2 * (lane & 3);
    *reinterpret_cast<float2*>(&so[(warp * 16 + r0) * 128 + col]) = make_float2(o[nb][0], o[nb][1]);
    *reinterpret_cast<float2*>(&so[(warp * 16 + r0 + 8) * 128 + col]) = make_float2(o[nb][2], o[nb][3]);
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (!ok) return;
  const int dcol = threadIdx.x;  // 0..127: one output dim per thread
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sml[(w * 16 + g) * 2]);
    float Lsum = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float mw = sml[(w * 16 + g) * 2];
      const float f = (mw == -INFINITY) ? 0.f : ex2d(mw - M);
      Lsum += f * sml[(w * 16 + g) * 2 + 1];
      acc += f * so[(w * 16 + g) * 128 + dcol];
    }
    const long long hq = static_cast<long long>(n) * p.Hq + h * G + g;
    p.part_o[(hq * p.n_split_max + s_idx) * kD + dcol] = acc / Lsum;
    if (dcol == 0) p.part_lse[hq * p.n_split_max + s_idx] = (M + log2f(Lsum)) * 0.693147180559945309f;
  }
  // The combine kernel may be scheduled once every CTA has got here or exited: it waits for
  // this grid's partials (griddepcontrol.wait) before reading them.
  griddep_launch_dependents();
}

struct CombineParams {
  const float* part_o;
  const float* part_lse;
  const int* cache_lens;
  uint4* out;  // [N, Hq, d] bf16
  float* lse;  // [N, Hq] or nullptr
  int Hq, Lmax, split, n_split_max;
  int window;  // as in DecodeParams: splits wholly before the window wrote nothing
};

// One CTA of 128 threads per (sequence, query head); thread i owns output dim i.  A
// programmatic dependent launch after the split kernel, whose partials it waits for.
__global__ void __launch_bounds__(128) decode_combine_kernel(const __grid_constant__ CombineParams p) {
  griddep_wait();
  const int hq = blockIdx.x;  // n * Hq + head
  const int n = hq / p.Hq;
  const int L = p.cache_lens[n];
  if (L < 0 || L >= p.Lmax) return;
  const int ns = L / p.split + 1;  // splits covering keys 0..L
  const int s0 = p.window > 0 ? max(0, L - p.window + 1) / p.split : 0;  // the first one in the window
  const float* lse_s = p.part_lse + static_cast<long long>(hq) * p.n_split_max;
  float M = -INFINITY;
#pragma unroll 8
  for (int s = s0; s < ns; ++s) M = fmaxf(M, lse_s[s]);
  const float kLog2e = 1.44269504088896341f;
  float z = 0.f, acc = 0.f;
  const float* po = p.part_o + static_cast<long long>(hq) * p.n_split_max * kD + threadIdx.x;
#pragma unroll 8
  for (int s = s0; s < ns; ++s) {
    const float w = ex2d((lse_s[s] - M) * kLog2e);
    z += w;
    acc += w * po[s * kD];
  }
  __shared__ float sv[128];
  sv[threadIdx.x] = acc / z;
  __syncthreads();
  if (threadIdx.x < 16) {
    uint4 w;
    const float* v = sv + threadIdx.x * 8;
    w.x = pack_bf16x2(v[0], v[1]);
    w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]);
    w.w = pack_bf16x2(v[6], v[7]);
    p.out[static_cast<long long>(hq) * (kD / 8) + threadIdx.x] = w;
  }
  if (p.lse != nullptr && threadIdx.x == 0) p.lse[hq] = M + logf(z);
}

}  // namespace q3
