// qkv_proj.cuh - the merged q/k/v projection with QK-Norm and RoPE in the GEMM epilogue.
//
// What it computes: y = x w_qkv^T for token hidden states x [M, hidden] and the stacked
// projection weights w_qkv [(Hq + 2 Hkv) d, hidden] (q, k and v in one GEMM: "LLM Internals -
// Assembling a large model from scratch", the comparison with inference engines: qkv_proj);
// the q and k heads of y then get QK-Norm and rotate-half RoPE at their token's position
// ("Hand-Writing a Vision-Language Model, Part 1", order of operations; "Qwen3 Architecture
// Layer-by-Layer", Qwen3RMSNorm and apply_rotary_pos_emb), v is stored as projected.
//
// A head is 128 columns of y, so the accumulator of an N tile holds whole head vectors and
// the norm needs no reduction across CTAs: the epilogue thread that owns a token row has its
// head's 128 values in registers.  Normalising the fp32 accumulator directly also skips the
// bf16 rounding the pages' path takes between the projection and q_norm.
//
// Tiles: 128 tokens x 256 columns (two heads), K in chunks of 64 (one 128B-swizzled row per
// token).  Persistent CTAs take contiguous runs of tiles in token-tile-major order, so a run
// mostly stays on one token tile.  Ten warps:
//   warp 0     TMA producer: x and w_qkv chunks into a 4-stage ring; owns TMEM.
//   warp 1     MMA issuer (one thread): tcgen05.mma M=128 N=256 K=16, 4 per chunk, into one
//              of two TMEM accumulators (256 columns each), so the epilogue of a tile
//              overlaps the next tile's MMAs.
//   warps 2-9  epilogue, two warps per TMEM lane quadrant (warp % 4), one per head of the
//              tile, one thread per token row: tcgen05.ld of the head's 128 fp32, then for
//              q and k heads the sum of squares, 1/rms, gain and the rotation; bf16 rows to
//              q_out / k_out / v_out.  The rotation's (cos, sin) come from the token tile's
//              RoPE table ([64][128] float2, 64 KB, built by qkv_rope_table_kernel): for one
//              frequency the 32 rows of a warp are one coalesced 256-byte read, and the
//              table stays in L2 for all the tile's column tiles.  Left out of shared
//              memory, it leaves room for a fourth stage.  The GEMM is a programmatic
//              dependent launch after the table kernel: its loads and MMAs start at once,
//              and only the epilogue warps wait for the table (griddep_wait).
//
// qkv_proj_pair_kernel is the same GEMM on SM pairs (tcgen05 cta_group::2): a cluster of two
// CTAs computes a 256-token x 256-column tile with M=256 MMAs, each CTA loading its own 128
// token rows and half of the tile's weight rows, so an SM streams 32 KB per K chunk instead
// of 48 KB for the same share of the MMAs.  The host takes it when each pair's run of tiles
// is long enough to repay its deeper ring and cross-CTA handoffs.
#pragma once
#include "common.cuh"

namespace q3 {

struct QkvParams {
  const float* q_norm_w;  // [d]
  const float* k_norm_w;  // [d]
  const float2* rope;     // [ceil(M/128)][64][128]: (cos, sin) x attention_scaling
  uint4* q_out;           // [M, Hq, d] bf16
  uint4* k_out;           // [M, Hkv, d]
  uint4* v_out;           // [M, Hkv, d]
  int M, hidden, Hq, Hkv, n_heads, n_mt, n_nt, n_tiles, n_k;
  int n_mp, n_tiles2;  // the SM-pair kernel: token-tile pairs, and pair tiles (n_mp * n_nt)
  float eps;
  WaitCfg wait;
};

// warp 0: TMA producer; warp 1: MMA issuer; warps 2-9: epilogue, two warps per TMEM lane
// quadrant, one for each of a tile's two heads
constexpr int kQkvThreads = 320;
constexpr int kQkvStages = 4;
constexpr uint32_t kQkA = 16384;                  // 128 tokens x 64 bf16
constexpr uint32_t kQkB = 32768;                  // 256 columns x 64 bf16
constexpr uint32_t kQkStage = kQkA + kQkB;
constexpr uint32_t kQkGain = kQkvStages * kQkStage;  // q gain, k gain: 2 x 512 B
constexpr uint32_t kQkBar = kQkGain + 1024;
// barrier block: full[stages], empty[stages], acc_full[2], acc_empty[2], done, tmem slot, abort flag
constexpr uint32_t kQbFull = 0, kQbEmpty = kQbFull + 8 * kQkvStages, kQbAccFull = kQbEmpty + 8 * kQkvStages,
                   kQbAccEmpty = kQbAccFull + 16, kQbDone = kQbAccEmpty + 16, kQbTmem = kQbDone + 8,
                   kQbAbort = kQbTmem + 4;
static_assert(kQbAbort + 4 <= 128, "the qkv barrier block is 128 bytes");
constexpr uint32_t kQkvSmemBytes = kQkBar + 128 + 1024;

// The RoPE table of every token tile: entry [mt][i][r] = (cos, sin)(pos[mt*128 + r] * inv_i)
// times attention_scaling; rows past M use position 0.
struct QkvRopeParams {
  const int* pos;
  float2* rope;
  int M, n_mt;
  float scale;
  RopeTable tab;
};

__global__ void __launch_bounds__(256) qkv_rope_table_kernel(const __grid_constant__ QkvRopeParams p) {
  // The projection launched next may start now: only its epilogue reads this table, and it
  // waits for this grid first (griddep_wait).
  griddep_launch_dependents();
  const long long total = static_cast<long long>(p.n_mt) * 64 * 128;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(e & 127);
    const int i = static_cast<int>((e >> 7) & 63);
    const long long m = (e >> 13) * 128 + r;
    const int ps = m < p.M ? p.pos[m] : 0;
    float s, c;
    rope_sincos(ps, p.tab.hi[i], p.tab.lo[i], s, c);
    p.rope[e] = make_float2(c * p.scale, s * p.scale);
  }
}

__device__ __forceinline__ void qkv_tile_coords(const QkvParams& p, int tile, int& mt, int& nt) {
  mt = tile / p.n_nt;
  nt = tile - mt * p.n_nt;
}

__global__ void __launch_bounds__(kQkvThreads, 1)
    qkv_proj_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const __grid_constant__ QkvParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sb - raw);
  const uint32_t bar = sb + kQkBar;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kQkBar + kQbAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + kQkBar + kQbTmem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // this CTA's run of tiles
  const int per = (p.n_tiles + gridDim.x - 1) / gridDim.x;
  const int t_begin = blockIdx.x * per;
  const int t_end = min(p.n_tiles, t_begin + per);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQkvStages; ++s) {
      mbar_init(bar + kQbFull + 8 * s, 1);
      mbar_init(bar + kQbEmpty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar + kQbAccFull + 8 * b, 1);
      mbar_init(bar + kQbAccEmpty + 8 * b, 256);
    }
    mbar_init(bar + kQbDone, 1);
    *abort_flag = 0;
    mbar_init_fence();
    fence_proxy_async_smem();
  }
  if (threadIdx.x < 128) {  // gains into shared memory
    float* sg = reinterpret_cast<float*>(sgen + kQkGain);
    sg[threadIdx.x] = p.q_norm_w[threadIdx.x];
    sg[128 + threadIdx.x] = p.k_norm_w[threadIdx.x];
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
      tma_prefetch_map(&tmX);
      tma_prefetch_map(&tmW);
      int last[kQkvStages];
      for (int s = 0; s < kQkvStages; ++s) last[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      for (int tile = t_begin; tile < t_end && ok; ++tile) {
        int mt, nt;
        qkv_tile_coords(p, tile, mt, nt);
        for (int kc = 0; kc < p.n_k; ++kc, ++it) {
          const int st = static_cast<int>(it % kQkvStages);
          const uint32_t ph = (it / kQkvStages) & 1;
          if (it >= kQkvStages &&
              !mbar_wait(bar + kQbEmpty + 8 * st, ph ^ 1, p.wait, abort_flag, kSiteQkvEmpty)) {
            ok = false;
            break;
          }
          const uint32_t dst = sb + st * kQkStage;
          mbar_arrive_expect_tx(bar + kQbFull + 8 * st, kQkStage);
          tma_load_2d(dst, &tmX, bar + kQbFull + 8 * st, kc * 64, mt * 128);
          tma_load_2d(dst + kQkA, &tmW, bar + kQbFull + 8 * st, kc * 64, nt * 256);
          last[st] = static_cast<int>(it);
        }
      }
      for (int s = 0; s < kQkvStages; ++s)
        if (last[s] >= 0)
          mbar_wait(bar + kQbFull + 8 * s, (last[s] / kQkvStages) & 1, p.wait, nullptr, kSiteQkvDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16(128, 256, false);  // A = x rows, B = w rows, both K-major
      uint32_t it = 0;
      bool ok = true;
      int n = 0;
      for (int tile = t_begin; tile < t_end && ok; ++tile, ++n) {
        const int buf = n & 1;
        if (n >= 2 && !mbar_wait(bar + kQbAccEmpty + 8 * buf, ((n >> 1) - 1) & 1, p.wait, abort_flag, kSiteQkvAcc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * 256);
        for (int kc = 0; kc < p.n_k; ++kc, ++it) {
          const int st = static_cast<int>(it % kQkvStages);
          if (!mbar_wait(bar + kQbFull + 8 * st, (it / kQkvStages) & 1, p.wait, abort_flag, kSiteQkvFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sb + st * kQkStage, sbw = sa + kQkA;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_ss(acc, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sbw + kk * 32, 16, 1024), kId,
                      (kc > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar + kQbEmpty + 8 * st);
        }
        if (!ok) break;
        tc_commit(bar + kQbAccFull + 8 * buf);
      }
      tc_commit(bar + kQbDone);
      mbar_wait(bar + kQbDone, 0, p.wait, nullptr, kSiteQkvDrain);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    griddep_wait();  // the RoPE table, written by the kernel launched before this one
    const int wq = warp & 3;
    const int hh = (warp - 2) >> 2;  // which of the tile's two heads this warp takes
    const int row = wq * 32 + lane;  // token row of the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float* sg = reinterpret_cast<const float*>(sgen + kQkGain);
    bool ok = true;
    int n = 0;
    for (int tile = t_begin; tile < t_end && ok; ++tile, ++n) {
      int mt, nt;
      qkv_tile_coords(p, tile, mt, nt);
      const int buf = n & 1;
      ok = mbar_wait(bar + kQbAccFull + 8 * buf, (n >> 1) & 1, p.wait, abort_flag, kSiteQkvAcc);
      if (!ok) break;
      tc_fence_after();
      const long long m = static_cast<long long>(mt) * 128 + row;
      {
        const int h = nt * 2 + hh;  // head index in [q heads | k heads | v heads]
        uint32_t y[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_off + static_cast<uint32_t>(buf * 256 + hh * 128 + c * 32), r);
#pragma unroll
          for (int i = 0; i < 32; ++i) y[c * 32 + i] = r[i];
        }
        // this head is in registers: once both heads' warps are here the accumulator is free
        tc_fence_before();
        mbar_arrive(bar + kQbAccEmpty + 8 * buf);
        if (h >= p.n_heads || m >= p.M) continue;
        uint4* dst;
        if (h < p.Hq + p.Hkv) {
          // QK-Norm: 1/rms of the fp32 row, then gain and rotate-half RoPE, pairs (i, i+64)
          const bool is_q = h < p.Hq;
          const float* g = sg + (is_q ? 0 : 128);
          float ss = 0.f;
#pragma unroll
          for (int i = 0; i < 128; ++i) ss = fmaf(__uint_as_float(y[i]), __uint_as_float(y[i]), ss);
          const float rn = rsqrtf(fmaf(ss, 1.0f / kD, p.eps));
          const float2* rope = p.rope + static_cast<size_t>(mt) * 64 * 128;  // this token tile's table
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const float2 cs = rope[i * 128 + row];
            const float a = g[i] * (__uint_as_float(y[i]) * rn);
            const float b = g[64 + i] * (__uint_as_float(y[64 + i]) * rn);
            y[i] = __float_as_uint(a * cs.x - b * cs.y);
            y[64 + i] = __float_as_uint(b * cs.x + a * cs.y);
          }
          dst = is_q ? p.q_out + (m * p.Hq + h) * (kD / 8) : p.k_out + (m * p.Hkv + (h - p.Hq)) * (kD / 8);
        } else {
          dst = p.v_out + (m * p.Hkv + (h - p.Hq - p.Hkv)) * (kD / 8);
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(y[8 * c + 0]), __uint_as_float(y[8 * c + 1]));
          w.y = pack_bf16x2(__uint_as_float(y[8 * c + 2]), __uint_as_float(y[8 * c + 3]));
          w.z = pack_bf16x2(__uint_as_float(y[8 * c + 4]), __uint_as_float(y[8 * c + 5]));
          w.w = pack_bf16x2(__uint_as_float(y[8 * c + 6]), __uint_as_float(y[8 * c + 7]));
          dst[c] = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ SM-pair variant
// Two CTAs of a cluster (one per SM of a pair) share each MMA: tcgen05.mma.cta_group::2
// with M = 256, the rows of CTA r being its own token tile 2*mp + r, and N = 256 split in
// halves, CTA r holding weight rows nt*256 + 128r .. +127.  Each SM so loads 32 KB per
// K-chunk instead of 48 KB for the same 128 x 256 x 64 share of the work.  CTA 0 (the
// leader) issues the MMAs; both CTAs' copies complete on the leader's stage barriers, the
// leader's commits arrive on the barriers of both CTAs, and each CTA's epilogue reads its
// own 128 rows of the accumulator from its own TMEM.
constexpr int kQk2Stages = 6;
constexpr uint32_t kQk2B = 16384;                   // 128 weight rows x 64 bf16 (this CTA's half)
constexpr uint32_t kQk2Stage = kQkA + kQk2B;
constexpr uint32_t kQk2Gain = kQk2Stages * kQk2Stage;
constexpr uint32_t kQk2Bar = kQk2Gain + 1024;
constexpr uint32_t kQ2Full = 0, kQ2Empty = kQ2Full + 8 * kQk2Stages, kQ2AccFull = kQ2Empty + 8 * kQk2Stages,
                   kQ2AccEmpty = kQ2AccFull + 16, kQ2Done = kQ2AccEmpty + 16, kQ2Tmem = kQ2Done + 8,
                   kQ2Abort = kQ2Tmem + 4;
static_assert(kQ2Abort + 4 <= 256, "the pair kernel's barrier block is 256 bytes");
constexpr uint32_t kQkv2SmemBytes = kQk2Bar + 256 + 1024;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Every thread of both CTAs.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The shared::cluster address of this CTA's shared variable at `addr` in the CTA of `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_init_fence_cluster() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// A TMA load into this CTA's shared memory whose bytes complete on `bar`, a barrier of
// either CTA of the pair (its shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(m), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tc_mma_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at `bar` in both CTAs of the pair when every MMA this thread
// has issued completes.
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(static_cast<unsigned short>(3))
      : "memory");
}
// The same, on this CTA's barrier only.
__device__ __forceinline__ void tc_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// Arrive on a barrier of either CTA of the pair (its shared::cluster address).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kQkvThreads, 1)
    qkv_proj_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                         const __grid_constant__ QkvParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sb - raw);
  const uint32_t bar = sb + kQk2Bar;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kQk2Bar + kQ2Abort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + kQk2Bar + kQ2Tmem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  // this pair's run of pair tiles (each: token tiles 2*mp and 2*mp + 1, column tile nt)
  const int n_pairs = static_cast<int>(gridDim.x >> 1), pid = static_cast<int>(blockIdx.x >> 1);
  const int per = (p.n_tiles2 + n_pairs - 1) / n_pairs;
  const int t_begin = pid * per;
  const int t_end = min(p.n_tiles2, t_begin + per);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQk2Stages; ++s) {
      mbar_init(bar + kQ2Full + 8 * s, 1);   // the leader's: its arrival + both CTAs' bytes
      mbar_init(bar + kQ2Empty + 8 * s, 1);  // the leader's commit, in each CTA
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar + kQ2AccFull + 8 * b, 1);    // the leader's commit, in each CTA
      mbar_init(bar + kQ2AccEmpty + 8 * b, 16);  // the leader's: one arrival per epilogue warp of both CTAs
    }
    mbar_init(bar + kQ2Done, 1);
    *abort_flag = 0;
    mbar_init_fence_cluster();
    fence_proxy_async_smem();
  }
  if (threadIdx.x < 128) {  // gains into shared memory
    float* sg = reinterpret_cast<float*>(sgen + kQk2Gain);
    sg[threadIdx.x] = p.q_norm_w[threadIdx.x];
    sg[128 + threadIdx.x] = p.k_norm_w[threadIdx.x];
  }
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any copy or commit reaches them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producers
    // Both CTAs load their own token rows and their half of the weight rows; the bytes
    // complete on the leader's stage barrier, whose one arrival (with the expected bytes of
    // both CTAs) is the leader's.
    if (lane == 0) {
      tma_prefetch_map(&tmX);
      tma_prefetch_map(&tmW);
      int last[kQk2Stages];
      for (int s = 0; s < kQk2Stages; ++s) last[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      for (int tile = t_begin; tile < t_end && ok; ++tile) {
        const int mp = tile / p.n_nt, nt = tile - (tile / p.n_nt) * p.n_nt;
        const int mt = 2 * mp + static_cast<int>(rank);
        for (int kc = 0; kc < p.n_k; ++kc, ++it) {
          const int st = static_cast<int>(it % kQk2Stages);
          const uint32_t ph = (it / kQk2Stages) & 1;
          if (it >= kQk2Stages &&
              !mbar_wait(bar + kQ2Empty + 8 * st, ph ^ 1, p.wait, abort_flag, kSiteQkvEmpty)) {
            ok = false;
            break;
          }
          const uint32_t dst = sb + st * kQk2Stage;
          const uint32_t full = map_to_rank(bar + kQ2Full + 8 * st, 0);
          if (leader) mbar_arrive_expect_tx(bar + kQ2Full + 8 * st, 2 * kQk2Stage);
          tma_load_2d_pair(dst, &tmX, full, kc * 64, mt * 128);
          tma_load_2d_pair(dst + kQkA, &tmW, full, kc * 64, nt * 256 + static_cast<int>(rank) * 128);
          last[st] = static_cast<int>(it);
        }
      }
      // The leader's barriers count both CTAs' copies: once they complete, nothing either
      // CTA issued is still in flight.  After an abort the odd CTA may have issued a few
      // copies beyond the leader's last phase; it gives them a bounded pause to land.
      if (leader) {
        for (int s = 0; s < kQk2Stages; ++s)
          if (last[s] >= 0)
            mbar_wait(bar + kQ2Full + 8 * s, (last[s] / kQk2Stages) & 1, p.wait, nullptr, kSiteQkvDrain);
      } else if (!ok) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 50000u) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && leader) {
      constexpr uint32_t kId = idesc_bf16(256, 256, false);  // M = 2 x 128 token rows, N = 256 columns
      uint32_t it = 0;
      bool ok = true;
      int n = 0;
      for (int tile = t_begin; tile < t_end && ok; ++tile, ++n) {
        const int buf = n & 1;
        if (n >= 2 && !mbar_wait(bar + kQ2AccEmpty + 8 * buf, ((n >> 1) - 1) & 1, p.wait, abort_flag, kSiteQkvAcc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * 256);
        for (int kc = 0; kc < p.n_k; ++kc, ++it) {
          const int st = static_cast<int>(it % kQk2Stages);
          if (!mbar_wait(bar + kQ2Full + 8 * st, (it / kQk2Stages) & 1, p.wait, abort_flag, kSiteQkvFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sb + st * kQk2Stage, sbw = sa + kQkA;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_ss_pair(acc, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sbw + kk * 32, 16, 1024), kId,
                           (kc > 0 || kk > 0) ? 1u : 0u);
          tc_commit_pair_both(bar + kQ2Empty + 8 * st);
        }
        if (!ok) break;
        tc_commit_pair_both(bar + kQ2AccFull + 8 * buf);
      }
      tc_commit_pair_local(bar + kQ2Done);
      mbar_wait(bar + kQ2Done, 0, p.wait, nullptr, kSiteQkvDrain);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    griddep_wait();  // the RoPE table, written by the kernel launched before this one
    const int wq = warp & 3;
    const int hh = (warp - 2) >> 2;  // which of the tile's two heads this warp takes
    const int row = wq * 32 + lane;  // token row of this CTA's tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float* sg = reinterpret_cast<const float*>(sgen + kQk2Gain);
    bool ok = true;
    int n = 0;
    for (int tile = t_begin; tile < t_end && ok; ++tile, ++n) {
      const int mp = tile / p.n_nt, nt = tile - (tile / p.n_nt) * p.n_nt;
      const int mt = 2 * mp + static_cast<int>(rank);
      const int buf = n & 1;
      ok = mbar_wait(bar + kQ2AccFull + 8 * buf, (n >> 1) & 1, p.wait, abort_flag, kSiteQkvAcc);
      if (!ok) break;
      tc_fence_after();
      const long long m = static_cast<long long>(mt) * 128 + row;
      const int h = nt * 2 + hh;  // head index in [q heads | k heads | v heads]
      uint32_t y[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + static_cast<uint32_t>(buf * 256 + hh * 128 + c * 32), r);
#pragma unroll
        for (int i = 0; i < 32; ++i) y[c * 32 + i] = r[i];
      }
      // this warp's rows are in registers: one arrival on the leader's barrier per warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(bar + kQ2AccEmpty + 8 * buf, 0));
      if (h >= p.n_heads || m >= p.M) continue;
      uint4* dst;
      if (h < p.Hq + p.Hkv) {
        const bool is_q = h < p.Hq;
        const float* g = sg + (is_q ? 0 : 128);
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 128; ++i) ss = fmaf(__uint_as_float(y[i]), __uint_as_float(y[i]), ss);
        const float rn = rsqrtf(fmaf(ss, 1.0f / kD, p.eps));
        const float2* rope = p.rope + static_cast<size_t>(mt) * 64 * 128;  // this token tile's table
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float2 cs = rope[i * 128 + row];
          const float a = g[i] * (__uint_as_float(y[i]) * rn);
          const float b = g[64 + i] * (__uint_as_float(y[64 + i]) * rn);
          y[i] = __float_as_uint(a * cs.x - b * cs.y);
          y[64 + i] = __float_as_uint(b * cs.x + a * cs.y);
        }
        dst = is_q ? p.q_out + (m * p.Hq + h) * (kD / 8) : p.k_out + (m * p.Hkv + (h - p.Hq)) * (kD / 8);
      } else {
        dst = p.v_out + (m * p.Hkv + (h - p.Hq - p.Hkv)) * (kD / 8);
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(y[8 * c + 0]), __uint_as_float(y[8 * c + 1]));
        w.y = pack_bf16x2(__uint_as_float(y[8 * c + 2]), __uint_as_float(y[8 * c + 3]));
        w.z = pack_bf16x2(__uint_as_float(y[8 * c + 4]), __uint_as_float(y[8 * c + 5]));
        w.w = pack_bf16x2(__uint_as_float(y[8 * c + 6]), __uint_as_float(y[8 * c + 7]));
        dst[c] = w;
      }
    }
  }

  // Neither CTA leaves while the other's MMAs may still read its shared memory or TMEM.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace q3
