// prefill.cuh - causal GQA flash attention for sm_100a with the Q half of the QK-Norm+RoPE
// prologue fused into the Q-tile load.
//
// What it computes: for every query row, softmax over keys j <= i of (q'.k'_j)/sqrt(d),
// times v_j, where q' and k' are the QK-Normed and rotated vectors and query head h reads
// KV head h/G ("Assembling a large model from scratch", Attention.forward: scores, tril
// mask, fp32 softmax, repeat_interleave of KV heads; "Hand-Writing a Vision-Language Model,
// Part 1", order of operations).  The online (running-max) logsumexp that lets the key
// axis be tiled is the technique named for the fused cross-entropy in "Qwen3 Architecture
// Layer-by-Layer", Liger fused linear cross-entropy.
//
// One CTA owns one 128-row query tile of one (batch row, KV head): rows are P = 128/G
// consecutive positions x the G query heads of the group, so each K/V tile is loaded once
// per GQA group and feeds 128 MMA rows.  Six warps:
//   warp 0      TMA producer: K'/V tiles (128 keys x 128 dims, two 128B-swizzled boxes
//               each) into a 2-stage ring; owns the TMEM allocation.
//   warp 1      MMA issuer (one thread): S = Q K^T into one of two TMEM S buffers, then
//               O += P V into the TMEM O accumulator; tcgen05.commit signals completion.
//   warps 2-5   one thread per query row: Q prologue (warp-cooperative, into swizzled
//               smem), then per key tile: tcgen05.ld of its S row, causal mask, exp2 online
//               softmax with a lazy rescale (O is rescaled only when the running max grows
//               by more than 2^8), bf16 P into swizzled smem; finally O/l and the LSE.
// TMEM: S0 cols [0,128), S1 [128,256), O [256,384) of a 512-column allocation.
// Every wait is bounded (see mbar_wait); on a timeout every role stops, copies and MMAs
// in flight are drained, TMEM is freed and the error is left in the status word.
#pragma once
#include "common.cuh"

namespace q3 {

struct PrefillParams {
  const uint32_t* q;  // [B, T, Hq, d] bf16 pairs
  const float* q_norm_w;
  const int* pos;  // [B, T]
  uint4* out;      // [B, T, Hq, d] bf16, 16-byte chunks
  float* lse;      // [B, Hq, T] or nullptr
  int B, T, Hq, Hkv, log2G, P, n_qt;
  float eps, scale_log2;
  WaitCfg wait;
  int fault;
  RopeTable rope;
};

constexpr uint32_t kPfTile = 32768;  // 128 rows x 128 bf16
constexpr uint32_t kPfBox = 16384;   // 128 rows x 64 bf16: one 128B-swizzled TMA box
constexpr uint32_t kPfQ = 0;
constexpr uint32_t kPfK = kPfTile;       // 2 stages
constexpr uint32_t kPfV = 3 * kPfTile;   // 2 stages
constexpr uint32_t kPfP = 5 * kPfTile;
constexpr uint32_t kPfBar = 6 * kPfTile;
// barrier block (byte offsets from kPfBar)
constexpr uint32_t kBKFull = 0, kBKEmpty = 16, kBVFull = 32, kBVEmpty = 48, kBSFull = 64, kBPReady = 80,
                   kBOFull = 88, kBQReady = 96, kBDone = 104, kBTmemSlot = 112, kBAbort = 116;
constexpr uint32_t kPrefillSmemBytes = kPfBar + 128 + 1024;  // + slack to align the base to 1024
constexpr int kPrefillThreads = 192;
constexpr float kLn2 = 0.693147180559945309f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kPrefillThreads, 1)
    fmha_prefill_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sb - raw);
  const uint32_t sQ = sb + kPfQ, sK = sb + kPfK, sV = sb + kPfV, sP = sb + kPfP, bar = sb + kPfBar;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kPfBar + kBAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + kPfBar + kBTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.B * p.Hkv;
  const int qt = p.n_qt - 1 - static_cast<int>(blockIdx.x) / BH;  // heaviest tiles first
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int b = bh / p.Hkv, hkv = bh % p.Hkv;
  const int G = 1 << p.log2G;
  const int t0 = qt * p.P;
  const int t_end = min(t0 + p.P, p.T);
  const int nkv = (t_end - 1) / 128 + 1;  // key tiles 0..nkv-1 hold every key some row sees

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar + kBKFull + 8 * s, 1);
      mbar_init(bar + kBKEmpty + 8 * s, 1);
      mbar_init(bar + kBVFull + 8 * s, 1);
      mbar_init(bar + kBVEmpty + 8 * s, 1);
      mbar_init(bar + kBSFull + 8 * s, 1);
    }
    mbar_init(bar + kBPReady, 128);
    mbar_init(bar + kBOFull, 1);
    mbar_init(bar + kBQReady, 128);
    mbar_init(bar + kBDone, 1);
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
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      int k_last[2] = {-1, -1}, v_last[2] = {-1, -1};
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (j >= 2 && !mbar_wait(bar + kBKEmpty + 8 * st, ph ^ 1, p.wait, abort_flag, kSitePrefillKEmpty)) break;
        if (!(p.fault != 0 && j == 0)) {
          mbar_arrive_expect_tx(bar + kBKFull + 8 * st, kPfTile);
          tma_load_4d(sK + st * kPfTile, &tmK, bar + kBKFull + 8 * st, 0, j * 128, hkv, b);
          tma_load_4d(sK + st * kPfTile + kPfBox, &tmK, bar + kBKFull + 8 * st, 64, j * 128, hkv, b);
          k_last[st] = j;
        }
        if (j >= 2 && !mbar_wait(bar + kBVEmpty + 8 * st, ph ^ 1, p.wait, abort_flag, kSitePrefillVEmpty)) break;
        mbar_arrive_expect_tx(bar + kBVFull + 8 * st, kPfTile);
        tma_load_4d(sV + st * kPfTile, &tmV, bar + kBVFull + 8 * st, 0, j * 128, hkv, b);
        tma_load_4d(sV + st * kPfTile + kPfBox, &tmV, bar + kBVFull + 8 * st, 64, j * 128, hkv, b);
        v_last[st] = j;
      }
      // Every issued copy must land before this CTA's shared memory is released.
      for (int s = 0; s < 2; ++s) {
        if (k_last[s] >= 0) mbar_wait(bar + kBKFull + 8 * s, (k_last[s] >> 1) & 1, p.wait, nullptr, kSitePrefillDrain);
        if (v_last[s] >= 0) mbar_wait(bar + kBVFull + 8 * s, (v_last[s] >> 1) & 1, p.wait, nullptr, kSitePrefillDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdQK = idesc_bf16(128, 128, false);  // B = K rows, K-major
      constexpr uint32_t kIdPV = idesc_bf16(128, 128, true);   // B = V, dims contiguous (MN-major)
      const uint32_t tO = tmem + 256;
      bool ok = mbar_wait(bar + kBQReady, 0, p.wait, abort_flag, kSitePrefillQReady);
      auto issue_s = [&](int j) {
        const int st = j & 1;
        ok = ok && mbar_wait(bar + kBKFull + 8 * st, (j >> 1) & 1, p.wait, abort_flag, kSitePrefillKFull);
        if (!ok) return;
        tc_fence_after();
        const uint32_t tS = tmem + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * kPfBox + (kk & 3) * 32;
          tc_mma_ss(tS, smem_desc_sw128(sQ + koff, 16, 1024), smem_desc_sw128(sK + st * kPfTile + koff, 16, 1024),
                    kIdQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar + kBSFull + 8 * (j & 1));
        tc_commit(bar + kBKEmpty + 8 * st);
      };
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; j < nkv && ok; ++j) {
        if (j + 1 < nkv) issue_s(j + 1);
        if (!ok) break;
        const int st = j & 1;
        ok = mbar_wait(bar + kBPReady, j & 1, p.wait, abort_flag, kSitePrefillPReady) &&
             mbar_wait(bar + kBVFull + 8 * st, (j >> 1) & 1, p.wait, abort_flag, kSitePrefillVFull);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * kPfBox + (kk & 3) * 32;
          tc_mma_ss(tO, smem_desc_sw128(sP + aoff, 16, 1024),
                    smem_desc_sw128(sV + st * kPfTile + kk * 2048, kPfBox, 1024), kIdPV,
                    (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar + kBOFull);
        tc_commit(bar + kBVEmpty + 8 * st);
      }
      // Drain: every MMA issued above has completed once this arrives.
      tc_commit(bar + kBDone);
      mbar_wait(bar + kBDone, 0, p.wait, nullptr, kSitePrefillDrain);
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroup
    const int wq = warp & 3;          // TMEM lane quadrant this warp may access
    const int row = wq * 32 + lane;   // query-tile row owned by this thread
    {
      // Q prologue: warp (warp-2) normalises and rotates rows [32*(warp-2), +32).
      const float2 ga = reinterpret_cast<const float2*>(p.q_norm_w)[lane];
      const float2 gb = reinterpret_cast<const float2*>(p.q_norm_w)[32 + lane];
      const float hi0 = p.rope.hi[2 * lane], lo0 = p.rope.lo[2 * lane];
      const float hi1 = p.rope.hi[2 * lane + 1], lo1 = p.rope.lo[2 * lane + 1];
      float s0 = 0.f, c0 = 1.f, s1 = 0.f, c1 = 1.f;
      int cur_t = -1;
      const int rbase = (warp - 2) * 32;
      for (int rr = 0; rr < 32; ++rr) {
        const int r = rbase + rr;
        const int t = t0 + (r >> p.log2G);
        uint32_t wa = 0u, wb = 0u;
        if (t < p.T) {  // uniform across the warp
          if (t != cur_t) {
            const int ps = p.pos[static_cast<long long>(b) * p.T + t];
            rope_sincos(ps, hi0, lo0, s0, c0);
            rope_sincos(ps, hi1, lo1, s1, c1);
            cur_t = t;
          }
          const int h = hkv * G + (r & (G - 1));
          const uint32_t* qs = p.q + (static_cast<long long>(b * p.T + t) * p.Hq + h) * (kD / 2);
          const uint32_t ua = qs[lane], ub = qs[32 + lane];
          float2 ya, yb;
          norm_rope_pairs(make_float2(bf16lo(ua), bf16hi(ua)), make_float2(bf16lo(ub), bf16hi(ub)), ga, gb, s0, c0,
                          s1, c1, p.eps, ya, yb);
          wa = pack_bf16x2(ya.x, ya.y);
          wb = pack_bf16x2(yb.x, yb.y);
        }
        const uint32_t off = sw128_offset(r, lane >> 2) + (lane & 3) * 4;
        st_shared_u32(sQ + off, wa);
        st_shared_u32(sQ + kPfBox + off, wb);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar + kBQReady);
    }

    const int t_row = t0 + (row >> p.log2G);
    const int lim = min(t_row, p.T - 1);  // last key index this row may see
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tO = tmem + 256 + lane_off;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      ok = mbar_wait(bar + kBSFull + 8 * (j & 1), (j >> 1) & 1, p.wait, abort_flag, kSitePrefillSFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float s[128];
      const uint32_t tS = tmem + lane_off + (j & 1) * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + c * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
      }
      const int kv0 = j * 128;
      if (kv0 + 127 > t0) {
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = (kv0 + c <= lim) ? s[c] : -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
      const float mt = mx * sl2;
      float m_new = m;
      bool resc = false;
      if (mt > m + 8.0f) {  // lazy rescale: keep a stale max while p stays <= 2^8
        m_new = mt;
        resc = (j > 0);
      }
      uint32_t pk[64];
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = ex2(fmaf(s[c], sl2, -m_new));
        const float p1 = ex2(fmaf(s[c + 1], sl2, -m_new));
        sum += p0 + p1;  // fp32 row sum; P.V uses the bf16-rounded p
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      if (j > 0) {
        ok = mbar_wait(bar + kBOFull, (j - 1) & 1, p.wait, abort_flag, kSitePrefillOFull);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, resc)) {
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
      l += sum;
      m = m_new;
#pragma unroll
      for (int cb = 0; cb < 16; ++cb)
        st_shared_v4(sP + (cb >> 3) * kPfBox + sw128_offset(row, cb & 7), pk[4 * cb], pk[4 * cb + 1], pk[4 * cb + 2],
                     pk[4 * cb + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar + kBPReady);
    }
    if (ok) {
      ok = mbar_wait(bar + kBOFull, (nkv - 1) & 1, p.wait, abort_flag, kSitePrefillOFull);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const int h = hkv * G + (row & (G - 1));
      const bool valid = t_row < p.T;
      const float inv_l = 1.0f / l;
      uint4* dst = p.out + (static_cast<long long>(b * p.T + (valid ? t_row : 0)) * p.Hq + h) * (kD / 8);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
        if (valid) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(r[8 * k + 0]) * inv_l, __uint_as_float(r[8 * k + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(r[8 * k + 2]) * inv_l, __uint_as_float(r[8 * k + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(r[8 * k + 4]) * inv_l, __uint_as_float(r[8 * k + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(r[8 * k + 6]) * inv_l, __uint_as_float(r[8 * k + 7]) * inv_l);
            dst[c * 4 + k] = w;
          }
        }
      }
      if (p.lse != nullptr && valid)
        p.lse[(static_cast<long long>(b) * p.Hq + h) * p.T + t_row] = (m + log2f(l)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace q3
