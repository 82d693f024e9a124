// prologue.cuh - QK-Norm + RoPE of raw head vectors, written straight into KV-cache layout.
//
// One warp per head vector (Qwen3 applies a per-head RMSNorm of width head_dim with a
// shared gain, then rotate-half RoPE: "Hand-Writing a Vision-Language Model, Part 1",
// RMSNorm / RotaryEmbedding; "Qwen3 Architecture Layer-by-Layer", Qwen3RMSNorm and
// apply_rotary_pos_emb).  Lane l loads dims {2l,2l+1} and {64+2l,65+2l} as two 4-byte
// words, so each half of the vector is one coalesced 128-byte access and both members of
// every RoPE pair (i, i+64) live in the same lane: no shuffle for the rotation, one
// 5-step butterfly for the sum of squares.  The result is rounded once to bf16.
#pragma once
#include "common.cuh"

namespace q3 {

struct PrologueParams {
  const uint32_t* x;   // [B, T, H, d] bf16 pairs
  const float* w;      // [d]
  const int* pos;      // [B, T]
  uint32_t* dst;       // [B, H, Tcap, d] bf16 pairs
  const uint2* v_src;  // optional [B, T, H, d], 4 bf16 per lane
  uint2* v_dst;        // optional [B, H, Tcap, d]
  int B, T, H, Tcap, write_at_pos;
  float eps;
  RopeTable rope;
};

constexpr int kPrologueUnroll = 4;  // vectors in flight per warp

__global__ void __launch_bounds__(256) qk_norm_rope_kernel(const __grid_constant__ PrologueParams p) {
  // The RoPE constants go through shared memory once per block: read from parameter space
  // with a lane-dependent index they would serialise.
  __shared__ float s_rope[2 * kHalf];
  if (threadIdx.x < 2 * kHalf)
    s_rope[threadIdx.x] = threadIdx.x < kHalf ? p.rope.hi[threadIdx.x] : p.rope.lo[threadIdx.x - kHalf];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const long long nwarps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long nvec = static_cast<long long>(p.B) * p.T * p.H;
  const float2 ga = reinterpret_cast<const float2*>(p.w)[lane];
  const float2 gb = reinterpret_cast<const float2*>(p.w)[32 + lane];
  const float hi0 = s_rope[2 * lane], hi1 = s_rope[2 * lane + 1];
  const float lo0 = s_rope[kHalf + 2 * lane], lo1 = s_rope[kHalf + 2 * lane + 1];
  for (long long v0 = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); v0 < nvec;
       v0 += nwarps * kPrologueUnroll) {
    uint32_t ua[kPrologueUnroll], ub[kPrologueUnroll];
    uint2 vv[kPrologueUnroll];
    int ps[kPrologueUnroll];
#pragma unroll
    for (int u = 0; u < kPrologueUnroll; ++u) {  // every load of the batch before any arithmetic
      const long long v = v0 + u * nwarps;
      ua[u] = ub[u] = 0u;
      ps[u] = 0;
      vv[u] = make_uint2(0u, 0u);
      if (v < nvec) {
        ps[u] = p.pos[v / p.H];
        ua[u] = p.x[v * (kD / 2) + lane];
        ub[u] = p.x[v * (kD / 2) + 32 + lane];
        if (p.v_src != nullptr) vv[u] = p.v_src[v * (kD / 4) + lane];
      }
    }
#pragma unroll
    for (int u = 0; u < kPrologueUnroll; ++u) {
      const long long v = v0 + u * nwarps;
      if (v >= nvec) break;  // uniform across the warp
      const int h = static_cast<int>(v % p.H);
      const long long bt = v / p.H;  // b*T + t
      const int t = static_cast<int>(bt % p.T);
      const int b = static_cast<int>(bt / p.T);
      const int row = p.write_at_pos ? ps[u] : t;
      if (row < 0 || row >= p.Tcap) {
        if (lane == 0) record_error(QWEN3_ERR_INVALID_ARG, kSitePrologueRow);
        continue;
      }
      float s0, c0, s1, c1;
      rope_sincos(ps[u], hi0, lo0, s0, c0);
      rope_sincos(ps[u], hi1, lo1, s1, c1);
      float2 ya, yb;
      norm_rope_pairs(make_float2(bf16lo(ua[u]), bf16hi(ua[u])), make_float2(bf16lo(ub[u]), bf16hi(ub[u])), ga, gb,
                      s0, c0, s1, c1, p.eps, ya, yb);
      const long long drow = (static_cast<long long>(b) * p.H + h) * p.Tcap + row;
      uint32_t* ds = p.dst + drow * (kD / 2);
      ds[lane] = pack_bf16x2(ya.x, ya.y);
      ds[32 + lane] = pack_bf16x2(yb.x, yb.y);
      if (p.v_src != nullptr) p.v_dst[drow * (kD / 4) + lane] = vv[u];
    }
  }
}

}  // namespace q3
