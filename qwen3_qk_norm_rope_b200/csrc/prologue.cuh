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

__global__ void __launch_bounds__(256) qk_norm_rope_kernel(const __grid_constant__ PrologueParams p) {
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  const long long nvec = static_cast<long long>(p.B) * p.T * p.H;
  const float2 ga = reinterpret_cast<const float2*>(p.w)[lane];
  const float2 gb = reinterpret_cast<const float2*>(p.w)[32 + lane];
  const float hi0 = p.rope.hi[2 * lane], lo0 = p.rope.lo[2 * lane];
  const float hi1 = p.rope.hi[2 * lane + 1], lo1 = p.rope.lo[2 * lane + 1];
  for (long long v = static_cast<long long>(blockIdx.x) * warps_per_block + (threadIdx.x >> 5); v < nvec;
       v += static_cast<long long>(gridDim.x) * warps_per_block) {
    const int h = static_cast<int>(v % p.H);
    const long long bt = v / p.H;  // b*T + t
    const int t = static_cast<int>(bt % p.T);
    const int b = static_cast<int>(bt / p.T);
    const int ps = p.pos[bt];
    const int row = p.write_at_pos ? ps : t;
    if (row < 0 || row >= p.Tcap) {
      if (lane == 0) record_error(QWEN3_ERR_INVALID_ARG, kSitePrologueRow);
      continue;
    }
    const uint32_t* xs = p.x + v * (kD / 2);
    const uint32_t ua = xs[lane], ub = xs[32 + lane];
    float s0, c0, s1, c1;
    rope_sincos(ps, hi0, lo0, s0, c0);
    rope_sincos(ps, hi1, lo1, s1, c1);
    float2 ya, yb;
    norm_rope_pairs(make_float2(bf16lo(ua), bf16hi(ua)), make_float2(bf16lo(ub), bf16hi(ub)), ga, gb, s0, c0, s1,
                    c1, p.eps, ya, yb);
    const long long drow = (static_cast<long long>(b) * p.H + h) * p.Tcap + row;
    uint32_t* ds = p.dst + drow * (kD / 2);
    ds[lane] = pack_bf16x2(ya.x, ya.y);
    ds[32 + lane] = pack_bf16x2(yb.x, yb.y);
    if (p.v_src != nullptr) p.v_dst[drow * (kD / 4) + lane] = p.v_src[v * (kD / 4) + lane];
  }
}

}  // namespace q3
