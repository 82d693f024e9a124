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
  // Optional queries of the same tokens (the prefill): raw xq [B, T, Hq, d] with gain wq,
  // written as Q' [B, H, T*G, d] with G = Hq / H: row t*G + g of KV head h holds query
  // head h*G + g, the row order of the attention kernel's GQA-packed query tiles.
  const uint32_t* xq;
  const float* wq;
  uint32_t* dstq;
  int B, T, H, Tcap, write_at_pos;
  int Hq, log2G;
  // Optional paged destination: dst and v_dst are page pools [num_pages, H, page, d]; key
  // index kk of batch row b (pos[b,t] when write_at_pos, else key0 + t) lives in page
  // block_table[b, kk / page] at offset kk % page.  page = 1 << log2_page.
  const int* block_table;
  int max_blocks, log2_page, num_pages, key0;
  // Optional varlen batch (B = 1, T = N packed tokens; sequence b owns tokens cu[b] ..
  // cu[b+1]-1).  Without pages, tokens before cu[0] or from cu[B] on belong to no sequence
  // and get zero keys and values (a sequence's last key tile reads past its end, and the
  // values there still enter P.V as 0 x value).  With pages, a token's keys go to its own
  // sequence's pages (seq[b] = {qoff, T, start, koff}: key index start + token - qoff), and
  // tokens of no valid sequence write no key or value.
  const int* vl_cu;
  const int4* vl_seq;
  int vl_B;
  float eps;
  float rope_scale;  // attention_scaling: multiplies cos and sin (1 for the default rope type)
  RopeTable rope;
};

constexpr int kPrologueHeads = 8;  // head vectors of one token in flight per warp

// One warp per token (b, t): its position and the sin/cos of its 64 angles are computed once
// and shared by the token's H key heads (and, for the prefill, its Hq query heads), whose
// loads are issued a batch at a time before any arithmetic.  Each warp's work is a fixed
// chain of dependent loads, so the kernel takes as many chain times as it has waves: at most
// 64 registers a thread keeps 4 blocks (32 warps) resident per SM, which holds the 4096
// tokens of a B=2, T=2048 prefill in one wave (at 80 registers only 3 blocks fit and 68
// blocks ran as a second wave).  kPerBatch: one warp per batch of kPrologueHeads head vectors
// of a token instead (its key batches, then its query batches), for calls whose tokens are
// few enough that all their batches fit one wave: the batches then run side by side rather
// than as one chain per token.
template <bool kPerBatch>
__global__ void __launch_bounds__(256, 4) qk_norm_rope_kernel(const __grid_constant__ PrologueParams p) {
  // The RoPE constants go through shared memory once per block: read from parameter space
  // with a lane-dependent index they would serialise.
  __shared__ float s_rope[2 * kHalf];
  // The attention kernel that follows may be scheduled now: it waits (griddep_wait) for
  // this grid's results before it reads them, and meanwhile sets up and loads its queries.
  griddep_launch_dependents();
  if (threadIdx.x < 2 * kHalf)
    s_rope[threadIdx.x] = threadIdx.x < kHalf ? p.rope.hi[threadIdx.x] : p.rope.lo[threadIdx.x - kHalf];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  const int ntok = p.B * p.T;
  const float2 ga = reinterpret_cast<const float2*>(p.w)[lane];
  const float2 gb = reinterpret_cast<const float2*>(p.w)[32 + lane];
  const float hi0 = s_rope[2 * lane], hi1 = s_rope[2 * lane + 1];
  const float lo0 = s_rope[kHalf + 2 * lane], lo1 = s_rope[kHalf + 2 * lane + 1];
  const int nbk = (p.H + kPrologueHeads - 1) / kPrologueHeads;
  const int nb = kPerBatch ? nbk + (p.xq != nullptr ? (p.Hq + kPrologueHeads - 1) / kPrologueHeads : 0) : 1;
  // units: ntok (one per token), or ntok * nb <= 32 warps per SM (one per batch of heads)
  const int nunits = ntok * nb;
  for (int unit = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); unit < nunits; unit += nwarps) {
    const int bt = kPerBatch ? unit / nb : unit;
    // the head batches of this unit: all of them, or key batch ub, or query batch ub - nbk
    const int ub = kPerBatch ? unit - bt * nb : -1;
    const int k_lo = ub < 0 ? 0 : (ub < nbk ? ub * kPrologueHeads : p.H);
    const int k_hi = ub < 0 ? p.H : k_lo + kPrologueHeads;
    const int q_lo = ub < 0 ? 0 : (ub < nbk ? p.Hq : (ub - nbk) * kPrologueHeads);
    const int q_hi = ub < 0 ? p.Hq : q_lo + kPrologueHeads;
    const int b = bt / p.T;
    const int t = bt - b * p.T;
    const int ps = p.pos[bt];
    // destination of head 0 and the distance between heads, in rows of d
    size_t row0 = 0, hstride = 0;
    bool kv_write = true, kv_zero = false;
    if (p.block_table == nullptr) {
      const int row = p.write_at_pos ? ps : t;
      if (row < 0 || row >= p.Tcap) {
        if (lane == 0) record_error(QWEN3_ERR_INVALID_ARG, kSitePrologueRow);
        continue;
      }
      row0 = static_cast<size_t>(b) * p.H * p.Tcap + row;
      hstride = p.Tcap;
      if (p.vl_cu != nullptr) kv_zero = bt < __ldg(p.vl_cu) || bt >= __ldg(p.vl_cu + p.vl_B);
    } else {
      int bs = b, kk = p.write_at_pos ? ps : p.key0 + t;
      if (p.vl_seq != nullptr) {
        // the token's sequence: the last b with cu[b] <= bt, checked against its metadata
        int lo = 0, hi = p.vl_B - 1;
        bs = -1;
        while (lo <= hi) {
          const int mid = (lo + hi) >> 1;
          if (__ldg(p.vl_cu + mid) <= bt) {
            bs = mid;
            lo = mid + 1;
          } else {
            hi = mid - 1;
          }
        }
        const int4 sq = bs >= 0 ? p.vl_seq[bs] : make_int4(0, 0, 0, 0);
        kv_write = bs >= 0 && bt >= sq.x && bt < sq.x + sq.y;
        kk = sq.z + (bt - sq.x);
      }
      if (kv_write) {
        const int blk = kk >> p.log2_page;
        const int page =
            (kk >= 0 && blk < p.max_blocks) ? p.block_table[static_cast<size_t>(bs) * p.max_blocks + blk] : -1;
        if (page < 0 || page >= p.num_pages) {
          if (lane == 0) record_error(QWEN3_ERR_INVALID_ARG, kSitePrologueRow);
          continue;
        }
        row0 = (static_cast<size_t>(page) * p.H << p.log2_page) + (kk & ((1 << p.log2_page) - 1));
        hstride = static_cast<size_t>(1) << p.log2_page;
      }
    }
    float s0, c0, s1, c1;
    rope_sincos(ps, hi0, lo0, s0, c0);
    rope_sincos(ps, hi1, lo1, s1, c1);
    s0 *= p.rope_scale;
    c0 *= p.rope_scale;
    s1 *= p.rope_scale;
    c1 *= p.rope_scale;
    for (int h0 = k_lo; kv_write && h0 < min(k_hi, p.H); h0 += kPrologueHeads) {
      uint32_t ua[kPrologueHeads], ub[kPrologueHeads];
      uint2 vv[kPrologueHeads];
#pragma unroll
      for (int u = 0; u < kPrologueHeads; ++u) {  // every load of the batch before any arithmetic
        ua[u] = ub[u] = 0u;
        vv[u] = make_uint2(0u, 0u);
        if (h0 + u < p.H) {
          const size_t v = static_cast<size_t>(bt) * p.H + h0 + u;
          ua[u] = p.x[v * (kD / 2) + lane];
          ub[u] = p.x[v * (kD / 2) + 32 + lane];
          if (p.v_src != nullptr) vv[u] = p.v_src[v * (kD / 4) + lane];
        }
      }
#pragma unroll
      for (int u = 0; u < kPrologueHeads; ++u) {
        if (h0 + u >= p.H) break;  // uniform across the warp
        float2 ya, yb;
        norm_rope_pairs(make_float2(bf16lo(ua[u]), bf16hi(ua[u])), make_float2(bf16lo(ub[u]), bf16hi(ub[u])), ga,
                        gb, s0, c0, s1, c1, p.eps, ya, yb);
        if (kv_zero) {
          ya = yb = make_float2(0.f, 0.f);
          vv[u] = make_uint2(0u, 0u);
        }
        const size_t drow = row0 + static_cast<size_t>(h0 + u) * hstride;
        uint32_t* ds = p.dst + drow * (kD / 2);
        ds[lane] = pack_bf16x2(ya.x, ya.y);
        ds[32 + lane] = pack_bf16x2(yb.x, yb.y);
        if (p.v_src != nullptr) p.v_dst[drow * (kD / 4) + lane] = vv[u];
      }
    }
    if (p.xq == nullptr) continue;
    const float2 qa = reinterpret_cast<const float2*>(p.wq)[lane];
    const float2 qb = reinterpret_cast<const float2*>(p.wq)[32 + lane];
    const int G = 1 << p.log2G;
    for (int h0 = q_lo; h0 < min(q_hi, p.Hq); h0 += kPrologueHeads) {
      uint32_t ua[kPrologueHeads], ub[kPrologueHeads];
#pragma unroll
      for (int u = 0; u < kPrologueHeads; ++u) {
        ua[u] = ub[u] = 0u;
        if (h0 + u < p.Hq) {
          const size_t v = static_cast<size_t>(bt) * p.Hq + h0 + u;
          ua[u] = p.xq[v * (kD / 2) + lane];
          ub[u] = p.xq[v * (kD / 2) + 32 + lane];
        }
      }
#pragma unroll
      for (int u = 0; u < kPrologueHeads; ++u) {
        const int h = h0 + u;
        if (h >= p.Hq) break;  // uniform across the warp
        float2 ya, yb;
        norm_rope_pairs(make_float2(bf16lo(ua[u]), bf16hi(ua[u])), make_float2(bf16lo(ub[u]), bf16hi(ub[u])), qa,
                        qb, s0, c0, s1, c1, p.eps, ya, yb);
        const size_t drow = ((static_cast<size_t>(b) * p.H + (h >> p.log2G)) * p.T + t) * G + (h & (G - 1));
        uint32_t* ds = p.dstq + drow * (kD / 2);
        ds[lane] = pack_bf16x2(ya.x, ya.y);
        ds[32 + lane] = pack_bf16x2(yb.x, yb.y);
      }
    }
  }
}

}  // namespace q3
