// paged.cuh - KV cache in pages (the block-table layout of paged serving engines: "LLM
// Internals - Assembling a large model from scratch", the notes below the code, on real
// systems replacing the append-by-concatenation cache with preallocated paged memory).
//
// A pool holds num_pages pages of `page` tokens for all KV heads, [num_pages, Hkv, page, d]
// bf16; key index j of batch row b lives in page block_table[b, j / page] at offset
// j % page.  The decode split kernel and the prefill attention kernel read pages of 64 keys
// or more in place; this file holds the gather for smaller pages, which copies a row's first
// n keys out of the pages into the contiguous layout [B, Hkv, n, d] that the prefill
// attention kernel then reads (a 128-key tile of 16-key pages would take 16 TMA boxes of
// 2 KB per operand, and the TMA box rate, not the bytes, would then bound the prefill).
#pragma once
#include "common.cuh"

namespace q3 {

struct GatherParams {
  const uint4* k_pages;  // [num_pages, Hkv, page, d] as 16-byte chunks
  const uint4* v_pages;
  const int* block_table;  // [B, max_blocks]
  uint4* k_out;            // [B, Hkv, n, d]
  uint4* v_out;
  int B, Hkv, n, max_blocks, log2_page, num_pages;
};

// One thread per 16-byte chunk of a (row, key, head) vector: 16 chunks per head vector.
__global__ void __launch_bounds__(256) paged_gather_kernel(const __grid_constant__ GatherParams p) {
  const long long total = static_cast<long long>(p.B) * p.n * p.Hkv * 16;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int c = static_cast<int>(i & 15);
    const long long v = i >> 4;  // ((b * n) + key) * Hkv + h
    const int h = static_cast<int>(v % p.Hkv);
    const long long bk = v / p.Hkv;
    const int key = static_cast<int>(bk % p.n);
    const int b = static_cast<int>(bk / p.n);
    const int blk = key >> p.log2_page;
    const int page = blk < p.max_blocks ? p.block_table[static_cast<long long>(b) * p.max_blocks + blk] : -1;
    const long long dst = ((static_cast<long long>(b) * p.Hkv + h) * p.n + key) * 16 + c;
    if (page < 0 || page >= p.num_pages) {
      if (c == 0 && h == 0) record_error(QWEN3_ERR_INVALID_ARG, kSitePagedTable);
      p.k_out[dst] = make_uint4(0u, 0u, 0u, 0u);
      p.v_out[dst] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const long long src =
        ((static_cast<long long>(page) * p.Hkv + h) << p.log2_page | (key & ((1 << p.log2_page) - 1))) * 16 + c;
    p.k_out[dst] = p.k_pages[src];
    p.v_out[dst] = p.v_pages[src];
  }
}

}  // namespace q3
