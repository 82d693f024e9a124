/*
 * qwen3_attn.h - C ABI of libqwen3attn.so, the Qwen3 attention core on B200 (sm_100a).
 *
 * The core takes projected q/k/v and computes, per head vector of head_dim d = 128:
 *   1. QK-Norm: y = g * x / sqrt(mean(x^2) + eps), fp32 statistics, learned gain g[d]
 *      ("Qwen3 Architecture Layer-by-Layer", Primitives: Qwen3RMSNorm; "Hand-Writing a
 *      Vision-Language Model, Part 1", RMSNorm and the order-of-operations list).
 *   2. RoPE, rotate-half pairing (dim i with dim i + d/2), inv_i = theta^(-2i/d), angle
 *      pos * inv_i ("Hand-Writing ... Part 1", RotaryEmbedding (RoPE); "Qwen3 Architecture
 *      Layer-by-Layer", apply_rotary_pos_emb and Qwen3RotaryEmbedding).
 *   3. Causal grouped-query attention, scale 1/sqrt(d), query head h reading KV head
 *      h / (Hq/Hkv) ("Assembling a large model from scratch", The complete code,
 *      Attention.forward; "Qwen3 Architecture Layer-by-Layer", The attention dispatch).
 * V is never normalised or rotated.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers to memory the caller owns; the library
 *     never frees or retains them.  bf16 tensors are passed as `qwen3_bf16` (uint16 bit
 *     patterns of IEEE bfloat16).  All tensors are dense row-major (C order) with the
 *     shapes stated below; base addresses must be 16-byte aligned.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream) and never
 *     synchronise, except qwen3_attn_device_status().  Host-side argument checks happen
 *     before any launch; a failed check launches nothing.
 *   - Functions return a qwen3_status and never abort or throw.
 *   - Inputs must not alias outputs.
 *   - Supported shapes: d == 128; Hkv >= 1; Hq % Hkv == 0 with G = Hq/Hkv a power of two,
 *     G <= 128 for prefill and G <= 16 for decode.  Other shapes return
 *     QWEN3_ERR_UNSUPPORTED.
 *   - Device waits are bounded.  If a kernel's internal wait runs out (a hardware or
 *     library fault, never a legal input), the kernel records QWEN3_ERR_DEVICE_TIMEOUT in a
 *     device-side status word and returns early; qwen3_attn_device_status() reports it.
 */
#ifndef QWEN3_ATTN_H_
#define QWEN3_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t qwen3_bf16;
typedef struct CUstream_st* qwen3_stream_t; /* same handle as cudaStream_t */

typedef enum {
  QWEN3_OK = 0,
  QWEN3_ERR_INVALID_ARG = 1,    /* NULL required pointer, non-positive size, misaligned pointer */
  QWEN3_ERR_UNSUPPORTED = 2,    /* d != 128, Hq % Hkv != 0, G not a supported power of two    */
  QWEN3_ERR_CUDA = 3,           /* a CUDA runtime/driver call or launch failed                */
  QWEN3_ERR_DEVICE_TIMEOUT = 4, /* a bounded device-side wait ran out                         */
  QWEN3_ERR_WORKSPACE = 5       /* workspace NULL or smaller than the *_workspace_size value  */
} qwen3_status;

/*
 * qwen3_attn_variant - the variants of the core that a Qwen3 configuration can select.
 * "Qwen3 Architecture Layer-by-Layer", Per-layer attention type: a layer is full or
 * sliding-window attention.  Qwen3RotaryEmbedding: the rope type fixes inv_freq (its
 * initialisation function) and an attention_scaling that multiplies cos and sin.  "Qwen 3
 * From Scratch": long context through rotary scaling (YaRN) in the config.
 *   theta              RoPE base: inv_i = theta^(-2i/d), used when inv_freq is NULL (> 0).
 *   inv_freq           optional HOST array of d/2 rotary frequencies, e.g. a YaRN or linear
 *                      scaling initialisation computed by the caller; it replaces theta.
 *                      Read during the call only.  Entries must be finite.
 *   attention_scaling  multiplies cos and sin, so q' and k' (and the keys the call writes to
 *                      a cache); 1 for the default rope type.  Finite, > 0.
 *   window             sliding window W >= 1: query at key index i sees keys i-W < j <= i,
 *                      its own key included; 0 = full causal attention.
 * An invalid variant returns QWEN3_ERR_INVALID_ARG.  The plain entry points are the
 * variant {theta, NULL, 1, 0}.
 */
typedef struct qwen3_attn_variant {
  float theta;
  const double* inv_freq;
  float attention_scaling;
  int window;
} qwen3_attn_variant;

/*
 * qwen3_qk_norm_rope - QK-Norm then RoPE of raw head vectors, written in cache layout.
 * Defined by steps 1-2 above ("Hand-Writing ... Part 1": q_norm/k_norm run right after the
 * projection and before RoPE).
 *   x      [B, T, H, d] bf16, raw projected head vectors (k, or q).
 *   w      [d] fp32 gain.
 *   pos    [B, T] int32 positions (the rotation angle of token t of row b is pos[b,t]*inv_i).
 *   dst    [B, H, Tcap, d] bf16: token t of row b, head h is written to slot
 *          dst[b, h, row, :] with row = t when write_at_pos == 0, row = pos[b,t] otherwise
 *          (the decode append: the new token of sequence b goes to index cache_len = pos).
 *   v_src  optional [B, T, H, d] bf16, copied unchanged to v_dst at the same slots
 *          (V is never normalised or rotated); pass NULL for both to skip.
 *   Rows must satisfy row < Tcap; an out-of-range row is skipped and recorded as
 *   QWEN3_ERR_INVALID_ARG in the device status word.  Results are rounded once to bf16.
 */
int qwen3_qk_norm_rope(const qwen3_bf16* x, const float* w, const int32_t* pos,
                       qwen3_bf16* dst, const qwen3_bf16* v_src, qwen3_bf16* v_dst,
                       int B, int T, int H, int d, int Tcap, int write_at_pos,
                       float theta, float eps, qwen3_stream_t stream);

/* qwen3_qk_norm_rope with a rope variant (inv_freq, attention_scaling; window unused). */
int qwen3_qk_norm_rope_variant(const qwen3_bf16* x, const float* w, const int32_t* pos,
                               qwen3_bf16* dst, const qwen3_bf16* v_src, qwen3_bf16* v_dst,
                               int B, int T, int H, int d, int Tcap, int write_at_pos,
                               const qwen3_attn_variant* variant, float eps,
                               qwen3_stream_t stream);

/*
 * qwen3_attn_prefill - causal GQA self-attention over T new tokens with the QK-Norm+RoPE
 * prologue ("Assembling a large model from scratch", Attention.forward with S == T; the
 * mask is tril on token index: token i sees tokens 0..i of its own batch row).
 *   q         [B, T, Hq, d] bf16 raw projected queries.
 *   k, v      [B, T, Hkv, d] bf16 raw projected keys and values.
 *   q_norm_w, k_norm_w  [d] fp32 gains.
 *   pos       [B, T] int32 RoPE positions.
 *   out       [B, T, Hq, d] bf16 attention output (heads not merged with o_proj).
 * The call needs qwen3_attn_prefill_workspace_size(B, T, Hq, Hkv, d) bytes of scratch (the
 * normed+rotated keys and queries), which it obtains stream-ordered with
 * cudaMallocAsync/cudaFreeAsync on `stream`.  Use qwen3_attn_prefill_ex to pass your own
 * workspace or to fill a KV cache instead.
 */
int qwen3_attn_prefill(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v,
                       const float* q_norm_w, const float* k_norm_w, const int32_t* pos,
                       qwen3_bf16* out, int B, int T, int Hq, int Hkv, int d,
                       float theta, float eps, qwen3_stream_t stream);

/*
 * qwen3_attn_prefill_ex - qwen3_attn_prefill with optional outputs and caller memory.
 *   lse       optional [B, Hq, T] fp32: natural-log logsumexp of the scaled logits of each
 *             query row (the logsumexp of "Qwen3 Architecture Layer-by-Layer", The
 *             cross-entropy math, applied to attention scores).  NULL to skip.
 *   k_cache, v_cache  optional [B, Hkv, Tcap, d] bf16 (Tcap >= T).  When given (both or
 *             neither), the normed+rotated keys and the raw values of tokens 0..T-1 are
 *             written to slots 0..T-1 and attention reads them from there, so the cache is
 *             ready for qwen3_attn_decode with cache_lens = T.
 *   workspace, ws_bytes  device scratch of at least
 *             qwen3_attn_prefill_workspace_size(B, T, Hq, Hkv, d) bytes, else
 *             QWEN3_ERR_WORKSPACE.  It holds the normed+rotated keys (unused when a cache is
 *             given) and queries, which one prologue pass per token writes before the
 *             attention kernel reads them.
 */
int qwen3_attn_prefill_ex(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v,
                          const float* q_norm_w, const float* k_norm_w, const int32_t* pos,
                          qwen3_bf16* out, float* lse,
                          qwen3_bf16* k_cache, qwen3_bf16* v_cache, int Tcap,
                          void* workspace, size_t ws_bytes,
                          int B, int T, int Hq, int Hkv, int d,
                          float theta, float eps, qwen3_stream_t stream);

/*
 * qwen3_attn_prefill_chunk - T new tokens per batch row over a KV cache that already holds
 * `start` tokens (chunked prefill).  "Assembling a large model from scratch",
 * Attention.forward with a cache and the notes below the code: the new keys are normed,
 * rotated and appended after the cached ones, S = start + T keys in all, and new token i
 * sees keys 0..start+i (the mask tril(diagonal = S - T)).  With start == 0 this is
 * qwen3_attn_prefill_ex with a cache; with T == 1 it is one decode step at length start.
 *   q, k, v, gains  as in qwen3_attn_prefill, for the T new tokens only.
 *   pos       [B, T] int32 RoPE positions of the new tokens (normally start..start+T-1;
 *             the mask uses the key index start+i, never pos).
 *   k_cache, v_cache  required [B, Hkv, Tcap, d] bf16.  Slots 0..start-1 are read: keys
 *             already normed and rotated, values raw, as qwen3_attn_prefill_ex and
 *             qwen3_attn_decode leave them.  The new keys' k' and raw v are written to slots
 *             start..start+T-1.  No other slot is touched.
 *   out       [B, T, Hq, d] bf16; lse optional [B, Hq, T] fp32 (NULL to skip).
 *   start     cached tokens, the same for every batch row; 0 <= start and
 *             start + T <= Tcap, else QWEN3_ERR_INVALID_ARG.
 *   workspace, ws_bytes  at least qwen3_attn_prefill_workspace_size(B, T, Hq, Hkv, d) bytes,
 *             else QWEN3_ERR_WORKSPACE.  With
 *             qwen3_attn_prefill_chunk_workspace_size(B, start, T, Hq, Hkv, d) bytes, a chunk
 *             whose work items are few next to the SMs (a short chunk over a long prefix)
 *             splits the key axis: each run of keys leaves its O/l and LSE as partials in the
 *             workspace and one more kernel merges them by logsumexp weight (the online
 *             logsumexp of "Qwen3 Architecture Layer-by-Layer", Liger fused linear
 *             cross-entropy).  With less, the call runs unsplit.  Sliding windows never split.
 * Other errors as in qwen3_attn_prefill_ex.  The caches must not alias q, k, v or out.
 */
int qwen3_attn_prefill_chunk(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v,
                             const float* q_norm_w, const float* k_norm_w, const int32_t* pos,
                             qwen3_bf16* out, float* lse,
                             qwen3_bf16* k_cache, qwen3_bf16* v_cache, int start, int Tcap,
                             void* workspace, size_t ws_bytes,
                             int B, int T, int Hq, int Hkv, int d,
                             float theta, float eps, qwen3_stream_t stream);

/*
 * qwen3_attn_decode - one new token per sequence attending over its KV cache
 * ("Assembling a large model from scratch", KVCache.update and Transformer.forward: the new
 * token sits at position cache.length and sees the whole history).
 *   q            [N, Hq, d] bf16 raw query of the new token.
 *   k_new, v_new [N, Hkv, d] bf16 raw key and value of the new token.
 *   q_norm_w, k_norm_w  [d] fp32 gains.
 *   k_cache, v_cache    [N, Hkv, Lmax, d] bf16.  Slots 0..L-1 of sequence n hold its
 *                normed+rotated keys and raw values.  This call writes the new token's
 *                normed+rotated key and raw value into slot L (L = cache_lens[n]).
 *   cache_lens   [N] int32 device array, L per sequence BEFORE the append; 0 <= L < Lmax.
 *                Not modified (the caller advances it, like the cache length that grows
 *                by the appended tokens).  A sequence with L >= Lmax is skipped and
 *                recorded as QWEN3_ERR_INVALID_ARG in the device status word.
 *   out          [N, Hq, d] bf16; lse optional [N, Hq] fp32 (NULL to skip).
 *   workspace    at least qwen3_attn_decode_workspace_size(N, Hq, d, Lmax) bytes of
 *                device scratch for the split-KV partials, else QWEN3_ERR_WORKSPACE.
 */
int qwen3_attn_decode(const qwen3_bf16* q, const qwen3_bf16* k_new, const qwen3_bf16* v_new,
                      const float* q_norm_w, const float* k_norm_w,
                      qwen3_bf16* k_cache, qwen3_bf16* v_cache, const int32_t* cache_lens,
                      qwen3_bf16* out, float* lse,
                      int N, int Hq, int Hkv, int d, int Lmax,
                      float theta, float eps, void* workspace, size_t ws_bytes,
                      qwen3_stream_t stream);

/*
 * qwen3_attn_decode_noalloc - qwen3_attn_decode for callers that cannot allocate device
 * memory.  The pages have no counterpart to this call; it exists for the host programs,
 * not for the method.  Some callers own no allocator: a plug-in that an inference engine
 * hands only its input and output buffers, or a serving loop whose device pool is managed
 * elsewhere and which must not call cudaMalloc on its hot path (cudaMalloc can
 * synchronise the device and bypasses that pool).  This call takes the same arguments as
 * qwen3_attn_decode minus the workspace and allocates nothing: its split-KV partials live
 * in one fixed region of QWEN3_ATTN_NOALLOC_SCRATCH_BYTES (48 MiB) of device memory that
 * the library declares statically, which every GPU that loads the library holds until
 * the process exits.
 *   - Limit: qwen3_attn_decode_workspace_size(N, Hq, d, Lmax) must not exceed
 *     QWEN3_ATTN_NOALLOC_SCRATCH_BYTES (64 sequences x 32 heads x Lmax 32769 need 34.9
 *     MB); larger requests return QWEN3_ERR_WORKSPACE and launch nothing.
 *   - The region's device address belongs to one CUDA context.  The first call in a
 *     context (the device's primary context, or another context the caller made current)
 *     looks that address up and keeps it for that context; after a device reset the new
 *     context's first call looks it up again.
 *   - Argument checks come first: a bad argument returns what qwen3_attn_decode returns
 *     for it, before the region is looked up.
 *   - Every call on a device shares the one region, and a call leaves its partials there.
 *     Nothing in it needs to start at zero (each split writes its partial before the
 *     combine reads it).  Calls whose kernels overlap on the GPU (other streams, other
 *     host threads) race on the region: serialise them.
 * All other arguments, outputs and errors are those of qwen3_attn_decode.
 */
#define QWEN3_ATTN_NOALLOC_SCRATCH_BYTES ((size_t)48 << 20)
int qwen3_attn_decode_noalloc(const qwen3_bf16* q, const qwen3_bf16* k_new, const qwen3_bf16* v_new,
                              const float* q_norm_w, const float* k_norm_w,
                              qwen3_bf16* k_cache, qwen3_bf16* v_cache, const int32_t* cache_lens,
                              qwen3_bf16* out, float* lse,
                              int N, int Hq, int Hkv, int d, int Lmax,
                              float theta, float eps, qwen3_stream_t stream);

/*
 * qwen3_attn_prefill_variant - the general prefill: qwen3_attn_prefill_ex (k_cache,
 * v_cache NULL and start 0) or qwen3_attn_prefill_chunk (caches given, `start` cached
 * tokens), with a qwen3_attn_variant in place of theta.  A sliding window keeps the last
 * `window` keys of each query; the key tiles wholly before every row's window are not read.
 */
int qwen3_attn_prefill_variant(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v,
                               const float* q_norm_w, const float* k_norm_w, const int32_t* pos,
                               qwen3_bf16* out, float* lse,
                               qwen3_bf16* k_cache, qwen3_bf16* v_cache, int start, int Tcap,
                               void* workspace, size_t ws_bytes,
                               int B, int T, int Hq, int Hkv, int d,
                               const qwen3_attn_variant* variant, float eps, qwen3_stream_t stream);

/*
 * qwen3_attn_decode_variant - qwen3_attn_decode with a qwen3_attn_variant in place of theta.
 * With a window the new token at position L attends to keys max(0, L-window+1)..L; the
 * splits wholly before the window are not read.
 */
int qwen3_attn_decode_variant(const qwen3_bf16* q, const qwen3_bf16* k_new, const qwen3_bf16* v_new,
                              const float* q_norm_w, const float* k_norm_w,
                              qwen3_bf16* k_cache, qwen3_bf16* v_cache, const int32_t* cache_lens,
                              qwen3_bf16* out, float* lse,
                              int N, int Hq, int Hkv, int d, int Lmax,
                              const qwen3_attn_variant* variant, float eps,
                              void* workspace, size_t ws_bytes, qwen3_stream_t stream);

/*
 * qwen3_paged_kv - a KV cache in pages, as paged serving engines keep it ("LLM Internals -
 * Assembling a large model from scratch", the notes below the code: real systems replace the
 * grow-by-concatenation cache with preallocated paged memory).
 *   k_pages, v_pages  [num_pages, Hkv, page_size, d] bf16 device pools (16-byte aligned).
 *   block_table       [rows, max_blocks] int32 device array: key index j of batch row (or
 *                     sequence) b lives in page block_table[b, j / page_size] at offset
 *                     j % page_size.  Only the blocks that hold keys the call reads or writes
 *                     are read; an entry outside [0, num_pages) is recorded as
 *                     QWEN3_ERR_INVALID_ARG in the device status word and its keys skipped.
 *   page_size         a power of two in [16, 1024].
 * The caller owns the pools and the table.
 */
typedef struct qwen3_paged_kv {
  qwen3_bf16* k_pages;
  qwen3_bf16* v_pages;
  const int32_t* block_table;
  int num_pages;
  int page_size;
  int max_blocks;
} qwen3_paged_kv;

/*
 * qwen3_attn_decode_paged - qwen3_attn_decode_variant over a paged cache: the new key and
 * value go to key index L = cache_lens[n] of sequence n (its page must be in the table), and
 * the split-KV kernel reads each 64-key chunk page by page with TMA.  L + 1 <=
 * max_blocks * page_size.  Workspace: qwen3_attn_decode_workspace_size(N, Hq, d,
 * max_blocks * page_size) bytes.
 */
int qwen3_attn_decode_paged(const qwen3_bf16* q, const qwen3_bf16* k_new, const qwen3_bf16* v_new,
                            const float* q_norm_w, const float* k_norm_w,
                            const qwen3_paged_kv* kv, const int32_t* cache_lens,
                            qwen3_bf16* out, float* lse,
                            int N, int Hq, int Hkv, int d,
                            const qwen3_attn_variant* variant, float eps,
                            void* workspace, size_t ws_bytes, qwen3_stream_t stream);

/*
 * qwen3_attn_prefill_paged - chunked prefill over a paged cache: T new tokens per batch row
 * after `start` cached ones (start = 0: a fresh prompt).  The new keys (normed, rotated) and
 * values are written into their pages at key indices start..start+T-1.  The attention
 * kernel then reads the row's start + T keys and values in place, one TMA box per page (or
 * per 128 rows of a larger page), as qwen3_attn_prefill_chunk reads a contiguous cache.
 * Pages under 64 keys would take too many small boxes: their keys and values are first
 * gathered into the workspace, where the attention kernel reads them.
 * start + T <= max_blocks * page_size.  A key index below start + T whose block-table entry
 * is out of range is recorded as QWEN3_ERR_INVALID_ARG in the device status word (read in
 * place, its rows are not read; gathered, they are zero) and the call's outputs for that row
 * are undefined.  Workspace: qwen3_attn_prefill_paged_workspace_size(B, start, T, Hq, Hkv, d)
 * bytes.
 */
int qwen3_attn_prefill_paged(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v,
                             const float* q_norm_w, const float* k_norm_w, const int32_t* pos,
                             qwen3_bf16* out, float* lse,
                             const qwen3_paged_kv* kv, int start,
                             void* workspace, size_t ws_bytes,
                             int B, int T, int Hq, int Hkv, int d,
                             const qwen3_attn_variant* variant, float eps, qwen3_stream_t stream);

/* Scratch bytes qwen3_attn_prefill_paged needs: K and V of start + T keys per row (used
 * for pages under 64 keys only), Q', the partials of a key-axis split when its work items
 * are few (as for qwen3_attn_prefill_chunk_workspace_size), and alignment slack; 0 when a
 * size is not positive (start may be 0).  A smaller workspace that still holds all but the
 * split partials runs the call unsplit. */
size_t qwen3_attn_prefill_paged_workspace_size(int B, int start, int T, int Hq, int Hkv, int d);

/*
 * qwen3_attn_prefill_varlen - prefill of B sequences packed on one token axis, the batching
 * of serving engines ("LLM Internals - Assembling a large model from scratch", the
 * comparison with inference engines: the tokens of many requests form one batch and
 * attention is computed per request; the review question on vLLM: flattened tokens plus
 * batching metadata).  Each sequence is an independent causal prefill, as
 * qwen3_attn_prefill_chunk computes it for one batch row.
 *   q          [N, Hq, d] bf16; k, v [N, Hkv, d]: the raw tokens of all sequences.
 *   pos        [N] int32 rotary positions (usually ctx_lens[b] + t for token t of b).
 *   cu_seqlens [B + 1] int32 device array: sequence b owns tokens cu_seqlens[b] ..
 *              cu_seqlens[b+1] - 1, with 0 <= cu_seqlens[b] <= cu_seqlens[b+1] <= N.
 *              Tokens before cu_seqlens[0] or from cu_seqlens[B] on belong to no
 *              sequence (padding); their rows of out and lse are not written.  An empty
 *              sequence is allowed.
 *   out        [N, Hq, d] bf16; lse [Hq, N] float (natural log) or NULL.
 *   kv         NULL: fresh prompts; the keys of a sequence are its own tokens, and ctx_lens
 *              must be NULL and key_cap 0.  Otherwise a paged cache (row b of the block
 *              table is sequence b): the sequence's new keys (normed, rotated) and values go
 *              to its key indices ctx_lens[b] .. ctx_lens[b] + T_b - 1, and its queries see
 *              its ctx_lens[b] cached keys first, as in qwen3_attn_prefill_paged.
 *   ctx_lens   [B] int32 device array of cached keys per sequence, or NULL (all 0).
 *   key_cap    with kv: a bound (> 0) on the sum over sequences of ctx_lens[b] + T_b.  The
 *              attention reads every sequence's keys and values in its own pages; pages
 *              under 64 keys are gathered first, into key_cap rows of the workspace.
 * The lengths stay on the device: the host reads none of them.  A sequence whose metadata
 * is out of range (offsets outside [0, N] or decreasing, a negative ctx_lens, keys past
 * max_blocks * page_size, or keys past key_cap) is recorded as QWEN3_ERR_INVALID_ARG in
 * the device status word and skipped.  Workspace:
 * qwen3_attn_prefill_varlen_workspace_size(B, N, key_cap, Hq, Hkv, d) bytes.
 */
int qwen3_attn_prefill_varlen(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v,
                              const float* q_norm_w, const float* k_norm_w, const int32_t* pos,
                              const int32_t* cu_seqlens, qwen3_bf16* out, float* lse,
                              const qwen3_paged_kv* kv, const int32_t* ctx_lens, long long key_cap,
                              void* workspace, size_t ws_bytes,
                              int B, int N, int Hq, int Hkv, int d,
                              const qwen3_attn_variant* variant, float eps, qwen3_stream_t stream);

/* Scratch bytes qwen3_attn_prefill_varlen needs: the sequence metadata and work list, Q',
 * and K' and V for N rows (key_cap = 0) or key_cap rows (used for pages under 64 keys
 * only); 0 for an unsupported shape. */
size_t qwen3_attn_prefill_varlen_workspace_size(int B, int N, long long key_cap, int Hq, int Hkv, int d);

/*
 * qwen3_qkv_proj_norm_rope - the merged q/k/v projection with QK-Norm and RoPE in the GEMM
 * epilogue.  y = x w_qkv^T ("LLM Internals - Assembling a large model from scratch": one
 * qkv_proj GEMM for the three projections), split into q [M, Hq, d], k [M, Hkv, d],
 * v [M, Hkv, d]; q and k get QK-Norm (fp32 statistics of the fp32 accumulator) and RoPE at
 * pos, then one bf16 rounding; v is stored as projected.
 *   x         [M, hidden] bf16 token hidden states (hidden a multiple of 8).
 *   w_qkv     [(Hq + 2 Hkv) d, hidden] bf16: q's Hq*d rows, then k's, then v's (the layout of
 *             a PyTorch Linear weight, out x in).
 *   pos       [M] int32 positions.
 *   q_out, k_out, v_out  [M, Hq, d], [M, Hkv, d], [M, Hkv, d] bf16.
 *   variant   the rope type (theta or a frequency table, attention_scaling); window unused.
 *   workspace at least qwen3_qkv_proj_workspace_size(M) bytes (the RoPE table of the
 *             tokens), else QWEN3_ERR_WORKSPACE.
 * q_out and k_out are the normed, rotated vectors the attention entry points compute
 * themselves from raw q and k.
 * All pointers are device pointers the caller owns: x, w_qkv and the outputs 16-byte
 * aligned, the gains 8-byte, pos 4-byte.  The call is asynchronous on `stream` (two
 * launches: the RoPE table, then the GEMM, on one SM per tile or, for long K runs, on SM
 * pairs; see qwen3_attn_set_sm_pairs).  Errors: QWEN3_ERR_INVALID_ARG for a null pointer,
 * a non-positive size, a misaligned pointer, eps < 0 or an invalid variant;
 * QWEN3_ERR_UNSUPPORTED for d != 128, hidden not a multiple of 8 or sizes past the 32-bit
 * index range; QWEN3_ERR_WORKSPACE as above; QWEN3_ERR_CUDA when a launch fails.
 */
int qwen3_qkv_proj_norm_rope(const qwen3_bf16* x, const qwen3_bf16* w_qkv,
                             const float* q_norm_w, const float* k_norm_w, const int32_t* pos,
                             qwen3_bf16* q_out, qwen3_bf16* k_out, qwen3_bf16* v_out,
                             int M, int hidden, int Hq, int Hkv, int d,
                             const qwen3_attn_variant* variant, float eps,
                             void* workspace, size_t ws_bytes, qwen3_stream_t stream);

/* Scratch bytes qwen3_qkv_proj_norm_rope needs: ceil(M/128) * 64 KB; 0 when M <= 0. */
size_t qwen3_qkv_proj_workspace_size(int M);

/* Scratch bytes qwen3_attn_prefill_ex and qwen3_attn_prefill_chunk need: B*T*Hkv*d*2
 * (normed, rotated keys) + B*T*Hq*d*2 (normed, rotated queries), plus alignment slack;
 * 0 when a size is not positive. */
size_t qwen3_attn_prefill_workspace_size(int B, int T, int Hq, int Hkv, int d);

/*
 * qwen3_attn_prefill_chunk_workspace_size - workspace bytes of a chunked prefill (or a
 * prefill_variant with caches) of T new tokens over `start` cached ones that let it split
 * the key axis when its work items are few: qwen3_attn_prefill_workspace_size plus the
 * split partials (fp32 O/l and LSEs of every new row and query head, for each run of
 * keys).  Equal to qwen3_attn_prefill_workspace_size when the shapes give no split.
 * 0 for invalid sizes.
 */
size_t qwen3_attn_prefill_chunk_workspace_size(int B, int start, int T, int Hq, int Hkv, int d);

/* Scratch bytes qwen3_attn_decode needs (split-KV partial outputs and logsumexps). */
size_t qwen3_attn_decode_workspace_size(int N, int Hq, int d, int Lmax);

/* Bytes of one layer's bf16 KV cache [2][N][Hkv][Lmax][d]: 2*Hkv*d values per token
 * ("Qwen 3 From Scratch", Worked example: 1024 values per token for Hkv=4, d=128). */
size_t qwen3_attn_kv_cache_bytes(int N, int Hkv, int Lmax, int d);

/* Static description of a status code (never NULL). */
const char* qwen3_attn_status_string(int status);

/*
 * qwen3_attn_device_status - synchronise `stream`, then return and optionally clear the
 * device-side status word of the current device (QWEN3_OK if no kernel recorded an
 * error).  When `site` is not NULL it receives a code naming the wait or check that fired.
 */
int qwen3_attn_device_status(qwen3_stream_t stream, int clear, int* site);

/*
 * qwen3_attn_set_wait_limit - bound, in nanoseconds, on every device-side wait of later
 * launches (default 2e9).  Returns the previous value.
 */
uint64_t qwen3_attn_set_wait_limit(uint64_t ns);

/*
 * qwen3_attn_set_fault_injection - test hook.  While flags == 1, every prefill launch's K/V
 * producer skips its first key-tile load, so the consumers' bounded waits run out and the
 * launch ends early, leaving QWEN3_ERR_DEVICE_TIMEOUT in the status word (outputs are not
 * written).  0 turns it off.  No memory outside the call's own buffers is touched.
 */
void qwen3_attn_set_fault_injection(int flags);

/*
 * qwen3_attn_set_softmax_path - test hook choosing the prefill softmax of later launches
 * (every prefill, chunk, paged and varlen call).  Both paths compute the same softmax
 * ("Assembling a large model from scratch", Attention.forward: fp32 softmax over the masked
 * scores; the online logsumexp of "Qwen3 Architecture Layer-by-Layer", Liger fused linear
 * cross-entropy); they differ in the reference exponent only.
 *   QWEN3_SOFTMAX_AUTO (0, the default): a launch whose gains bound every logit
 *       (sqrt(d) * max|g_q| * max|g_k| * attention_scaling^2 * log2(e) <= 60) uses that
 *       bound as a fixed reference; larger gains take the running-max path.
 *   QWEN3_SOFTMAX_RUNNING_MAX (1): every launch takes the running-max path (a row max per
 *       key tile, lazy rescale of the accumulator), whatever the gains.
 * Returns the previous setting, or -1 (nothing changed) for any other value.
 */
#define QWEN3_SOFTMAX_AUTO 0
#define QWEN3_SOFTMAX_RUNNING_MAX 1
int qwen3_attn_set_softmax_path(int path);

/*
 * qwen3_attn_set_sm_pairs - test hook choosing how later qkv projections
 * (qwen3_qkv_proj_norm_rope) use the SMs.  The projection has a variant in which the two
 * SMs of a pair share every tensor-core MMA (tcgen05 with cta_group::2, a cluster of two
 * CTAs, each loading its own token rows and half of the tile's weight rows).  It computes
 * the same results as the one-SM kernel, in the same precision.
 *   QWEN3_SM_PAIRS_AUTO (0, the default): SM pairs when each pair's run of tiles reaches
 *       128 K chunks of 64 (hidden >= 2048 at 4096 tokens), one SM per tile otherwise.
 *   QWEN3_SM_PAIRS_OFF (1): one SM per tile.
 *   QWEN3_SM_PAIRS_ALWAYS (2): SM pairs whatever the size.
 * Returns the previous setting, or -1 (nothing changed) for any other value.
 */
#define QWEN3_SM_PAIRS_AUTO 0
#define QWEN3_SM_PAIRS_OFF 1
#define QWEN3_SM_PAIRS_ALWAYS 2
int qwen3_attn_set_sm_pairs(int mode);

/* Library version string. */
const char* qwen3_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QWEN3_ATTN_H_ */
