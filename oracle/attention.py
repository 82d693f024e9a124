"""fp64 CPU oracle for the Qwen3 attention core (QK-Norm, RoPE, causal GQA).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the CUDA
library: it is a plain restatement of the definitions on the pages, in numpy
float64, with one matrix product per block of query rows as the only library
step.

What it computes, and where each step is defined:

  1. QK-Norm, per head vector x of length d:
        y = g * x / sqrt(mean(x^2) + eps)
     "Qwen3 Architecture Layer-by-Layer", Primitives: Qwen3RMSNorm;
     "Hand-Writing a Vision-Language Model, Part 1", RMSNorm (the formula is
     stated there in words: no mean subtraction, eps inside the root);
     "Qwen 3 From Scratch", In code.  It runs after the projection and before
     RoPE ("Hand-Writing ... Part 1", step list 3-5).
  2. RoPE, rotate-half pairing, for i < d/2:
        inv_i = theta^(-2i/d),  a = pos * inv_i
        y_i       = x_i cos a - x_{i+d/2} sin a
        y_{i+d/2} = x_{i+d/2} cos a + x_i sin a
     "Hand-Writing ... Part 1", RotaryEmbedding (RoPE); "Assembling a large
     model from scratch", The complete code (rope_cos_sin, rotate_half,
     apply_rope); "Qwen3 Architecture Layer-by-Layer", apply_rotary_pos_emb and
     Qwen3RotaryEmbedding (inv_freq formula).  Angles are exact fp64 here.
  3. Scores s_ij = q'_i . k'_j / sqrt(d); query head h reads KV head h // G,
     G = Hq / Hkv ("Hand-Writing ... Part 1", repeat_kv; "Assembling a large
     model", Attention.forward with repeat_interleave).
  4. Causal mask on index: key j is visible to query i iff j <= i + (S - T),
     i.e. tril(diagonal = S - T) ("Assembling a large model", Attention.forward
     and the implementation notes below the code).
  5. Softmax over visible keys, out_i = sum_j p_ij v_j; lse_i = natural log of
     sum_j exp(s_ij) (the logsumexp of "Qwen3 Architecture Layer-by-Layer",
     The cross-entropy math, applied to the scaled logits).
  6. Decode: the new token sits at position L = cached length; its k is
     normalised, rotated at L and appended, its v appended raw, and the query
     attends to all L+1 keys ("Assembling a large model", KVCache.update and
     Transformer.forward, start = cache.length).

  7. Variants ("Qwen3 Architecture Layer-by-Layer", Per-layer attention type
     and Qwen3RotaryEmbedding; "Qwen 3 From Scratch", long context with rotary
     scaling): a sliding-window layer lets query i see only the last W keys,
     i - W < j <= i; another rope type brings its own inv_freq and an
     attention_scaling that multiplies cos and sin.
  8. Varlen batches: several sequences packed on one token axis with offsets
     cu_seqlens, each an independent (chunked) causal prefill ("Assembling a large
     model", the comparison with inference engines and the review question on
     vLLM: flattened tokens plus batching metadata, attention per request).

Readings where the pages leave a step open:
  * No intermediate rounding: the pages' HF path casts to bf16 between the
    norm and the gain; the oracle keeps everything in fp64.  `staged=True`
    rounds q' and k' to bf16 once after RoPE, which is where the GPU path
    rounds them before its bf16 MMAs; it is used only for the logsumexp bound.
    That rounding decides a discrete code, so it is taken from the value held
    in float32 (the precision in which the kernels, like the pages' RMSNorm
    with its x.float(), hold q' and k' before the cast): fp64 -> fp32 -> bf16.
  * Rotate-half with theta from the argument (the page prose that speaks of
    adjacent pairs and base 10000 contradicts every code block on the pages).
  * The sliding window counts the query's own key: W keys, i - W < j <= i (the
    pages name the windowed mask but print no formula; this is the usual
    reading of a window of W tokens).  YaRN's frequency formula is not on the
    pages, so the variant takes any inv_freq table as an input.
"""
from __future__ import annotations

import numpy as np


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), as float64.

    bfloat16 keeps 8 significant bits.  With x = m * 2^e, 0.5 <= |m| < 1, the
    representable neighbours are multiples of 2^(e-8); rint rounds half to even.
    Normal-range values only (the inputs here never approach under/overflow).
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """QK-Norm over the last axis: g * x / sqrt(mean(x^2) + eps)."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return np.asarray(g, dtype=np.float64) * (x / np.sqrt(ms + eps))


def rope_inv_freq(d: int, theta: float) -> np.ndarray:
    """inv_i = theta^(-2i/d) for i = 0 .. d/2-1."""
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * i / d)


def rope(x: np.ndarray, pos: np.ndarray, theta: float, inv_freq=None, scaling: float = 1.0) -> np.ndarray:
    """Rotate-half RoPE.  x [..., T, H, d]; pos broadcastable to [..., T].

    inv_freq: optional d/2 rotary frequencies (any rope type's initialisation) in place of
    theta^(-2i/d); scaling: the attention_scaling that multiplies cos and sin
    ("Qwen3 Architecture Layer-by-Layer", Qwen3RotaryEmbedding; 1 for the default type)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    inv = rope_inv_freq(d, theta) if inv_freq is None else np.asarray(inv_freq, dtype=np.float64)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv  # [..., T, d/2]
    c = (np.cos(ang) * scaling)[..., None, :]  # broadcast over heads
    s = (np.sin(ang) * scaling)[..., None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def qk_prologue(x: np.ndarray, g: np.ndarray, pos: np.ndarray, theta: float, eps: float,
                staged: bool = False, inv_freq=None, scaling: float = 1.0) -> np.ndarray:
    """QK-Norm then RoPE of raw head vectors x [..., T, H, d] at positions pos [..., T].

    staged=True returns the bf16 value the result rounds to when held in float32."""
    y = rope(rms_norm(x, g, eps), pos, theta, inv_freq, scaling)
    return bf16_round(y.astype(np.float32).astype(np.float64)) if staged else y


def _attend(qg: np.ndarray, kk: np.ndarray, vv: np.ndarray, limit: np.ndarray, window: int = 0):
    """Softmax attention of query rows over keys 0..limit[r] (inclusive); with a sliding
    window W > 0 only keys limit[r]-W < j <= limit[r] (the last W, the query's own key
    included: the sliding-window causal mask of "Qwen3 Architecture Layer-by-Layer",
    Per-layer attention type).

    qg [R, d] already-normed/rotated queries; kk, vv [S, d]; limit [R] int.
    Returns out [R, d] and lse [R] (natural log, scaled logits).
    """
    d = qg.shape[-1]
    s = (qg @ kk.T) / np.sqrt(np.float64(d))  # [R, S]
    j = np.arange(kk.shape[0])
    visible = j[None, :] <= limit[:, None]
    if window > 0:
        visible &= j[None, :] > limit[:, None] - window
    s = np.where(visible, s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    z = np.sum(e, axis=1, keepdims=True)
    out = (e / z) @ vv
    lse = (m + np.log(z))[:, 0]
    return out, lse


def prefill_ref(q, k, v, q_norm_w, k_norm_w, pos, theta: float, eps: float,
                rows=None, staged: bool = False, block: int = 256, window: int = 0, inv_freq=None,
                scaling: float = 1.0):
    """Causal GQA prefill with the QK-Norm + RoPE prologue, in fp64.

    q [B,T,Hq,d], k and v [B,T,Hkv,d], gains [d], pos [B,T] (any real arrays;
    they are widened exactly to float64).  Returns out [B,T,Hq,d] and lse
    [B,Hq,T].  With `rows` (a sorted int array of query indices) only those
    rows are computed and the returned arrays are [B,len(rows),Hq,d] and
    [B,Hq,len(rows)]; keys still run over every position the mask admits.
    Query rows are processed in blocks so no T x T matrix is ever held.  window, inv_freq
    and scaling select the variants (a sliding window; another rope type's frequencies and
    attention_scaling); the defaults are Qwen3's full causal attention and default RoPE.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((B, rows.size, Hq, d))
    lse = np.zeros((B, Hq, rows.size))
    for b in range(B):
        kp = qk_prologue(k[b], k_norm_w, pos[b], theta, eps, staged, inv_freq, scaling)  # [T, Hkv, d]
        qp = qk_prologue(q[b, rows], q_norm_w, np.asarray(pos[b])[rows], theta, eps, staged, inv_freq, scaling)
        for h in range(Hq):
            hk = h // G
            for r0 in range(0, rows.size, block):
                rr = rows[r0:r0 + block]
                top = int(rr.max()) + 1
                o, l = _attend(qp[r0:r0 + block, h], kp[:top, hk], v[b, :top, hk], rr, window)
                out[b, r0:r0 + block, h] = o
                lse[b, h, r0:r0 + block] = l
    return out, lse


def chunk_prefill_ref(q, k, v, q_norm_w, k_norm_w, pos, k_cache, v_cache, start: int,
                      theta: float, eps: float, rows=None, staged: bool = False, block: int = 256,
                      window: int = 0, inv_freq=None, scaling: float = 1.0):
    """T new tokens per batch row over a cache that already holds `start` tokens, in fp64.

    "Assembling a large model from scratch", Attention.forward and the notes below
    the code: the new q and k get QK-Norm and RoPE at their positions, the new k and
    v are appended after the cached ones (S = start + T keys), and new row i sees key
    j iff j <= i + (S - T) = i + start, the mask tril(diagonal = S - T).

    q [B,T,Hq,d], k and v [B,T,Hkv,d] raw new tokens at positions pos [B,T];
    k_cache and v_cache indexable as [b][Hkv, >=start, d]: cached keys as stored
    (already normed and rotated), cached values raw.  Returns out [B,len(rows),Hq,d]
    and lse [B,Hq,len(rows)] for the new rows in `rows` (default: all T).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((B, rows.size, Hq, d))
    lse = np.zeros((B, Hq, rows.size))
    for b in range(B):
        kp = qk_prologue(k[b], k_norm_w, pos[b], theta, eps, staged, inv_freq, scaling)  # [T, Hkv, d]
        qp = qk_prologue(q[b, rows], q_norm_w, np.asarray(pos[b])[rows], theta, eps, staged, inv_freq, scaling)
        kc = np.asarray(k_cache[b], dtype=np.float64)[:, :start]     # [Hkv, start, d]
        vc = np.asarray(v_cache[b], dtype=np.float64)[:, :start]
        for h in range(Hq):
            hk = h // G
            keys = np.concatenate([kc[hk], kp[:, hk]], axis=0)          # [start + T, d]
            vals = np.concatenate([vc[hk], v[b, :, hk]], axis=0)
            for r0 in range(0, rows.size, block):
                rr = rows[r0:r0 + block]
                top = start + int(rr.max()) + 1
                o, l = _attend(qp[r0:r0 + block, h], keys[:top], vals[:top], rr + start, window)
                out[b, r0:r0 + block, h] = o
                lse[b, h, r0:r0 + block] = l
    return out, lse


def varlen_prefill_ref(q, k, v, q_norm_w, k_norm_w, pos, cu_seqlens, theta: float, eps: float,
                       k_prefix=None, v_prefix=None, staged: bool = False, window: int = 0, inv_freq=None,
                       scaling: float = 1.0):
    """Prefill of several sequences packed on one token axis, in fp64.

    The batching of serving engines ("Assembling a large model from scratch", the
    comparison with inference engines: the tokens of many requests form one batch and
    attention is computed per request; and the review question on vLLM: one forward pass
    over a variable-length batch, flattened tokens plus batching metadata): q [N,Hq,d], k
    and v [N,Hkv,d] and pos [N] hold the tokens of all sequences back to back, and sequence
    b owns tokens cu_seqlens[b] .. cu_seqlens[b+1]-1.
    Each sequence is an independent causal prefill: its tokens see only keys of their own
    sequence.  With k_prefix and v_prefix (per sequence [Hkv, ctx_b, d]: cached keys as
    stored, values raw) sequence b's new tokens follow its ctx_b cached ones, as in the
    chunked prefill; without them every sequence is a fresh prompt.

    Returns out [N,Hq,d] and lse [Hq,N]; rows of tokens that belong to no sequence are NaN.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    pos = np.asarray(pos)
    out = np.full((N, Hq, d), np.nan)
    lse = np.full((Hq, N), np.nan)
    for b in range(cu.size - 1):
        lo, hi = int(cu[b]), int(cu[b + 1])
        if hi == lo:
            continue
        if k_prefix is None:
            kc = np.zeros((1, Hkv, 0, d))
            vc = np.zeros((1, Hkv, 0, d))
        else:
            kc = np.asarray(k_prefix[b], dtype=np.float64)[None]
            vc = np.asarray(v_prefix[b], dtype=np.float64)[None]
        o, l = chunk_prefill_ref(q[None, lo:hi], k[None, lo:hi], v[None, lo:hi], q_norm_w, k_norm_w,
                                 pos[None, lo:hi], kc, vc, kc.shape[2], theta, eps, staged=staged, window=window,
                                 inv_freq=inv_freq, scaling=scaling)
        out[lo:hi] = o[0]
        lse[:, lo:hi] = l[0]
    return out, lse


def build_cache_k(k_hist, k_norm_w, theta: float, eps: float, inv_freq=None, scaling: float = 1.0) -> np.ndarray:
    """Cache contents for a raw key history k_hist [L,Hkv,d]: QK-Norm and RoPE at
    positions 0..L-1, rounded to bf16 (the cache's storage type), as float64."""
    L = np.asarray(k_hist).shape[0]
    return bf16_round(qk_prologue(k_hist, k_norm_w, np.arange(L), theta, eps, inv_freq=inv_freq, scaling=scaling))


def decode_ref(q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache, cache_lens,
               theta: float, eps: float, seqs=None, staged: bool = False, window: int = 0, inv_freq=None,
               scaling: float = 1.0):
    """One decode step over a KV cache, in fp64.

    q [N,Hq,d], k_new and v_new [N,Hkv,d] raw; k_cache/v_cache indexable as
    [n][Hkv, >=L_n, d] holding the already-normed/rotated keys and raw values;
    cache_lens [N].  The new token sits at position L_n.  Returns out [n_sel,Hq,d]
    and lse [n_sel,Hq] for the sequences in `seqs` (default: all).
    """
    q = np.asarray(q, dtype=np.float64)
    N, Hq, d = q.shape
    Hkv = np.asarray(k_new).shape[1]
    G = Hq // Hkv
    seqs = range(N) if seqs is None else seqs
    outs, lses = [], []
    for n in seqs:
        L = int(cache_lens[n])
        qp = qk_prologue(q[n][None], q_norm_w, np.array([L]), theta, eps, staged, inv_freq, scaling)[0]  # [Hq, d]
        kn = qk_prologue(np.asarray(k_new[n], dtype=np.float64)[None], k_norm_w, np.array([L]),
                         theta, eps, staged, inv_freq, scaling)[0]                                    # [Hkv, d]
        kc = np.asarray(k_cache[n], dtype=np.float64)
        vc = np.asarray(v_cache[n], dtype=np.float64)
        o = np.zeros((Hq, d))
        ls = np.zeros(Hq)
        for h in range(Hq):
            hk = h // G
            keys = np.concatenate([kc[hk, :L], kn[hk][None]], axis=0)
            vals = np.concatenate([vc[hk, :L], np.asarray(v_new[n], dtype=np.float64)[hk][None]], axis=0)
            oo, ll = _attend(qp[h][None], keys, vals, np.array([L]), window)
            o[h], ls[h] = oo[0], ll[0]
        outs.append(o)
        lses.append(ls)
    return np.stack(outs), np.stack(lses)


def qkv_proj_norm_rope_ref(x, w_qkv, q_norm_w, k_norm_w, pos, Hq: int, Hkv: int, theta: float, eps: float,
                           staged: bool = False, inv_freq=None, scaling: float = 1.0):
    """The merged qkv projection followed by QK-Norm and RoPE, in fp64.

    x [M, hidden] token hidden states; w_qkv [(Hq + 2 Hkv) d, hidden], the q, k and v
    projection weights stacked in that order (one GEMM for the three: "Assembling a large
    model from scratch", the comparison with inference engines, qkv_proj); pos [M].
    y = x w_qkv^T splits into q [M, Hq, d], k [M, Hkv, d], v [M, Hkv, d]; q and k get
    QK-Norm then RoPE at pos ("Hand-Writing ... Part 1", order of operations), v is
    returned as projected.  Returns (q', k', v).
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_qkv, dtype=np.float64)
    d = w.shape[0] // (Hq + 2 * Hkv)
    y = x @ w.T
    M = x.shape[0]
    q = y[:, :Hq * d].reshape(M, Hq, d)
    k = y[:, Hq * d:(Hq + Hkv) * d].reshape(M, Hkv, d)
    v = y[:, (Hq + Hkv) * d:].reshape(M, Hkv, d)
    pos = np.asarray(pos)
    qp = qk_prologue(q, q_norm_w, pos, theta, eps, staged, inv_freq, scaling)
    kp = qk_prologue(k, k_norm_w, pos, theta, eps, staged, inv_freq, scaling)
    return qp, kp, v


def paged_gather(pages, block_table_row, n: int, page_size: int) -> np.ndarray:
    """The first n keys of one sequence out of a paged pool, as [Hkv, n, d].

    pages [num_pages, Hkv, page_size, d]; key j lives in page block_table_row[j // page_size]
    at offset j % page_size (the block-table layout of paged KV caches, which "Assembling a
    large model from scratch" names as what real systems use instead of concatenation)."""
    pages = np.asarray(pages)
    out = np.empty((pages.shape[1], n, pages.shape[3]), dtype=np.float64)
    for j in range(n):
        out[:, j] = pages[int(block_table_row[j // page_size]), :, j % page_size]
    return out


def kv_cache_values_per_token(Hkv: int, d: int) -> int:
    """Values one layer's cache holds per token: a key and a value per KV head
    ("Qwen 3 From Scratch", Worked example: 2 x Hkv x d_head)."""
    return 2 * Hkv * d
