"""Brute-force scalar-loop restatement of the attention core, for tiny shapes.

TEST INFRASTRUCTURE ONLY (tests import it to pin the vectorised oracle).  Pure
Python floats (IEEE double) and the math module; no numpy arithmetic.  Every
step is written element by element in the order the pages give it:
QK-Norm ("Qwen3 Architecture Layer-by-Layer", Qwen3RMSNorm), rotate-half RoPE
("Hand-Writing a Vision-Language Model, Part 1", RotaryEmbedding), scores with
the 1/sqrt(d) scale, the tril(diagonal=S-T) mask and an fp64 softmax
("Assembling a large model from scratch", Attention.forward).
"""
from __future__ import annotations

import math


def _norm_rope(vec, gain, pos, theta, eps, inv_freq=None, scaling=1.0):
    d = len(vec)
    ms = sum(x * x for x in vec) / d
    r = 1.0 / math.sqrt(ms + eps)
    y = [gain[i] * vec[i] * r for i in range(d)]
    half = d // 2
    out = [0.0] * d
    for i in range(half):
        a = pos * (theta ** (-2.0 * i / d) if inv_freq is None else float(inv_freq[i]))
        c, s = math.cos(a) * scaling, math.sin(a) * scaling
        out[i] = y[i] * c - y[i + half] * s
        out[i + half] = y[i + half] * c + y[i] * s
    return out


def prefill_loops(q, k, v, gq, gk, pos, theta, eps, S_minus_T=0, window=0, inv_freq=None, scaling=1.0):
    """q[b][t][h][i], k/v[b][t][hk][i] nested lists (or arrays); returns
    out[b][t][h][i] and lse[b][h][t] as nested lists.  window > 0: query t sees only keys
    j with t - window < j <= t; inv_freq / scaling: another rope type's frequencies and
    the attention_scaling on cos and sin."""
    B, T, Hq, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0][0])
    G = Hq // Hkv
    out = [[[[0.0] * d for _ in range(Hq)] for _ in range(T)] for _ in range(B)]
    lse = [[[0.0] * T for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        kk = [[_norm_rope([float(x) for x in k[b][t][h]], gk, float(pos[b][t]), theta, eps, inv_freq, scaling)
               for h in range(Hkv)] for t in range(T)]
        for t in range(T):
            for h in range(Hq):
                qq = _norm_rope([float(x) for x in q[b][t][h]], gq, float(pos[b][t]), theta, eps, inv_freq, scaling)
                hk = h // G
                scores, seen = [], []
                for j in range(T):
                    if j <= t + S_minus_T and (window == 0 or j > t + S_minus_T - window):
                        scores.append(sum(qq[i] * kk[j][hk][i] for i in range(d)) / math.sqrt(d))
                        seen.append(j)
                m = max(scores)
                w = [math.exp(s - m) for s in scores]
                z = sum(w)
                for i in range(d):
                    out[b][t][h][i] = sum(w[n] * float(v[b][seen[n]][hk][i]) for n in range(len(w))) / z
                lse[b][h][t] = m + math.log(z)
    return out, lse


def decode_loops(q, k_new, v_new, gq, gk, k_cache, v_cache, lens, theta, eps):
    """Decode one token per sequence, element by element.  k_cache[n][hk][j][i]
    holds normed/rotated keys for j < lens[n]."""
    N, Hq, d = len(q), len(q[0]), len(q[0][0])
    Hkv = len(k_new[0])
    G = Hq // Hkv
    out = [[[0.0] * d for _ in range(Hq)] for _ in range(N)]
    lse = [[0.0] * Hq for _ in range(N)]
    for n in range(N):
        L = int(lens[n])
        kn = [_norm_rope([float(x) for x in k_new[n][hk]], gk, float(L), theta, eps) for hk in range(Hkv)]
        for h in range(Hq):
            hk = h // G
            qq = _norm_rope([float(x) for x in q[n][h]], gq, float(L), theta, eps)
            keys = [[float(x) for x in k_cache[n][hk][j]] for j in range(L)] + [kn[hk]]
            vals = [[float(x) for x in v_cache[n][hk][j]] for j in range(L)] + [[float(x) for x in v_new[n][hk]]]
            scores = [sum(qq[i] * key[i] for i in range(d)) / math.sqrt(d) for key in keys]
            m = max(scores)
            w = [math.exp(s - m) for s in scores]
            z = sum(w)
            for i in range(d):
                out[n][h][i] = sum(w[j] * vals[j][i] for j in range(len(w))) / z
            lse[n][h] = m + math.log(z)
    return out, lse


def chunk_prefill_loops(q, k, v, gq, gk, pos, k_cache, v_cache, start, theta, eps):
    """T new tokens per batch row over `start` cached ones, element by element.
    k_cache[b][hk][j][i] holds normed/rotated keys and v_cache[b][hk][j][i] raw
    values for j < start; new key t sits at index start + t and new row t sees
    keys 0..start + t."""
    B, T, Hq, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0][0])
    G = Hq // Hkv
    out = [[[[0.0] * d for _ in range(Hq)] for _ in range(T)] for _ in range(B)]
    lse = [[[0.0] * T for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            keys = [[float(x) for x in k_cache[b][hk][j]] for j in range(start)]
            vals = [[float(x) for x in v_cache[b][hk][j]] for j in range(start)]
            for t in range(T):
                keys.append(_norm_rope([float(x) for x in k[b][t][hk]], gk, float(pos[b][t]), theta, eps))
                vals.append([float(x) for x in v[b][t][hk]])
            for t in range(T):
                qq = _norm_rope([float(x) for x in q[b][t][h]], gq, float(pos[b][t]), theta, eps)
                scores = [sum(qq[i] * keys[j][i] for i in range(d)) / math.sqrt(d) for j in range(start + t + 1)]
                m = max(scores)
                w = [math.exp(s - m) for s in scores]
                z = sum(w)
                for i in range(d):
                    out[b][t][h][i] = sum(w[j] * vals[j][i] for j in range(len(w))) / z
                lse[b][h][t] = m + math.log(z)
    return out, lse


def varlen_prefill_loops(q, k, v, gq, gk, pos, cu_seqlens, theta, eps, k_prefix=None, v_prefix=None):
    """Packed sequences, token by token.  Token n belongs to the sequence b with
    cu_seqlens[b] <= n < cu_seqlens[b+1]; its keys are that sequence's ctx_b cached keys
    (k_prefix[b][hk][j], already normed and rotated; values v_prefix[b][hk][j] raw) followed
    by the sequence's own new tokens up to n.  Tokens in no sequence get None."""
    N, Hq, d = len(q), len(q[0]), len(q[0][0])
    Hkv = len(k[0])
    G = Hq // Hkv
    out = [None] * N
    lse = [[None] * N for _ in range(Hq)]
    for n in range(N):
        owner = [b for b in range(len(cu_seqlens) - 1) if cu_seqlens[b] <= n < cu_seqlens[b + 1]]
        if not owner:
            continue
        b = owner[0]
        first = int(cu_seqlens[b])
        ctx = 0 if k_prefix is None else len(k_prefix[b][0])
        row = [[0.0] * d for _ in range(Hq)]
        for h in range(Hq):
            hk = h // G
            keys = [[float(x) for x in k_prefix[b][hk][j]] for j in range(ctx)]
            vals = [[float(x) for x in v_prefix[b][hk][j]] for j in range(ctx)]
            for m in range(first, n + 1):
                keys.append(_norm_rope([float(x) for x in k[m][hk]], gk, float(pos[m]), theta, eps))
                vals.append([float(x) for x in v[m][hk]])
            qq = _norm_rope([float(x) for x in q[n][h]], gq, float(pos[n]), theta, eps)
            scores = [sum(qq[i] * key[i] for i in range(d)) / math.sqrt(d) for key in keys]
            mx = max(scores)
            w = [math.exp(x - mx) for x in scores]
            z = sum(w)
            for i in range(d):
                row[h][i] = sum(w[j] * vals[j][i] for j in range(len(w))) / z
            lse[h][n] = mx + math.log(z)
        out[n] = row
    return out, lse


def qkv_proj_norm_rope_loops(x, w_qkv, gq, gk, pos, Hq, Hkv, theta, eps):
    """The merged projection element by element, then QK-Norm and RoPE per head vector.
    x[m][i], w_qkv[o][i]; returns q'[m][h][i], k'[m][h][i], v[m][h][i]."""
    M, hidden = len(x), len(x[0])
    n_out = len(w_qkv)
    d = n_out // (Hq + 2 * Hkv)
    y = [[sum(float(x[m][i]) * float(w_qkv[o][i]) for i in range(hidden)) for o in range(n_out)] for m in range(M)]
    q = [[_norm_rope(y[m][h * d:(h + 1) * d], gq, float(pos[m]), theta, eps) for h in range(Hq)] for m in range(M)]
    k = [[_norm_rope(y[m][(Hq + h) * d:(Hq + h + 1) * d], gk, float(pos[m]), theta, eps) for h in range(Hkv)]
         for m in range(M)]
    v = [[y[m][(Hq + Hkv + h) * d:(Hq + Hkv + h + 1) * d] for h in range(Hkv)] for m in range(M)]
    return q, k, v
