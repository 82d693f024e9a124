"""Plant plausible mistakes in the oracle (on the CPU) and confirm the pins catch
each one: a wrong RoPE sign, adjacent-pair RoPE, RoPE frequencies theta^(-i/d), RoPE
before QK-Norm, a missing eps, eps outside the square root, mean-centering, bf16 ties
rounded away from zero, a KV cache kept unrounded, h mod Hkv head mapping, an off-by-one
causal mask, a missing 1/sqrt(d) scale, a base-2 logsumexp, in decode the new token
rotated one position late or its value never appended, a paged gather that ignores the
block table, in the chunked prefill a mask without the cached-prefix offset or cached
keys rotated a second time, in the variants a sliding window one key too wide,
attention_scaling applied to cos only and a caller's inv_freq ignored, in the varlen
batch one causal mask over the whole packed token axis or the cached prefixes dropped,
and in the merged projection the k and v blocks swapped."""
import numpy as np
import pytest

import oracle.attention as A
from tests import oracle_checks as C


def _inv(x, theta, inv_freq):
    return A.rope_inv_freq(x.shape[-1], theta) if inv_freq is None else np.asarray(inv_freq, dtype=np.float64)


def _rope_wrong_sign(x, pos, theta, inv_freq=None, scaling=1.0):
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * _inv(x, theta, inv_freq)
    c, s = scaling * np.cos(ang)[..., None, :], scaling * np.sin(ang)[..., None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)


def _rope_adjacent_pairs(x, pos, theta, inv_freq=None, scaling=1.0):
    x = np.asarray(x, dtype=np.float64)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * _inv(x, theta, inv_freq)
    c, s = scaling * np.cos(ang)[..., None, :], scaling * np.sin(ang)[..., None, :]
    xe, xo = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = xe * c - xo * s
    y[..., 1::2] = xo * c + xe * s
    return y


def _norm_no_eps(x, g, eps):
    x = np.asarray(x, dtype=np.float64)
    return g * x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True))


def _norm_centered(x, g, eps):
    x = np.asarray(x, dtype=np.float64)
    x = x - x.mean(axis=-1, keepdims=True)
    return g * x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def _attend_off_by_one(qg, kk, vv, limit, window=0):
    return _ORIG_ATTEND(qg, kk, vv, limit - 1 + (limit == 0), window)


def _attend_no_scale(qg, kk, vv, limit, window=0):
    return _ORIG_ATTEND(qg * np.sqrt(qg.shape[-1]), kk, vv, limit, window)


def _attend_log2(qg, kk, vv, limit, window=0):
    o, l = _ORIG_ATTEND(qg, kk, vv, limit, window)
    return o, l / np.log(2.0)


def _attend_window_one_wider(qg, kk, vv, limit, window=0):
    # the window lets in one key too many (i - W <= j instead of i - W < j)
    return _ORIG_ATTEND(qg, kk, vv, limit, window + 1 if window > 0 else 0)


def _rope_scaling_on_cos_only(x, pos, theta, inv_freq=None, scaling=1.0):
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * _inv(x, theta, inv_freq)
    c, s = scaling * np.cos(ang)[..., None, :], np.sin(ang)[..., None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def _rope_ignores_inv_freq(x, pos, theta, inv_freq=None, scaling=1.0):
    return _ORIG_ROPE(x, pos, theta, None, scaling)


def _qkv_swapped_kv(x, w_qkv, gq, gk, pos, Hq, Hkv, theta, eps, **kw):
    # the k and v blocks of the merged weight taken in the wrong order
    w = np.asarray(w_qkv, dtype=np.float64)
    d = w.shape[0] // (Hq + 2 * Hkv)
    w2 = np.concatenate([w[:Hq * d], w[(Hq + Hkv) * d:], w[Hq * d:(Hq + Hkv) * d]], axis=0)
    return _ORIG_QKV(x, w2, gq, gk, pos, Hq, Hkv, theta, eps, **kw)


_ORIG_ATTEND = A._attend
_ORIG_ROPE = A.rope
_ORIG_QKV = A.qkv_proj_norm_rope_ref


def _prefill_mod_mapping(q, k, v, gq, gk, pos, theta, eps, rows=None, staged=False, block=256, **kw):
    # h -> h % Hkv instead of h // G: permute the query heads so the oracle's
    # h // G lookup lands on h % Hkv, then undo the permutation on the output.
    q = np.asarray(q, dtype=np.float64)
    Hq, Hkv = q.shape[2], np.asarray(k).shape[2]
    G = Hq // Hkv
    perm = np.array([(h % Hkv) * G + h // Hkv for h in range(Hq)])
    qq = np.empty_like(q)
    qq[:, :, perm] = q
    o, l = _ORIG_PREFILL(qq, k, v, gq, gk, pos, theta, eps, rows=rows, staged=staged, block=block, **kw)
    return o[:, :, perm], l[:, perm]


_ORIG_CHUNK = A.chunk_prefill_ref


def _chunk_no_offset(q, k, v, gq, gk, pos, k_cache, v_cache, start, theta, eps, rows=None, staged=False, block=256,
                     window=0, inv_freq=None, scaling=1.0):
    # the mask forgets the cached prefix: new row i sees keys 0..i of the concatenation
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, T, Hq, d = q.shape
    G = Hq // k.shape[2]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    out, lse = np.zeros((B, rows.size, Hq, d)), np.zeros((B, Hq, rows.size))
    for b in range(B):
        kp = A.qk_prologue(k[b], gk, pos[b], theta, eps, staged, inv_freq, scaling)
        qp = A.qk_prologue(q[b, rows], gq, np.asarray(pos[b])[rows], theta, eps, staged, inv_freq, scaling)
        for h in range(Hq):
            keys = np.concatenate([np.asarray(k_cache[b])[h // G, :start], kp[:, h // G]])
            vals = np.concatenate([np.asarray(v_cache[b])[h // G, :start], v[b, :, h // G]])
            o, l = A._attend(qp[:, h], keys, vals, rows, window)
            out[b, :, h], lse[b, h] = o, l
    return out, lse


def _chunk_rerotates_cache(q, k, v, gq, gk, pos, k_cache, v_cache, start, theta, eps, **kw):
    # the cached keys get RoPE a second time at their positions 0..start-1
    kc = np.stack([A.rope(np.asarray(k_cache[b])[:, :start].transpose(1, 0, 2), np.arange(start), theta)
                   .transpose(1, 0, 2) for b in range(len(k_cache))])
    return _ORIG_CHUNK(q, k, v, gq, gk, pos, kc, v_cache, start, theta, eps, **kw)


_ORIG_VARLEN = A.varlen_prefill_ref


def _varlen_one_causal_axis(q, k, v, gq, gk, pos, cu_seqlens, theta, eps, k_prefix=None, v_prefix=None, **kw):
    # attention runs causally over the whole packed axis: a token also sees the tokens of
    # the sequences packed before it
    cu = np.asarray(cu_seqlens)
    whole = np.array([cu[0], cu[-1]])
    return _ORIG_VARLEN(q, k, v, gq, gk, pos, whole, theta, eps,
                        k_prefix=None if k_prefix is None else k_prefix[:1],
                        v_prefix=None if v_prefix is None else v_prefix[:1], **kw)


_ORIG_PREFILL = A.prefill_ref

def _inv_freq_half_exponent(d, theta):
    # theta^(-i/d) instead of theta^(-2i/d)
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(np.float64(theta), -i / d)


def _norm_eps_outside_root(x, g, eps):
    x = np.asarray(x, dtype=np.float64)
    return g * x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps)


def _prologue_rope_before_norm(x, g, pos, theta, eps, staged=False, inv_freq=None, scaling=1.0):
    # RoPE first, then QK-Norm: the per-channel gain lands on rotated channels
    y = A.rms_norm(A.rope(x, pos, theta, inv_freq, scaling), g, eps) * scaling
    return A.bf16_round(y.astype(np.float32).astype(np.float64)) if staged else y


def _bf16_ties_away(x):
    # round to nearest with ties away from zero instead of ties to even
    x = np.asarray(x, dtype=np.float64).astype(np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = ((b + 0x8000) & 0xFFFF0000).astype(np.uint32)
    return b.view(np.float32).astype(np.float64)


def _cache_not_rounded(k_hist, k_norm_w, theta, eps, inv_freq=None, scaling=1.0):
    # the cache keeps the fp64 keys instead of their bf16 storage values
    L = np.asarray(k_hist).shape[0]
    return A.qk_prologue(k_hist, k_norm_w, np.arange(L), theta, eps, inv_freq=inv_freq, scaling=scaling)


def _decode_one_position_late(q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache, cache_lens, theta, eps,
                              seqs=None, staged=False, window=0, inv_freq=None, scaling=1.0):
    # the new token is rotated at L + 1 (positions counted from one) instead of at L
    q = np.asarray(q, dtype=np.float64)
    N, Hq, d = q.shape
    G = Hq // np.asarray(k_new).shape[1]
    outs, lses = [], []
    for n in (range(N) if seqs is None else seqs):
        L = int(cache_lens[n])
        qp = A.qk_prologue(q[n][None], q_norm_w, np.array([L + 1]), theta, eps, staged, inv_freq, scaling)[0]
        kn = A.qk_prologue(np.asarray(k_new[n], dtype=np.float64)[None], k_norm_w, np.array([L + 1]), theta, eps,
                           staged, inv_freq, scaling)[0]
        kc, vc = np.asarray(k_cache[n], dtype=np.float64), np.asarray(v_cache[n], dtype=np.float64)
        o, ls = np.zeros((Hq, d)), np.zeros(Hq)
        for h in range(Hq):
            keys = np.concatenate([kc[h // G, :L], kn[h // G][None]], axis=0)
            vals = np.concatenate([vc[h // G, :L], np.asarray(v_new[n], dtype=np.float64)[h // G][None]], axis=0)
            oo, ll = A._attend(qp[h][None], keys, vals, np.array([L]), window)
            o[h], ls[h] = oo[0], ll[0]
        outs.append(o)
        lses.append(ls)
    return np.stack(outs), np.stack(lses)


def _decode_drops_new_value(q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache, cache_lens, theta, eps, **kw):
    # the new token's value is never appended: its slot reads as zeros
    return _ORIG_DECODE(q, k_new, np.zeros_like(np.asarray(v_new, dtype=np.float64)), q_norm_w, k_norm_w, k_cache,
                        v_cache, cache_lens, theta, eps, **kw)


def _paged_gather_ignores_table(pages, block_table_row, n, page_size):
    # block index taken as the page index, as if the table were the identity
    return _ORIG_GATHER(pages, list(range(len(block_table_row))), n, page_size)


def _varlen_drops_prefixes(q, k, v, gq, gk, pos, cu_seqlens, theta, eps, k_prefix=None, v_prefix=None, **kw):
    # the cached prefixes are ignored: every sequence attends to its new tokens only
    return _ORIG_VARLEN(q, k, v, gq, gk, pos, cu_seqlens, theta, eps, **kw)


_ORIG_DECODE = A.decode_ref
_ORIG_GATHER = A.paged_gather


MUTANTS = [
    ("rope", _rope_wrong_sign),
    ("rope", _rope_adjacent_pairs),
    ("rms_norm", _norm_no_eps),
    ("rms_norm", _norm_centered),
    ("_attend", _attend_off_by_one),
    ("_attend", _attend_no_scale),
    ("_attend", _attend_log2),
    ("_attend", _attend_window_one_wider),
    ("rope", _rope_scaling_on_cos_only),
    ("rope", _rope_ignores_inv_freq),
    ("qkv_proj_norm_rope_ref", _qkv_swapped_kv),
    ("prefill_ref", _prefill_mod_mapping),
    ("chunk_prefill_ref", _chunk_no_offset),
    ("chunk_prefill_ref", _chunk_rerotates_cache),
    ("varlen_prefill_ref", _varlen_one_causal_axis),
    ("rope_inv_freq", _inv_freq_half_exponent),
    ("rms_norm", _norm_eps_outside_root),
    ("qk_prologue", _prologue_rope_before_norm),
    ("bf16_round", _bf16_ties_away),
    ("build_cache_k", _cache_not_rounded),
    ("decode_ref", _decode_one_position_late),
    ("decode_ref", _decode_drops_new_value),
    ("paged_gather", _paged_gather_ignores_table),
    ("varlen_prefill_ref", _varlen_drops_prefixes),
]


@pytest.mark.parametrize("name,fn", MUTANTS, ids=[m[1].__name__.strip("_") for m in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, name, fn):
    monkeypatch.setattr(A, name, fn)
    failed = []
    for check in C.ALL_CHECKS:
        try:
            check()
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no pin caught the planted mistake in {name}"
