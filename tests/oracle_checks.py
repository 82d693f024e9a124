"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each check raises AssertionError on failure.  They look the oracle's functions
up at call time (`A.<name>`), so `test_oracle_mutants.py` can plant a plausible
mistake in the oracle and confirm that some check catches it.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle.attention as A
import oracle.loops as Lp

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")
THETA, EPS, D = 1.0e6, 1.0e-6, 128


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _gain(seed, d=D):
    return 1.0 + 0.1 * np.random.default_rng(seed).standard_normal(d)


def _inputs(B, T, Hq, Hkv, seed=0, d=D):
    q = _rand((B, T, Hq, d), seed)
    k = _rand((B, T, Hkv, d), seed + 1)
    v = _rand((B, T, Hkv, d), seed + 2)
    pos = np.broadcast_to(np.arange(T), (B, T)).copy()
    return q, k, v, _gain(seed + 3, d), _gain(seed + 4, d), pos


# ---------------------------------------------------------------- bf16 rounding
def check_bf16_round_matches_torch():
    """The oracle's own bf16 rounding equals torch's float32->bfloat16 conversion
    (round to nearest even) on float32-representable values, ties included."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(50.0)
    ties = (np.arange(1, 2001, dtype=np.float32) * np.float32(2 ** -8) + np.float32(1.0)).astype(np.float32)
    x = np.concatenate([x, ties, -ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = A.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, ref), np.flatnonzero(got != ref)[:5]


# ---------------------------------------------------------------- RMSNorm
def check_rmsnorm_unit_gain_closed_form():
    """With unit gain the output RMS is sqrt(ms / (ms + eps)) exactly."""
    for seed, scale in [(0, 1.0), (1, 1e-3), (2, 30.0)]:
        x = _rand((64, D), seed, scale)
        y = A.rms_norm(x, np.ones(D), EPS)
        ms = np.mean(x * x, axis=-1)
        rms_y = np.sqrt(np.mean(y * y, axis=-1))
        assert np.allclose(rms_y, np.sqrt(ms / (ms + EPS)), rtol=1e-13, atol=0)


def check_rmsnorm_gain_and_no_centering():
    """The gain multiplies channel-wise, and there is no mean subtraction: a
    constant vector c*1 maps to sign(c) * g * |c|/sqrt(c^2+eps)."""
    g = _gain(5)
    for c in (2.0, -0.5):
        y = A.rms_norm(np.full((1, D), c), g, EPS)
        assert np.allclose(y[0], g * c / math.sqrt(c * c + EPS), rtol=1e-14)
    x = _rand((3, D), 9)
    assert np.allclose(A.rms_norm(x, g, EPS), g * A.rms_norm(x, np.ones(D), EPS), rtol=1e-14)


# ---------------------------------------------------------------- RoPE
def check_rope_inv_freq_golden():
    gold = json.load(open(GOLDEN))["rope_inv_freq"]
    inv = A.rope_inv_freq(gold["head_dim"], float(gold["rope_theta"]))
    assert inv.shape == (gold["n_frequencies"],)
    i = np.arange(gold["n_frequencies"])
    assert np.allclose(inv, 10.0 ** (gold["base10_exponent_per_i"] * i), rtol=1e-13)
    assert inv[0] == 1.0 and abs(inv[63] / 1.2409e-6 - 1) < 1e-4


def check_rope_identity_at_pos0():
    x = _rand((1, 4, 3, D), 11)
    assert np.allclose(A.rope(x, np.zeros((1, 4)), THETA), x, rtol=0, atol=0)


def check_rope_plane_rotation():
    """Unit vector e_i (i < d/2) at position p is rotated in the (i, i+d/2) plane
    by angle p*inv_i, counter-clockwise: the textbook matrix [[c,-s],[s,c]]."""
    p = 37.0
    for i in (0, 5, 31, 63):
        a = p * THETA ** (-2.0 * i / D)
        Rm = np.array([[math.cos(a), -math.sin(a)], [math.sin(a), math.cos(a)]])
        for col, unit in enumerate((i, i + D // 2)):
            x = np.zeros((1, 1, D))
            x[0, 0, unit] = 1.0
            y = A.rope(x, np.array([p]), THETA)[0, 0]
            assert abs(y[i] - Rm[0, col]) < 1e-14 and abs(y[i + D // 2] - Rm[1, col]) < 1e-14
            others = np.delete(y, [i, i + D // 2])
            assert np.all(others == 0.0)


def check_rope_preserves_norm():
    x = _rand((2, 16, 4, D), 12, 3.0)
    pos = np.random.default_rng(13).integers(0, 40000, size=(2, 16))
    y = A.rope(x, pos, THETA)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def check_rope_relative_position():
    """<R(m) q, R(n) k> depends only on m - n."""
    q = _rand((1, 1, D), 14)
    k = _rand((1, 1, D), 15)
    base = None
    for m, n in [(10, 3), (107, 100), (32767, 32760)]:
        dq = A.rope(q, np.array([m]), THETA)[0, 0]
        dk = A.rope(k, np.array([n]), THETA)[0, 0]
        val = float(dq @ dk)
        if base is None:
            base = val
        assert abs(val - base) < 1e-9 * max(1.0, abs(base))


def check_rope_relative_position_printed_pairs():
    """The pages' own example: token 5 attending to token 3 and token 50 attending to token
    48 get the same score, for every query and key vector and every frequency."""
    pairs = json.load(open(GOLDEN))["rope_relative_position"]["same_signal_pairs"]
    q = _rand((8, 1, D), 16)
    k = _rand((8, 1, D), 17)
    vals = []
    for m, n in pairs:
        dq = A.rope(q, np.full(8, m), THETA)[:, 0]
        dk = A.rope(k, np.full(8, n), THETA)[:, 0]
        vals.append(np.sum(dq * dk, axis=-1))
    assert np.allclose(vals[0], vals[1], rtol=1e-12, atol=1e-12)
    # and the signal does change with the distance (the pin would pass for a RoPE that
    # ignored positions altogether otherwise)
    m, n = pairs[0]
    far = np.sum(A.rope(q, np.full(8, m), THETA)[:, 0] * A.rope(k, np.full(8, n + 7), THETA)[:, 0], axis=-1)
    assert np.max(np.abs(far - vals[0])) > 1e-3


# ---------------------------------------------------------------- attention
def check_row0_is_v0():
    """Prefill row 0 sees only key 0: out = v_0 of KV head h//G, lse = s_00."""
    q, k, v, gq, gk, pos = _inputs(2, 9, 4, 2, seed=20)
    out, lse = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
    G = 2
    for b in range(2):
        qp = A.qk_prologue(q[b, :1], gq, pos[b, :1], THETA, EPS)[0]
        kp = A.qk_prologue(k[b, :1], gk, pos[b, :1], THETA, EPS)[0]
        for h in range(4):
            assert np.array_equal(out[b, 0, h], v[b, 0, h // G])
            assert abs(lse[b, h, 0] - qp[h] @ kp[h // G] / math.sqrt(D)) < 1e-12


def check_constant_v():
    """If every value vector equals c, every output equals c (rows sum to 1)."""
    q, k, _, gq, gk, pos = _inputs(1, 40, 4, 2, seed=21)
    c = _rand((D,), 22)
    v = np.broadcast_to(c, (1, 40, 2, D)).copy()
    out, _ = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS, block=16)
    assert np.allclose(out, c, rtol=0, atol=1e-13)


def check_gqa_equals_mha_on_repeated_kv():
    """GQA with G = Hq/Hkv equals MHA run on KV heads repeated G times each
    (repeat_interleave along the head axis)."""
    q, k, v, gq, gk, pos = _inputs(1, 24, 8, 2, seed=23)
    out_g, lse_g = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
    kr, vr = np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2)
    out_m, lse_m = A.prefill_ref(q, kr, vr, gq, gk, pos, THETA, EPS)
    assert np.allclose(out_g, out_m, rtol=0, atol=1e-14) and np.allclose(lse_g, lse_m, atol=1e-14)


def check_against_torch_sdpa():
    """The attention part equals torch's fp64 scaled_dot_product_attention
    (causal, enable_gqa) applied to the oracle's normed and rotated q, k."""
    B, T, Hq, Hkv = 2, 33, 8, 2
    q, k, v, gq, gk, pos = _inputs(B, T, Hq, Hkv, seed=24)
    out, _ = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS, block=8)
    qp = np.stack([A.qk_prologue(q[b], gq, pos[b], THETA, EPS) for b in range(B)])
    kp = np.stack([A.qk_prologue(k[b], gk, pos[b], THETA, EPS) for b in range(B)])
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).transpose(1, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(t(qp), t(kp), t(v), is_causal=True, enable_gqa=True)
    assert np.allclose(out, ref.transpose(1, 2).numpy(), rtol=0, atol=1e-12)


def check_causality():
    """Changing keys/values after row i leaves rows <= i unchanged."""
    q, k, v, gq, gk, pos = _inputs(1, 30, 4, 2, seed=25)
    out1, lse1 = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
    k2, v2 = k.copy(), v.copy()
    k2[:, 18:] += 5.0
    v2[:, 18:] -= 3.0
    out2, lse2 = A.prefill_ref(q, k2, v2, gq, gk, pos, THETA, EPS)
    assert np.array_equal(out1[:, :18], out2[:, :18]) and np.array_equal(lse1[:, :, :18], lse2[:, :, :18])
    assert not np.allclose(out1[:, 18:], out2[:, 18:])


def check_brute_force_prefill():
    for (T, Hq, Hkv, seed) in [(5, 2, 1, 30), (16, 4, 2, 31), (9, 4, 1, 32)]:
        q, k, v, gq, gk, pos = _inputs(1, T, Hq, Hkv, seed=seed)
        pos = pos + 3 * seed  # arbitrary, non-zero start
        out, lse = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS, block=4)
        out_l, lse_l = Lp.prefill_loops(q.tolist(), k.tolist(), v.tolist(), gq.tolist(), gk.tolist(),
                                        pos.tolist(), THETA, EPS)
        assert np.allclose(out, np.array(out_l), rtol=0, atol=1e-12)
        assert np.allclose(lse, np.array(lse_l), rtol=0, atol=1e-12)


def _tiny_decode(seed, N=2, Hq=4, Hkv=2, lens=(5, 9)):
    rng = np.random.default_rng(seed)
    Lmax = max(lens) + 1
    q = rng.standard_normal((N, Hq, D))
    kn = rng.standard_normal((N, Hkv, D))
    vn = rng.standard_normal((N, Hkv, D))
    kh = rng.standard_normal((N, Lmax, Hkv, D))
    vc = rng.standard_normal((N, Hkv, Lmax, D))
    gq, gk = _gain(seed + 1), _gain(seed + 2)
    kc = np.stack([A.qk_prologue(kh[n], gk, np.arange(Lmax), THETA, EPS).transpose(1, 0, 2) for n in range(N)])
    return q, kn, vn, gq, gk, kc, vc, np.array(lens), kh


def check_brute_force_decode():
    q, kn, vn, gq, gk, kc, vc, lens, _ = _tiny_decode(40)
    out, lse = A.decode_ref(q, kn, vn, gq, gk, kc, vc, lens, THETA, EPS)
    out_l, lse_l = Lp.decode_loops(q.tolist(), kn.tolist(), vn.tolist(), gq.tolist(), gk.tolist(),
                                   kc.tolist(), vc.tolist(), lens.tolist(), THETA, EPS)
    assert np.allclose(out, np.array(out_l), rtol=0, atol=1e-12)
    assert np.allclose(lse, np.array(lse_l), rtol=0, atol=1e-12)


def check_decode_equals_last_prefill_row():
    """Decode at cached length L over a cache of keys normed/rotated at 0..L-1
    equals row L of a prefill over the same L+1 raw tokens."""
    rng = np.random.default_rng(41)
    L, Hq, Hkv = 23, 8, 2
    q = rng.standard_normal((1, L + 1, Hq, D))
    k = rng.standard_normal((1, L + 1, Hkv, D))
    v = rng.standard_normal((1, L + 1, Hkv, D))
    gq, gk = _gain(42), _gain(43)
    pos = np.arange(L + 1)[None]
    out_p, lse_p = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
    kc = A.qk_prologue(k[0, :L], gk, np.arange(L), THETA, EPS).transpose(1, 0, 2)[None]
    vc = v[0, :L].transpose(1, 0, 2)[None]
    out_d, lse_d = A.decode_ref(q[:, L], k[:, L], v[:, L], gq, gk, kc, vc, np.array([L]), THETA, EPS)
    assert np.allclose(out_d[0], out_p[0, L], rtol=0, atol=1e-13)
    assert np.allclose(lse_d[0], lse_p[0, :, L], rtol=0, atol=1e-13)


# ---------------------------------------------------------------- chunked prefill
def _chunk_split(q, k, v, gk, pos, start):
    """Split a full prompt into a cache of its first `start` tokens (keys normed and
    rotated at their positions, kept in fp64) and the remaining new tokens."""
    B = q.shape[0]
    kc = np.stack([A.qk_prologue(k[b, :start], gk, pos[b, :start], THETA, EPS).transpose(1, 0, 2) for b in range(B)])
    vc = v[:, :start].transpose(0, 2, 1, 3)
    return q[:, start:], k[:, start:], v[:, start:], pos[:, start:], kc, vc


def check_brute_force_chunk_prefill():
    for (start, T, Hq, Hkv, seed) in [(3, 4, 2, 1, 70), (7, 5, 4, 2, 71), (0, 6, 4, 1, 72), (9, 1, 4, 2, 73)]:
        q, k, v, gq, gk, pos = _inputs(2, start + T, Hq, Hkv, seed=seed)
        pos = pos + seed
        qn, kn, vn, pn, kc, vc = _chunk_split(q, k, v, gk, pos, start)
        out, lse = A.chunk_prefill_ref(qn, kn, vn, gq, gk, pn, kc, vc, start, THETA, EPS, block=2)
        out_l, lse_l = Lp.chunk_prefill_loops(qn.tolist(), kn.tolist(), vn.tolist(), gq.tolist(), gk.tolist(),
                                              pn.tolist(), kc.tolist(), vc.tolist(), start, THETA, EPS)
        assert np.allclose(out, np.array(out_l), rtol=0, atol=1e-12)
        assert np.allclose(lse, np.array(lse_l), rtol=0, atol=1e-12)


def check_chunk_equals_tail_of_full_prefill():
    """tril(diagonal = S - T) lets the new tokens see the whole history, so a chunk over
    a cache of the first `start` tokens reproduces rows start.. of a prefill over all
    of them ("Assembling a large model from scratch", notes below the code)."""
    for (start, T, Hq, Hkv, seed) in [(37, 29, 8, 2, 74), (64, 64, 4, 4, 75), (5, 70, 8, 1, 76)]:
        q, k, v, gq, gk, pos = _inputs(2, start + T, Hq, Hkv, seed=seed)
        full_o, full_l = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
        qn, kn, vn, pn, kc, vc = _chunk_split(q, k, v, gk, pos, start)
        out, lse = A.chunk_prefill_ref(qn, kn, vn, gq, gk, pn, kc, vc, start, THETA, EPS, block=16)
        assert np.allclose(out, full_o[:, start:], rtol=0, atol=1e-13)
        assert np.allclose(lse, full_l[:, :, start:], rtol=0, atol=1e-13)
        rows = np.array([0, T // 2, T - 1])
        out_s, lse_s = A.chunk_prefill_ref(qn, kn, vn, gq, gk, pn, kc, vc, start, THETA, EPS, rows=rows, block=2)
        assert np.allclose(out_s, full_o[:, start + rows], rtol=0, atol=1e-13)
        assert np.allclose(lse_s, full_l[:, :, start + rows], rtol=0, atol=1e-13)


def check_chunk_of_one_token_is_decode():
    """A chunk of one new token over a cache of L tokens is one decode step at L."""
    q, kn, vn, gq, gk, kc, vc, lens, _ = _tiny_decode(77, N=1, lens=(11,))
    L = int(lens[0])
    out_d, lse_d = A.decode_ref(q, kn, vn, gq, gk, kc, vc, lens, THETA, EPS)
    out_c, lse_c = A.chunk_prefill_ref(q[:, None], kn[:, None], vn[:, None], gq, gk, np.array([[L]]), kc, vc, L,
                                       THETA, EPS)
    assert np.allclose(out_c[:, 0], out_d, rtol=0, atol=1e-13)
    assert np.allclose(lse_c[:, :, 0], lse_d, rtol=0, atol=1e-13)


def check_chunk_over_empty_cache_is_prefill():
    q, k, v, gq, gk, pos = _inputs(2, 33, 8, 2, seed=78)
    empty = np.zeros((2, 2, 0, D))
    out, lse = A.chunk_prefill_ref(q, k, v, gq, gk, pos, empty, empty, 0, THETA, EPS)
    ref_o, ref_l = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
    assert np.allclose(out, ref_o, rtol=0, atol=1e-14) and np.allclose(lse, ref_l, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- varlen batches
def _packed(lens, Hq, Hkv, seed, lead=0, tail=0, ctx=None):
    """Sequences of the given lengths packed back to back after `lead` unowned tokens and
    before `tail` more; positions run from ctx_b (0 without a prefix) within each sequence.
    With ctx, also the cached prefixes: keys normed and rotated at 0..ctx_b-1, values raw."""
    cu = np.concatenate([[lead], lead + np.cumsum(lens)]).astype(np.int64)
    N = int(cu[-1]) + tail
    c = [0] * len(lens) if ctx is None else list(ctx)
    pos = np.zeros(N, dtype=np.int64)
    for b, L in enumerate(lens):
        pos[cu[b]:cu[b + 1]] = c[b] + np.arange(L)
    q, k, v = _rand((N, Hq, D), seed), _rand((N, Hkv, D), seed + 1), _rand((N, Hkv, D), seed + 2)
    gq, gk = _gain(seed + 3), _gain(seed + 4)
    kp = vp = None
    if ctx is not None:
        kp = [A.qk_prologue(_rand((n, Hkv, D), seed + 10 + b), gk, np.arange(n), THETA, EPS).transpose(1, 0, 2)
              for b, n in enumerate(ctx)]
        vp = [_rand((Hkv, n, D), seed + 40 + b) for b, n in enumerate(ctx)]
    return q, k, v, gq, gk, pos, cu, kp, vp


def check_brute_force_varlen_prefill():
    """Ragged sequences (an empty one, a single token, unowned tokens before and after),
    fresh and over cached prefixes, against the token-by-token loops."""
    for (lens, Hq, Hkv, seed, lead, tail, ctx) in [((3, 0, 1, 5), 4, 2, 90, 0, 0, None),
                                                   ((4, 2), 2, 1, 91, 2, 1, (3, 0)),
                                                   ((1, 6, 2), 4, 1, 92, 0, 3, (2, 5, 1))]:
        q, k, v, gq, gk, pos, cu, kp, vp = _packed(lens, Hq, Hkv, seed, lead, tail, ctx)
        out, lse = A.varlen_prefill_ref(q, k, v, gq, gk, pos, cu, THETA, EPS, k_prefix=kp, v_prefix=vp)
        lp = None if kp is None else [x.tolist() for x in kp]
        lv = None if vp is None else [x.tolist() for x in vp]
        out_l, lse_l = Lp.varlen_prefill_loops(q.tolist(), k.tolist(), v.tolist(), gq.tolist(), gk.tolist(),
                                               pos.tolist(), cu.tolist(), THETA, EPS, k_prefix=lp, v_prefix=lv)
        for n in range(q.shape[0]):
            if out_l[n] is None:
                assert np.isnan(out[n]).all() and np.isnan(lse[:, n]).all()
            else:
                assert np.allclose(out[n], np.array(out_l[n]), rtol=0, atol=1e-12)
                assert np.allclose(lse[:, n], [lse_l[h][n] for h in range(Hq)], rtol=0, atol=1e-12)


def check_varlen_of_equal_lengths_is_the_batch():
    """Packing B sequences of equal length T on one token axis gives the batched prefill
    [B, T] row for row (the token axis is the batch axis flattened)."""
    B, T, Hq, Hkv = 3, 37, 8, 2
    q, k, v, gq, gk, pos = _inputs(B, T, Hq, Hkv, seed=93)
    ref_o, ref_l = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
    cu = np.arange(B + 1) * T
    out, lse = A.varlen_prefill_ref(q.reshape(B * T, Hq, D), k.reshape(B * T, Hkv, D), v.reshape(B * T, Hkv, D), gq,
                                    gk, pos.reshape(-1), cu, THETA, EPS)
    assert np.allclose(out, ref_o.reshape(B * T, Hq, D), rtol=0, atol=1e-14)
    assert np.allclose(lse, ref_l.transpose(1, 0, 2).reshape(Hq, B * T), rtol=0, atol=1e-14)


def check_varlen_sequences_are_independent():
    """Attention stays inside each sequence: reversing the order of the packed sequences
    moves their outputs with them and changes nothing else; a prefixed sequence equals the
    chunked prefill over its prefix."""
    lens, ctx = (5, 9, 1, 4), (0, 6, 3, 2)
    q, k, v, gq, gk, pos, cu, kp, vp = _packed(lens, 4, 2, 94, ctx=ctx)
    out, lse = A.varlen_prefill_ref(q, k, v, gq, gk, pos, cu, THETA, EPS, k_prefix=kp, v_prefix=vp)
    order = list(range(len(lens)))[::-1]
    idx = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in order])
    cu_r = np.concatenate([[0], np.cumsum([lens[b] for b in order])])
    out_r, lse_r = A.varlen_prefill_ref(q[idx], k[idx], v[idx], gq, gk, pos[idx], cu_r, THETA, EPS,
                                        k_prefix=[kp[b] for b in order], v_prefix=[vp[b] for b in order])
    assert np.array_equal(out_r, out[idx]) and np.array_equal(lse_r, lse[:, idx])
    b = 1
    sl = slice(cu[b], cu[b + 1])
    o1, l1 = A.chunk_prefill_ref(q[None, sl], k[None, sl], v[None, sl], gq, gk, pos[None, sl], kp[b][None],
                                 vp[b][None], ctx[b], THETA, EPS)
    assert np.array_equal(o1[0], out[sl]) and np.array_equal(l1[0], lse[:, sl])


# ---------------------------------------------------------------- variants
def check_brute_force_variants():
    """Sliding window, another rope type's frequencies and attention_scaling against the
    scalar loops."""
    inv = 1.0 / (1.0 + np.arange(D // 2)) ** 1.3  # any decreasing table of frequencies
    for (T, Hq, Hkv, seed, window, inv_freq, scaling) in [(9, 4, 2, 80, 3, None, 1.0), (7, 2, 1, 81, 1, inv, 1.0),
                                                          (8, 4, 1, 82, 0, inv, 1.25), (10, 4, 2, 83, 4, None, 0.8)]:
        q, k, v, gq, gk, pos = _inputs(1, T, Hq, Hkv, seed=seed)
        out, lse = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS, block=3, window=window, inv_freq=inv_freq,
                                 scaling=scaling)
        out_l, lse_l = Lp.prefill_loops(q.tolist(), k.tolist(), v.tolist(), gq.tolist(), gk.tolist(), pos.tolist(),
                                        THETA, EPS, window=window, inv_freq=inv_freq, scaling=scaling)
        assert np.allclose(out, np.array(out_l), rtol=0, atol=1e-12)
        assert np.allclose(lse, np.array(lse_l), rtol=0, atol=1e-12)


def check_window_special_cases():
    """W >= T is full causal attention; W = 1 leaves each query its own key, so out_i is
    v_i of its KV head and lse_i is s_ii; a window of W over a long prompt gives row i the
    result of a causal prefill over just tokens i-W+1..i (positions kept)."""
    q, k, v, gq, gk, pos = _inputs(2, 40, 8, 2, seed=84)
    full_o, full_l = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
    o, l = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS, window=40)
    assert np.array_equal(o, full_o) and np.array_equal(l, full_l)
    o1, l1 = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS, window=1)
    G = 4
    for h in range(8):
        assert np.allclose(o1[:, :, h], v[:, :, h // G], rtol=0, atol=1e-14)
    qp = A.qk_prologue(q, gq, pos, THETA, EPS)
    kp = A.qk_prologue(k, gk, pos, THETA, EPS)
    for b in range(2):
        for h in range(8):
            s = np.sum(qp[b, :, h] * kp[b, :, h // G], axis=-1) / np.sqrt(D)
            assert np.allclose(l1[b, h], s, rtol=0, atol=1e-12)
    W = 7
    ow, lw = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS, window=W)
    for i in (0, 3, 6, 7, 20, 39):
        lo = max(0, i - W + 1)
        os_, ls_ = A.prefill_ref(q[:, lo:i + 1], k[:, lo:i + 1], v[:, lo:i + 1], gq, gk, pos[:, lo:i + 1], THETA, EPS)
        assert np.allclose(ow[:, i], os_[:, -1], rtol=0, atol=1e-13)
        assert np.allclose(lw[:, :, i], ls_[:, :, -1], rtol=0, atol=1e-13)


def check_window_chunk_and_decode_agree_with_prefill():
    """With a window, a chunk over a cached prefix reproduces the windowed prefill's tail
    rows, and a decode step reproduces its last row."""
    start, T, W = 30, 21, 9
    q, k, v, gq, gk, pos = _inputs(1, start + T, 8, 2, seed=85)
    full_o, full_l = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS, window=W)
    qn, kn, vn, pn, kc, vc = _chunk_split(q, k, v, gk, pos, start)
    o, l = A.chunk_prefill_ref(qn, kn, vn, gq, gk, pn, kc, vc, start, THETA, EPS, window=W)
    assert np.allclose(o, full_o[:, start:], rtol=0, atol=1e-13) and np.allclose(l, full_l[:, :, start:], atol=1e-13)
    L = start + T - 1
    od, ld = A.decode_ref(q[:, L], k[:, L], v[:, L], gq, gk,
                          A.qk_prologue(k[:, :L], gk, pos[:, :L], THETA, EPS).transpose(0, 2, 1, 3),
                          v[:, :L].transpose(0, 2, 1, 3), np.array([L]), THETA, EPS, window=W)
    assert np.allclose(od[0], full_o[0, L], rtol=0, atol=1e-13) and np.allclose(ld[0], full_l[0, :, L], atol=1e-13)


def check_rope_variant_closed_forms():
    """inv_freq = theta^(-2i/d) is the default; attention_scaling s multiplies the rotated
    vector by s; a constant table c rotates every pair by pos*c (a plane rotation)."""
    x = _rand((3, 5, 2, D), 86)
    pos = np.array([[0, 1, 7, 100, 32768]] * 3)
    assert np.array_equal(A.rope(x, pos, THETA, inv_freq=A.rope_inv_freq(D, THETA)), A.rope(x, pos, THETA))
    assert np.allclose(A.rope(x, pos, THETA, scaling=1.7), 1.7 * A.rope(x, pos, THETA), rtol=1e-14, atol=1e-15)
    c = 0.37
    y = A.rope(x, pos, THETA, inv_freq=np.full(D // 2, c))
    ang = pos[..., None, None] * c
    assert np.allclose(y[..., :64], x[..., :64] * np.cos(ang) - x[..., 64:] * np.sin(ang), rtol=0, atol=1e-12)
    assert np.allclose(y[..., 64:], x[..., 64:] * np.cos(ang) + x[..., :64] * np.sin(ang), rtol=0, atol=1e-12)


def check_attention_scaling_against_torch_sdpa():
    """attention_scaling s scales q' and k' by s, so the logits scale by s^2: torch fp64
    SDPA with scale s^2/sqrt(d) on the default q', k' gives the same rows."""
    q, k, v, gq, gk, pos = _inputs(1, 24, 4, 2, seed=87)
    sc = 1.3
    o, _ = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS, scaling=sc)
    qp = torch.from_numpy(A.qk_prologue(q, gq, pos, THETA, EPS)).permute(0, 2, 1, 3)
    kp = torch.from_numpy(A.qk_prologue(k, gk, pos, THETA, EPS)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(qp, kp, vt, is_causal=True, enable_gqa=True,
                                                           scale=sc * sc / np.sqrt(D))
    assert np.allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def check_build_cache_k_stores_bf16():
    """The cache holds bf16 values: each key element is exactly representable in bf16 (a
    float32 whose low 16 bits are zero) and lies within half a bf16 ulp (at most 2^-8 of its
    magnitude: bf16 keeps 8 significant bits) of
    the normed, rotated fp64 key."""
    k = _rand((40, 2, D), 95, 3.0)
    g = _gain(96)
    c = A.build_cache_k(k, g, THETA, EPS)
    f32 = c.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), c)
    assert np.all((f32.view(np.uint32) & 0xFFFF) == 0)
    exact = A.qk_prologue(k, g, np.arange(40), THETA, EPS)
    assert np.all(np.abs(c - exact) <= np.abs(exact) * 2.0 ** -8)
    assert np.any(c != exact)


def check_paged_gather_addressing():
    """A pool whose every slot holds 1000*page + offset (per head and dim) gathers, for a
    hand-written block table, to 1000*table[j // size] + j % size at key j."""
    num_pages, Hkv, size, d = 7, 2, 4, 3
    pages = np.zeros((num_pages, Hkv, size, d))
    for pg in range(num_pages):
        for off in range(size):
            pages[pg, :, off] = 1000 * pg + off
    table = [5, 0, 3, 6]
    got = A.paged_gather(pages, table, 14, size)
    want = np.array([1000 * table[j // size] + j % size for j in range(14)], dtype=np.float64)
    assert got.shape == (Hkv, 14, d)
    assert np.array_equal(got, np.broadcast_to(want[None, :, None], (Hkv, 14, d)))


# ---------------------------------------------------------------- merged qkv projection
def check_qkv_projection_brute_force_and_identity():
    """The merged projection against scalar loops; with w_qkv = the identity on each head's
    block it reduces to QK-Norm + RoPE of x itself (the prologue pinned above)."""
    rng = np.random.default_rng(90)
    Hq, Hkv, hidden, M = 2, 1, 16, 3
    d = D
    x = rng.standard_normal((M, hidden))
    w = rng.standard_normal(((Hq + 2 * Hkv) * d, hidden)) / 4
    gq, gk = _gain(91), _gain(92)
    pos = np.array([0, 5, 300])
    q, k, v = A.qkv_proj_norm_rope_ref(x, w, gq, gk, pos, Hq, Hkv, THETA, EPS)
    ql, kl, vl = Lp.qkv_proj_norm_rope_loops(x.tolist(), w.tolist(), gq.tolist(), gk.tolist(), pos.tolist(), Hq, Hkv,
                                             THETA, EPS)
    assert np.allclose(q, np.array(ql), rtol=0, atol=1e-12)
    assert np.allclose(k, np.array(kl), rtol=0, atol=1e-12)
    assert np.allclose(v, np.array(vl), rtol=0, atol=1e-12)
    xh = rng.standard_normal((M, d))
    eye = np.concatenate([np.eye(d)] * (Hq + 2 * Hkv), axis=0)  # every head projects x itself
    q2, k2, v2 = A.qkv_proj_norm_rope_ref(xh, eye, gq, gk, pos, Hq, Hkv, THETA, EPS)
    want_q = A.qk_prologue(np.repeat(xh[:, None], Hq, axis=1), gq, pos, THETA, EPS)
    assert np.allclose(q2, want_q, rtol=0, atol=1e-13) and np.allclose(v2[:, 0], xh, rtol=0, atol=0)


def check_qkv_projection_scale_invariance():
    """Scaling the hidden states scales v and leaves q', k' unchanged up to the eps term."""
    rng = np.random.default_rng(93)
    x = rng.standard_normal((5, 64))
    w = rng.standard_normal(((4 + 4) * D, 64)) / 8
    gq, gk = _gain(94), _gain(95)
    pos = np.arange(5) * 7
    q1, k1, v1 = A.qkv_proj_norm_rope_ref(x, w, gq, gk, pos, 4, 2, THETA, 0.0)
    q2, k2, v2 = A.qkv_proj_norm_rope_ref(3.0 * x, w, gq, gk, pos, 4, 2, THETA, 0.0)
    assert np.allclose(q1, q2, rtol=0, atol=1e-12) and np.allclose(k1, k2, rtol=0, atol=1e-12)
    assert np.allclose(3.0 * v1, v2, rtol=1e-12, atol=1e-13)


def check_position_shift_invariance():
    """Shifting every position by a constant leaves outputs unchanged (RoPE is relative)."""
    q, k, v, gq, gk, pos = _inputs(1, 20, 4, 2, seed=50)
    o1, l1 = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
    o2, l2 = A.prefill_ref(q, k, v, gq, gk, pos + 12345, THETA, EPS)
    assert np.allclose(o1, o2, rtol=0, atol=1e-9) and np.allclose(l1, l2, atol=1e-9)


def check_qk_scale_invariance():
    """Scaling raw q or k by c > 0 leaves the output unchanged up to the eps term."""
    q, k, v, gq, gk, pos = _inputs(1, 20, 4, 2, seed=51)
    o1, _ = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
    o2, _ = A.prefill_ref(q * 7.5, k * 0.25, v, gq, gk, pos, THETA, EPS)
    # eps moves a normalised k by ~eps / (2 * mean(k^2)) ~ 8e-6 relative here.
    assert np.allclose(o1, o2, rtol=0, atol=2e-4)
    o3, _ = A.prefill_ref(q * 7.5, k * 0.25, v, gq, gk, pos, THETA, 0.0)
    o4, _ = A.prefill_ref(q, k, v, gq, gk, pos, THETA, 0.0)
    assert np.allclose(o3, o4, rtol=0, atol=1e-12)


def check_row_subset_equals_full():
    q, k, v, gq, gk, pos = _inputs(2, 50, 4, 1, seed=52)
    out, lse = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS)
    rows = np.array([0, 7, 31, 49])
    out_s, lse_s = A.prefill_ref(q, k, v, gq, gk, pos, THETA, EPS, rows=rows, block=3)
    assert np.allclose(out_s, out[:, rows], rtol=0, atol=1e-14)
    assert np.allclose(lse_s, lse[:, :, rows], rtol=0, atol=1e-14)


def check_worked_example_kv_cache():
    gold = json.load(open(GOLDEN))["wide_gqa_block"]
    vals = A.kv_cache_values_per_token(gold["n_kv_heads"], gold["head_dim"])
    assert vals == gold["kv_cache_values_per_token_per_layer"]
    mha = A.kv_cache_values_per_token(gold["n_query_heads"], gold["head_dim"])
    assert vals / mha == gold["fraction_of_full_multi_head_cache"]
    assert gold["key_value_projection"][1] == gold["n_kv_heads"] * gold["head_dim"]
    assert gold["query_projection"][1] == gold["n_query_heads"] * gold["head_dim"]


def check_worked_example_logit_scale():
    """Unit-RMS head vectors have raw dot products of RMS ~ sqrt(128) ~ 11.3."""
    gold = json.load(open(GOLDEN))["wide_gqa_block"]
    x = _rand((20000, D), 60, 3.0)
    y = _rand((20000, D), 61, 0.2)
    qn = A.rms_norm(x, np.ones(D), EPS)
    kn = A.rms_norm(y, np.ones(D), EPS)
    rms = float(np.sqrt(np.mean(np.sum(qn * kn, axis=-1) ** 2)))
    assert abs(rms - gold["raw_dot_rms_of_unit_rms_vectors"]) < 0.03 * 11.3


ALL_CHECKS = [v for k, v in sorted(globals().items()) if k.startswith("check_")]
