"""Variants through the C ABI against the fp64 oracle: sliding-window attention in prefill,
chunked prefill and decode, and another rope type's frequency table with an
attention_scaling on cos/sin ("Qwen3 Architecture Layer-by-Layer", Per-layer attention
type and Qwen3RotaryEmbedding)."""
import numpy as np
import pytest
import torch

import oracle
import qwen3_qk_norm_rope_b200 as qa
from synthetic import ChunkShape, DecodeShape, PrefillShape, as_f64, chunk_inputs, decode_history, \
    decode_step_inputs, prefill_inputs
from tests.gpu_common import (LSE_PURE_TOL, LSE_TOL, MAX_TOL, MEAN_TOL, assert_status_ok, compare, dev,
                              prefill_lse_bound, to_np)

pytestmark = pytest.mark.gpu
NAN16 = 0x7FC1
THETA, EPS = 1.0e6, 1.0e-6


def _yarn_like_table(d=128, theta=THETA, factor=4.0, lo=1.0, hi=32.0, orig=4096):
    """A frequency table shaped like YaRN's: frequencies whose wavelength fits the original
    context many times keep theta^(-2i/d), the longest wavelengths are divided by `factor`,
    and a linear ramp blends the two.  (Any table serves the test: the library takes it as
    given.)"""
    i = np.arange(d // 2, dtype=np.float64)
    base = theta ** (-2.0 * i / d)
    rot = orig * base / (2 * np.pi)  # rotations over the original context
    ramp = np.clip((rot - lo) / (hi - lo), 0.0, 1.0)
    return base * ramp + (base / factor) * (1.0 - ramp)


def _prefill_case(B, T, Hq, Hkv, seed, window=0, inv_freq=None, scaling=1.0, gain_mul=1.0):
    inp = prefill_inputs(PrefillShape("variant", B, T, Hq, Hkv), seed=seed)
    inp["q_norm_w"] = inp["q_norm_w"] * gain_mul
    inp["k_norm_w"] = inp["k_norm_w"] * gain_mul
    d = dev()
    t = {k: v.to(d) for k, v in inp.items()}
    lse = torch.full((B, Hq, T), float("nan"), dtype=torch.float32, device=d)
    out = qa.prefill(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], lse=lse, window=window,
                     inv_freq=inv_freq, attention_scaling=scaling)
    torch.cuda.synchronize()
    assert_status_ok()
    args = (as_f64(inp["q"]), as_f64(inp["k"]), as_f64(inp["v"]), as_f64(inp["q_norm_w"]), as_f64(inp["k_norm_w"]),
            inp["pos"].numpy(), THETA, EPS)
    kw = dict(window=window, inv_freq=inv_freq, scaling=scaling)
    ref, ref_lse = oracle.prefill_ref(*args, **kw)
    ref_st, st_lse = oracle.prefill_ref(*args, staged=True, **kw)
    return out, lse, ref, ref_lse, ref_st, st_lse


WINDOWS = [
    # (B, T, Hq, Hkv, window): windows of 1 key, under a tile, a tile exactly, over a tile,
    # not a multiple of 128, and wider than T; G in {1, 2, 4, 16}
    (2, 700, 16, 8, 1),
    (1, 900, 32, 8, 100),
    (2, 641, 8, 8, 128),
    (1, 1000, 16, 1, 300),
    (1, 777, 32, 8, 513),
    (2, 300, 16, 4, 5000),
]


# The logsumexp bound against the staged oracle (1e-3) is set for rows whose LSE is a soft
# maximum over many keys.  With a window of one key every row's LSE IS one logit, and rows
# under a short window with large gains are nearly so: a single bf16 rounding-boundary
# straddle of one q' or k' element (the kernel's fp32 value a few ulp from the correctly
# rounded one) moves that element by one bf16 ulp, at most 2^-7 of it, and the LSE by up to
# 2^-7 |q'_i k'_i| / sqrt(d), with nothing to average it out.  The straddles measured at the
# element sizes of these inputs stayed near 3e-3 at most.  Those cases are held to 4e-3
# (times the gain product squared where the gains are scaled).
SINGLE_LOGIT_LSE_TOL = 4e-3


@pytest.mark.parametrize("B,T,Hq,Hkv,window", WINDOWS)
def test_prefill_sliding_window(B, T, Hq, Hkv, window):
    out, lse, ref, ref_lse, _, st_lse = _prefill_case(B, T, Hq, Hkv, seed=T + window, window=window)
    what = f"window {window} B{B} T{T} Hq{Hq} Hkv{Hkv}"
    if window > 1:
        compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, what)
        return
    # Every row sees only its own key.  out = v of its KV head (up to the bf16 P); the LSE is
    # the logit s = q'.k'/sqrt(d) itself, which the bf16 rounding of q' and k' (unit roundoff
    # u = 2^-8 each) and the fp32 accumulation move by less than
    # (2^-7 + 2^-15) sum_i |q'_i k'_i| / sqrt(d) (prefill_lse_bound in gpu_common): that
    # per-row bound holds against the pure oracle, one straddle's worth against the staged one.
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, what, lse_tol=SINGLE_LOGIT_LSE_TOL,
            lse_pure_tol=float("inf"))
    inp = prefill_inputs(PrefillShape("variant", B, T, Hq, Hkv), seed=T + window)
    G = Hq // Hkv
    v = inp["v"].float().numpy()
    # P is bf16(p) against the fp32 l, and out is rounded to bf16: two roundings of at most
    # 2^-8 each (with one visible key p = l = 1 and out is v exactly)
    assert np.allclose(to_np(out), np.repeat(v, G, axis=2), rtol=2.0 ** -7, atol=1e-6)
    qp = oracle.qk_prologue(as_f64(inp["q"]), as_f64(inp["q_norm_w"]), inp["pos"].numpy(), THETA, EPS)
    kp = np.repeat(oracle.qk_prologue(as_f64(inp["k"]), as_f64(inp["k_norm_w"]), inp["pos"].numpy(), THETA, EPS),
                   G, axis=2)
    bound = (2.0 ** -7 + 2.0 ** -15) * np.abs(qp * kp).sum(-1) / np.sqrt(128.0) + 1e-5  # [B, T, Hq]
    err = np.abs(to_np(lse) - ref_lse)  # [B, Hq, T]
    assert np.all(err <= bound.transpose(0, 2, 1)), (err - bound.transpose(0, 2, 1)).max()


def test_prefill_window_running_max_path():
    """Large gains take the running-max softmax, where the first key tiles of an item can be
    wholly outside some rows' windows (no max yet for those rows)."""
    out, lse, ref, ref_lse, ref_st, st_lse = _prefill_case(2, 800, 16, 8, seed=41, window=200, gain_mul=1.6)
    compare(to_np(out), to_np(lse), ref_st, st_lse, st_lse, "window 200, large gains (staged)",
            lse_tol=SINGLE_LOGIT_LSE_TOL * 1.6 ** 2)
    # against the pure oracle: the default output bounds times the gain product 1.6^2, and
    # the LSE of every row within the rigorous per-row bound over the keys in its window
    inp = prefill_inputs(PrefillShape("variant", 2, 800, 16, 8), seed=41)
    inp["q_norm_w"] = inp["q_norm_w"] * 1.6
    inp["k_norm_w"] = inp["k_norm_w"] * 1.6
    g2 = 1.6 ** 2
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, "window 200, large gains (pure)",
            lse_tol=SINGLE_LOGIT_LSE_TOL * g2, max_tol=MAX_TOL * g2, mean_tol=MEAN_TOL * g2,
            lse_pure_bound=prefill_lse_bound(inp, np.arange(800), window=200))


def test_prefill_rope_variant():
    inv = _yarn_like_table()
    out, lse, ref, ref_lse, _, st_lse = _prefill_case(2, 600, 16, 8, seed=42, inv_freq=inv, scaling=1.1)
    # attention_scaling s scales the logits by s^2, and with them the logit error from the
    # single bf16 rounding of q', k'
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, "yarn-like table, scaling 1.1", lse_tol=1e-3 * 1.1 ** 2)


def test_qk_norm_rope_variant_kernel():
    d = dev()
    rng = np.random.default_rng(43)
    B, T, H = 2, 129, 8
    x = torch.from_numpy(rng.standard_normal((B, T, H, 128)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy((1 + 0.1 * rng.standard_normal(128)).astype(np.float32))
    pos = torch.from_numpy(rng.integers(0, 40000, size=(B, T)).astype(np.int32))
    inv = _yarn_like_table()
    dst = torch.zeros((B, H, T, 128), dtype=torch.bfloat16, device=d)
    qa.qk_norm_rope(x.to(d), w.to(d), pos.to(d), dst, inv_freq=inv, attention_scaling=1.25)
    torch.cuda.synchronize()
    assert_status_ok()
    ref = oracle.qk_prologue(as_f64(x), as_f64(w), pos.numpy(), THETA, EPS, inv_freq=inv, scaling=1.25)
    got = to_np(dst.permute(0, 2, 1, 3))
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 3e-5), np.abs(got - ref).max()


def test_chunk_sliding_window():
    shape = ChunkShape("window chunk", 1, 1000, 300, 32, 8)
    inp = chunk_inputs(shape, seed=44)
    window = 400
    d = dev()
    Tcap = shape.start + shape.T + 16
    kc = torch.empty((1, 8, Tcap, 128), dtype=torch.bfloat16)
    kc.view(torch.int16).fill_(NAN16)
    vc = kc.clone()
    gk = as_f64(inp["k_norm_w"])
    kb = oracle.build_cache_k(as_f64(inp["k_hist"][0]), gk, THETA, EPS)
    kc[0, :, :shape.start] = torch.from_numpy(kb.transpose(1, 0, 2).copy()).to(torch.bfloat16)
    vc[0, :, :shape.start] = inp["v_hist"][0].permute(1, 0, 2)
    t = {k: inp[k].to(d) for k in ("q", "k", "v", "q_norm_w", "k_norm_w", "pos")}
    kcd, vcd = kc.to(d), vc.to(d)
    lse = torch.full((1, 32, shape.T), float("nan"), dtype=torch.float32, device=d)
    out = qa.prefill_chunk(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], kcd, vcd, shape.start,
                           lse=lse, window=window)
    torch.cuda.synchronize()
    assert_status_ok()
    args = (as_f64(inp["q"]), as_f64(inp["k"]), as_f64(inp["v"]), as_f64(inp["q_norm_w"]), gk, inp["pos"].numpy(),
            as_f64(kc[:, :, :shape.start]), as_f64(vc[:, :, :shape.start]), shape.start, THETA, EPS)
    ref, ref_lse = oracle.chunk_prefill_ref(*args, window=window)
    _, st_lse = oracle.chunk_prefill_ref(*args, window=window, staged=True)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, "chunk, window 400")


@pytest.mark.parametrize("window,inv,scaling", [(1, False, 1.0), (1024, False, 1.0), (3000, False, 1.0),
                                                (2500, True, 1.1)])
def test_decode_variants(window, inv, scaling):
    """Windows that end inside a split, on a split boundary, and over several splits; and a
    rope variant on top of a window.  Stale slots hold NaN patterns."""
    shape = DecodeShape("decode variants", 6, 32, 8)
    lens = [5000, 2047, 1024, 3000, 0, 7777]
    Lmax = 8192
    inv_freq = _yarn_like_table() if inv else None
    d = dev()
    step = decode_step_inputs(shape, seed=45)
    step["cache_lens"] = torch.as_tensor(np.asarray(lens, dtype=np.int32))
    kc = torch.empty((6, 8, Lmax, 128), dtype=torch.bfloat16, device=d)
    vc = torch.empty_like(kc)
    kc.view(torch.int16).fill_(NAN16)
    vc.view(torch.int16).fill_(NAN16)
    gq, gk = as_f64(step["q_norm_w"]), as_f64(step["k_norm_w"])
    host = {}
    for n, L in enumerate(lens):
        if L == 0:
            continue
        hist = decode_history(shape, n, L, step["s_k"], seed=45)
        kcache = oracle.build_cache_k(as_f64(hist["k_hist"]), gk, THETA, EPS, inv_freq=inv_freq, scaling=scaling)
        kc[n, :, :L] = torch.from_numpy(kcache.transpose(1, 0, 2)).to(torch.bfloat16).to(d)
        vc[n, :, :L] = hist["v_hist"].permute(1, 0, 2).to(d)
        host[n] = (kcache.transpose(1, 0, 2), as_f64(hist["v_hist"]).transpose(1, 0, 2))
    host[4] = (np.zeros((8, 0, 128)), np.zeros((8, 0, 128)))
    t = {k: v.to(d) for k, v in step.items()}
    lse = torch.full((6, 32), float("nan"), dtype=torch.float32, device=d)
    out = qa.decode(t["q"], t["k_new"], t["v_new"], t["q_norm_w"], t["k_norm_w"], kc, vc, t["cache_lens"], lse=lse,
                    window=window, inv_freq=inv_freq, attention_scaling=scaling)
    torch.cuda.synchronize()
    assert_status_ok()
    lse_tol = (SINGLE_LOGIT_LSE_TOL if window == 1 else LSE_TOL) * scaling ** 2
    for n, (kh, vh) in host.items():
        L = lens[n]
        args = (as_f64(step["q"])[n:n + 1], as_f64(step["k_new"])[n:n + 1], as_f64(step["v_new"])[n:n + 1], gq, gk,
                [kh], [vh], [L], THETA, EPS)
        kw = dict(window=window, inv_freq=inv_freq, scaling=scaling)
        ref, ref_lse = oracle.decode_ref(*args, **kw)
        _, st_lse = oracle.decode_ref(*args, staged=True, **kw)
        o = to_np(out[n:n + 1])
        err = np.abs(o - ref)
        assert np.isfinite(o).all(), f"window {window} seq {n}: non-finite"
        assert err.max() <= MAX_TOL and err.mean() <= MEAN_TOL, f"window {window} seq {n} L={L}: {err.max():.3e}"
        l = to_np(lse[n:n + 1])
        assert np.abs(l - st_lse).max() <= lse_tol, f"window {window} seq {n}: lse {np.abs(l - st_lse).max():.3e}"
        assert np.abs(l - ref_lse).max() <= LSE_PURE_TOL
