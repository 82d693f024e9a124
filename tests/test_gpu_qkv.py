"""The merged qkv projection with QK-Norm + RoPE in the GEMM epilogue, through the C ABI,
against the fp64 oracle (oracle.qkv_proj_norm_rope_ref) on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import qwen3_qk_norm_rope_b200 as qa
from synthetic import QKV_SHAPES, QkvShape, as_f64, qkv_proj_inputs
from tests.gpu_common import assert_status_ok, dev, to_np

pytestmark = pytest.mark.gpu
THETA, EPS = 1.0e6, 1.0e-6


def _run(shape: QkvShape, seed: int, inv_freq=None, scaling=1.0, pos=None):
    inp = qkv_proj_inputs(shape, seed=seed)
    if pos is not None:
        inp["pos"] = pos
    d = dev()
    t = {k: v.to(d) for k, v in inp.items()}
    q, k, v = qa.qkv_proj_norm_rope(t["x"], t["w_qkv"], t["q_norm_w"], t["k_norm_w"], t["pos"], shape.Hq, shape.Hkv,
                                    inv_freq=inv_freq, attention_scaling=scaling)
    torch.cuda.synchronize()
    assert_status_ok()
    ref = oracle.qkv_proj_norm_rope_ref(as_f64(inp["x"]), as_f64(inp["w_qkv"]), as_f64(inp["q_norm_w"]),
                                        as_f64(inp["k_norm_w"]), inp["pos"].numpy(), shape.Hq, shape.Hkv, THETA, EPS,
                                        inv_freq=inv_freq, scaling=scaling)
    return (to_np(q), to_np(k), to_np(v)), ref


def _check(got, ref, what):
    # fp32 accumulation of exact bf16 products (relative error ~ hidden * 2^-24), the norm and
    # rotation in fp32, then one bf16 rounding (unit roundoff 2^-8): 2^-8 |ref| plus a small
    # absolute term for entries near zero, scaled to the tensor's RMS.  Round-to-nearest errors
    # average about a quarter ulp, under 2^-9 of the magnitude: the bound on the mean.
    for name, g, r in zip("qkv", got, ref):
        assert np.isfinite(g).all(), f"{what} {name}: non-finite"
        rms = np.sqrt(np.mean(r * r))
        err = np.abs(g - r)
        bound = np.abs(r) * 2.0 ** -8 + 2e-3 * rms
        assert np.all(err <= bound), f"{what} {name}: worst excess {(err - bound).max():.3e} (rms {rms:.3f})"
        assert err.mean() <= 2.0 ** -9 * np.mean(np.abs(r)) + 1e-4 * rms, f"{what} {name}: mean {err.mean():.3e}"


@pytest.fixture
def sm_pairs(request):
    """The SM-pair setting for the test (the default rule, or one kernel forced), restored after."""
    old = qa.set_sm_pairs(request.param)
    yield request.param
    qa.set_sm_pairs(old)


@pytest.mark.parametrize("sm_pairs", [qa.SM_PAIRS_AUTO, qa.SM_PAIRS_ALWAYS], indirect=True, ids=["auto", "pairs"])
@pytest.mark.parametrize("M,hidden,Hq,Hkv", [
    (300, 256, 4, 2),    # M off the 128-row tile, hidden a few chunks
    (128, 200, 3, 3),    # an odd head count (the last tile holds one head), hidden off the 64-chunk
    (1000, 512, 16, 8),  # several token tiles per CTA run
    (1, 64, 1, 1),       # one token, one head of each kind, one K chunk
])
def test_qkv_proj_small(M, hidden, Hq, Hkv, sm_pairs):
    """Short K runs take the one-SM kernel by default; forced, the SM-pair kernel on the same
    shapes (a single token tile, whose pair partner has no rows; an odd head count)."""
    shape = QkvShape("qkv small", M, hidden, Hq, Hkv)
    got, ref = _run(shape, seed=M + hidden)
    _check(got, ref, f"M{M} hidden{hidden} Hq{Hq} Hkv{Hkv}")


def test_qkv_proj_full_size():
    shape = QKV_SHAPES["qwen3-0.6b-qkv"]
    got, ref = _run(shape, seed=0)
    _check(got, ref, shape.name)


@pytest.mark.parametrize("M,hidden,Hq,Hkv", [
    (300, 8192, 4, 2),   # three token tiles: the last pair's second CTA has no rows
    (200, 8200, 3, 3),   # an odd head count, and hidden off the 64-chunk
    (2400, 4096, 16, 8),  # three pair tiles per SM pair, 19 token tiles, rows off the tile
])
@pytest.mark.parametrize("sm_pairs", [qa.SM_PAIRS_AUTO, qa.SM_PAIRS_OFF], indirect=True, ids=["auto", "one-sm"])
def test_qkv_proj_long_k_runs(M, hidden, Hq, Hkv, sm_pairs):
    """Runs of 128 K chunks or more per SM pair, which the library computes by default with
    both SMs of a pair on each MMA (M = 256 rows split across the two CTAs, each holding half
    of the tile's weight rows); forced, the one-SM kernel on the same shapes."""
    shape = QkvShape("qkv long K", M, hidden, Hq, Hkv)
    got, ref = _run(shape, seed=M + hidden + 1)
    _check(got, ref, f"M{M} hidden{hidden} Hq{Hq} Hkv{Hkv}")


@pytest.mark.parametrize("M,hidden,Hq,Hkv", [(300, 2048, 4, 2), (4096, 1024, 16, 8)])
def test_qkv_proj_sm_pair_and_one_sm_kernels_agree_bit_for_bit(M, hidden, Hq, Hkv):
    """Both kernels multiply the same bf16 operands in the same K order into fp32 and apply
    the same epilogue, so they must return identical bits."""
    shape = QkvShape("qkv kernels", M, hidden, Hq, Hkv)
    inp = qkv_proj_inputs(shape, seed=17)
    d = dev()
    t = {k: v.to(d) for k, v in inp.items()}
    res = {}
    for mode in (qa.SM_PAIRS_OFF, qa.SM_PAIRS_ALWAYS):
        old = qa.set_sm_pairs(mode)
        try:
            res[mode] = qa.qkv_proj_norm_rope(t["x"], t["w_qkv"], t["q_norm_w"], t["k_norm_w"], t["pos"], Hq, Hkv)
            torch.cuda.synchronize()
            assert_status_ok()
        finally:
            qa.set_sm_pairs(old)
    for name, a, b in zip("qkv", res[qa.SM_PAIRS_OFF], res[qa.SM_PAIRS_ALWAYS]):
        assert torch.equal(a, b), f"{name}: max diff {(a.float() - b.float()).abs().max().item():.3e}"


def test_qkv_proj_full_size_4b_sampled_rows():
    """The 4B-shaped projection (M=8192, hidden=2560, 48 heads) at full size, checked on 640
    sampled token rows (every row's output depends on that row alone): rows of both CTAs of
    several SM pairs, the first and the last token tile."""
    shape = QKV_SHAPES["qwen3-4b-qkv"]
    inp = qkv_proj_inputs(shape, seed=3)
    d = dev()
    t = {k: v.to(d) for k, v in inp.items()}
    q, k, v = qa.qkv_proj_norm_rope(t["x"], t["w_qkv"], t["q_norm_w"], t["k_norm_w"], t["pos"], shape.Hq, shape.Hkv)
    torch.cuda.synchronize()
    assert_status_ok()
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([np.arange(128), np.arange(shape.M - 128, shape.M),
                                     rng.choice(shape.M, size=384, replace=False)]))
    ref = oracle.qkv_proj_norm_rope_ref(as_f64(inp["x"])[rows], as_f64(inp["w_qkv"]), as_f64(inp["q_norm_w"]),
                                        as_f64(inp["k_norm_w"]), inp["pos"].numpy()[rows], shape.Hq, shape.Hkv,
                                        THETA, EPS)
    got = tuple(to_np(a)[rows] for a in (q, k, v))
    _check(got, ref, shape.name + " (sampled rows)")


def test_qkv_proj_rope_variant_and_positions():
    shape = QkvShape("qkv variant", 384, 256, 8, 4)
    i = np.arange(64, dtype=np.float64)
    inv = (1e6 ** (-2.0 * i / 128)) / np.where(i > 40, 4.0, 1.0)  # a rescaled table
    pos = torch.from_numpy(np.random.default_rng(5).integers(0, 40000, size=384).astype(np.int32))
    got, ref = _run(shape, seed=7, inv_freq=inv, scaling=1.1, pos=pos)
    _check(got, ref, "table + scaling, gapped positions")


def test_qkv_proj_feeds_the_prologue_definition():
    """Its q', k' are the normed, rotated vectors the attention entry points build from raw q
    and k: applying the standalone prologue kernel to the projection's raw output (taken
    from the oracle's fp64 product, rounded to bf16) agrees within the two bf16 roundings."""
    shape = QkvShape("qkv vs prologue", 256, 256, 4, 2)
    inp = qkv_proj_inputs(shape, seed=11)
    (q, k, v), _ = _run(shape, seed=11)
    y = as_f64(inp["x"]) @ as_f64(inp["w_qkv"]).T
    d = dev()
    qraw = torch.from_numpy(y[:, :4 * 128].reshape(1, 256, 4, 128).astype(np.float32)).to(torch.bfloat16).to(d)
    dst = torch.empty((1, 4, 256, 128), dtype=torch.bfloat16, device=d)
    qa.qk_norm_rope(qraw, inp["q_norm_w"].to(d), inp["pos"][None].to(d), dst)
    torch.cuda.synchronize()
    assert_status_ok()
    via_prologue = to_np(dst[0].permute(1, 0, 2))
    assert np.allclose(q, via_prologue, rtol=2.0 ** -6, atol=2e-2)
