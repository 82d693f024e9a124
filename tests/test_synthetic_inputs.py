"""The seeded input recipe that every parity case and benchmark draws from: q and k are
N(0,1) times per-channel scales that are log-uniform in [0.5, 4], v is unscaled, the
QK-Norm gains are 1 + 0.1 N(0,1) in fp32, positions run 0..T-1, cached decode lengths are
uniform in [1024, 32768], all values are bf16, and the same seed gives the same tensors."""
import numpy as np
import torch

from synthetic import (CHUNK_SHAPES, DECODE_SHAPES, VARLEN_SHAPES, PrefillShape, chunk_inputs, decode_step_inputs,
                       prefill_inputs, varlen_inputs)


def _channel_rms(t: torch.Tensor) -> np.ndarray:
    x = t.float().numpy().reshape(-1, t.shape[-1])
    return np.sqrt(np.mean(x * x, axis=0))


def test_prefill_recipe():
    shape = PrefillShape("recipe", 2, 512, 16, 8)
    inp = prefill_inputs(shape, seed=0)
    assert inp["q"].dtype == inp["k"].dtype == inp["v"].dtype == torch.bfloat16
    assert tuple(inp["q"].shape) == (2, 512, 16, 128) and tuple(inp["k"].shape) == (2, 512, 8, 128)
    assert inp["q_norm_w"].dtype == torch.float32 and tuple(inp["q_norm_w"].shape) == (128,)
    assert inp["pos"].dtype == torch.int32 and torch.equal(inp["pos"], torch.arange(512, dtype=torch.int32).repeat(2, 1))
    # per-channel scales: 16384 (q) and 8192 (k) samples per channel estimate each scale to ~1%
    for name in ("q", "k"):
        s = _channel_rms(inp[name])
        assert s.min() > 0.5 * 0.95 and s.max() < 4.0 * 1.05, name
        # log-uniform: the log-scales spread over [ln 0.5, ln 4] with mean near their midpoint
        ls = np.log(s)
        assert abs(ls.mean() - 0.5 * (np.log(0.5) + np.log(4.0))) < 0.2
        assert ls.max() - ls.min() > 0.8 * (np.log(4.0) - np.log(0.5))
    assert np.all(np.abs(_channel_rms(inp["v"]) - 1.0) < 0.05)  # v carries no scale
    # q and k draw their scale vectors independently
    assert np.corrcoef(_channel_rms(inp["q"]), _channel_rms(inp["k"]))[0, 1] < 0.5
    for g in (inp["q_norm_w"].numpy(), inp["k_norm_w"].numpy()):
        assert abs(g.mean() - 1.0) < 0.05 and 0.07 < g.std() < 0.13


def test_same_seed_same_inputs():
    shape = PrefillShape("seeds", 1, 64, 4, 2)
    a, b, c = prefill_inputs(shape, seed=3), prefill_inputs(shape, seed=3), prefill_inputs(shape, seed=4)
    for key in a:
        assert torch.equal(a[key], b[key]), key
    assert not torch.equal(a["q"], c["q"])


def test_decode_recipe():
    shape = DECODE_SHAPES["batched-decode"]
    step = decode_step_inputs(shape, seed=0)
    lens = step["cache_lens"].numpy()
    assert lens.dtype == np.int32 and lens.shape == (64,)
    assert lens.min() >= 1024 and lens.max() <= 32768
    assert shape.cache_capacity >= lens.max() + 1  # room for the appended token
    assert tuple(step["q"].shape) == (64, 32, 128) and tuple(step["k_new"].shape) == (64, 8, 128)
    assert torch.equal(step["cache_lens"], decode_step_inputs(shape, seed=0)["cache_lens"])


def test_chunk_is_the_tail_of_one_prompt():
    shape = CHUNK_SHAPES["qwen3-4b-second-chunk"]
    small = type(shape)(shape.name, 1, 48, 80, shape.Hq, shape.Hkv)
    ch = chunk_inputs(small, seed=5)
    full = prefill_inputs(PrefillShape("full", 1, 48 + 80, shape.Hq, shape.Hkv), seed=5)
    assert torch.equal(torch.cat([ch["k_hist"], ch["k"]], dim=1), full["k"])
    assert torch.equal(torch.cat([ch["v_hist"], ch["v"]], dim=1), full["v"])
    assert torch.equal(ch["q"], full["q"][:, 48:]) and torch.equal(ch["pos"], full["pos"][:, 48:])


def test_varlen_packing():
    for shape in VARLEN_SHAPES.values():
        inp = varlen_inputs(shape, seed=0)
        cu = inp["cu_seqlens"].numpy()
        assert cu[0] == shape.lead and np.array_equal(np.diff(cu), np.asarray(shape.lens))
        assert cu[-1] + shape.tail == shape.N == inp["q"].shape[0]
        pos = inp["pos"].numpy()
        for b, (T, c) in enumerate(zip(shape.lens, shape.contexts)):
            assert np.array_equal(pos[cu[b]:cu[b + 1]], c + np.arange(T))
            assert inp["k_hist"][b].shape[0] == c
