"""The running-max softmax of the prefill kernel, held to the stated tolerances against the
pure fp64 oracle.

The kernel has two softmax paths that compute the same function ("Assembling a large model
from scratch", Attention.forward: fp32 softmax over the masked scores; the online
logsumexp of "Qwen3 Architecture Layer-by-Layer", Liger fused linear cross-entropy).  When
the gains bound every logit (QK-Norm fixes each head vector's RMS, "Qwen3 Architecture
Layer-by-Layer", Qwen3RMSNorm), that bound is the reference exponent; larger gains, such as
trained q_norm/k_norm weights can have, take the running-max path (a row max per key tile
and a lazy rescale of the accumulator).  The default inputs (gains 1 + 0.1 N(0,1)) never
reach that path on their own, so these tests force it with the library's test hook
(qwen3_attn_set_softmax_path) and hold it to the same bounds as the default path: outputs
within max 2e-2 / mean 2e-3 of the pure oracle, the LSE within 1e-3 of the staged oracle
(and within 1e-2 of the pure one, or its rigorous per-row bound where rows see few keys).
"""
import numpy as np
import pytest
import torch

import qwen3_qk_norm_rope_b200 as qa
from synthetic import PREFILL_SHAPES, ChunkShape, PrefillShape, chunk_inputs, prefill_inputs
from tests.gpu_common import (check_lse_straddle, compare, prefill_gpu, prefill_lse_bound, prefill_oracle,
                              to_np)
from tests.test_gpu_chunk import _caches, _oracle, _run
from tests.test_gpu_prefill import _sampled_rows
from tests.test_gpu_variants import _prefill_case

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def running_max_path():
    old = qa.set_softmax_path(qa.SOFTMAX_RUNNING_MAX)
    yield
    qa.set_softmax_path(old)


@pytest.mark.parametrize("name", ["tiny", "qwen3-0.6b", "qwen3-4b"])
def test_running_max_full_parity(name):
    inp = prefill_inputs(PREFILL_SHAPES[name], seed=0)
    out, lse = prefill_gpu(inp)
    ref, ref_lse, st_lse = prefill_oracle(inp)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, name + ", running max")


def test_running_max_long_wide_gqa_sampled_rows():
    shape = PREFILL_SHAPES["long-wide-gqa"]
    inp = prefill_inputs(shape, seed=0)
    out, lse = prefill_gpu(inp)
    rows = _sampled_rows(shape.T, 256, 1024, 256, seed=1)
    ref, ref_lse, st_lse = prefill_oracle(inp, rows=rows)
    idx = torch.from_numpy(rows).to(out.device)
    compare(to_np(out[:, idx]), None, ref, None, None, "long-wide-gqa sampled rows, running max")
    check_lse_straddle(to_np(lse[:, :, idx]), ref_lse, st_lse, prefill_lse_bound(inp, rows),
                       "long-wide-gqa sampled rows, running max")
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("B,start,T,Hq,Hkv,slack", [(2, 200, 300, 16, 8, 40), (1, 9000, 40, 32, 8, 100),
                                                    (2, 333, 517, 64, 4, 11)])
def test_running_max_chunk(B, start, T, Hq, Hkv, slack):
    shape = ChunkShape("chunk", B, start, T, Hq, Hkv)
    inp = chunk_inputs(shape, seed=start + T)
    kc, vc = _caches(inp, shape, start + T + slack)
    out, lse, _, _ = _run(inp, shape, kc, vc)
    ref, ref_lse, _, st_lse = _oracle(inp, shape, kc, vc)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, f"chunk B{B} start{start} T{T} Hq{Hq}, running max")


@pytest.mark.parametrize("B,T,Hq,Hkv,window", [(1, 900, 32, 8, 100), (1, 1000, 16, 1, 300), (1, 777, 32, 8, 513)])
def test_running_max_window(B, T, Hq, Hkv, window):
    """Windows leave the first key tiles of an item wholly outside some rows' windows: those
    rows have no max yet and must keep p = 0."""
    out, lse, ref, ref_lse, _, st_lse = _prefill_case(B, T, Hq, Hkv, seed=T + window, window=window)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, f"window {window} B{B} T{T} Hq{Hq}, running max")


def test_hook_switches_the_path():
    """The two paths round P to bf16 against different reference exponents, so the forced
    path gives other bits than the default one; both are the same softmax within the
    tolerances."""
    inp = prefill_inputs(PREFILL_SHAPES["qwen3-0.6b"], seed=0)
    out_r, lse_r = prefill_gpu(inp)
    qa.set_softmax_path(qa.SOFTMAX_AUTO)
    out_f, lse_f = prefill_gpu(inp)
    assert not torch.equal(out_r, out_f)
    diff = (out_r.float() - out_f.float()).abs()
    assert diff.max().item() <= 2e-2 and diff.mean().item() <= 2e-3
    assert (lse_r - lse_f).abs().max().item() <= 1e-3
