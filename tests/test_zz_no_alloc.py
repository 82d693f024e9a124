"""qwen3_attn_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a plug-in handed only its input and output buffers, or a serving loop
that must not call cudaMalloc on its hot path).  Its split-KV partials live in the
library's fixed device region instead of a caller workspace.

It is checked through the C ABI against qwen3_attn_decode, the entry point that takes a
caller workspace, on two calls in a row with different lengths, so contents the first
call leaves in the shared region cannot leak into the second.  This file is collected
last so that a run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import qwen3_qk_norm_rope_b200 as qa
from synthetic import DECODE_SHAPES, decode_step_inputs
from tests.gpu_common import MAX_TOL, MEAN_TOL, assert_status_ok, dev

pytestmark = pytest.mark.gpu


def _case(N, lens, Lmax, seed):
    d = dev()
    shape = DECODE_SHAPES["batched-decode"]
    step = decode_step_inputs(shape, seed=seed)
    t = {k: (v[:N] if k in ("q", "k_new", "v_new") else v).contiguous().to(d) for k, v in step.items()}
    t["cache_lens"] = torch.tensor(lens, dtype=torch.int32, device=d)
    g = torch.Generator(device=d)
    g.manual_seed(seed)
    kc = torch.randn((N, shape.Hkv, Lmax, 128), generator=g, device=d).to(torch.bfloat16)
    vc = torch.randn((N, shape.Hkv, Lmax, 128), generator=g, device=d).to(torch.bfloat16)
    return t, kc, vc


def _both(t, kc, vc):
    N, Hq = t["q"].shape[0], t["q"].shape[1]
    d = t["q"].device
    lse_ref = torch.empty((N, Hq), dtype=torch.float32, device=d)
    ref = qa.decode(t["q"], t["k_new"], t["v_new"], t["q_norm_w"], t["k_norm_w"], kc, vc, t["cache_lens"],
                    lse=lse_ref)
    out = torch.full_like(ref, float("nan"))
    lse = torch.full_like(lse_ref, float("nan"))
    qa.decode_noalloc(t["q"], t["k_new"], t["v_new"], t["q_norm_w"], t["k_norm_w"], kc, vc, t["cache_lens"],
                      out=out, lse=lse)
    torch.cuda.synchronize()
    assert_status_ok()
    return out, lse, ref, lse_ref


def test_decode_noalloc_matches_workspace_entry_point_on_two_calls():
    Lmax = 32769
    runs = [(_case(16, [int(x) for x in np.random.default_rng(1).integers(1024, 32768, 16)], Lmax, 3)),
            (_case(9, [0, 1, 63, 1023, 1024, 4095, 20000, 32767, 32768], Lmax, 4))]
    for i, (t, kc, vc) in enumerate(runs):
        out, lse, ref, lse_ref = _both(t, kc, vc)
        err = (out.float() - ref.float()).abs()
        assert torch.isfinite(out.float()).all(), f"call {i}: non-finite output"
        assert err.max().item() <= MAX_TOL and err.mean().item() <= MEAN_TOL, f"call {i}: {err.max().item():.3e}"
        assert (lse - lse_ref).abs().max().item() <= 1e-3, f"call {i}: lse"


def test_decode_noalloc_rejects_requests_beyond_its_region():
    d = dev()
    shape = DECODE_SHAPES["batched-decode"]
    N, Lmax = 128, 32769  # needs about 70 MB of partials, more than the 48 MiB region
    assert qa.decode_workspace_size(N, shape.Hq, Lmax) > qa.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((N, shape.Hq, 128), dtype=torch.bfloat16, device=d)
    kv = torch.zeros((N, shape.Hkv, 128), dtype=torch.bfloat16, device=d)
    w = torch.ones(128, dtype=torch.float32, device=d)
    cache = torch.zeros((N, shape.Hkv, 1, 128), dtype=torch.bfloat16, device=d).expand(N, shape.Hkv, Lmax, 128)
    lens = torch.zeros(N, dtype=torch.int32, device=d)
    out = torch.empty_like(q)
    st = qa.lib().qwen3_attn_decode_noalloc(q.data_ptr(), kv.data_ptr(), kv.data_ptr(), w.data_ptr(), w.data_ptr(),
                                            cache.data_ptr(), cache.data_ptr(), lens.data_ptr(), out.data_ptr(),
                                            None, N, shape.Hq, shape.Hkv, 128, Lmax, 1e6, 1e-6, None)
    assert st == qa.ERR_WORKSPACE
