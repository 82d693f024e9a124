"""qwen3_attn_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a plug-in handed only its input and output buffers, or a serving loop
that must not call cudaMalloc on its hot path).  Its split-KV partials live in the
library's fixed device region instead of a caller workspace.

It is checked through the C ABI against qwen3_attn_decode, the entry point that takes a
caller workspace, on three calls in a row with different sizes (the last one smaller, so
its partials sit in a region the earlier calls left full of their own), so contents a call
leaves in the shared region cannot leak into the next.  Both entry points run the same
kernels with the same split layout, so their outputs must agree bit for bit.  One sequence
is also checked against the fp64 oracle.  This file is collected last so that a run
stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import qwen3_qk_norm_rope_b200 as qa
from synthetic import DECODE_SHAPES, as_f64, decode_step_inputs
from tests.gpu_common import LSE_PURE_TOL, LSE_TOL, MAX_TOL, MEAN_TOL, assert_status_ok, dev, to_np

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


def test_decode_noalloc_matches_workspace_entry_point_on_successive_calls():
    runs = [(_case(16, [int(x) for x in np.random.default_rng(1).integers(1024, 32768, 16)], 32769, 3)),
            (_case(9, [0, 1, 63, 1023, 1024, 4095, 20000, 32767, 32768], 32769, 4)),
            (_case(5, [700, 2047, 0, 3000, 4095], 4096, 5))]
    for i, (t, kc, vc) in enumerate(runs):
        out, lse, ref, lse_ref = _both(t, kc, vc)
        assert torch.isfinite(out.float()).all(), f"call {i}: non-finite output"
        assert torch.equal(out, ref), f"call {i}: out differs, max {(out.float() - ref.float()).abs().max().item():.3e}"
        assert torch.equal(lse, lse_ref), f"call {i}: lse differs"


def test_decode_noalloc_against_the_oracle():
    """One sequence of a no-allocation call against the fp64 oracle over the same cache
    contents (random bf16 keys and values read back from the device, the appended slot
    included)."""
    t, kc, vc = _case(4, [5000, 1500, 32768, 1], 32769, 6)
    shape = DECODE_SHAPES["batched-decode"]
    out = torch.full_like(t["q"], float("nan"))
    lse = torch.full((4, shape.Hq), float("nan"), dtype=torch.float32, device=out.device)
    qa.decode_noalloc(t["q"], t["k_new"], t["v_new"], t["q_norm_w"], t["k_norm_w"], kc, vc, t["cache_lens"],
                      out=out, lse=lse)
    torch.cuda.synchronize()
    assert_status_ok()
    for n, L in enumerate([5000, 1500, 32768, 1]):
        kh = as_f64(kc[n, :, :L].cpu())
        vh = as_f64(vc[n, :, :L].cpu())
        q, kn, vn = (as_f64(t[k][n:n + 1].cpu()) for k in ("q", "k_new", "v_new"))
        args = (q, kn, vn, as_f64(t["q_norm_w"].cpu()), as_f64(t["k_norm_w"].cpu()), [kh], [vh], [L], shape.theta,
                shape.eps)
        ref, ref_lse = oracle.decode_ref(*args)
        _, st_lse = oracle.decode_ref(*args, staged=True)
        err = np.abs(to_np(out[n:n + 1]) - ref)
        assert err.max() <= MAX_TOL and err.mean() <= MEAN_TOL, f"seq {n} L={L}: {err.max():.3e}"
        assert np.abs(to_np(lse[n:n + 1]) - st_lse).max() <= LSE_TOL
        assert np.abs(to_np(lse[n:n + 1]) - ref_lse).max() <= LSE_PURE_TOL


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
