"""Shared helpers of the GPU parity tests: run the CUDA path through the binding (C ABI)
and compare with the fp64 oracle on the same seeded inputs.

Tolerances (bf16 outputs, fp32 softmax statistics): max |out - oracle| <= 2e-2 and mean
<= 2e-3 against the pure fp64 oracle; |lse - oracle| <= 1e-3 against the oracle's staged
mode, which rounds q' and k' to bf16 once after RoPE as the kernels do before their bf16
MMAs (a single bf16 rounding of q', k' moves a logit by ~1.6e-3 RMS, which is why the
pure-oracle LSE error is reported but bounded only loosely).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import qwen3_qk_norm_rope_b200 as qa
from synthetic import as_f64

MAX_TOL, MEAN_TOL, LSE_TOL = 2e-2, 2e-3, 1e-3
LSE_PURE_TOL = 1e-2


def dev():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    return torch.device("cuda", 0)


def assert_status_ok():
    st, site = qa.device_status(clear=True)
    assert st == qa.OK, f"device status {qa.status_string(st)} at site {site}"


def prefill_gpu(inp: dict, theta=1e6, eps=1e-6, want_lse=True, caches=None):
    d = dev()
    t = {k: v.to(d) for k, v in inp.items()}
    B, T, Hq, _ = t["q"].shape
    lse = torch.full((B, Hq, T), float("nan"), dtype=torch.float32, device=d) if want_lse else None
    kc = vc = None
    if caches is not None:
        kc, vc = caches
    out = qa.prefill(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], theta=theta, eps=eps, lse=lse,
                     k_cache=kc, v_cache=vc)
    torch.cuda.synchronize()
    assert_status_ok()
    return out, lse


def prefill_oracle(inp: dict, theta=1e6, eps=1e-6, rows=None):
    args = (as_f64(inp["q"]), as_f64(inp["k"]), as_f64(inp["v"]), as_f64(inp["q_norm_w"]),
            as_f64(inp["k_norm_w"]), inp["pos"].numpy(), theta, eps)
    ref, ref_lse = oracle.prefill_ref(*args, rows=rows)
    _, st_lse = oracle.prefill_ref(*args, rows=rows, staged=True)
    return ref, ref_lse, st_lse


def compare(out: np.ndarray, lse, ref, ref_lse, st_lse, what: str, lse_tol: float = LSE_TOL,
            lse_pure_tol: float = LSE_PURE_TOL):
    err = np.abs(out - ref)
    msg = f"{what}: max {err.max():.3e} mean {err.mean():.3e}"
    assert np.isfinite(out).all(), what + ": non-finite output"
    assert err.max() <= MAX_TOL and err.mean() <= MEAN_TOL, msg
    if lse is not None:
        e_st = np.abs(lse - st_lse).max()
        e_pure = np.abs(lse - ref_lse).max()
        assert e_st <= lse_tol, f"{what}: lse vs staged oracle {e_st:.3e}"
        assert e_pure <= lse_pure_tol, f"{what}: lse vs pure oracle {e_pure:.3e}"
    return err.max(), err.mean()


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
