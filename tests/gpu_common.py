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

# Every comparison appends its maxima here; tests/conftest.py prints the table at the end of
# the run, so each workload's errors against the pure and the staged oracle are on record.
PARITY_LOG: list = []


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


def record(what: str, **vals):
    PARITY_LOG.append(dict(what=what, **{k: (None if v is None else float(v)) for k, v in vals.items()}))


def compare(out: np.ndarray, lse, ref, ref_lse, st_lse, what: str, lse_tol: float = LSE_TOL,
            lse_pure_tol: float = LSE_PURE_TOL, max_tol: float = MAX_TOL, mean_tol: float = MEAN_TOL,
            lse_pure_bound=None):
    """Outputs against `ref` (the pure oracle unless a caller says otherwise), the LSE against
    the staged oracle (st_lse) and the pure one (ref_lse): within lse_pure_tol, or row by row
    within the array lse_pure_bound when one is given."""
    err = np.abs(out - ref)
    msg = f"{what}: max {err.max():.3e} mean {err.mean():.3e}"
    assert np.isfinite(out).all(), what + ": non-finite output"
    e_st = e_pure = None
    if lse is not None:
        e_st = np.abs(lse - st_lse).max()
        e_pure = np.abs(lse - ref_lse).max()
    record(what, out_max=err.max(), out_mean=err.mean(), lse_pure=e_pure, lse_staged=e_st)
    assert err.max() <= max_tol and err.mean() <= mean_tol, msg
    if lse is not None:
        assert e_st <= lse_tol, f"{what}: lse vs staged oracle {e_st:.3e}"
        if lse_pure_bound is None:
            assert e_pure <= lse_pure_tol, f"{what}: lse vs pure oracle {e_pure:.3e}"
        else:
            over = np.abs(lse - ref_lse) - lse_pure_bound
            assert np.all(over <= 0), f"{what}: lse vs pure oracle {over.max():.3e} over the rigorous bound"
    return err.max(), err.mean()


# The straddle rule for LSE checks over many rows that see few keys.  Against the staged
# oracle (q', k' rounded to bf16 as the kernels round them) the kernel differs only where its
# fp32 q' or k' element lands on the other side of a bf16 rounding boundary: rare, and one
# bf16 ulp (at most 2^-7 of the element) moves a logit by at most 2^-7 |q'_i k'_i| / sqrt(d),
# which reaches the LSE in a row whose softmax that key dominates.  Such rows
# (the first rows of a causal prefill) may reach STRADDLE_TOL on at most STRADDLE_FRACTION of
# the row-heads; the rest stay within LSE_TOL.  Against the pure oracle every row is held to
# the rigorous bound of prefill_lse_bound.
STRADDLE_TOL, STRADDLE_FRACTION = 4e-3, 1e-4


def lse_bound(qp_abs: np.ndarray, kp_abs: np.ndarray, visible: np.ndarray, G: int) -> np.ndarray:
    """The rigorous per-row LSE bound of prefill_lse_bound for one batch row, from the
    magnitudes of the exact normed, rotated queries [R, Hq, d] and keys [S, Hkv, d] and the
    [R, S] mask of keys each row sees; [Hq, R].  Keys that are already bf16 (a cache) are
    not rounded again, so the bound holds for them too, with room to spare."""
    R, Hq, d = qp_abs.shape
    out = np.empty((Hq, R))
    for h in range(Hq):
        a = np.where(visible, qp_abs[:, h] @ kp_abs[:, h // G].T, 0.0)
        out[h] = (2.0 ** -7 + 2.0 ** -15) * a.max(-1) / np.sqrt(d) + 1e-5 + visible.sum(-1) * 2.0 ** -24
    return out


def prefill_lse_bound(inp: dict, rows: np.ndarray, theta=1e6, eps=1e-6, window: int = 0) -> np.ndarray:
    """Rigorous bound on |LSE_kernel - LSE_pure| for query rows `rows` of a uniform causal
    prefill, [B, Hq, len(rows)].  The LSE is 1-Lipschitz in the largest change of any
    logit.  Rounding q' and k' to bf16 (unit roundoff u = 2^-8 each) changes each product
    q'_i k'_ji by at most (2u + u^2) |q'_i k'_ji|, and fp32 accumulation of the 128 products
    adds at most 128 x 2^-24 = 2^-17 of sum_i |q'_i k'_ji|: together less than
    (2^-7 + 2^-15) sum_i |q'_i k'_ji| / sqrt(d) on logit j.  The fp32 softmax sum adds at
    most keys x 2^-24."""
    B, T, Hq, d = inp["q"].shape
    G = Hq // inp["k"].shape[2]
    gq, gk = as_f64(inp["q_norm_w"]), as_f64(inp["k_norm_w"])
    bound = np.empty((B, Hq, len(rows)))
    for b in range(B):
        pos = inp["pos"][b].numpy()
        qp = np.abs(oracle.qk_prologue(as_f64(inp["q"][b, torch.from_numpy(rows)]), gq, pos[rows], theta, eps))
        kp = np.abs(oracle.qk_prologue(as_f64(inp["k"][b]), gk, pos, theta, eps))  # [T, Hkv, d]
        j = np.arange(T)[None, :]
        visible = j <= rows[:, None]
        if window:
            visible &= j > rows[:, None] - window
        bound[b] = lse_bound(qp, kp, visible, G)
    return bound


def chunk_lse_bound(inp: dict, start: int, k_cached: np.ndarray, rows=None, theta=1e6, eps=1e-6,
                    window: int = 0) -> np.ndarray:
    """prefill_lse_bound for a chunk of T new rows over `start` cached keys (k_cached
    [B, Hkv, start, d], already normed, rotated and bf16): row i sees keys j <= start + i
    (and j > start + i - window with a window).  [B, Hq, len(rows)]."""
    B, T, Hq, d = inp["q"].shape
    G = Hq // inp["k"].shape[2]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    gq, gk = as_f64(inp["q_norm_w"]), as_f64(inp["k_norm_w"])
    bound = np.empty((B, Hq, len(rows)))
    for b in range(B):
        pos = inp["pos"][b].numpy()
        qp = np.abs(oracle.qk_prologue(as_f64(inp["q"][b, torch.from_numpy(rows)]), gq, pos[rows], theta, eps))
        kn = np.abs(oracle.qk_prologue(as_f64(inp["k"][b]), gk, pos, theta, eps))  # [T, Hkv, d]
        kp = np.concatenate([np.abs(k_cached[b]).transpose(1, 0, 2), kn], axis=0)  # [start + T, Hkv, d]
        j = np.arange(start + T)[None, :]
        i = start + rows[:, None]
        visible = j <= i
        if window:
            visible &= j > i - window
        bound[b] = lse_bound(qp, kp, visible, G)
    return bound


def check_lse_straddle(lse: np.ndarray, ref_lse, st_lse, bound, what: str):
    """The LSE by the rigorous bound against the pure oracle and by the straddle rule
    against the staged one."""
    e_pure = np.abs(lse - ref_lse)
    e_st = np.abs(lse - st_lse)
    record(what + " (lse)", lse_pure=e_pure.max(), lse_staged=e_st.max())
    assert np.all(e_pure <= bound), f"{what}: lse vs pure oracle {(e_pure - bound).max():.3e} over the rigorous bound"
    assert e_st.max() <= STRADDLE_TOL, f"{what}: lse vs staged oracle {e_st.max():.3e}"
    frac = float(np.mean(e_st > LSE_TOL))
    assert frac <= STRADDLE_FRACTION, f"{what}: {frac:.2e} of row-heads over {LSE_TOL} against the staged oracle"
    return e_st.max(), frac


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
