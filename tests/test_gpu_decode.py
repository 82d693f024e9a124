"""Decode parity: append + split-KV attention + LSE combine (through the C ABI) against the
fp64 oracle, on caches the oracle builds from seeded raw histories.  Stale cache slots are
filled with NaN patterns, so any read past a sequence's end would show."""
import numpy as np
import pytest
import torch

import oracle
import qwen3_qk_norm_rope_b200 as qa
from synthetic import DECODE_SHAPES, DecodeShape, as_f64, decode_history, decode_step_inputs, prefill_inputs, \
    PrefillShape
from tests.gpu_common import (LSE_PURE_TOL, LSE_TOL, MAX_TOL, MEAN_TOL, assert_status_ok, dev, prefill_gpu,
                              to_np)

pytestmark = pytest.mark.gpu
NAN16 = 0x7FC1


def _setup(shape: DecodeShape, lens, Lmax, seed, checked):
    """Inputs, device caches (oracle-built for the `checked` sequences, random for the rest,
    NaN in every slot >= L), and the host copies the oracle needs."""
    d = dev()
    step = decode_step_inputs(shape, seed=seed)
    step["cache_lens"] = torch.as_tensor(np.asarray(lens, dtype=np.int32))
    N, Hkv = shape.N, shape.Hkv
    kc = torch.empty((N, Hkv, Lmax, 128), dtype=torch.bfloat16, device=d)
    vc = torch.empty_like(kc)
    kc.view(torch.int16).fill_(NAN16)
    vc.view(torch.int16).fill_(NAN16)
    g = torch.Generator(device=d)
    g.manual_seed(seed)
    host = {}
    gk = as_f64(step["k_norm_w"])
    for n in range(N):
        L = int(lens[n])
        if L < 0 or L >= Lmax:
            continue
        if n in checked:
            hist = decode_history(shape, n, L, step["s_k"], seed=seed)
            kcache = oracle.build_cache_k(as_f64(hist["k_hist"]), gk, shape.theta, shape.eps)  # [L,Hkv,d]
            kc[n, :, :L] = torch.from_numpy(kcache.transpose(1, 0, 2)).to(torch.bfloat16).to(d)
            vc[n, :, :L] = hist["v_hist"].permute(1, 0, 2).to(d)
            host[n] = (kcache.transpose(1, 0, 2), as_f64(hist["v_hist"]).transpose(1, 0, 2))
        elif L > 0:
            kc[n, :, :L] = torch.randn((Hkv, L, 128), generator=g, device=d).to(torch.bfloat16)
            vc[n, :, :L] = torch.randn((Hkv, L, 128), generator=g, device=d).to(torch.bfloat16)
    return step, kc, vc, host


def _run(shape, step, kc, vc, Lmax):
    d = dev()
    t = {k: v.to(d) for k, v in step.items()}
    lse = torch.full((shape.N, shape.Hq), float("nan"), dtype=torch.float32, device=d)
    out = qa.decode(t["q"], t["k_new"], t["v_new"], t["q_norm_w"], t["k_norm_w"], kc, vc, t["cache_lens"],
                    theta=shape.theta, eps=shape.eps, lse=lse)
    torch.cuda.synchronize()
    return out, lse


def _check(shape, step, out, lse, kc, vc, host, what):
    gq, gk = as_f64(step["q_norm_w"]), as_f64(step["k_norm_w"])
    lens = step["cache_lens"].numpy()
    for n, (kh, vh) in host.items():
        L = int(lens[n])
        args = (as_f64(step["q"])[n:n + 1], as_f64(step["k_new"])[n:n + 1], as_f64(step["v_new"])[n:n + 1], gq, gk,
                [kh], [vh], [L], shape.theta, shape.eps)
        ref, ref_lse = oracle.decode_ref(*args)
        _, st_lse = oracle.decode_ref(*args, staged=True)
        o = to_np(out[n:n + 1])
        err = np.abs(o - ref)
        assert np.isfinite(o).all(), f"{what} seq {n}: non-finite"
        assert err.max() <= MAX_TOL and err.mean() <= MEAN_TOL, f"{what} seq {n} L={L}: {err.max():.3e}"
        l = to_np(lse[n:n + 1])
        assert np.abs(l - st_lse).max() <= LSE_TOL, f"{what} seq {n}: lse {np.abs(l - st_lse).max():.3e}"
        assert np.abs(l - ref_lse).max() <= LSE_PURE_TOL
        # the appended slot: normed+rotated new key, raw new value
        kref = oracle.qk_prologue(as_f64(step["k_new"])[n][None], gk, np.array([L]), shape.theta, shape.eps)[0]
        kgot = to_np(kc[n, :, L])
        assert np.all(np.abs(kgot - kref) <= np.abs(kref) * 2.0 ** -8 + 2e-5)
        assert torch.equal(vc[n, :, L].cpu(), step["v_new"][n])


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (16, 16), (64, 4), (8, 4)])
def test_decode_small_edge_lengths(Hq, Hkv):
    Lmax = 3000
    shape = DecodeShape("small", 6, Hq, Hkv, lmin=0, lmax=Lmax - 1)
    lens = [0, 1, 63, 1023, 1024, Lmax - 1]  # empty history, split and chunk boundaries, full cache
    step, kc, vc, host = _setup(shape, lens, Lmax, seed=Hq + Hkv, checked=set(range(6)))
    out, lse = _run(shape, step, kc, vc, Lmax)
    assert_status_ok()
    _check(shape, step, out, lse, kc, vc, host, f"Hq{Hq} Hkv{Hkv}")


def test_decode_batched_full_size_all_sequences():
    """The batched-decode workload at full size (64 sequences, L ~ U[1024, 32768]), every
    sequence checked against the oracle.  Four sequences (the longest, the shortest and two
    seeded picks) carry caches the oracle builds from raw histories (normed, rotated keys);
    the other 60 carry random bf16 caches, which the oracle reads back from the device one
    sequence at a time as its cache history."""
    shape = DECODE_SHAPES["batched-decode"]
    Lmax = shape.cache_capacity
    step0 = decode_step_inputs(shape, seed=0)
    lens = step0["cache_lens"].numpy()
    rng = np.random.default_rng(2)
    checked = {int(np.argmax(lens)), int(np.argmin(lens))} | set(int(x) for x in rng.choice(64, 2, replace=False))
    step, kc, vc, host = _setup(shape, lens, Lmax, seed=0, checked=checked)
    out, lse = _run(shape, step, kc, vc, Lmax)
    assert_status_ok()
    assert torch.isfinite(out.float()).all()
    _check(shape, step, out, lse, kc, vc, host, "batched-decode")
    for n in range(shape.N):
        if n in checked:
            continue
        L = int(lens[n])
        one = {n: (to_np(kc[n, :, :L]), to_np(vc[n, :, :L]))}
        _check(shape, step, out, lse, kc, vc, one, "batched-decode random cache")


def test_decode_after_prefill_equals_last_prefill_row():
    """Prefill T tokens into a cache, then decode token T: equals row T of a prefill over
    T+1 tokens (oracle) and agrees with the GPU prefill of T+1 tokens."""
    d = dev()
    T, Hq, Hkv = 700, 32, 8
    full = prefill_inputs(PrefillShape("p", 1, T + 1, Hq, Hkv), seed=11)
    head = {k: (v[:, :T].contiguous() if k in ("q", "k", "v", "pos") else v) for k, v in full.items()}
    Lmax = 1024
    kc = torch.empty((1, Hkv, Lmax, 128), dtype=torch.bfloat16, device=d)
    vc = torch.empty_like(kc)
    kc.view(torch.int16).fill_(NAN16)
    vc.view(torch.int16).fill_(NAN16)
    prefill_gpu(head, caches=(kc, vc))
    t = {k: v.to(d) for k, v in full.items()}
    lens = torch.tensor([T], dtype=torch.int32, device=d)
    lse = torch.empty((1, Hq), dtype=torch.float32, device=d)
    out = qa.decode(t["q"][:, T].contiguous(), t["k"][:, T].contiguous(), t["v"][:, T].contiguous(),
                    t["q_norm_w"], t["k_norm_w"], kc, vc, lens, lse=lse)
    torch.cuda.synchronize()
    assert_status_ok()
    rows = np.array([T])
    ref, ref_lse = oracle.prefill_ref(as_f64(full["q"]), as_f64(full["k"]), as_f64(full["v"]),
                                      as_f64(full["q_norm_w"]), as_f64(full["k_norm_w"]), full["pos"].numpy(),
                                      1e6, 1e-6, rows=rows)
    err = np.abs(to_np(out) - ref[0, 0])
    assert err.max() <= MAX_TOL and err.mean() <= MEAN_TOL
    assert np.abs(to_np(lse)[0] - ref_lse[0, :, 0]).max() <= LSE_PURE_TOL
    out_p, _ = prefill_gpu(full)
    assert (out_p[0, T].float() - out[0].float()).abs().max().item() <= 2 * MAX_TOL


def test_decode_rejects_out_of_range_length_on_device():
    """A sequence with L >= Lmax is skipped and reported; the others are still computed."""
    Lmax = 2048
    shape = DecodeShape("bad", 3, 32, 8, lmin=0, lmax=Lmax - 1)
    lens = [500, Lmax, 1500]
    step, kc, vc, host = _setup(shape, lens, Lmax, seed=4, checked={0, 2})
    out, lse = _run(shape, step, kc, vc, Lmax)
    st, site = qa.device_status(clear=True)
    assert st == qa.ERR_INVALID_ARG, (st, site)
    _check(shape, step, out, lse, kc, vc, host, "with a bad length")
