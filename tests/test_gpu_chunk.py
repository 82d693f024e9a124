"""Chunked prefill parity: T new tokens over a KV cache that already holds `start` tokens
("Assembling a large model from scratch", Attention.forward with a cache: the mask
tril(diagonal = S - T)).  The cached prefix is built by the oracle (QK-Norm + RoPE of the
raw history, rounded to bf16); the CUDA path runs through the C ABI and is compared with
the fp64 oracle on the same inputs.  The caches are checked slot by slot afterwards."""
import numpy as np
import pytest
import torch

import oracle
import qwen3_qk_norm_rope_b200 as qa
from synthetic import CHUNK_SHAPES, ChunkShape, PrefillShape, as_f64, chunk_inputs, prefill_inputs
from tests.gpu_common import MAX_TOL, MEAN_TOL, assert_status_ok, chunk_lse_bound, compare, dev, prefill_gpu, to_np

pytestmark = pytest.mark.gpu

CANARY = 0x7FC1  # a bf16 NaN bit pattern in every slot the call must not write


def _caches(inp: dict, shape: ChunkShape, Tcap: int):
    """bf16 caches [B,Hkv,Tcap,d]: slots < start hold the oracle's cache contents (keys
    normed and rotated at 0..start-1, raw values), every other slot the canary."""
    B, Hkv, s = shape.B, shape.Hkv, shape.start
    kc = torch.empty((B, Hkv, Tcap, shape.d), dtype=torch.bfloat16)
    kc.view(torch.int16).fill_(CANARY)
    vc = kc.clone()
    gk = as_f64(inp["k_norm_w"])
    for b in range(B):
        if s:
            kb = oracle.build_cache_k(as_f64(inp["k_hist"][b]), gk, shape.theta, shape.eps)  # [s,Hkv,d]
            kc[b, :, :s] = torch.from_numpy(kb.transpose(1, 0, 2).copy()).to(torch.bfloat16)
            vc[b, :, :s] = inp["v_hist"][b].permute(1, 0, 2)
    return kc, vc


def _run(inp: dict, shape: ChunkShape, kc: torch.Tensor, vc: torch.Tensor):
    d = dev()
    t = {k: inp[k].to(d) for k in ("q", "k", "v", "q_norm_w", "k_norm_w", "pos")}
    kcd, vcd = kc.to(d), vc.to(d)
    lse = torch.full((shape.B, shape.Hq, shape.T), float("nan"), dtype=torch.float32, device=d)
    out = qa.prefill_chunk(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], kcd, vcd, shape.start,
                           theta=shape.theta, eps=shape.eps, lse=lse)
    torch.cuda.synchronize()
    assert_status_ok()
    return out, lse, kcd, vcd


def _oracle(inp: dict, shape: ChunkShape, kc: torch.Tensor, vc: torch.Tensor, rows=None):
    s = shape.start
    args = (as_f64(inp["q"]), as_f64(inp["k"]), as_f64(inp["v"]), as_f64(inp["q_norm_w"]), as_f64(inp["k_norm_w"]),
            inp["pos"].numpy(), as_f64(kc[:, :, :s]), as_f64(vc[:, :, :s]), s, shape.theta, shape.eps)
    ref, ref_lse = oracle.chunk_prefill_ref(*args, rows=rows)
    ref_st, st_lse = oracle.chunk_prefill_ref(*args, rows=rows, staged=True)
    return ref, ref_lse, ref_st, st_lse


def _check_caches(inp, shape, kc_before, vc_before, kc_after, vc_after):
    s, T = shape.start, shape.T
    ka, va = kc_after.cpu(), vc_after.cpu()
    # the cached prefix and the slots past the chunk are untouched
    assert torch.equal(ka[:, :, :s].view(torch.int16), kc_before[:, :, :s].view(torch.int16))
    assert torch.equal(va[:, :, :s].view(torch.int16), vc_before[:, :, :s].view(torch.int16))
    assert torch.equal(ka[:, :, s + T:].view(torch.int16), kc_before[:, :, s + T:].view(torch.int16))
    assert torch.equal(va[:, :, s + T:].view(torch.int16), vc_before[:, :, s + T:].view(torch.int16))
    # the new keys: QK-Norm + RoPE at their positions, one bf16 rounding; values bit-exact
    kref = oracle.qk_prologue(as_f64(inp["k"]), as_f64(inp["k_norm_w"]), inp["pos"].numpy(), shape.theta, shape.eps)
    kgot = to_np(ka[:, :, s:s + T].permute(0, 2, 1, 3))
    assert np.all(np.abs(kgot - kref) <= np.abs(kref) * 2.0 ** -8 + 2e-5), np.abs(kgot - kref).max()
    assert torch.equal(va[:, :, s:s + T].permute(0, 2, 1, 3), inp["v"])


CASES = [
    # (B, start, T, Hq, Hkv, slack): start and T off the tile grid, G in {1, 2, 4, 16, 32},
    # one-token chunks (a decode step through the prefill kernel), a short chunk over a long
    # prefix (few work items, many key tiles each), B > 1
    (2, 200, 300, 16, 8, 40),
    (1, 128, 128, 8, 8, 0),
    (1, 1000, 77, 32, 1, 5),
    (3, 1500, 1, 32, 8, 3),
    (1, 9000, 40, 32, 8, 100),
    (2, 333, 517, 64, 4, 11),
]


@pytest.mark.parametrize("B,start,T,Hq,Hkv,slack", CASES)
def test_chunk_parity(B, start, T, Hq, Hkv, slack):
    shape = ChunkShape("chunk", B, start, T, Hq, Hkv)
    inp = chunk_inputs(shape, seed=start + T)
    kc, vc = _caches(inp, shape, start + T + slack)
    out, lse, kca, vca = _run(inp, shape, kc, vc)
    ref, ref_lse, _, st_lse = _oracle(inp, shape, kc, vc)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, f"chunk B{B} start{start} T{T} Hq{Hq} Hkv{Hkv}")
    _check_caches(inp, shape, kc, vc, kca, vca)


def test_chunk_full_size_sampled_rows():
    shape = CHUNK_SHAPES["qwen3-4b-second-chunk"]
    inp = chunk_inputs(shape, seed=0)
    kc, vc = _caches(inp, shape, shape.start + shape.T)
    out, lse, _, _ = _run(inp, shape, kc, vc)
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([np.arange(128), rng.choice(np.arange(128, shape.T - 128), 256, replace=False),
                                     np.arange(shape.T - 128, shape.T)]))
    ref, ref_lse, _, st_lse = _oracle(inp, shape, kc, vc, rows=rows)
    idx = torch.from_numpy(rows).to(out.device)
    compare(to_np(out[:, idx]), to_np(lse[:, :, idx]), ref, ref_lse, st_lse, "4B second chunk, sampled rows")
    assert torch.isfinite(out.float()).all()


def test_chunk_over_empty_cache_equals_prefill_into_cache():
    shape = ChunkShape("empty prefix", 2, 0, 300, 16, 8)
    inp = chunk_inputs(shape, seed=8)
    kc, vc = _caches(inp, shape, 320)
    out, lse, kca, vca = _run(inp, shape, kc, vc)
    pinp = {k: inp[k] for k in ("q", "k", "v", "q_norm_w", "k_norm_w", "pos")}
    kc2, vc2 = kc.to(dev()), vc.to(dev())
    out_p, lse_p = prefill_gpu(pinp, caches=(kc2, vc2))
    assert torch.equal(out, out_p) and torch.equal(lse, lse_p)
    assert torch.equal(kca.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vca.view(torch.int16), vc2.view(torch.int16))


def test_two_chunks_equal_one_prefill():
    """Prefill of the first 256 tokens into a cache, then a chunk of the next 300 over it,
    gives the rows a single prefill of all 556 tokens gives: same key tiles in the same
    order, same per-row limits, same softmax reference, so the same bits."""
    d = dev()
    full = prefill_inputs(PrefillShape("two chunks", 1, 556, 32, 8), seed=12)
    kc = torch.zeros((1, 8, 600, 128), dtype=torch.bfloat16, device=d)
    vc = torch.zeros_like(kc)
    first = {k: (v[:, :256].contiguous() if v.dim() > 1 else v) for k, v in full.items()}
    prefill_gpu(first, caches=(kc, vc))
    t = {k: v.to(d) for k, v in full.items()}
    lse2 = torch.empty((1, 32, 300), dtype=torch.float32, device=d)
    out2 = qa.prefill_chunk(t["q"][:, 256:].contiguous(), t["k"][:, 256:].contiguous(), t["v"][:, 256:].contiguous(),
                            t["q_norm_w"], t["k_norm_w"], t["pos"][:, 256:].contiguous(), kc, vc, 256, lse=lse2)
    torch.cuda.synchronize()
    assert_status_ok()
    out_f, lse_f = prefill_gpu(full)
    diff = (out2.float() - out_f[:, 256:].float()).abs().max().item()
    assert torch.equal(out2, out_f[:, 256:]), f"max diff {diff:.3e}"
    assert torch.equal(lse2, lse_f[:, :, 256:])


def test_chunk_large_gains_running_max_path():
    shape = ChunkShape("large gains", 1, 450, 260, 16, 8)
    inp = chunk_inputs(shape, seed=31)
    inp["q_norm_w"] = inp["q_norm_w"] * 1.6
    inp["k_norm_w"] = inp["k_norm_w"] * 1.6
    kc, vc = _caches(inp, shape, 710)
    out, lse, _, _ = _run(inp, shape, kc, vc)
    _, _, ref_st, st_lse = _oracle(inp, shape, kc, vc)
    # the same staged comparison and gain-scaled LSE bound as the prefill large-gains test
    compare(to_np(out), to_np(lse), ref_st, st_lse, st_lse, "chunk large gains (staged)", lse_tol=1e-3 * 1.6 ** 2)
    # and against the pure oracle, with the bounds of the prefill large-gains test
    ref, ref_lse, _, _ = _oracle(inp, shape, kc, vc)
    g2 = 1.6 ** 2
    bound = chunk_lse_bound(inp, shape.start, as_f64(kc[:, :, :shape.start]), theta=shape.theta, eps=shape.eps)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, "chunk large gains (pure)", lse_tol=1e-3 * g2,
            max_tol=MAX_TOL * g2, mean_tol=MEAN_TOL * g2, lse_pure_bound=bound)


SHORT_OVER_LONG = [
    # (T, start): a few new tokens over a long cached prefix, the case the key-axis split is
    # for: B * Hkv work items are far below the SM count, each with ~235 key tiles
    (1, 30000),
    (16, 30011),
    (64, 29950),
]


@pytest.mark.parametrize("T,start", SHORT_OVER_LONG)
def test_short_chunk_over_long_prefix_splits_the_keys(T, start):
    """The key-axis split (each run of keys leaves O/l and its LSE; one more kernel merges
    them by logsumexp weight) against the oracle, and against the same call run unsplit
    (a workspace without room for the partials)."""
    shape = ChunkShape("short chunk", 1, start, T, 32, 8)
    assert qa.prefill_chunk_workspace_size(1, start, T, 32, 8) > qa.prefill_workspace_size(1, T, 32, 8)
    inp = chunk_inputs(shape, seed=T)
    kc, vc = _caches(inp, shape, start + T + 7)
    out, lse, kca, vca = _run(inp, shape, kc, vc)
    ref, ref_lse, _, st_lse = _oracle(inp, shape, kc, vc)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, f"short chunk T{T} over {start}, key split")
    _check_caches(inp, shape, kc, vc, kca, vca)
    # unsplit: the plain prefill workspace has no room for the partials
    d = dev()
    t = {k: inp[k].to(d) for k in ("q", "k", "v", "q_norm_w", "k_norm_w", "pos")}
    lse1 = torch.empty_like(lse)
    ws = torch.empty(qa.prefill_workspace_size(1, T, 32, 8), dtype=torch.uint8, device=d)
    out1 = qa.prefill_chunk(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], kc.to(d), vc.to(d), start,
                            lse=lse1, workspace=ws)
    torch.cuda.synchronize()
    assert_status_ok()
    compare(to_np(out1), to_np(lse1), ref, ref_lse, st_lse, f"short chunk T{T} over {start}, unsplit")
    diff = (out.float() - out1.float()).abs()
    assert diff.max().item() <= 2e-2 and (lse - lse1).abs().max().item() <= 1e-3


@pytest.mark.parametrize("B,start,T,Hq,Hkv", [(1, 5200, 16, 32, 8), (2, 8000, 16, 32, 8), (1, 20000, 1, 64, 4),
                                             (1, 3000, 128, 8, 8), (3, 1500, 5, 16, 2)])
def test_single_query_tile_chunk_takes_two_runs_per_item(B, start, T, Hq, Hkv):
    """A chunk whose every KV head has a single query tile (T * G <= 128): each work item
    takes two runs of keys, one per softmax group over the same query rows.  Against the
    oracle, and against the same call run unsplit.  5200 + 16 keys make 41 tiles in 5 item
    runs, the last of 9 tiles, so its halves differ in length."""
    shape = ChunkShape("single query tile", B, start, T, Hq, Hkv)
    assert T * (Hq // Hkv) <= 128
    assert qa.prefill_chunk_workspace_size(B, start, T, Hq, Hkv) > qa.prefill_workspace_size(B, T, Hq, Hkv)
    inp = chunk_inputs(shape, seed=start + T + B)
    kc, vc = _caches(inp, shape, start + T + 3)
    out, lse, _, _ = _run(inp, shape, kc, vc)
    ref, ref_lse, _, st_lse = _oracle(inp, shape, kc, vc)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, f"one query tile B{B} T{T} over {start}, two runs per item")
    d = dev()
    t = {k: inp[k].to(d) for k in ("q", "k", "v", "q_norm_w", "k_norm_w", "pos")}
    lse1 = torch.empty_like(lse)
    ws = torch.empty(qa.prefill_workspace_size(B, T, Hq, Hkv), dtype=torch.uint8, device=d)
    out1 = qa.prefill_chunk(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], kc.to(d), vc.to(d), start,
                            lse=lse1, workspace=ws)
    torch.cuda.synchronize()
    assert_status_ok()
    diff = (out.float() - out1.float()).abs()
    assert diff.max().item() <= 2e-2 and (lse - lse1).abs().max().item() <= 1e-3


def test_short_chunk_key_split_running_max_path():
    shape = ChunkShape("short chunk", 1, 20000, 48, 16, 4)
    inp = chunk_inputs(shape, seed=5)
    kc, vc = _caches(inp, shape, 20100)
    old = qa.set_softmax_path(qa.SOFTMAX_RUNNING_MAX)
    try:
        out, lse, _, _ = _run(inp, shape, kc, vc)
    finally:
        qa.set_softmax_path(old)
    ref, ref_lse, _, st_lse = _oracle(inp, shape, kc, vc)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, "short chunk over 20000, key split, running max")
    # a single query tile per KV head: two runs per item on the running-max path
    shape = ChunkShape("short chunk", 1, 20000, 16, 16, 4)
    inp = chunk_inputs(shape, seed=6)
    kc, vc = _caches(inp, shape, 20020)
    old = qa.set_softmax_path(qa.SOFTMAX_RUNNING_MAX)
    try:
        out, lse, _, _ = _run(inp, shape, kc, vc)
    finally:
        qa.set_softmax_path(old)
    ref, ref_lse, _, st_lse = _oracle(inp, shape, kc, vc)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, "one query tile over 20000, two runs per item, running max")


@pytest.mark.parametrize("start,T,Hq,Hkv", [(0, 1024, 2, 1), (200, 1000, 4, 2)])
def test_key_split_with_runs_a_pair_does_not_reach(start, T, Hq, Hkv):
    """Few work items split into runs of the longest pair's key tiles; the lightest pairs
    read fewer tiles than there are runs, so some of their runs hold no key at all and leave
    an empty partial (LSE -inf) that the combine must weigh by zero."""
    shape = ChunkShape("split, empty runs", 1, start, T, Hq, Hkv)
    assert qa.prefill_chunk_workspace_size(1, start, T, Hq, Hkv) > qa.prefill_workspace_size(1, T, Hq, Hkv)
    inp = chunk_inputs(shape, seed=start + 3)
    kc, vc = _caches(inp, shape, start + T)
    out, lse, _, _ = _run(inp, shape, kc, vc)
    ref, ref_lse, _, st_lse = _oracle(inp, shape, kc, vc)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, f"key split, empty runs, start {start} T {T} Hq {Hq}")
