"""Paged KV cache through the C ABI: decode and chunked prefill over page pools addressed by
a block table, against the fp64 oracle on the same cache contents read in key order
(oracle.paged_gather).  Pages are dealt to sequences in a seeded random order; pages no
sequence owns hold NaN patterns and must stay untouched."""
import numpy as np
import pytest
import torch

import oracle
import qwen3_qk_norm_rope_b200 as qa
from synthetic import ChunkShape, DecodeShape, as_f64, chunk_inputs, decode_history, decode_step_inputs
from tests.gpu_common import (LSE_PURE_TOL, LSE_TOL, MAX_TOL, MEAN_TOL, assert_status_ok, compare, dev, to_np)

pytestmark = pytest.mark.gpu
NAN16 = 0x7FC1
THETA, EPS = 1.0e6, 1.0e-6


def _tables(rows, blocks_needed, max_blocks, num_pages, seed):
    """A block table [rows, max_blocks] dealing distinct pages in a random order; unused
    entries are -1.  Returns the table and the set of pages in use."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(num_pages)
    table = np.full((rows, max_blocks), -1, dtype=np.int32)
    k = 0
    for r in range(rows):
        for b in range(blocks_needed[r]):
            table[r, b] = perm[k]
            k += 1
    return table, set(int(x) for x in perm[:k])


def _scatter(pool, table_row, keys, page):
    """Write keys [Hkv, n, d] into the pool along one table row (test-side setup)."""
    n = keys.shape[1]
    for j in range(n):
        pool[int(table_row[j // page]), :, j % page] = keys[:, j]


@pytest.mark.parametrize("page,window", [(16, 0), (32, 0), (64, 0), (256, 0), (128, 700), (16, 700)])
def test_decode_paged(page, window):
    shape = DecodeShape("paged decode", 5, 32, 8)
    lens = [3000, page - 1, 1023, 4095, 100]
    max_blocks = 4096 // page + 1
    blocks = [(L + 1 + page - 1) // page for L in lens]  # the new token's block included
    num_pages = sum(blocks) + 7
    table, used = _tables(5, blocks, max_blocks, num_pages, seed=page)
    d = dev()
    step = decode_step_inputs(shape, seed=50 + page)
    step["cache_lens"] = torch.as_tensor(np.asarray(lens, dtype=np.int32))
    kp = torch.empty((num_pages, 8, page, 128), dtype=torch.bfloat16)
    kp.view(torch.int16).fill_(NAN16)
    vp = kp.clone()
    gq, gk = as_f64(step["q_norm_w"]), as_f64(step["k_norm_w"])
    host = {}
    for n, L in enumerate(lens):
        hist = decode_history(shape, n, L, step["s_k"], seed=50 + page)
        kc = oracle.build_cache_k(as_f64(hist["k_hist"]), gk, THETA, EPS).transpose(1, 0, 2)  # [Hkv, L, d]
        vc = as_f64(hist["v_hist"]).transpose(1, 0, 2)
        _scatter(kp, table[n], torch.from_numpy(kc.copy()).to(torch.bfloat16), page)
        _scatter(vp, table[n], torch.from_numpy(vc.copy()).to(torch.bfloat16), page)
        host[n] = (kc, vc)
    before_k, before_v = kp.clone(), vp.clone()
    kpd, vpd = kp.to(d), vp.to(d)
    t = {k: v.to(d) for k, v in step.items()}
    tab = torch.from_numpy(table).to(d)
    lse = torch.full((5, 32), float("nan"), dtype=torch.float32, device=d)
    out = qa.decode_paged(t["q"], t["k_new"], t["v_new"], t["q_norm_w"], t["k_norm_w"], kpd, vpd, tab,
                          t["cache_lens"], lse=lse, window=window)
    torch.cuda.synchronize()
    assert_status_ok()
    ka, va = kpd.cpu(), vpd.cpu()
    for n, L in enumerate(lens):
        kc, vc = host[n]
        args = (as_f64(step["q"])[n:n + 1], as_f64(step["k_new"])[n:n + 1], as_f64(step["v_new"])[n:n + 1], gq, gk,
                [kc], [vc], [L], THETA, EPS)
        ref, ref_lse = oracle.decode_ref(*args, window=window)
        _, st_lse = oracle.decode_ref(*args, window=window, staged=True)
        o = to_np(out[n:n + 1])
        err = np.abs(o - ref)
        assert np.isfinite(o).all() and err.max() <= MAX_TOL and err.mean() <= MEAN_TOL, (n, err.max())
        l = to_np(lse[n:n + 1])
        assert np.abs(l - st_lse).max() <= LSE_TOL and np.abs(l - ref_lse).max() <= LSE_PURE_TOL
        # the new token went to key index L of its pages: normed+rotated key, raw value
        pg, off = int(table[n, L // page]), L % page
        kref = oracle.qk_prologue(as_f64(step["k_new"])[n][None], gk, np.array([L]), THETA, EPS)[0]
        assert np.all(np.abs(to_np(ka[pg, :, off]) - kref) <= np.abs(kref) * 2.0 ** -8 + 2e-5)
        assert torch.equal(va[pg, :, off], step["v_new"][n])
        # and read back in key order the pages hold the history unchanged
        assert np.array_equal(oracle.paged_gather(to_np(ka), table[n], L, page), kc)
    # pages no sequence owns, and every other slot, are untouched
    mask = torch.ones_like(ka, dtype=torch.bool)
    for n, L in enumerate(lens):
        pg, off = int(table[n, L // page]), L % page
        mask[pg, :, off] = False
    assert torch.equal(ka.view(torch.int16)[mask], before_k.view(torch.int16)[mask])
    assert torch.equal(va.view(torch.int16)[mask], before_v.view(torch.int16)[mask])


@pytest.mark.parametrize("page", [64, 16])
def test_decode_paged_equals_contiguous(page):
    """The same caches, once contiguous and once in pages, give the same bits (pages under
    64 keys are read one box per page for both 64-dim halves, larger ones a box per half)."""
    shape = DecodeShape("paged vs contiguous", 3, 32, 8)
    lens = [2500, 64, 1000]
    Lmax = 2560
    max_blocks = Lmax // page
    blocks = [(L + 1 + page - 1) // page for L in lens]
    table, _ = _tables(3, blocks, max_blocks, sum(blocks), seed=9)
    d = dev()
    step = decode_step_inputs(shape, seed=60)
    step["cache_lens"] = torch.as_tensor(np.asarray(lens, dtype=np.int32))
    g = torch.Generator().manual_seed(3)
    kc = torch.randn((3, 8, Lmax, 128), generator=g).to(torch.bfloat16)
    vc = torch.randn((3, 8, Lmax, 128), generator=g).to(torch.bfloat16)
    kp = torch.zeros((sum(blocks), 8, page, 128), dtype=torch.bfloat16)
    vp = torch.zeros_like(kp)
    for n, L in enumerate(lens):
        _scatter(kp, table[n], kc[n, :, :L], page)
        _scatter(vp, table[n], vc[n, :, :L], page)
    t = {k: v.to(d) for k, v in step.items()}
    out_c = qa.decode(t["q"], t["k_new"], t["v_new"], t["q_norm_w"], t["k_norm_w"], kc.to(d), vc.to(d),
                      t["cache_lens"])
    out_p = qa.decode_paged(t["q"], t["k_new"], t["v_new"], t["q_norm_w"], t["k_norm_w"], kp.to(d), vp.to(d),
                            torch.from_numpy(table).to(d), t["cache_lens"])
    torch.cuda.synchronize()
    assert_status_ok()
    assert torch.equal(out_c, out_p)


@pytest.mark.parametrize("start,T,page", [(0, 300, 64), (777, 300, 16), (1000, 129, 256), (5000, 32, 64),
                                          (3000, 20, 16), (4090, 7, 256)])
def test_prefill_paged(start, T, page):
    shape = ChunkShape("paged chunk", 2, start, T, 16, 8)
    inp = chunk_inputs(shape, seed=start + T)
    n = start + T
    max_blocks = (n + page - 1) // page + 2
    blocks = [(n + page - 1) // page] * 2
    num_pages = sum(blocks) + 5
    table, _ = _tables(2, blocks, max_blocks, num_pages, seed=page + start)
    kp = torch.empty((num_pages, 8, page, 128), dtype=torch.bfloat16)
    kp.view(torch.int16).fill_(NAN16)
    vp = kp.clone()
    gk = as_f64(inp["k_norm_w"])
    prefix_k, prefix_v = [], []
    for b in range(2):
        kb = oracle.build_cache_k(as_f64(inp["k_hist"][b]), gk, THETA, EPS).transpose(1, 0, 2) if start else \
            np.zeros((8, 0, 128))
        vb = as_f64(inp["v_hist"][b]).transpose(1, 0, 2) if start else np.zeros((8, 0, 128))
        _scatter(kp, table[b], torch.from_numpy(kb.copy()).to(torch.bfloat16), page)
        _scatter(vp, table[b], torch.from_numpy(vb.copy()).to(torch.bfloat16), page)
        prefix_k.append(kb)
        prefix_v.append(vb)
    before_k, before_v = kp.clone(), vp.clone()
    d = dev()
    t = {k: inp[k].to(d) for k in ("q", "k", "v", "q_norm_w", "k_norm_w", "pos")}
    kpd, vpd = kp.to(d), vp.to(d)
    lse = torch.full((2, 16, T), float("nan"), dtype=torch.float32, device=d)
    out = qa.prefill_paged(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], kpd, vpd,
                           torch.from_numpy(table).to(d), start, lse=lse)
    torch.cuda.synchronize()
    assert_status_ok()
    kcache = np.stack([np.asarray(prefix_k[b], dtype=np.float64) for b in range(2)])
    vcache = np.stack([np.asarray(prefix_v[b], dtype=np.float64) for b in range(2)])
    args = (as_f64(inp["q"]), as_f64(inp["k"]), as_f64(inp["v"]), as_f64(inp["q_norm_w"]), gk, inp["pos"].numpy(),
            kcache, vcache, start, THETA, EPS)
    ref, ref_lse = oracle.chunk_prefill_ref(*args)
    _, st_lse = oracle.chunk_prefill_ref(*args, staged=True)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, f"paged prefill start {start} T {T} page {page}")
    # the new keys and values are in their pages, in key order; nothing else changed
    ka, va = kpd.cpu(), vpd.cpu()
    kref = oracle.qk_prologue(as_f64(inp["k"]), gk, inp["pos"].numpy(), THETA, EPS)  # [B, T, Hkv, d]
    written = torch.zeros_like(ka, dtype=torch.bool)
    for b in range(2):
        got = oracle.paged_gather(to_np(ka), table[b], n, page)[:, start:]  # [Hkv, T, d]
        want = kref[b].transpose(1, 0, 2)
        assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -8 + 2e-5)
        gotv = oracle.paged_gather(to_np(va), table[b], n, page)[:, start:]
        assert np.array_equal(gotv, as_f64(inp["v"][b]).transpose(1, 0, 2))
        for j in range(start, n):
            written[int(table[b, j // page]), :, j % page] = True
    keep = ~written
    assert torch.equal(ka.view(torch.int16)[keep], before_k.view(torch.int16)[keep])
    assert torch.equal(va.view(torch.int16)[keep], before_v.view(torch.int16)[keep])
