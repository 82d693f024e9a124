"""Benchmark of the Qwen3 attention core on B200: prints ONE JSON line.

One step is one pass of the whole hot path over one batch of synthetic input:
  * prefill of the long-context wide-GQA workload (B=1, T=32768, Hq=64, Hkv=4, d=128), the
    largest prefill that fits one GPU: QK-Norm + RoPE prologue and causal GQA attention, and
  * one batched decode step (64 sequences, cached lengths ~ U[1024, 32768], Hq=32,
    Hkv=8): append of the new normed/rotated key, split-KV attention, LSE combine.
`value` is the prefill throughput in TFLOP/s (causal flops 4*B*Hq*d*T(T+1)/2; the
prologue is counted as free work); the decode throughput in GB/s rides along under
"decode", and the Qwen3-0.6B- and 4B-shaped prefills, each timed alone over as many
calls, under "prefill_shapes".  Inputs are resident in HBM before the timed region; L2 is
flushed (a 256 MiB write) before every step and every call, outside the per-call CUDA-event
windows.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    python bench.py --prefill qwen3-0.6b          # another prefill workload in the step
    python bench.py --workload chunked-prefill    # the chunked-prefill call alone
    python bench.py --workload qkv-proj           # the merged qkv projection + QK-Norm/RoPE
    python bench.py --workload varlen-prefill     # a ragged batch of prompts on one token axis

The chunked-prefill workload times qwen3_attn_prefill_chunk on the Qwen3-4B-shaped
second chunk (B=1, 4096 new tokens over 4096 cached, Hq=32, Hkv=8) and prints its own
line in the same format (causal flops: new row i sees start + i + 1 keys).

Multi-GPU (torchrun, one rank per GPU): every rank runs its own replica of the step
(weak scaling, no collective on the data path); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic import CHUNK_SHAPES, DECODE_SHAPES, PREFILL_SHAPES, QKV_SHAPES, VARLEN_SHAPES, chunk_inputs, \
    decode_step_inputs, prefill_inputs, qkv_proj_inputs, varlen_inputs  # noqa: E402

METRIC = "causal GQA attn TFLOP/s (+QK-Norm/RoPE) % bf16 peak; decode HBM GB/s"
# The step's prefill: the largest single-GPU prefill workload (B=1, T=32768, Hq=64, Hkv=4).
HEADLINE_PREFILL = "long-wide-gqa"
# Prefill workloads timed beside the step, each alone, reported under "prefill_shapes".
OTHER_PREFILLS = ("qwen3-0.6b", "qwen3-4b")
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
# A device-side spin of about 0.1 ms after each L2 flush, outside the timed window: the GPU
# stays busy while the host enqueues the call, so a short call's window holds its device
# time and not the host's enqueue (the blocking-kernel practice of GPU benchmark harnesses).
# The end-to-end legs leave it out: there the host's part belongs to the figure.
HOLD_CYCLES = 200_000
L2_NOTE = "flushed before every step (256 MiB write, then a ~0.1 ms device-side spin, both outside the timed windows)"
L2_NOTE_STEP = ("flushed before every step and every call (256 MiB write, then a ~0.1 ms device-side spin, both "
                "outside the timed windows)")


def hold_device():
    torch.cuda._sleep(HOLD_CYCLES)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in PEAKS_FALLBACK}, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def decode_bytes(lens: np.ndarray, Hq: int, Hkv: int, d: int = 128) -> int:
    """Algorithmic HBM bytes of one decode step: every cached K and V row read once
    (L per sequence), the new token's q read, out written, k/v_new read and written."""
    lens = lens.astype(np.int64)
    kv = int(lens.sum()) * Hkv * d * 2 * 2
    qo = lens.size * Hq * d * 2 * 2
    new = lens.size * Hkv * d * 2 * 2 * 2
    return kv + qo + new


# DRAM traffic of the decode split-KV kernel per cached token (dram__bytes_read.sum +
# dram__bytes_write.sum of one ncu capture of a smaller case, divided by its cached tokens),
# valid only for the kernel source it was measured on.  Refreshed with each new capture.
DECODE_TRAFFIC = {"src_sha256": "9c02d49265cc31c08af603737c19fb9d763c26ee719b5caaedf0dad97588df61",
                  "bytes_per_cached_token": (630.657280e6 + 5.152512e6) / 153639}


def decode_src_sha256() -> str:
    import hashlib

    h = hashlib.sha256()
    for f in ("decode.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "qwen3_qk_norm_rope_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def decode_traffic(lens: np.ndarray):
    if DECODE_TRAFFIC["src_sha256"] is None or DECODE_TRAFFIC["src_sha256"] != decode_src_sha256():
        return None
    return DECODE_TRAFFIC["bytes_per_cached_token"] * float(lens.astype(np.int64).sum())


# DRAM traffic of the prefill attention kernel per launch on a workload (dram__bytes_read.sum
# + dram__bytes_write.sum of one ncu capture of that launch), valid only for the kernel
# source it was measured on.  Refreshed with each new capture.
PREFILL_TRAFFIC = {"src_sha256": "9bb0814517d2b15eb41681e1cdb1a8f53d0d1d314898fccbedcaa03ebe37c3d0",
                   "bytes": {"long-context wide-GQA prefill B=1 T=32768 Hq=64 Hkv=4": 1.22407e9 + 0.51934e9}}


def prefill_src_sha256() -> str:
    import hashlib

    h = hashlib.sha256()
    for f in ("prefill.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "qwen3_qk_norm_rope_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def prefill_traffic(ps):
    if PREFILL_TRAFFIC["src_sha256"] is None or PREFILL_TRAFFIC["src_sha256"] != prefill_src_sha256():
        return None
    return PREFILL_TRAFFIC["bytes"].get(ps.name)


def decode_flops(lens: np.ndarray, Hq: int, d: int = 128) -> float:
    return 4.0 * Hq * d * float((lens.astype(np.int64) + 1).sum())


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.path is None or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[4], f[5], f[6], f[7], f[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        sm = [r[0] for r in rows]
        loaded = [r for r in rows if r[2] > 200.0] or rows
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            for name, flag in zip(names, r[4:8]):
                if flag.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r[0] for r in loaded])), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "sm_mhz_min": min(sm)}


# ------------------------------------------------------------------------------ workload
class Workload:
    """Device-resident inputs of one step, built once."""

    def __init__(self, dev: torch.device, seed: int = 0, prefill: str = HEADLINE_PREFILL, decode_seqs: int = 64,
                 others=()):
        import dataclasses

        import qwen3_qk_norm_rope_b200 as qa

        self.qa = qa
        self.dev = dev
        self.ps = PREFILL_SHAPES[prefill]
        # the other prefill workloads, timed alone: (shape, device inputs, out, workspace)
        self.others = []
        for name in others:
            if name == prefill:
                continue
            sh = PREFILL_SHAPES[name]
            t = {k: v.to(dev) for k, v in prefill_inputs(sh, seed=seed).items()}
            self.others.append((name, sh, t, torch.empty_like(t["q"]),
                                torch.empty(qa.prefill_workspace_size(sh.B, sh.T, sh.Hq, sh.Hkv), dtype=torch.uint8,
                                            device=dev)))
        full = DECODE_SHAPES["batched-decode"]
        self.ds = full if decode_seqs == full.N else dataclasses.replace(
            full, name=f"first {decode_seqs} sequences of the {full.name}", N=decode_seqs)
        p = prefill_inputs(self.ps, seed=seed)
        self.p_host = p
        self.p = {k: v.to(dev) for k, v in p.items()}
        self.p_out = torch.empty_like(self.p["q"])
        self.p_ws = torch.empty(qa.prefill_workspace_size(self.ps.B, self.ps.T, self.ps.Hq, self.ps.Hkv), dtype=torch.uint8,
                                device=dev)
        d = decode_step_inputs(full, seed=seed)
        d = {k: (v[:decode_seqs].contiguous() if k in ("q", "k_new", "v_new", "cache_lens") else v)
             for k, v in d.items()}
        self.d_host = d
        self.d = {k: v.to(dev) for k, v in d.items()}
        self.lens = d["cache_lens"].numpy()
        N, Hkv, Lmax = self.ds.N, self.ds.Hkv, self.ds.cache_capacity
        self.Lmax = Lmax
        self.kc = torch.empty((N, Hkv, Lmax, 128), dtype=torch.bfloat16, device=dev)
        self.vc = torch.empty_like(self.kc)
        # Cache history: raw keys drawn like the prefill keys (N(0,1) times the per-channel
        # scale s_k), normed and rotated at positions 0..L-1 by the library's own prologue;
        # raw values N(0,1).  Drawn on the device with a seeded generator.
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 1)
        s_k = d["s_k"].to(dev)
        Lmax_hist = int(self.lens.max())
        pos = torch.arange(Lmax_hist, dtype=torch.int32, device=dev)[None]
        for n in range(N):
            L = int(self.lens[n])
            kh = (torch.randn((1, L, Hkv, 128), generator=g, device=dev) * s_k).to(torch.bfloat16)
            vh = torch.randn((1, L, Hkv, 128), generator=g, device=dev).to(torch.bfloat16)
            qa.qk_norm_rope(kh, self.d["k_norm_w"], pos[:, :L].contiguous(), self.kc[n:n + 1], v_src=vh,
                            v_dst=self.vc[n:n + 1], theta=self.ds.theta, eps=self.ds.eps)
        self.d_out = torch.empty_like(self.d["q"])
        self.d_ws = torch.empty(qa.decode_workspace_size(N, self.ds.Hq, Lmax), dtype=torch.uint8, device=dev)
        self.flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        torch.cuda.synchronize(dev)
        st, site = qa.device_status(clear=True, device=dev)
        if st != qa.OK:
            raise RuntimeError(f"cache build failed: {qa.status_string(st)} at site {site}")

    def prefill(self):
        p = self.p
        self.qa.prefill(p["q"], p["k"], p["v"], p["q_norm_w"], p["k_norm_w"], p["pos"], out=self.p_out,
                        workspace=self.p_ws)

    def decode(self):
        d = self.d
        self.qa.decode(d["q"], d["k_new"], d["v_new"], d["q_norm_w"], d["k_norm_w"], self.kc, self.vc,
                       d["cache_lens"], out=self.d_out, workspace=self.d_ws)

    def flush_l2(self):
        self.flush.fill_(1.0)

    def prefill_other(self, i: int):
        _, _, t, out, ws = self.others[i]
        self.qa.prefill(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], out=out, workspace=ws)

    # launches of this library's kernels per step: prefill (prologue + attention) and
    # decode (append + split-KV attention + combine)
    LAUNCHES_PER_STEP = 5


def time_steps(w: Workload, steps: int):
    """Per-step CUDA events on the launching stream; the L2 flush sits between windows."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(steps):
        w.flush_l2()
        hold_device()
        ev[i][0].record()
        w.prefill()
        ev[i][1].record()
        w.decode()
        ev[i][2].record()
    torch.cuda.synchronize(w.dev)
    pre = sum(e[0].elapsed_time(e[1]) for e in ev)
    dec = sum(e[1].elapsed_time(e[2]) for e in ev)
    return pre, dec


def time_other_prefills(w: Workload, steps: int, warmup: int):
    """Each other prefill workload alone: `warmup` untimed calls, then `steps` calls with L2
    flushed before each, outside the per-call CUDA-event windows.  Milliseconds per call."""
    res = []
    for i in range(len(w.others)):
        for _ in range(warmup):
            w.flush_l2()
            w.prefill_other(i)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for j in range(steps):
            w.flush_l2()
            hold_device()
            ev[j][0].record()
            w.prefill_other(i)
            ev[j][1].record()
        torch.cuda.synchronize(w.dev)
        res.append(sum(e[0].elapsed_time(e[1]) for e in ev) / steps)
    return res


def time_e2e(w: Workload, steps: int):
    """The same step through the public API with host buffers: pinned host -> device copies
    of the step's inputs, the calls, and device -> host copies of the outputs, all inside
    the event window."""
    ph = {k: v.pin_memory() for k, v in w.p_host.items()}
    dh = {k: w.d_host[k].pin_memory() for k in ("q", "k_new", "v_new", "q_norm_w", "k_norm_w", "cache_lens")}
    out_p = torch.empty(w.p_out.shape, dtype=torch.bfloat16).pin_memory()
    out_d = torch.empty(w.d_out.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in ph.values()) + sum(t.numel() * t.element_size()
                                                                       for t in dh.values())
    d2h = out_p.numel() * 2 + out_d.numel() * 2
    pre_ms = 0.0
    tot_ms = 0.0
    for i in range(steps):
        w.flush_l2()
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        for k, v in ph.items():
            w.p[k].copy_(v, non_blocking=True)
        w.prefill()
        out_p.copy_(w.p_out, non_blocking=True)
        e1.record()
        for k, v in dh.items():
            w.d[k].copy_(v, non_blocking=True)
        w.decode()
        out_d.copy_(w.d_out, non_blocking=True)
        e2.record()
        torch.cuda.synchronize(w.dev)
        pre_ms += e0.elapsed_time(e1)
        tot_ms += e0.elapsed_time(e2)
    return pre_ms, tot_ms, h2d, d2h


def time_e2e_pipelined(w: Workload, steps: int):
    """The prefill call through the public API over a stream of steps, as a serving loop runs
    it: step i's inputs are copied in from pinned host memory on one copy stream while step
    i-1 computes, and each step's output is copied back on another copy stream while the
    next one computes; two device buffer sets alternate.  One event window covers every
    step's copies and calls, the first copy in and the last copy out included.  The inputs
    are larger than L2, so nothing is flushed between steps."""
    dev = w.dev
    ph = {k: v.pin_memory() for k, v in w.p_host.items()}
    bufs = [w.p, {k: torch.empty_like(v) for k, v in w.p.items()}]
    outs = [w.p_out, torch.empty_like(w.p_out)]
    host_out = [torch.empty(w.p_out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in ph.values())
    d2h = host_out[0].numel() * 2
    s_c = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(steps)]
    done = [torch.cuda.Event() for _ in range(steps)]
    out_done = [torch.cuda.Event() for _ in range(steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(s_c)
    s_in.wait_stream(s_c)
    s_out.wait_stream(s_c)
    qa = w.qa
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(done[i - 2])  # step i-2 has read buffer set b
            for k, v in ph.items():
                bufs[b][k].copy_(v, non_blocking=True)
            in_ready[i].record(s_in)
        s_c.wait_event(in_ready[i])
        if i >= 2:
            s_c.wait_event(out_done[i - 2])  # step i-2's output has left buffer b
        t = bufs[b]
        qa.prefill(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], out=outs[b], workspace=w.p_ws)
        done[i].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[i])
            host_out[b].copy_(outs[b], non_blocking=True)
            out_done[i].record(s_out)
    s_c.wait_stream(s_in)
    s_c.wait_stream(s_out)
    e1.record(s_c)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1), h2d, d2h


# ------------------------------------------------------------------------------ CPU oracle
def oracle_threads() -> int:
    """BLAS threads the oracle's numpy runs on: the cores a CPU-baseline figure used."""
    try:
        from threadpoolctl import threadpool_info

        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # noqa: BLE001
        return os.cpu_count()


def prefill_oracle(name: str = HEADLINE_PREFILL, batch_rows: int = 1, seed: int = 0):
    """The fp64 oracle on a prefill workload with its inputs built once: the returned
    run(rows) times one oracle call on the last `rows` query rows (every head) of the first
    `batch_rows` batch rows and returns its seconds, causal flops and a description of the
    sample.  run.full_flops is the whole workload's causal flops."""
    import oracle
    from synthetic import as_f64

    ps = PREFILL_SHAPES[name]
    batch_rows = min(batch_rows, ps.B)
    inp = prefill_inputs(ps, seed=seed)
    args = (as_f64(inp["q"][:batch_rows]), as_f64(inp["k"][:batch_rows]), as_f64(inp["v"][:batch_rows]),
            as_f64(inp["q_norm_w"]), as_f64(inp["k_norm_w"]), inp["pos"][:batch_rows].numpy(), ps.theta, ps.eps)
    del inp

    def run(rows: int) -> dict:
        sel = np.arange(ps.T - rows, ps.T)
        t0 = time.perf_counter()
        oracle.prefill_ref(*args, rows=sel)
        secs = time.perf_counter() - t0
        flops = batch_rows * 4.0 * ps.Hq * ps.d * float((sel + 1).sum())
        return {"seconds": secs, "flops": flops,
                "sample": (f"prefill: last {rows} of {ps.T} query rows x {ps.Hq} heads of {batch_rows} of {ps.B} "
                           f"batch rows of the {ps.name} ({flops:.3g} causal flops)")}

    run.max_rows = ps.T
    run.full_flops = ps.causal_flops()
    return run


def decode_oracle_sample(decode_seqs: int = 16, seed: int = 0) -> dict:
    """The oracle's decode of the first `decode_seqs` sequences of the batched decode; their
    caches are built (normed and rotated keys) before the timed call."""
    import oracle
    from synthetic import as_f64, decode_history

    ds = DECODE_SHAPES["batched-decode"]
    step = decode_step_inputs(ds, seed=seed)
    lens = step["cache_lens"].numpy()
    sel = list(range(decode_seqs))
    kh, vh = [], []
    for n in sel:
        h = decode_history(ds, n, int(lens[n]), step["s_k"], seed=seed)
        kh.append(oracle.build_cache_k(as_f64(h["k_hist"]), as_f64(step["k_norm_w"]), ds.theta,
                                       ds.eps).transpose(1, 0, 2))
        vh.append(as_f64(h["v_hist"]).transpose(1, 0, 2))
    t0 = time.perf_counter()
    oracle.decode_ref(as_f64(step["q"])[sel], as_f64(step["k_new"])[sel], as_f64(step["v_new"])[sel],
                      as_f64(step["q_norm_w"]), as_f64(step["k_norm_w"]), kh, vh, lens[sel], ds.theta, ds.eps)
    secs = time.perf_counter() - t0
    return {"seconds": secs, "gbs": decode_bytes(lens[sel], ds.Hq, ds.Hkv) / secs / 1e9,
            "sample": f"decode: first {decode_seqs} of 64 sequences ({int(lens[sel].sum())} cached tokens)"}


def cpu_oracle_sample(name: str = HEADLINE_PREFILL, rows_per_head: int = 512, batch_rows: int = 1,
                      decode_seqs: int = 16, seed: int = 0):
    """The fp64 oracle, as it stands, on a bounded sample of the same workload: the last
    `rows_per_head` query rows (every head) of the first `batch_rows` batch rows of the
    prefill `name`, and the first `decode_seqs` sequences of the batched decode.  Returns
    TFLOP/s on the prefill sample, the whole prefill's time extrapolated from it by the
    exact flop ratio, GB/s on the decode sample, the seconds each took and the BLAS thread
    count."""
    run = prefill_oracle(name, batch_rows, seed)
    pre = run(min(rows_per_head, run.max_rows))
    dec = decode_oracle_sample(decode_seqs, seed) if decode_seqs > 0 else \
        {"seconds": 0.0, "gbs": 0.0, "sample": "no decode"}
    return {"tflops": pre["flops"] / pre["seconds"] / 1e12, "gbs": dec["gbs"], "t_prefill_s": pre["seconds"],
            "t_decode_s": dec["seconds"], "threads": oracle_threads(), "sample": pre["sample"] + "; " + dec["sample"],
            "flops": pre["flops"], "prefill_full_s_extrapolated": pre["seconds"] * run.full_flops / pre["flops"]}


# The reference arm times the oracle for about this many seconds in all (warm-up and timed
# steps together), whatever --steps and --warmup ask for: each step's sample is sized to fit.
REFERENCE_BUDGET_S = 120.0


def reference_steps(run, steps: int, warmup: int, budget_s: float = REFERENCE_BUDGET_S):
    """The reference arm's loop over an oracle whose inputs are already built: calibrate its
    cost per query row from two sample sizes (so a fixed per-call cost is not taken for a
    per-row one), size each step's sample so that `warmup` + `steps` calls take about
    `budget_s` seconds (one row at least), then run the untimed warm-up calls and
    the timed steps.  Only the oracle calls themselves are timed.  Returns the timed
    seconds, the flops, the rows per step and the last step's sample description."""
    lo, hi = min(8, run.max_rows), min(264, run.max_rows)
    t_lo = min(run(lo)["seconds"] for _ in range(2))  # the better of two calls: the first is a warm-up too
    t_hi = min(run(hi)["seconds"] for _ in range(2))
    per_row = max((t_hi - t_lo) / max(hi - lo, 1), 1e-7)
    fixed = max(t_lo - lo * per_row, 0.0)
    per_step = budget_s / max(steps + warmup, 1)
    rows = int(max(1, min(run.max_rows, (per_step - fixed) / per_row)))
    for _ in range(warmup):
        run(rows)
    secs = flops = 0.0
    res = None
    for _ in range(steps):
        res = run(rows)
        secs += res["seconds"]
        flops += res["flops"]
    return secs, flops, rows, res["sample"]


# ------------------------------------------------------------------------------ chunked prefill
CHUNK_METRIC = "chunked-prefill causal GQA attn TFLOP/s (+QK-Norm/RoPE, cache append) % bf16 peak"
SHORT_CHUNK_METRIC = "short-chunk prefill over a long cached prefix: HBM GB/s (K/V read, +QK-Norm/RoPE, cache append)"
CHUNKS = {"second": "qwen3-4b-second-chunk", "short": "qwen3-4b-short-chunk"}


def chunk_bytes(cs) -> float:
    """Algorithmic HBM bytes of a chunked prefill: every cached and new key and value row
    read once by the attention (start + T keys of Hkv heads), the new q, k, v read and the
    new k', v written to the cache, and out written."""
    d2 = cs.d * 2
    kv_read = 2.0 * cs.B * (cs.start + cs.T) * cs.Hkv * d2
    new_in = cs.B * cs.T * (cs.Hq + 2 * cs.Hkv) * d2
    new_out = cs.B * cs.T * (2 * cs.Hkv + cs.Hq) * d2
    return kv_read + new_in + new_out


def paged_copy(caches, n: int, page: int, seed: int, dev):
    """Page pools [num_pages, Hkv, page, d] holding the first n rows of each [B, Hkv, >=n, d]
    cache, pages dealt in a seeded random order, and the [B, ceil(n/page)] block table."""
    B, Hkv, _, d = caches[0].shape
    nb = -(-n // page)
    g = torch.Generator().manual_seed(seed + 77)
    table = torch.randperm(B * nb, generator=g).to(torch.int32).view(B, nb)
    pools = []
    for c in caches:
        pool = torch.zeros((B * nb, Hkv, page, d), dtype=c.dtype, device=dev)
        src = torch.zeros((B, Hkv, nb * page, d), dtype=c.dtype, device=dev)
        src[:, :, :n] = c[:, :, :n]
        pool[table.view(-1).long().to(dev)] = src.view(B, Hkv, nb, page, d).permute(0, 2, 1, 3, 4).reshape(
            B * nb, Hkv, page, d)
        pools.append(pool)
    return pools[0], pools[1], table.to(dev)


class ChunkWorkload:
    """Device-resident inputs of the chunked-prefill call: the new tokens, and caches whose
    first `start` slots hold the prefix (normed and rotated by the library's prologue)."""

    LAUNCHES_PER_STEP = 2  # K prologue (cache append) + attention

    def __init__(self, dev: torch.device, name: str = "qwen3-4b-second-chunk", seed: int = 0, page: int = 0):
        self.name = name
        import qwen3_qk_norm_rope_b200 as qa

        self.qa, self.dev, self.page = qa, dev, page
        self.cs = cs = CHUNK_SHAPES[name]
        inp = chunk_inputs(cs, seed=seed)
        self.host = {k: inp[k] for k in ("q", "k", "v", "q_norm_w", "k_norm_w", "pos")}
        self.t = {k: v.to(dev) for k, v in self.host.items()}
        Tcap = cs.start + cs.T
        self.kc = torch.zeros((cs.B, cs.Hkv, Tcap, cs.d), dtype=torch.bfloat16, device=dev)
        self.vc = torch.zeros_like(self.kc)
        pos = torch.arange(cs.start, dtype=torch.int32, device=dev)[None].expand(cs.B, cs.start).contiguous()
        qa.qk_norm_rope(inp["k_hist"].to(dev), self.t["k_norm_w"], pos, self.kc, v_src=inp["v_hist"].to(dev),
                        v_dst=self.vc, theta=cs.theta, eps=cs.eps)
        self.out = torch.empty_like(self.t["q"])
        self.ws = torch.empty(qa.prefill_chunk_workspace_size(cs.B, cs.start, cs.T, cs.Hq, cs.Hkv), dtype=torch.uint8,
                              device=dev)
        if page:
            # the same caches in pages of `page` tokens, dealt to the rows in a seeded random order
            self.k_pages, self.v_pages, self.table = paged_copy([self.kc, self.vc], Tcap, page, seed, dev)
            self.ws = torch.empty(qa.prefill_paged_workspace_size(cs.B, cs.start, cs.T, cs.Hq, cs.Hkv),
                                  dtype=torch.uint8, device=dev)
        # the call splits the key axis when the shapes give its workspace split partials
        self.split = (qa.prefill_chunk_workspace_size(cs.B, cs.start, cs.T, cs.Hq, cs.Hkv) >
                      qa.prefill_workspace_size(cs.B, cs.T, cs.Hq, cs.Hkv))
        self.flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        torch.cuda.synchronize(dev)
        st, site = qa.device_status(clear=True, device=dev)
        if st != qa.OK:
            raise RuntimeError(f"cache build failed: {qa.status_string(st)} at site {site}")

    def step(self):
        t, cs = self.t, self.cs
        if self.page:
            self.qa.prefill_paged(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], self.k_pages,
                                  self.v_pages, self.table, cs.start, out=self.out, workspace=self.ws,
                                  theta=cs.theta, eps=cs.eps)
            return
        self.qa.prefill_chunk(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], self.kc, self.vc,
                              cs.start, out=self.out, workspace=self.ws, theta=cs.theta, eps=cs.eps)

    def config(self):
        cs = self.cs
        return {"workload": cs.name + (f", cache in pages of {self.page}" if self.page else ""), "B": cs.B,
                "start": cs.start, "T": cs.T, "Hq": cs.Hq, "Hkv": cs.Hkv, "page": self.page or None,
                "d": cs.d, "rope_theta": cs.theta, "rms_eps": cs.eps, "seed": 0,
                "l2": L2_NOTE,
                "parallelism": "replicas (one independent workload per GPU)"}


def chunk_oracle(name: str = "qwen3-4b-second-chunk", seed: int = 0):
    """The oracle's chunked prefill with its inputs and cached prefix built once: run(rows)
    times one call on the last `rows` new rows (every head) of the chunk."""
    import oracle
    from synthetic import as_f64

    cs = CHUNK_SHAPES[name]
    inp = chunk_inputs(cs, seed=seed)
    kc = np.stack([oracle.build_cache_k(as_f64(inp["k_hist"][b]), as_f64(inp["k_norm_w"]), cs.theta, cs.eps)
                   .transpose(1, 0, 2) for b in range(cs.B)])
    vc = as_f64(inp["v_hist"]).transpose(0, 2, 1, 3)
    args = (as_f64(inp["q"]), as_f64(inp["k"]), as_f64(inp["v"]), as_f64(inp["q_norm_w"]), as_f64(inp["k_norm_w"]),
            inp["pos"].numpy(), kc, vc, cs.start, cs.theta, cs.eps)

    def run(rows: int) -> dict:
        sel = np.arange(cs.T - rows, cs.T)
        t0 = time.perf_counter()
        oracle.chunk_prefill_ref(*args, rows=sel)
        secs = time.perf_counter() - t0
        flops = cs.B * 4.0 * cs.Hq * cs.d * float((cs.start + sel + 1).sum())
        return {"seconds": secs, "flops": flops,
                "sample": f"last {rows} of {cs.T} new rows x {cs.Hq} heads of the {cs.name} ({flops:.3g} causal flops)"}

    run.max_rows = cs.T
    return run


def cpu_oracle_chunk_sample(name: str = "qwen3-4b-second-chunk", rows: int = 512, seed: int = 0):
    """The oracle's chunked prefill on the last `rows` new rows (every head) of the chunk."""
    res = chunk_oracle(name, seed)(rows)
    return dict(res, tflops=res["flops"] / res["seconds"] / 1e12, threads=oracle_threads(), rows=rows)


def run_chunk(args, world, rank, local):
    name = CHUNKS[args.chunk]
    cs = CHUNK_SHAPES[name]
    short = args.chunk == "short"
    if args.impl == "reference":
        if rank != 0:
            return
        run = chunk_oracle(name)
        secs, flops, rows, sample = reference_steps(run, args.steps, args.warmup, args.reference_budget)
        value = flops / secs / 1e12
        unit = "TFLOP/s"
        if short:
            # GB/s over the rows the oracle ran: the whole chunk's bytes scaled by its rows
            value = chunk_bytes(cs) * rows / cs.T * args.steps / secs / 1e9
            unit = "GB/s"
        line = {"impl": "reference", "metric": SHORT_CHUNK_METRIC if short else CHUNK_METRIC, "value": value,
                "unit": unit, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": cs.name},
                "cpu_baseline": {"value": value, "unit": unit, "cores": oracle_threads(), "kind": "oracle",
                                 "sample": "per step, " + sample},
                "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    w = ChunkWorkload(dev, name=name, page=args.paged)
    for _ in range(args.warmup):
        w.flush.fill_(1.0)
        w.step()
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    with ClockSampler(local) as clk:
        for i in range(K):
            w.flush.fill_(1.0)
            hold_device()
            ev[i][0].record()
            w.step()
            ev[i][1].record()
        torch.cuda.synchronize(dev)
        barrier(world)
        torch.cuda.synchronize(dev)
    st, site = w.qa.device_status(clear=True, device=dev)
    if st != w.qa.OK:
        raise RuntimeError(f"device status {w.qa.status_string(st)} at site {site}")
    ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    # e2e: pinned host inputs in, the call, the output back, inside one event window
    ph = {k: v.pin_memory() for k, v in w.host.items()}
    out_h = torch.empty(w.out.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in ph.values())
    e_steps = max(1, min(K, 200))
    e_ms = 0.0
    for _ in range(e_steps):
        w.flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for k, v in ph.items():
            w.t[k].copy_(v, non_blocking=True)
        w.step()
        out_h.copy_(w.out, non_blocking=True)
        e1.record()
        torch.cuda.synchronize(dev)
        e_ms += e0.elapsed_time(e1)
    ms, e_ms = max_over_ranks(world, [ms, e_ms], dev)
    if rank != 0:
        return
    flops = w.cs.causal_flops()
    per_s = ms * 1e-3 / K
    achieved = flops / per_s / 1e12
    launches = ChunkWorkload.LAUNCHES_PER_STEP + (1 if w.split else 0)
    kernel = ("chunked-prefill call (K prologue + cache append + attention)" if not w.page
              else "paged chunked-prefill call (K prologue into pages + attention reading the pages in place)")
    if w.split:
        kernel = kernel[:-1] + " with a key-axis split + logsumexp combine)"
    e2e_flops = world * flops * e_steps / (e_ms * 1e-3) / 1e12
    if short:
        # HBM bound: the K/V read of the whole prefix dominates the bytes
        nbytes = chunk_bytes(w.cs)
        gbs = nbytes / per_s / 1e9
        line = {"metric": SHORT_CHUNK_METRIC, "value": world * gbs, "unit": "GB/s", "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": w.config(),
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / peaks["hbm_gbs"], "traffic": None, "kernel": kernel,
                             "algorithmic_bytes": nbytes, "peak_source": peak_src},
                "tflops": world * achieved, "gpu_launches": launches * K, "clocks": clk.summary(),
                "e2e": {"value": world * nbytes * e_steps / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
                        "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(out_h.numel() * 2),
                        "ms_per_step": e_ms / e_steps}}
    else:
        line = {"metric": CHUNK_METRIC, "value": world * achieved, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": w.config(),
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": achieved / peaks["bf16_tflops"], "traffic": None, "kernel": kernel,
                             "algorithmic_flops": flops, "peak_source": peak_src + " burst"},
                "gpu_launches": launches * K, "clocks": clk.summary(),
                "e2e": {"value": e2e_flops, "unit": "TFLOP/s",
                        "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(out_h.numel() * 2),
                        "ms_per_step": e_ms / e_steps}}
    if world == 1 and not args.no_cpu_baseline:
        cb = cpu_oracle_chunk_sample(name, rows=min(2048, w.cs.T))
        if short:
            gb = chunk_bytes(w.cs) * cb["rows"] / w.cs.T / cb["seconds"] / 1e9
            line["cpu_baseline"] = {"value": gb, "unit": "GB/s", "cores": cb["threads"], "kind": "oracle",
                                    "sample": cb["sample"], "seconds": cb["seconds"]}
        else:
            line["cpu_baseline"] = {"value": cb["tflops"], "unit": "TFLOP/s", "cores": cb["threads"], "kind": "oracle",
                                    "sample": cb["sample"], "seconds": cb["seconds"]}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ qkv projection
QKV_METRIC = "merged qkv projection GEMM TFLOP/s (QK-Norm + RoPE epilogue) % bf16 peak"


def qkv_oracle(name: str, seed: int = 0):
    """The oracle's projection + QK-Norm + RoPE with its inputs built once: run(rows) times
    one call on the first `rows` tokens of the workload."""
    import oracle
    from synthetic import as_f64

    sh = QKV_SHAPES[name]
    inp = qkv_proj_inputs(sh, seed=seed)
    x, w = as_f64(inp["x"]), as_f64(inp["w_qkv"])
    gq, gk, pos = as_f64(inp["q_norm_w"]), as_f64(inp["k_norm_w"]), inp["pos"].numpy()

    def run(rows: int) -> dict:
        t0 = time.perf_counter()
        oracle.qkv_proj_norm_rope_ref(x[:rows], w, gq, gk, pos[:rows], sh.Hq, sh.Hkv, sh.theta, sh.eps)
        secs = time.perf_counter() - t0
        flops = 2.0 * rows * sh.hidden * (sh.Hq + 2 * sh.Hkv) * sh.d
        return {"seconds": secs, "flops": flops,
                "sample": f"first {rows} of {sh.M} tokens of the {sh.name} ({flops:.3g} flops)"}

    run.max_rows = sh.M
    return run


def cpu_oracle_qkv_sample(name: str, rows: int = 256, seed: int = 0):
    """The oracle's projection + QK-Norm + RoPE on the first `rows` tokens of the workload."""
    res = qkv_oracle(name, seed)(rows)
    return dict(res, tflops=res["flops"] / res["seconds"] / 1e12, threads=oracle_threads())


def run_qkv(args, world, rank, local):
    name = args.qkv
    sh = QKV_SHAPES[name]
    if args.impl == "reference":
        if rank != 0:
            return
        secs, flops, _, sample = reference_steps(qkv_oracle(name), args.steps, args.warmup)
        value = flops / secs / 1e12
        line = {"impl": "reference", "metric": QKV_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": sh.name},
                "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                                 "sample": "per step, " + sample},
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    import qwen3_qk_norm_rope_b200 as qa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    host = qkv_proj_inputs(sh, seed=0)
    t = {k: v.to(dev) for k, v in host.items()}
    outs = (torch.empty((sh.M, sh.Hq, sh.d), dtype=torch.bfloat16, device=dev),
            torch.empty((sh.M, sh.Hkv, sh.d), dtype=torch.bfloat16, device=dev),
            torch.empty((sh.M, sh.Hkv, sh.d), dtype=torch.bfloat16, device=dev))
    ws = torch.empty(qa.qkv_proj_workspace_size(sh.M), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        qa.qkv_proj_norm_rope(t["x"], t["w_qkv"], t["q_norm_w"], t["k_norm_w"], t["pos"], sh.Hq, sh.Hkv,
                              q_out=outs[0], k_out=outs[1], v_out=outs[2], workspace=ws)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    with ClockSampler(local) as clk:
        for i in range(K):
            flush.fill_(1.0)
            hold_device()
            ev[i][0].record()
            step()
            ev[i][1].record()
        torch.cuda.synchronize(dev)
        barrier(world)
        torch.cuda.synchronize(dev)
    st, site = qa.device_status(clear=True, device=dev)
    if st != qa.OK:
        raise RuntimeError(f"device status {qa.status_string(st)} at site {site}")
    ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    ph = {k: v.pin_memory() for k, v in host.items()}
    oh = [torch.empty(o.shape, dtype=torch.bfloat16).pin_memory() for o in outs]
    h2d = sum(v.numel() * v.element_size() for v in ph.values())
    d2h = sum(o.numel() * 2 for o in oh)
    e_steps = max(1, min(K, 100))
    e_ms = 0.0
    for _ in range(e_steps):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for k, v in ph.items():
            t[k].copy_(v, non_blocking=True)
        step()
        for o, h in zip(outs, oh):
            h.copy_(o, non_blocking=True)
        e1.record()
        torch.cuda.synchronize(dev)
        e_ms += e0.elapsed_time(e1)
    ms, e_ms = max_over_ranks(world, [ms, e_ms], dev)
    if rank != 0:
        return
    flops = sh.flops()
    achieved = flops / (ms * 1e-3 / K) / 1e12
    line = {"metric": QKV_METRIC, "value": world * achieved, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": sh.name, "M": sh.M, "hidden": sh.hidden, "Hq": sh.Hq, "Hkv": sh.Hkv, "d": sh.d,
                       "l2": L2_NOTE,
                       "parallelism": "replicas (one independent workload per GPU)"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                         "kernel": "qkv projection call (RoPE table + GEMM with the norm/rope epilogue)",
                         "algorithmic_flops": flops, "peak_source": peak_src + " burst"},
            "gpu_launches": 2 * K, "clocks": clk.summary(),
            "e2e": {"value": world * flops * e_steps / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": e_ms / e_steps}}
    if world == 1 and not args.no_cpu_baseline:
        cb = cpu_oracle_qkv_sample(name, rows=sh.M)
        line["cpu_baseline"] = {"value": cb["tflops"], "unit": "TFLOP/s", "cores": cb["threads"], "kind": "oracle",
                                "sample": cb["sample"], "seconds": cb["seconds"]}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ varlen prefill
VARLEN_METRIC = "varlen batched causal GQA prefill TFLOP/s (+QK-Norm/RoPE) % bf16 peak"


def varlen_oracle(name: str, seed: int = 0):
    """The oracle's prefill of the batch's longest sequence (over its cached keys, if any)
    with its inputs built once: run(rows) times one call on the last `rows` query rows
    (every head), keys over the whole sequence."""
    import oracle
    from synthetic import as_f64

    sh = VARLEN_SHAPES[name]
    inp = varlen_inputs(sh, seed=seed)
    b = int(np.argmax(sh.lens))
    cu = inp["cu_seqlens"].numpy()
    sl = slice(int(cu[b]), int(cu[b + 1]))
    T, c = sh.lens[b], sh.contexts[b]
    kc = oracle.build_cache_k(as_f64(inp["k_hist"][b]), as_f64(inp["k_norm_w"]), sh.theta, sh.eps).transpose(1, 0, 2)
    vc = as_f64(inp["v_hist"][b]).transpose(1, 0, 2)
    args = (as_f64(inp["q"][sl])[None], as_f64(inp["k"][sl])[None], as_f64(inp["v"][sl])[None],
            as_f64(inp["q_norm_w"]), as_f64(inp["k_norm_w"]), inp["pos"][sl].numpy()[None], kc[None], vc[None], c,
            sh.theta, sh.eps)

    def run(rows: int) -> dict:
        rows = min(rows, T)
        sel = np.arange(T - rows, T)
        t0 = time.perf_counter()
        oracle.chunk_prefill_ref(*args, rows=sel)
        secs = time.perf_counter() - t0
        flops = 4.0 * sh.Hq * sh.d * float((c + sel + 1).sum())
        sample = (f"last {rows} of {T} query rows x {sh.Hq} heads of the longest sequence of the {sh.name}"
                  + (f" (over its {c} cached keys)" if c else "") + f" ({flops:.3g} causal flops)")
        return {"seconds": secs, "flops": flops, "sample": sample}

    run.max_rows = T
    return run


def cpu_oracle_varlen_sample(name: str, rows: int = 256, seed: int = 0):
    """The oracle's prefill of the last `rows` query rows (every head) of the batch's longest
    sequence, keys over the whole sequence."""
    res = varlen_oracle(name, seed)(rows)
    return dict(res, tflops=res["flops"] / res["seconds"] / 1e12, threads=oracle_threads())


def time_call(step, flush, host: dict, dev_inputs: dict, outputs: list, K: int, warmup: int, world, local, dev,
              e2e_steps: int):
    """Time K calls of `step` (L2 flushed before each, outside the event windows) and the same
    call end to end: pinned host inputs in, the call, its outputs back, inside one window."""
    import qwen3_qk_norm_rope_b200 as qa

    for _ in range(warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    with ClockSampler(local) as clk:
        for i in range(K):
            flush.fill_(1.0)
            hold_device()
            ev[i][0].record()
            step()
            ev[i][1].record()
        torch.cuda.synchronize(dev)
        barrier(world)
        torch.cuda.synchronize(dev)
    st, site = qa.device_status(clear=True, device=dev)
    if st != qa.OK:
        raise RuntimeError(f"device status {qa.status_string(st)} at site {site}")
    ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    ph = {k: v.pin_memory() for k, v in host.items()}
    oh = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outputs]
    h2d = sum(v.numel() * v.element_size() for v in ph.values())
    d2h = sum(o.numel() * o.element_size() for o in oh)
    e_ms = 0.0
    for _ in range(e2e_steps):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for k, v in ph.items():
            dev_inputs[k].copy_(v, non_blocking=True)
        step()
        for o, h in zip(outputs, oh):
            h.copy_(o, non_blocking=True)
        e1.record()
        torch.cuda.synchronize(dev)
        e_ms += e0.elapsed_time(e1)
    ms, e_ms = max_over_ranks(world, [ms, e_ms], dev)
    return ms, e_ms, h2d, d2h, clk


def run_varlen(args, world, rank, local):
    name = args.varlen
    sh = VARLEN_SHAPES[name]
    if args.impl == "reference":
        if rank != 0:
            return
        secs, flops, _, sample = reference_steps(varlen_oracle(name), args.steps, args.warmup)
        value = flops / secs / 1e12
        line = {"impl": "reference", "metric": VARLEN_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": sh.name},
                "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                                 "sample": "per step, " + sample},
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    import qwen3_qk_norm_rope_b200 as qa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    inp = varlen_inputs(sh, seed=0)
    host = {k: inp[k] for k in ("q", "k", "v", "q_norm_w", "k_norm_w", "pos", "cu_seqlens")}
    t = {k: v.to(dev) for k, v in host.items()}
    out = torch.empty((sh.N, sh.Hq, sh.d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    cached = any(sh.contexts)
    page = (args.paged or 64) if cached else 0
    kv = {}
    key_cap = 0
    if cached:
        # each sequence's prefix, normed and rotated by the library's prologue, in pages of
        # `page` tokens dealt in a seeded random order; the call appends the new keys after it
        need = [-(-(c + T) // page) for T, c in zip(sh.lens, sh.contexts)]
        g = torch.Generator().manual_seed(78)
        perm = torch.randperm(sum(need), generator=g).to(torch.int32)
        table = torch.full((sh.B, max(need)), -1, dtype=torch.int32)
        off = 0
        for b, nb in enumerate(need):
            table[b, :nb] = perm[off:off + nb]
            off += nb
        k_pages = torch.zeros((sum(need), sh.Hkv, page, sh.d), dtype=torch.bfloat16, device=dev)
        v_pages = torch.zeros_like(k_pages)
        for b, c in enumerate(sh.contexts):
            if c == 0:
                continue
            nb = -(-c // page)
            kc = torch.zeros((1, sh.Hkv, nb * page, sh.d), dtype=torch.bfloat16, device=dev)
            vc = torch.zeros_like(kc)
            pos_b = torch.arange(c, dtype=torch.int32, device=dev)[None]
            qa.qk_norm_rope(inp["k_hist"][b][None].to(dev), t["k_norm_w"], pos_b, kc,
                            v_src=inp["v_hist"][b][None].to(dev), v_dst=vc, theta=sh.theta, eps=sh.eps)
            rows = table[b, :nb].long().to(dev)
            k_pages[rows] = kc[0].view(sh.Hkv, nb, page, sh.d).permute(1, 0, 2, 3)
            v_pages[rows] = vc[0].view(sh.Hkv, nb, page, sh.d).permute(1, 0, 2, 3)
        key_cap = sum(sh.lens) + sum(sh.contexts)
        kv = dict(k_pages=k_pages, v_pages=v_pages, block_table=table.to(dev), ctx_lens=inp["ctx_lens"].to(dev),
                  key_cap=key_cap)
        torch.cuda.synchronize(dev)
        st, site = qa.device_status(clear=True, device=dev)
        if st != qa.OK:
            raise RuntimeError(f"cache build failed: {qa.status_string(st)} at site {site}")
    ws = torch.empty(qa.prefill_varlen_workspace_size(sh.B, sh.N, sh.Hq, sh.Hkv, key_cap=key_cap),
                     dtype=torch.uint8, device=dev)

    def step():
        qa.prefill_varlen(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"], t["cu_seqlens"], out=out,
                          workspace=ws, theta=sh.theta, eps=sh.eps, **kv)

    K = args.steps
    ms, e_ms, h2d, d2h, clk = time_call(step, flush, host, t, [out], K, args.warmup, world, local, dev,
                                        max(1, min(K, 100)))
    if rank != 0:
        return
    flops = sh.causal_flops()
    achieved = flops / (ms * 1e-3 / K) / 1e12
    line = {"metric": VARLEN_METRIC, "value": world * achieved, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": sh.name + (f", pages of {page}" if page else ""), "lens": list(sh.lens),
                       "ctx": list(sh.contexts) if cached else None, "N": sh.N, "Hq": sh.Hq, "Hkv": sh.Hkv, "d": sh.d,
                       "rope_theta": sh.theta, "rms_eps": sh.eps, "seed": 0,
                       "l2": L2_NOTE,
                       "parallelism": "replicas (one independent workload per GPU)"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                         "kernel": "varlen prefill call (metadata + QK prologue + attention)" if not cached
                         else "paged varlen prefill call (metadata + QK prologue into pages + attention reading the "
                              "pages in place)",
                         "algorithmic_flops": flops, "peak_source": peak_src + " burst"},
            "gpu_launches": 3 * K, "clocks": clk.summary(),
            "e2e": {"value": world * flops * max(1, min(K, 100)) / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "ms_per_step": e_ms / max(1, min(K, 100))}}
    if world == 1 and not args.no_cpu_baseline:
        cb = cpu_oracle_varlen_sample(name, rows=512)
        line["cpu_baseline"] = {"value": cb["tflops"], "unit": "TFLOP/s", "cores": cb["threads"], "kind": "oracle",
                                "sample": cb["sample"], "seconds": cb["seconds"]}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ main
def dist_setup(backend: str = "nccl"):
    """One process per GPU (torchrun env).  The process group only carries the timing
    plumbing (barriers and the max over ranks); the data path has no collective."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        timeout = datetime.timedelta(seconds=120)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(world, vals, dev):
    if world == 1:
        return vals
    import torch.distributed as dist

    t = torch.tensor(vals, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle on the host cores, as it stands, on the step's
    prefill workload.  Its inputs are built once; each step is the oracle's prefill of the
    last rows (every head) of the workload, sized so that the warm-up and the K steps take
    about `--reference-budget` seconds of oracle time.  The oracle's decode of one sequence
    takes longer than such a step, so its GB/s comes from one separate call."""
    if rank != 0:
        return
    secs, flops, rows, sample = reference_steps(prefill_oracle(args.prefill, batch_rows=1), args.steps, args.warmup,
                                                args.reference_budget)
    dec = decode_oracle_sample(decode_seqs=1)
    value = flops / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(PREFILL_SHAPES[args.prefill]),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                             "sample": f"per step, {sample}; {dec['sample']} once, outside the steps"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "decode": {"value": dec["gbs"], "unit": "GB/s"}}
    print(json.dumps(line), flush=True)


def config_dict(ps=None, ds=None):
    ps = ps or PREFILL_SHAPES[HEADLINE_PREFILL]
    ds = ds or DECODE_SHAPES["batched-decode"]
    return {"workload": f"{ps.name} + {ds.name}",
            "prefill": {"B": ps.B, "T": ps.T, "Hq": ps.Hq, "Hkv": ps.Hkv, "d": ps.d, "causal": True},
            "decode": {"N": ds.N, "Hq": ds.Hq, "Hkv": ds.Hkv, "d": ds.d, "L": f"U[{ds.lmin},{ds.lmax}]",
                       "Lmax": ds.cache_capacity},
            "rope_theta": ps.theta, "rms_eps": ps.eps, "seed": 0,
            "l2": L2_NOTE_STEP + "; "
                  "decode K/V 4.4 GB > L2",
            "parallelism": "replicas (one independent workload per GPU)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill", default=HEADLINE_PREFILL, choices=sorted(PREFILL_SHAPES),
                    help="prefill workload of the step (default: the long-context wide-GQA prefill)")
    ap.add_argument("--no-other-prefills", action="store_true",
                    help="skip timing the other prefill workloads beside the step")
    ap.add_argument("--reference-budget", type=float, default=REFERENCE_BUDGET_S,
                    help="--impl reference: seconds of oracle time for the warm-up and timed steps together")
    ap.add_argument("--decode-seqs", type=int, default=64,
                    help="decode the first n of the 64 sequences (small cases for ncu captures)")
    ap.add_argument("--workload", default="step", choices=["step", "chunked-prefill", "qkv-proj", "varlen-prefill"],
                    help="step: long-context prefill + batched decode (default); chunked-prefill: the chunk call alone; "
                         "qkv-proj: the merged projection with the QK-Norm/RoPE epilogue; varlen-prefill: a "
                         "ragged batch of prompts packed on one token axis")
    ap.add_argument("--chunk", default="second", choices=sorted(CHUNKS),
                    help="chunked-prefill: second (4096 new tokens over 4096 cached) or short (16 over 32752)")
    ap.add_argument("--qkv", default="qwen3-0.6b-qkv", choices=sorted(QKV_SHAPES),
                    help="the qkv-proj workload's shape")
    ap.add_argument("--varlen", default="qwen3-4b-varlen", choices=sorted(VARLEN_SHAPES),
                    help="the varlen-prefill workload's shape")
    ap.add_argument("--paged", type=int, default=0,
                    help="chunked-prefill: keep the cache in pages of this many tokens (0: contiguous); "
                         "varlen-prefill: the page size of a shape with cached prefixes (default 64)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup("nccl")
    legs = {"chunked-prefill": run_chunk, "qkv-proj": run_qkv, "varlen-prefill": run_varlen}
    if args.workload in legs:
        legs[args.workload](args, world, rank, local)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    w = Workload(dev, prefill=args.prefill, decode_seqs=args.decode_seqs,
                 others=() if args.no_other_prefills else OTHER_PREFILLS)
    for _ in range(args.warmup):
        w.flush_l2()
        w.prefill()
        w.decode()
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        pre_ms, dec_ms = time_steps(w, args.steps)
        barrier(world)
        torch.cuda.synchronize(dev)
    st, site = w.qa.device_status(clear=True, device=dev)
    if st != w.qa.OK:
        raise RuntimeError(f"device status {w.qa.status_string(st)} at site {site}")
    other_ms = time_other_prefills(w, args.steps, args.warmup)
    st, site = w.qa.device_status(clear=True, device=dev)
    if st != w.qa.OK:
        raise RuntimeError(f"device status {w.qa.status_string(st)} at site {site}")
    res = max_over_ranks(world, [pre_ms, dec_ms] + other_ms, dev)
    pre_ms, dec_ms, other_ms = res[0], res[1], res[2:]
    e2e = None
    if not args.no_e2e:
        e_steps = max(1, min(args.steps, 200))
        e_pre, e_tot, h2d, d2h = time_e2e(w, e_steps)
        p_ms, p_h2d, p_d2h = time_e2e_pipelined(w, e_steps)
        e_pre, e_tot, p_ms = max_over_ranks(world, [e_pre, e_tot, p_ms], dev)
        flops = w.ps.causal_flops()
        e2e = {"value": world * flops * e_steps / (p_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(p_h2d), "d2h_bytes_per_step": int(p_d2h), "ms_per_step": p_ms / e_steps,
               "steps": e_steps,
               "schedule": "prefill calls through the public API, each step's inputs copied in from pinned host "
                           "memory and its output copied back on two copy streams that overlap the neighbouring "
                           "steps' compute; one event window over all steps",
               "serial": {"value": world * flops * e_steps / (e_pre * 1e-3) / 1e12, "unit": "TFLOP/s",
                          "ms_per_step": e_pre / e_steps, "step_with_decode_ms": e_tot / e_steps,
                          "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                          "schedule": "one step at a time on one stream: the prefill's inputs in, the call, its "
                                      "output out, then the same for the decode; L2 flushed before each step"}}
    if rank != 0:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return
    K = args.steps
    pre_s, dec_s = pre_ms * 1e-3 / K, dec_ms * 1e-3 / K
    tflops = world * w.ps.causal_flops() / pre_s / 1e12
    dbytes = decode_bytes(w.lens, w.ds.Hq, w.ds.Hkv)
    gbs = world * dbytes / dec_s / 1e9
    clocks = clk.summary()
    dominant_is_decode = dec_s >= pre_s
    rl_dec = {"bound": "hbm", "achieved": dbytes / dec_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
              "frac": dbytes / dec_s / 1e9 / peaks["hbm_gbs"], "traffic": decode_traffic(w.lens),
              "kernel": "decode call (append + split-KV attention + combine)",
              "algorithmic_bytes": dbytes, "peak_source": peak_src}
    # The step's prefill runs back to back for the whole timed region.  When the clock samples
    # taken during it show the power cap, its denominator is the dense bf16 peak measured
    # under the same cap (the sustained figure); otherwise the burst figure.  Both fractions
    # are reported.
    capped = bool(clocks) and "sw_power_cap" in clocks.get("reasons", [])
    pre_tf = w.ps.causal_flops() / pre_s / 1e12
    peak_pre = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
    rl_pre = {"bound": "tensor", "achieved": pre_tf, "peak": peak_pre, "unit": "TFLOP/s", "frac": pre_tf / peak_pre,
              "traffic": prefill_traffic(w.ps), "kernel": "prefill call (K prologue + attention)",
              "algorithmic_flops": w.ps.causal_flops(),
              "peak_source": peak_src + (" sustained (sw_power_cap seen in the timed region)" if capped else " burst"),
              "frac_of_burst": pre_tf / peaks["bf16_tflops"],
              "frac_of_sustained": pre_tf / peaks["bf16_tflops_sustained"]}
    line = {"metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": (pre_ms + dec_ms) / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(w.ps, w.ds),
            "prefill": {"value": tflops, "unit": "TFLOP/s", "ms": pre_s * 1e3, "frac_of_peak": rl_pre["frac"]},
            "decode": {"value": gbs, "unit": "GB/s", "ms": dec_s * 1e3, "frac_of_peak": rl_dec["frac"],
                       "bytes": dbytes, "tflops": world * decode_flops(w.lens, w.ds.Hq) / dec_s / 1e12},
            "roofline": rl_dec if dominant_is_decode else rl_pre,
            "roofline_other": rl_pre if dominant_is_decode else rl_dec,
            "prefill_shapes": {
                name: {"workload": sh.name, "value": world * sh.causal_flops() / (ms * 1e-3) / 1e12,
                       "unit": "TFLOP/s", "ms": ms,
                       "frac_of_peak": sh.causal_flops() / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                       "calls": K, "timing": "alone, L2 flushed before each call, CUDA events"}
                for (name, sh, *_), ms in zip(w.others, other_ms)},
            "gpu_launches": Workload.LAUNCHES_PER_STEP * K,
            "clocks": clocks, "e2e": e2e}
    if world == 1 and not args.no_cpu_baseline:
        cb = cpu_oracle_sample(args.prefill, rows_per_head=512, batch_rows=1, decode_seqs=16)
        line["cpu_baseline"] = {"value": cb["tflops"], "unit": "TFLOP/s", "cores": cb["threads"], "kind": "oracle",
                                "sample": cb["sample"], "decode_gbs": cb["gbs"],
                                "seconds": cb["t_prefill_s"] + cb["t_decode_s"],
                                "prefill_full_s_extrapolated": cb["prefill_full_s_extrapolated"]}
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
