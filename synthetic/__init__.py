"""Seeded synthetic inputs for the Qwen3 attention core.

This module only draws random numbers and rounds them to the storage dtypes.
It holds none of the attention arithmetic (no normalisation, no rotation, no
softmax): both the fp64 oracle and the CUDA path consume what it returns, and
neither of them is imported here.

Workload shapes follow the Qwen3 models described on the pages:
  * Qwen3-0.6B: 16 query heads, 8 KV heads, head_dim 128 ("Qwen3 Architecture
    Layer-by-Layer", config values; "Assembling a large model from scratch",
    shape table).
  * Qwen3-4B: 32 query heads, 8 KV heads, head_dim 128 ("Hand-Writing a
    Vision-Language Model, Part 1", Attention: Grouped-Query Attention).
  * The wide-GQA block of "Qwen 3 From Scratch", Worked example: 64 query
    heads over 4 KV heads, head_dim 128.

Value recipe (one numpy Generator, draws in this order): q, k, v ~ N(0,1);
per-channel scales s_q, s_k with log(s) ~ U(log 0.5, log 4), shared by every
head, token and batch row; gains g_q, g_k = 1 + 0.1 N(0,1) in fp32; then (for
decode) the cached lengths L ~ U{1024..32768}.  q and k are multiplied by
their scale vector, then q, k, v are rounded to bf16.  Positions are 0..T-1.
Draws are made in float32 (numpy's float32 normal stream) to halve host memory
on the 32768-token workload.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

HEAD_DIM = 128
ROPE_THETA = 1.0e6
RMS_EPS = 1.0e-6


@dataclass(frozen=True)
class PrefillShape:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    d: int = HEAD_DIM
    theta: float = ROPE_THETA
    eps: float = RMS_EPS

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def causal_flops(self) -> float:
        """QK^T and PV over the causal triangle only: 4*B*Hq*d*T(T+1)/2."""
        return 4.0 * self.B * self.Hq * self.d * self.T * (self.T + 1) / 2.0


@dataclass(frozen=True)
class DecodeShape:
    name: str
    N: int
    Hq: int
    Hkv: int
    d: int = HEAD_DIM
    lmin: int = 1024
    lmax: int = 32768
    theta: float = ROPE_THETA
    eps: float = RMS_EPS

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def cache_capacity(self) -> int:
        """Slots per (sequence, KV head): the longest history plus the appended token."""
        return self.lmax + 1


@dataclass(frozen=True)
class ChunkShape:
    """T new tokens per batch row after `start` cached ones (chunked prefill)."""
    name: str
    B: int
    start: int
    T: int
    Hq: int
    Hkv: int
    d: int = HEAD_DIM
    theta: float = ROPE_THETA
    eps: float = RMS_EPS

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def causal_flops(self) -> float:
        """QK^T and PV over the visible keys: new row i sees start + i + 1 of them."""
        return 4.0 * self.B * self.Hq * self.d * (self.T * self.start + self.T * (self.T + 1) / 2.0)


PREFILL_SHAPES = {
    "tiny": PrefillShape("tiny prefill B=1 T=128 Hq=16 Hkv=8", 1, 128, 16, 8),
    "qwen3-0.6b": PrefillShape("Qwen3-0.6B-shaped prefill B=2 T=2048 Hq=16 Hkv=8", 2, 2048, 16, 8),
    "qwen3-4b": PrefillShape("Qwen3-4B-shaped prefill B=1 T=8192 Hq=32 Hkv=8", 1, 8192, 32, 8),
    "long-wide-gqa": PrefillShape("long-context wide-GQA prefill B=1 T=32768 Hq=64 Hkv=4", 1, 32768, 64, 4),
}

DECODE_SHAPES = {
    "batched-decode": DecodeShape("batched decode N=64 Hq=32 Hkv=8 L~U[1024,32768]", 64, 32, 8),
}


CHUNK_SHAPES = {
    "qwen3-4b-second-chunk": ChunkShape("Qwen3-4B-shaped chunked prefill B=1 start=4096 T=4096 Hq=32 Hkv=8",
                                        1, 4096, 4096, 32, 8),
    # a few new tokens over a long cached prefix (the prefix fills the 32768-token context)
    "qwen3-4b-short-chunk": ChunkShape("Qwen3-4B-shaped short chunk B=1 start=32752 T=16 Hq=32 Hkv=8",
                                       1, 32752, 16, 32, 8),
}


@dataclass(frozen=True)
class VarlenShape:
    """B sequences packed on one token axis: new lengths `lens`, cached prefix lengths `ctx`
    (empty: fresh prompts), and `lead` / `tail` padding tokens that belong to no sequence."""
    name: str
    lens: tuple
    Hq: int
    Hkv: int
    ctx: tuple = ()
    lead: int = 0
    tail: int = 0
    d: int = HEAD_DIM
    theta: float = ROPE_THETA
    eps: float = RMS_EPS

    @property
    def B(self) -> int:
        return len(self.lens)

    @property
    def N(self) -> int:
        return self.lead + sum(self.lens) + self.tail

    @property
    def contexts(self) -> tuple:
        return self.ctx if self.ctx else (0,) * self.B

    def causal_flops(self) -> float:
        """QK^T and PV over each sequence's visible keys (new row i sees ctx + i + 1)."""
        return sum(4.0 * self.Hq * self.d * (T * c + T * (T + 1) / 2.0) for T, c in zip(self.lens, self.contexts))


def ragged_lengths(B: int, lo: int, hi: int, seed: int) -> tuple:
    """B lengths log-uniform in [lo, hi] (a serving batch's mix of short and long prompts)."""
    rng = np.random.default_rng(seed)
    return tuple(int(x) for x in np.exp(rng.uniform(np.log(lo), np.log(hi), size=B)).round())


VARLEN_SHAPES = {
    "qwen3-4b-varlen": VarlenShape("Qwen3-4B-shaped varlen prefill, 16 prompts of log-uniform length in "
                                   "[128, 8192], Hq=32 Hkv=8", ragged_lengths(16, 128, 8192, 2024), 32, 8),
    # continuous batching: new chunks of 64..2048 tokens over cached prefixes of 256..16384
    "qwen3-4b-varlen-cached": VarlenShape("Qwen3-4B-shaped varlen prefill over a paged cache, 16 chunks of "
                                          "log-uniform length in [64, 2048] after cached prefixes of log-uniform "
                                          "length in [256, 16384], Hq=32 Hkv=8",
                                          ragged_lengths(16, 64, 2048, 7), 32, 8,
                                          ctx=ragged_lengths(16, 256, 16384, 8)),
}


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _scales(rng: np.random.Generator, d: int) -> np.ndarray:
    return np.exp(rng.uniform(np.log(0.5), np.log(4.0), size=d)).astype(np.float32)


def _gains(rng: np.random.Generator, d: int) -> np.ndarray:
    return (1.0 + 0.1 * rng.standard_normal(d)).astype(np.float32)


def prefill_inputs(shape: PrefillShape, seed: int = 0) -> dict:
    """Raw prefill inputs as CPU tensors.

    q [B,T,Hq,d], k and v [B,T,Hkv,d] bf16; q_norm_w and k_norm_w [d] fp32;
    pos [B,T] int32 holding 0..T-1 for every batch row.
    """
    B, T, Hq, Hkv, d = shape.B, shape.T, shape.Hq, shape.Hkv, shape.d
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, Hq, d), dtype=np.float32)
    k = rng.standard_normal((B, T, Hkv, d), dtype=np.float32)
    v = rng.standard_normal((B, T, Hkv, d), dtype=np.float32)
    s_q, s_k = _scales(rng, d), _scales(rng, d)
    g_q, g_k = _gains(rng, d), _gains(rng, d)
    q *= s_q
    k *= s_k
    pos = np.broadcast_to(np.arange(T, dtype=np.int32), (B, T)).copy()
    return {
        "q": _bf16(q), "k": _bf16(k), "v": _bf16(v),
        "q_norm_w": torch.from_numpy(g_q), "k_norm_w": torch.from_numpy(g_k),
        "pos": torch.from_numpy(pos),
    }


def chunk_inputs(shape: ChunkShape, seed: int = 0) -> dict:
    """A prompt of start + T tokens drawn exactly as prefill_inputs draws it, split in two:
    the raw history k_hist, v_hist [B,start,Hkv,d] (the cache stores k_hist only after
    QK-Norm and RoPE at positions 0..start-1) and the T new tokens q, k, v at positions
    start..start+T-1, with the gains."""
    full = prefill_inputs(PrefillShape(shape.name, shape.B, shape.start + shape.T, shape.Hq, shape.Hkv,
                                       shape.d, shape.theta, shape.eps), seed)
    s = shape.start
    return {
        "q": full["q"][:, s:].contiguous(), "k": full["k"][:, s:].contiguous(), "v": full["v"][:, s:].contiguous(),
        "pos": full["pos"][:, s:].contiguous(), "q_norm_w": full["q_norm_w"], "k_norm_w": full["k_norm_w"],
        "k_hist": full["k"][:, :s].contiguous(), "v_hist": full["v"][:, :s].contiguous(),
    }


@dataclass(frozen=True)
class QkvShape:
    """A merged qkv projection: M tokens of `hidden` features to Hq + 2 Hkv heads of d."""
    name: str
    M: int
    hidden: int
    Hq: int
    Hkv: int
    d: int = HEAD_DIM
    theta: float = ROPE_THETA
    eps: float = RMS_EPS

    def flops(self) -> float:
        return 2.0 * self.M * self.hidden * (self.Hq + 2 * self.Hkv) * self.d


QKV_SHAPES = {
    "qwen3-0.6b-qkv": QkvShape("Qwen3-0.6B-shaped qkv projection M=4096 hidden=1024 Hq=16 Hkv=8", 4096, 1024, 16, 8),
    "qwen3-4b-qkv": QkvShape("Qwen3-4B-shaped qkv projection M=8192 hidden=2560 Hq=32 Hkv=8", 8192, 2560, 32, 8),
}


def qkv_proj_inputs(shape: QkvShape, seed: int = 0) -> dict:
    """Hidden states x ~ N(0,1) [M, hidden] and stacked weights w_qkv ~ N(0, 1/hidden)
    [(Hq + 2 Hkv) d, hidden], the q and k rows multiplied per output channel by scale
    vectors s_q, s_k (log-uniform in [0.5, 4], as the prefill recipe scales q and k), all
    bf16; gains 1 + 0.1 N(0,1) fp32; positions 0..M-1 int32."""
    rng = np.random.default_rng(seed)
    d = shape.d
    x = rng.standard_normal((shape.M, shape.hidden), dtype=np.float32)
    w = rng.standard_normal(((shape.Hq + 2 * shape.Hkv) * d, shape.hidden), dtype=np.float32)
    w *= np.float32(1.0 / np.sqrt(shape.hidden))
    s_q, s_k = _scales(rng, d), _scales(rng, d)
    g_q, g_k = _gains(rng, d), _gains(rng, d)
    nq, nk = shape.Hq * d, shape.Hkv * d
    w[:nq] *= np.tile(s_q, shape.Hq)[:, None]
    w[nq:nq + nk] *= np.tile(s_k, shape.Hkv)[:, None]
    return {"x": _bf16(x), "w_qkv": _bf16(w), "q_norm_w": torch.from_numpy(g_q), "k_norm_w": torch.from_numpy(g_k),
            "pos": torch.arange(shape.M, dtype=torch.int32)}


def decode_step_inputs(shape: DecodeShape, seed: int = 0) -> dict:
    """The new token of every sequence plus the cached lengths.

    q [N,Hq,d], k_new and v_new [N,Hkv,d] bf16 (raw, before QK-Norm/RoPE);
    gains [d] fp32; cache_lens [N] int32 ~ U{lmin..lmax}; the scale vector
    s_k is returned too so that cache histories can be drawn like config k.
    """
    N, Hq, Hkv, d = shape.N, shape.Hq, shape.Hkv, shape.d
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((N, Hq, d), dtype=np.float32)
    k = rng.standard_normal((N, Hkv, d), dtype=np.float32)
    v = rng.standard_normal((N, Hkv, d), dtype=np.float32)
    s_q, s_k = _scales(rng, d), _scales(rng, d)
    g_q, g_k = _gains(rng, d), _gains(rng, d)
    lens = rng.integers(shape.lmin, shape.lmax, size=N, endpoint=True).astype(np.int32)
    q *= s_q
    k *= s_k
    return {
        "q": _bf16(q), "k_new": _bf16(k), "v_new": _bf16(v),
        "q_norm_w": torch.from_numpy(g_q), "k_norm_w": torch.from_numpy(g_k),
        "cache_lens": torch.from_numpy(lens), "s_k": torch.from_numpy(s_k),
    }


def decode_history(shape: DecodeShape, n: int, length: int, s_k: torch.Tensor, seed: int = 0) -> dict:
    """Raw history of sequence n: k_hist (scaled like k) and v_hist [length,Hkv,d] bf16.

    Each sequence has its own child stream (seed, 1, n), so one sequence can be
    drawn without drawing the others.  k_hist is raw: the cache stores it only
    after QK-Norm and RoPE at positions 0..length-1.
    """
    rng = np.random.default_rng([seed, 1, n])
    k = rng.standard_normal((length, shape.Hkv, shape.d), dtype=np.float32)
    v = rng.standard_normal((length, shape.Hkv, shape.d), dtype=np.float32)
    k *= s_k.numpy()
    return {"k_hist": _bf16(k), "v_hist": _bf16(v)}


def as_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16/fp32/int tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def varlen_inputs(shape: VarlenShape, seed: int = 0) -> dict:
    """Packed inputs as CPU tensors: q [N,Hq,d], k and v [N,Hkv,d] drawn as one prompt of N
    tokens by the recipe above; cu_seqlens [B+1] int32 (the first sequence starts after the
    lead padding); pos [N] int32, ctx_b + t for token t of sequence b and 0 for padding;
    ctx_lens [B] int32; and per sequence the raw history k_hist[b], v_hist[b] [ctx_b,Hkv,d]
    (drawn after the gains, N(0,1), k scaled by s_k), which a cache holds after QK-Norm and
    RoPE at positions 0..ctx_b-1."""
    N, Hq, Hkv, d = shape.N, shape.Hq, shape.Hkv, shape.d
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((N, Hq, d), dtype=np.float32)
    k = rng.standard_normal((N, Hkv, d), dtype=np.float32)
    v = rng.standard_normal((N, Hkv, d), dtype=np.float32)
    s_q, s_k = _scales(rng, d), _scales(rng, d)
    g_q, g_k = _gains(rng, d), _gains(rng, d)
    q *= s_q
    k *= s_k
    cu = np.concatenate([[shape.lead], shape.lead + np.cumsum(shape.lens, dtype=np.int64)]).astype(np.int32)
    pos = np.zeros(N, dtype=np.int32)
    k_hist, v_hist = [], []
    for b, (T, c) in enumerate(zip(shape.lens, shape.contexts)):
        pos[cu[b]:cu[b + 1]] = c + np.arange(T, dtype=np.int32)
        kh = rng.standard_normal((c, Hkv, d), dtype=np.float32) * s_k
        vh = rng.standard_normal((c, Hkv, d), dtype=np.float32)
        k_hist.append(_bf16(kh))
        v_hist.append(_bf16(vh))
    return {
        "q": _bf16(q), "k": _bf16(k), "v": _bf16(v),
        "q_norm_w": torch.from_numpy(g_q), "k_norm_w": torch.from_numpy(g_k),
        "pos": torch.from_numpy(pos), "cu_seqlens": torch.from_numpy(cu),
        "ctx_lens": torch.from_numpy(np.asarray(shape.contexts, dtype=np.int32)),
        "k_hist": k_hist, "v_hist": v_hist,
    }
