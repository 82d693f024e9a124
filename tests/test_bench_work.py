"""The algorithmic work that bench.py divides by measured time (the roofline numerators):
causal prefill flops 4*B*Hq*d*T(T+1)/2 and decode bytes (every cached K/V row once, q in,
out, the new k and v read and written), checked against hand-computed values and the
per-workload totals they must give."""
import numpy as np

import bench
from synthetic import DECODE_SHAPES, PREFILL_SHAPES, decode_step_inputs


def test_prefill_causal_flops():
    # 4 flops per (query row, visible key, dim): QK^T and PV, masked work excluded
    assert PREFILL_SHAPES["tiny"].causal_flops() == 4 * 1 * 16 * 128 * 128 * 129 / 2
    expected = {"tiny": 6.76e7, "qwen3-0.6b": 3.44e10, "qwen3-4b": 5.50e11, "long-wide-gqa": 1.759e13}
    for name, flops in expected.items():
        assert abs(PREFILL_SHAPES[name].causal_flops() / flops - 1) < 2e-3, name


def test_decode_bytes_by_hand():
    # one sequence of 1024 cached tokens, Hq = 32, Hkv = 8, d = 128, bf16:
    #   K and V rows: 1024 x 2 x 8 x 128 x 2 B; q in and out: 2 x 32 x 128 x 2 B;
    #   new k and v read and written: 2 x 2 x 8 x 128 x 2 B
    want = 1024 * 2 * 8 * 128 * 2 + 2 * 32 * 128 * 2 + 2 * 2 * 8 * 128 * 2
    assert bench.decode_bytes(np.array([1024]), 32, 8) == want
    assert bench.decode_bytes(np.array([1024, 3]), 32, 8) == want + 3 * 4096 + 2 * 32 * 128 * 2 + 8192


def test_batched_decode_totals():
    shape = DECODE_SHAPES["batched-decode"]
    lens = decode_step_inputs(shape, seed=0)["cache_lens"].numpy()
    total = bench.decode_bytes(lens, shape.Hq, shape.Hkv)
    assert total == 4096 * int(lens.astype(np.int64).sum()) + 64 * (16384 + 8192)
    assert 4.3e9 < total < 4.5e9  # about 4.4 GB of K/V streamed per step at the seed-0 lengths
    # 4 flops per (query head, key, dim), the new key included: ~4 flops per byte, HBM bound
    assert abs(bench.decode_flops(lens, shape.Hq) / total - 4.0) < 0.1
