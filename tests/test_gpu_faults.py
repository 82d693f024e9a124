"""Failure detection without a GPU fault: the fault-injection hook makes the prefill
producer skip its first key-tile load, so the consumers' bounded waits run out (limit set
to 50 ms).  The kernel must end on its own, report QWEN3_ERR_DEVICE_TIMEOUT through the
status word, and leave the context usable for a correct run right after."""
import pytest
import torch

import qwen3_qk_norm_rope_b200 as qa
from synthetic import PREFILL_SHAPES, prefill_inputs
from tests.gpu_common import compare, dev, prefill_gpu, prefill_oracle, to_np

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    d = dev()
    inp = prefill_inputs(PREFILL_SHAPES["tiny"], seed=0)
    t = {k: v.to(d) for k, v in inp.items()}
    qa.device_status(clear=True)
    old = qa.set_wait_limit(50_000_000)
    qa.set_fault_injection(1)
    try:
        qa.prefill(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["pos"])
        st, site = qa.device_status(clear=True)
    finally:
        qa.set_fault_injection(0)
        qa.set_wait_limit(old)
    assert st == qa.ERR_DEVICE_TIMEOUT, (st, site)
    assert 20 <= site <= 29, site
    out, lse = prefill_gpu(inp)
    ref, ref_lse, st_lse = prefill_oracle(inp)
    compare(to_np(out), to_np(lse), ref, ref_lse, st_lse, "after the injected timeout")
