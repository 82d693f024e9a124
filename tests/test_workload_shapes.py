"""The synthetic workloads take their head counts, head size, hidden size, RMSNorm eps and
RoPE base from the model configurations the pages print (tests/golden/worked_examples.json,
each entry citing its page and section), so a benchmark or parity case named after a model
has that model's attention shapes."""
import json
import os

from synthetic import (DECODE_SHAPES, HEAD_DIM, PREFILL_SHAPES, QKV_SHAPES, RMS_EPS, ROPE_THETA, VARLEN_SHAPES,
                       CHUNK_SHAPES)

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def test_qwen3_0p6b_shapes():
    g = GOLDEN["qwen3_0p6b"]
    assert HEAD_DIM == g["head_dim"] and RMS_EPS == g["rms_norm_eps"] and ROPE_THETA == g["rope_theta"]
    for s in (PREFILL_SHAPES["qwen3-0.6b"], QKV_SHAPES["qwen3-0.6b-qkv"]):
        assert (s.Hq, s.Hkv, s.d) == (g["n_query_heads"], g["n_kv_heads"], g["head_dim"])
        assert s.Hq // s.Hkv == g["num_key_value_groups"]
    qkv = QKV_SHAPES["qwen3-0.6b-qkv"]
    assert qkv.hidden == g["hidden_size"]
    assert [qkv.Hq * qkv.d, qkv.hidden] == g["q_proj_weight"]
    assert [qkv.Hkv * qkv.d, qkv.hidden] == g["k_proj_weight"]
    assert [qkv.d] == g["q_norm_weight"]


def test_qwen3_4b_shapes():
    g = GOLDEN["qwen3_4b"]
    shapes = [PREFILL_SHAPES["qwen3-4b"], QKV_SHAPES["qwen3-4b-qkv"], DECODE_SHAPES["batched-decode"],
              *CHUNK_SHAPES.values(), *VARLEN_SHAPES.values()]
    for s in shapes:
        assert (s.Hq, s.Hkv, s.d) == (g["n_query_heads"], g["n_kv_heads"], g["head_dim"]), s.name
        assert s.Hq // s.Hkv == g["n_rep"]
    qkv = QKV_SHAPES["qwen3-4b-qkv"]
    assert [qkv.Hq * qkv.d, qkv.hidden] == g["q_proj_weight"]


def test_wide_gqa_block_shapes():
    g = GOLDEN["wide_gqa_block"]
    s = PREFILL_SHAPES["long-wide-gqa"]
    assert (s.Hq, s.Hkv, s.d) == (g["n_query_heads"], g["n_kv_heads"], g["head_dim"])
    assert g["query_projection"][1] == s.Hq * s.d and g["key_value_projection"][1] == s.Hkv * s.d
