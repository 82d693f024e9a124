"""fp64 CPU oracle for the Qwen3 attention core.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg, never by the library.  It shares no code with
the CUDA path.  Every function is pinned by `tests/test_oracle_pins.py`
(closed forms, invariants, special cases and brute force).
"""
from .attention import (  # noqa: F401
    bf16_round,
    build_cache_k,
    chunk_prefill_ref,
    decode_ref,
    kv_cache_values_per_token,
    paged_gather,
    prefill_ref,
    qk_prologue,
    qkv_proj_norm_rope_ref,
    rms_norm,
    rope,
    rope_inv_freq,
    varlen_prefill_ref,
)
from .loops import (  # noqa: F401
    chunk_prefill_loops,
    decode_loops,
    prefill_loops,
    qkv_proj_norm_rope_loops,
    varlen_prefill_loops,
)
