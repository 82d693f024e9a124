"""The fp64 oracle against closed forms, invariants, special cases, a library
routine (torch fp64 SDPA for the attention part, torch's bf16 conversion for
rounding), brute-force loops and the numbers the pages print."""
import pytest

from tests import oracle_checks as C


@pytest.mark.parametrize("check", C.ALL_CHECKS, ids=lambda f: f.__name__[len("check_"):])
def test_oracle_pin(check):
    check()
