"""The oracle against facts outside itself (CPU only).

Covers the four self-checks the layer must pass before any GPU comparison:
sharded == unsharded for every N, GeLU against its closed forms, finite
differences on tiny shapes, and the embedding equal to a plain row lookup bit
for bit; plus the worked examples the pages print and closed-form cases.
"""
import pytest

import oracle
from tests import oracle_checks as C


@pytest.mark.parametrize("check", C.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(oracle.tp_oracle)
