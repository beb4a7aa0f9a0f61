"""The fp64 oracle, pinned to closed forms, library routines, brute force and
the method's invariants (CPU only)."""
import numpy as np
import pytest

import oracle as O
from tests import oracle_pins as P


@pytest.fixture(scope="module")
def ora():
    return O.default()


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(ora, pin):
    pin(ora)


def test_bad_inherited_index_rejected(ora):
    rng = np.random.default_rng(0)
    st = P.rand_stack(rng, L=1, B=1, Hq=2, Hkv=1, d=4, n=10, role=np.array([[1, 0]]))
    S_in = np.array([[[0, 1, 2], [3, 4, 10]]], dtype=np.int32)   # 10 >= n
    with pytest.raises(ValueError):
        ora.layer(st, 0, 3, S_in, all_retrieval=False)


def test_bf16_rounding_helper():
    # the test helper rounds to nearest even like torch's bf16 cast
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e-3], dtype=np.float32)
    import torch
    exp = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(P.bf16_bits(x), exp)
