"""The oracle against the hand-worked examples in tests/golden/ (their README
says where each comes from)."""
import json
import math
import os

import numpy as np
import pytest

import oracle as O

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _expr(s: str) -> float:
    return float(eval(s, {"__builtins__": {}}, {"e": math.e}))


def test_worked_tie_example():
    with open(os.path.join(HERE, "worked_tie_example.json")) as f:
        g = json.load(f)
    L, B, Hq, Hkv, d, n, k = (g[x] for x in ("L", "B", "Hq", "Hkv", "d", "n", "k"))
    q = np.zeros((L, B, Hq, d), dtype=np.float32)
    K = np.zeros((L, B, Hkv, n, d), dtype=np.float32)
    V = np.zeros((L, B, Hkv, n, d), dtype=np.float32)
    q[:, 0, 0] = g["q"]
    K[:, 0, 0] = g["K"]
    V[:, 0, 0] = g["V"]
    st = O.Stack(q, K, V, np.array(g["role"], dtype=np.uint8))
    out, S, trace = O.decode_step(st, k, trace=True)
    want = np.array([[_expr(x) for x in row] for row in g["expect_out"]])
    np.testing.assert_allclose(out[:, 0, 0], want, rtol=0, atol=1e-15)
    assert trace[:, 0, 0].tolist() == g["expect_trace"]
    assert S[0, 0].tolist() == g["expect_trace"][-1]
