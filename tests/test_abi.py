"""The C-ABI library loads and exports every entry point include/lyc.h
declares; host-only arithmetic of the ABI (no GPU needed)."""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lyc():
    from hybrid_head_sparse_b200 import build as B
    B.build()
    from hybrid_head_sparse_b200 import lyc as m
    m.load()
    return m


def declared_functions():
    src = open(os.path.join(ROOT, "include", "lyc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lyc_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lyc):
    names = declared_functions()
    assert len(names) >= 12
    lib = lyc.load()
    for name in names:
        assert hasattr(lib, name), f"{name} declared in lyc.h but not exported"
    assert sorted(lyc.EXPORTED) == names


def test_status_strings(lyc):
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert lyc.lyc_status_string(code)


def test_create_rejects_bad_config(lyc):
    bad = [
        lyc.lyc_config(0, 1, 4, 2, 64, 128, 8, 0, 0, 0, 0),      # no layers
        lyc.lyc_config(1, 1, 6, 4, 64, 128, 8, 0, 0, 0, 0),      # Hq % Hkv != 0
        lyc.lyc_config(1, 1, 4, 2, 96, 128, 8, 0, 0, 0, 0),      # head_dim 96
        lyc.lyc_config(1, 1, 32, 2, 64, 128, 8, 0, 0, 0, 0),     # group of 16
        lyc.lyc_config(1, 1, 4, 2, 64, 1 << 21, 8, 0, 0, 0, 0),  # context too long
        lyc.lyc_config(1, 1, 4, 2, 64, 128, 0, 0, 0, 0, 0),      # k budget 0
    ]
    for cfg in bad:
        with pytest.raises(lyc.LycError) as e:
            lyc.lyc_create(cfg)
        assert e.value.code in (lyc.LYC_ERR_INVALID_ARG, lyc.LYC_ERR_UNSUPPORTED)


def ref_bytes(L, Hq, Hkv, d, es, B, role, n, k, kvmode, s_in=False):
    """Byte counts written out directly from their definitions."""
    G = Hq // Hkv
    keff = min(k, n)
    row = d * es * 2
    a = dist = 0
    for l in range(L):
        for g in range(Hkv):
            heads = range(g * G, (g + 1) * G)
            ret = [(l == 0 and not s_in) or role[l, h] for h in heads]
            nsp = sum(1 for r in ret if not r)
            if any(ret):
                a += n * row
                dist += n * row
            else:
                a += keff * row
            dist += (keff * row if nsp else 0) if kvmode else nsp * keff * row
    return a * B, dist * B


@pytest.mark.parametrize("kvmode", [0, 1])
def test_step_bytes(lyc, kvmode):
    rng = np.random.default_rng(0)
    L, Hq, Hkv, d = 32, 32, 8, 128
    role = (rng.random((L, Hq)) < 0.07).astype(np.uint8)
    cfg = lyc.lyc_config(L, 1, Hq, Hkv, d, 131072, 4096, lyc.LYC_BF16, kvmode, 0, 0)
    for n, k in ((131072, 4096), (1000, 4096), (32768, 1)):
        got = lyc.lyc_step_bytes(cfg, role, n, k)
        assert got == ref_bytes(L, Hq, Hkv, d, 2, 1, role, n, k, kvmode)
    # the headline layout: layer 0 dense, then two retrieval heads in distinct groups
    role = np.zeros((L, Hq), dtype=np.uint8)
    role[1:, 0] = 1
    role[1:, 5] = 1
    a, _ = lyc.lyc_step_bytes(cfg, role, 131072, 4096)
    assert a == (8 * 131072 + 31 * (2 * 131072 + 6 * 4096)) * 512
