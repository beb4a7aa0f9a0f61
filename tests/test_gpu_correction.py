"""Cache Correction's dense causal attention (lyc_cache_correction) on a B200
against the fp64 oracle (oracle.correction), with the tolerances of
tests/parity.py.  The refreshed K/V rows are written by the library first;
the oracle gets the same cache with those rows written on the host."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from hybrid_head_sparse_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lyc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from hybrid_head_sparse_b200 import lyc as lycmod
    lycmod.load()
    return lycmod


def correction_case(L, B, Hq, Hkv, n, T, seed, rows=None):
    spec = W.StackSpec(f"corr-{L}L-{B}b-n{n}", L=L, B=B, Hq=Hq, Hkv=Hkv, d=128, n=n, k=64,
                       planted="heavy", n_planted=min(64, max(1, n - 8)), seed=seed, n_max=rows)
    data = W.make_stack(spec, "cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 1)
    q = torch.randn((L, B, Hq, T, 128), generator=g, device="cuda").to(torch.bfloat16)
    k_new = torch.randn((L, B, Hkv, T, 128), generator=g, device="cuda").to(torch.bfloat16)
    v_new = torch.randn((L, B, Hkv, T, 128), generator=g, device="cuda").to(torch.bfloat16)
    return spec, data, q, k_new, v_new


def expected(spec, data, q, k_new, v_new, n, T, layers=None):
    """The oracle on the host copy of the cache with the refreshed rows written."""
    idx = list(range(spec.L)) if layers is None else list(layers)
    sel = torch.tensor(idx, device=data["k"].device)
    K = W.host_view(data["k"].index_select(0, sel)[:, :, :, :n]).copy()
    V = W.host_view(data["v"].index_select(0, sel)[:, :, :, :n]).copy()
    if k_new is not None:
        K[:, :, :, n - T:n] = W.host_view(k_new.index_select(0, sel))
        V[:, :, :, n - T:n] = W.host_view(v_new.index_select(0, sel))
    st = O.Stack(W.host_view(data["q"].index_select(0, sel)), np.ascontiguousarray(K),
                 np.ascontiguousarray(V), np.ones((len(idx), spec.Hq), dtype=np.uint8))
    return O.correction(st, W.host_view(q.index_select(0, sel)))


def run(lyc, spec, data, q, k_new, v_new, n, T):
    ctx = lyc.Lyc(spec.L, spec.B, spec.Hq, spec.Hkv, 128, spec.rows, spec.k)
    out = torch.full((spec.L, spec.B, spec.Hq, T, 128), float("nan"), device="cuda")
    ctx.cache_correction(q, data["k"], data["v"], n, out, k_new=k_new, v_new=v_new)
    rc = ctx.sync_status()
    torch.cuda.synchronize()
    ctx.close()
    return rc, out.cpu().numpy()


@pytest.mark.parametrize("L,B,Hq,Hkv,n,T", [
    (2, 2, 8, 2, 1000, 32),   # G*T = 128 rows, ragged last tile
    (2, 1, 8, 2, 300, 8),     # 32 query rows (96 padding rows)
    (1, 2, 8, 2, 32, 32),     # n = T: one tile, the mask inside it
    (2, 1, 8, 2, 129, 32),    # last tile of one row: fully masked for most queries
    (4, 2, 4, 2, 1024, 16),   # 16 groups x 8 tiles < one CTA per tile: groups split in pieces
    (1, 1, 32, 8, 5000, 32),  # Llama3-8B heads
])
def test_correction_matches_oracle(lyc, L, B, Hq, Hkv, n, T):
    spec, data, q, k_new, v_new = correction_case(L, B, Hq, Hkv, n, T, seed=7 * n + T)
    exp = expected(spec, data, q, k_new, v_new, n, T)
    rc, out = run(lyc, spec, data, q, k_new, v_new, n, T)
    assert rc == 0, lyc.status_string(rc)
    assert np.isfinite(out).all()
    P.check_out(out, exp, "bf16", f"correction n={n} T={T}")
    # the refreshed rows are in the cache
    assert torch.equal(data["k"][:, :, :, n - T:n], k_new)
    assert torch.equal(data["v"][:, :, :, n - T:n], v_new)


def test_correction_without_new_rows_and_padded_cache(lyc):
    """No refreshed rows passed (the cache already holds them); the cache has
    more rows allocated than n, so rows past n must not be read."""
    spec, data, q, _, _ = correction_case(2, 2, 8, 2, 700, 24, seed=3, rows=900)
    data["k"][:, :, :, 700:] = 1e4
    data["v"][:, :, :, 700:] = float("nan")
    exp = expected(spec, data, q, None, None, 700, 24)
    rc, out = run(lyc, spec, data, q, None, None, 700, 24)
    assert rc == 0
    P.check_out(out, exp, "bf16", "correction, padded cache")


def test_correction_unsupported_shapes(lyc):
    ctx = lyc.Lyc(1, 1, 8, 2, 128, 256, 64)
    q = torch.zeros((1, 1, 8, 33, 128), dtype=torch.bfloat16, device="cuda")  # G*T = 132 > 128
    K = torch.zeros((1, 1, 2, 256, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((1, 1, 8, 33, 128), device="cuda")
    with pytest.raises(lyc.LycError) as e:
        ctx.cache_correction(q, K, K, 256, out)
    assert e.value.code == lyc.LYC_ERR_UNSUPPORTED
    q = torch.zeros((1, 1, 8, 8, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lyc.LycError) as e:
        ctx.cache_correction(q, K, K, 4, out)  # T > n
    assert e.value.code == lyc.LYC_ERR_INVALID_ARG
    ctx.close()
    ctx = lyc.Lyc(1, 1, 8, 2, 64, 256, 64, dtype="fp32")
    with pytest.raises(lyc.LycError) as e:
        ctx.cache_correction(q, K, K, 256, out)
    assert e.value.code == lyc.LYC_ERR_UNSUPPORTED
    ctx.close()


def test_correction_full_size_llama3_8b_128k(lyc):
    """The 128K Llama3-8B stack with T = 32: layers 0 and 31 checked in full
    against the oracle."""
    L, n, T = 32, 131072, 32
    spec, data, q, k_new, v_new = correction_case(L, 1, 32, 8, n, T, seed=11)
    rc, out = run(lyc, spec, data, q, k_new, v_new, n, T)
    assert rc == 0, lyc.status_string(rc)
    exp = expected(spec, data, q, k_new, v_new, n, T, layers=[0, L - 1])
    P.check_out(out[[0, L - 1]], exp, "bf16", "correction 128K layers 0, 31")
