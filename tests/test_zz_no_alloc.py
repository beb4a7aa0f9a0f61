"""lyc_sparse_attention_noalloc, the entry point for callers that cannot
allocate device memory (a framework whose caching allocator owns the GPU's
memory, a serving path where cudaMalloc may synchronize the device), against
the existing entry point, lyc_decode_step, and against the fp64 oracle, on
the same inputs.

A one-layer step whose every head is sparse and whose sets are handed in
(LYC_STEP_S_IN) computes the same thing for every head: attention over the
rows of the head's set.  Calls in a row, with different inputs and shapes,
check that the shared scratch array's leftover contents (counters, partial
states, work list) do not leak into the next call.  The file name makes
pytest collect it last; it also passes alone.
"""
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
    from hybrid_head_sparse_b200 import lyc as m
    m.load()
    return m


def reference(lyc, data, S0, n, k):
    """The existing entry point: a one-layer step, every head sparse."""
    spec = data["spec"]
    ctx = lyc.Lyc(1, spec.B, spec.Hq, spec.Hkv, spec.d, n, k)
    out = torch.full((1, spec.B, spec.Hq, spec.d), float("nan"), device="cuda")
    S = S0.clone()
    role = np.zeros((1, spec.Hq), dtype=np.uint8)
    ctx.decode_step(data["q"], data["k"], data["v"], n, role, k, out, S, s_in=True)
    assert ctx.sync_status() == 0
    torch.cuda.synchronize()
    ctx.close()
    return out[0].cpu().numpy()


def oracle_sparse(data, S0, n, k):
    """The fp64 oracle's layer with every head sparse over the given sets."""
    spec = data["spec"]
    st = O.Stack(W.host_view(data["q"][:1]), W.host_view(data["k"][:1, :, :, :n]),
                 W.host_view(data["v"][:1, :, :, :n]), np.zeros((1, spec.Hq), dtype=np.uint8))
    o, S_out, _, fresh = O.layer(st, 0, k, S0.cpu().numpy(), all_retrieval=False, n=n)
    assert not fresh.any() and np.array_equal(S_out, S0.cpu().numpy())
    return o


def noalloc(lyc, data, S0, n, k, expect_status=0):
    spec = data["spec"]
    out = torch.full((spec.B, spec.Hq, spec.d), float("nan"), device="cuda")
    status = torch.full((1,), 0x5A5A, dtype=torch.int32, device="cuda")
    # layer 0 of the [1][B][Hkv][n][d] cache: strides (batch, head, token)
    kv = lyc.lyc_kv_cache(data["k"].data_ptr(), data["v"].data_ptr(), n, 0,
                          *data["k"].stride()[1:4])
    S = S0.contiguous()
    stream = torch.cuda.current_stream().cuda_stream
    rc = lyc.lyc_sparse_attention_noalloc(data["q"].data_ptr(), kv, spec.B, spec.Hq, spec.Hkv,
                                          spec.d, S.data_ptr(), k, out.data_ptr(),
                                          status.data_ptr(), stream)
    assert rc == lyc.LYC_OK, lyc.lyc_status_string(rc)
    torch.cuda.synchronize()
    assert int(status.item()) == expect_status
    return out.cpu().numpy()


def padded_sets(B, Hq, n, k):
    """k > n: every set holds all n rows, then -1 up to k."""
    S = torch.full((B, Hq, k), -1, dtype=torch.int32)
    S[:, :, :n] = torch.arange(n, dtype=torch.int32)
    return S.cuda()


CASES = [
    # (spec, k, pattern): calls in a row with different shapes and sets
    (W.StackSpec("na-llama", L=1, B=2, Hq=32, Hkv=8, d=128, n=5000, k=1024,
                 planted="heavy", n_planted=32, seed=21), 1024, "scattered"),
    (W.StackSpec("na-small", L=1, B=1, Hq=8, Hkv=2, d=64, n=700, k=200,
                 planted="none", seed=22), 200, "scattered"),
    # 256 sets of 32 tiles: segments cut over many CTAs, the combine launch
    (W.StackSpec("na-many", L=1, B=8, Hq=32, Hkv=8, d=128, n=9000, k=2048,
                 planted="heavy", n_planted=32, seed=23), 2048, "blocks"),
    # head_dim 64 with a GQA group of 8
    (W.StackSpec("na-gqa8", L=1, B=2, Hq=16, Hkv=2, d=64, n=3000, k=516,
                 planted="none", seed=24), 516, "scattered"),
    # k > n: the sets are all n rows, padded with -1
    (W.StackSpec("na-kgtn", L=1, B=1, Hq=4, Hkv=2, d=128, n=100, k=128,
                 planted="none", seed=25), 128, "padded"),
]


def test_noalloc_matches_existing_entry_point_and_oracle(lyc):
    atol, rtol = P.TOL["bf16"]
    for spec, k, pattern in CASES:
        data = W.make_stack(spec, "cuda")
        if pattern == "padded":
            S0 = padded_sets(spec.B, spec.Hq, spec.n, k)
        else:
            S0 = W.inherited_sets(spec.B, spec.Hq, spec.n, k, pattern, seed=spec.seed, device="cuda")
        want = reference(lyc, data, S0, spec.n, k)
        ora = oracle_sparse(data, S0, spec.n, k)
        for call in range(2):  # two calls in a row on the same inputs
            got = noalloc(lyc, data, S0, spec.n, k)
            assert np.isfinite(got).all()
            np.testing.assert_allclose(got, want, rtol=rtol, atol=atol,
                                       err_msg=f"{spec.name} call {call} vs lyc_decode_step")
            P.check_out(got, ora, "bf16", f"{spec.name} call {call} vs the oracle")


def test_noalloc_reports_an_index_past_n(lyc):
    """An index outside [0, n) is skipped and reported in the status word;
    the output stays finite and the next call is clean again."""
    spec = W.StackSpec("na-bad", L=1, B=1, Hq=4, Hkv=2, d=128, n=300, k=64, planted="none", seed=26)
    data = W.make_stack(spec, "cuda")
    S0 = W.inherited_sets(spec.B, spec.Hq, spec.n, 64, "scattered", seed=5, device="cuda")
    bad = S0.clone()
    bad[0, 2, 63] = spec.n + 7
    got = noalloc(lyc, data, bad, spec.n, 64, expect_status=1)
    assert np.isfinite(got).all()
    got = noalloc(lyc, data, S0, spec.n, 64)
    P.check_out(got, oracle_sparse(data, S0, spec.n, 64), "bf16", "after the bad call")


def test_noalloc_rejects_requests_past_its_scratch(lyc):
    spec = W.StackSpec("na-big", L=1, B=9, Hq=32, Hkv=8, d=64, n=256, k=64, planted="none")
    data = W.make_stack(spec, "cuda")
    S0 = W.inherited_sets(spec.B, spec.Hq, spec.n, 64, "scattered", seed=1, device="cuda")
    out = torch.empty((spec.B, spec.Hq, spec.d), device="cuda")
    kv = lyc.lyc_kv_cache(data["k"].data_ptr(), data["v"].data_ptr(), spec.n, 0,
                          *data["k"].stride()[1:4])
    assert spec.B * spec.Hq > lyc.LYC_NOALLOC_MAX_SETS
    rc = lyc.lyc_sparse_attention_noalloc(data["q"].data_ptr(), kv, spec.B, spec.Hq, spec.Hkv,
                                          spec.d, S0.data_ptr(), 64, out.data_ptr(), None,
                                          torch.cuda.current_stream().cuda_stream)
    assert rc == lyc.LYC_ERR_SCRATCH_LIMIT
    assert "scratch" in lyc.lyc_status_string(rc)
