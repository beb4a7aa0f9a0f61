"""lyc_sparse_attention_noalloc (the allocation-free entry point) against the
existing entry point, lyc_decode_step, on the same inputs.

A one-layer step whose every head is sparse and whose sets are handed in
(LYC_STEP_S_IN) computes the same thing, section 3.4 Eq. 3 of the
LycheeDecode summary page, for every head.  Two calls in a row, with
different inputs and shapes, check that the shared scratch array's leftover
contents (counters, partial states, work list) do not leak into the next
call.  The file name makes pytest collect it last; it also passes alone.
"""
import numpy as np
import pytest
import torch

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


def noalloc(lyc, data, S0, n, k):
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
    assert int(status.item()) == 0
    return out.cpu().numpy()


CASES = [
    # (spec, k, pattern): two calls in a row with different shapes and sets
    (W.StackSpec("na-llama", L=1, B=2, Hq=32, Hkv=8, d=128, n=5000, k=1024,
                 planted="heavy", n_planted=32, seed=21), 1024, "scattered"),
    (W.StackSpec("na-small", L=1, B=1, Hq=8, Hkv=2, d=64, n=700, k=200,
                 planted="none", seed=22), 200, "scattered"),
]


def test_noalloc_matches_existing_entry_point_two_calls(lyc):
    atol, rtol = P.TOL["bf16"]
    for spec, k, pattern in CASES:
        data = W.make_stack(spec, "cuda")
        S0 = W.inherited_sets(spec.B, spec.Hq, spec.n, k, pattern, seed=spec.seed, device="cuda")
        want = reference(lyc, data, S0, spec.n, k)
        got = noalloc(lyc, data, S0, spec.n, k)
        assert np.isfinite(got).all()
        np.testing.assert_allclose(got, want, rtol=rtol, atol=atol)


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
