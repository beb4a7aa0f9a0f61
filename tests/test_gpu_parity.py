"""The CUDA library (through its C ABI) against the fp64 oracle, on a B200."""
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


# bf16 attention kernels: "cp_async" (mma.sync with cp.async gathers, the
# default), "tma" (mma.sync with TMA gathers), "tc" (tcgen05, head_dim 128)
GATHERS = ["cp_async", "tma", "tc"]


def run_step(lyc, spec: W.StackSpec, select_mode="per_qhead", data=None, s_in=None,
             no_graph=False, k=None, n=None, gather="cp_async"):
    """One library step on the spec's inputs; returns (data, out, S, trace) on the host.
    gather: "cp_async" (the default mma.sync kernel), "tma" (the mma.sync kernel
    with four-row TMA gathers where the layout allows) or "tc" (the tcgen05 kernel)."""
    data = data or W.make_stack(spec, "cuda")
    k = k or spec.k
    n = n or spec.n
    flags = {"cp_async": 0, "tma": lyc.LYC_CFG_TMA_GATHER, "tc": lyc.LYC_CFG_TCGEN05}[gather]
    ctx = lyc.Lyc(spec.L, spec.B, spec.Hq, spec.Hkv, spec.d, max(spec.rows, n), k,
                  dtype=spec.dtype, select_mode=select_mode, flags=flags)
    Hs = ctx.Hs
    out = torch.full((spec.L, spec.B, spec.Hq, spec.d), float("nan"), device="cuda")
    S = torch.full((spec.B, Hs, k), -7, dtype=torch.int32, device="cuda")
    if s_in is not None:
        S.copy_(s_in)
    trace = torch.full((spec.L, spec.B, Hs, k), -7, dtype=torch.int32, device="cuda")
    ctx.set_trace(trace)
    ctx.decode_step(data["q"], data["k"], data["v"], n, data["role"], k, out, S,
                    s_in=s_in is not None, no_graph=no_graph)
    assert ctx.sync_status() == 0, lyc.lyc_last_error(ctx.ctx)
    torch.cuda.synchronize()
    res = (out.cpu().numpy(), S.cpu().numpy(), trace.cpu().numpy())
    ctx.close()
    return (data,) + res


# ---------------------------------------------------------------- selection kernel


# Every launch form of the selection kernel that a step uses: clusters of 4
# (a layer with many sets), 8 (beside the next attention) and 16 (alone),
# each in the fixed-k instantiation and in the one that carries the size rules.
TOPK_FORMS = [(cl, v) for cl in (4, 8, 16) for v in ("fixed", "rules")]


@pytest.mark.parametrize("n,k", [(1, 1), (5, 3), (64, 64), (100, 7), (513, 64), (4096, 1000),
                                 (131072, 4096), (131071, 4097), (1000, 999), (777, 800)])
def test_topk_bitexact_integer_keys(lyc, n, k):
    """Integer-valued keys with many ties: every launch form of the GPU
    selection is bit-exact against the oracle's argsTopK."""
    rng = np.random.default_rng(n * 7 + k)
    x = rng.integers(-6, 7, size=n).astype(np.float32)
    x[rng.random(n) < 0.1] = -0.0
    ctx = lyc.Lyc(1, 1, 1, 1, 64, max(n, 1), k, dtype="fp32")
    keys = torch.from_numpy(x).cuda()
    exp = O.topk(x.astype(np.float64), k)
    S = torch.full((k,), -7, dtype=torch.int32, device="cuda")
    ctx.topk_f32(keys, n, k, S)
    assert ctx.sync_status() == 0
    assert np.array_equal(S.cpu().numpy(), exp), "default launch form"
    for cl, variant in TOPK_FORMS:
        S.fill_(-7)
        v = lyc.LYC_TOPK_FIXED if variant == "fixed" else lyc.LYC_TOPK_RULES
        ctx.topk_f32(keys, n, k, S, cluster=cl, variant=v)
        assert ctx.sync_status() == 0
        assert np.array_equal(S.cpu().numpy(), exp), f"cluster {cl}, {variant} instantiation"
    ctx.close()


@pytest.mark.parametrize("cl,variant", TOPK_FORMS)
def test_topk_forms_heavy_ties_and_distinct(lyc, cl, variant):
    """Distinct fp32 keys, all-equal keys (every candidate tied: the radix
    fallback) and -inf halves, per launch form, at the step's 128K size."""
    n = 131072
    ctx = lyc.Lyc(1, 1, 1, 1, 64, n, 5000, dtype="fp32")
    rng = np.random.default_rng(cl * 10 + (variant == "rules"))
    v = lyc.LYC_TOPK_FIXED if variant == "fixed" else lyc.LYC_TOPK_RULES
    for x in (rng.standard_normal(n).astype(np.float32),
              np.full(n, 0.5, dtype=np.float32),
              np.concatenate([np.full(n // 2, -np.inf), rng.standard_normal(n // 2)]).astype(np.float32),
              rng.integers(-2, 3, size=n).astype(np.float32)):
        keys = torch.from_numpy(x).cuda()
        for k in (1, 4096, 5000):
            S = torch.full((k,), -7, dtype=torch.int32, device="cuda")
            ctx.topk_f32(keys, n, k, S, cluster=cl, variant=v)
            assert ctx.sync_status() == 0
            assert np.array_equal(S.cpu().numpy(), O.topk(x.astype(np.float64), k)), (cl, variant, k)
    ctx.close()


def test_topk_distinct_and_all_equal(lyc):
    ctx = lyc.Lyc(1, 1, 1, 1, 64, 200000, 5000, dtype="fp32")
    rng = np.random.default_rng(3)
    for x in (rng.standard_normal(200000).astype(np.float32),
              np.full(200000, 0.5, dtype=np.float32),
              np.concatenate([np.full(100000, -np.inf), rng.standard_normal(100000)]).astype(np.float32)):
        for k in (1, 4096, 5000):
            keys = torch.from_numpy(x).cuda()
            S = torch.full((k,), -7, dtype=torch.int32, device="cuda")
            ctx.topk_f32(keys, x.size, k, S)
            assert ctx.sync_status() == 0
            assert np.array_equal(S.cpu().numpy(), O.topk(x.astype(np.float64), k))
    ctx.close()


# ---------------------------------------------------------------- whole steps


def test_tiny_stack_fp32(lyc):
    spec = W.TINY
    data, out, S, tr = run_step(lyc, spec)
    P.check_layers(data, out, tr, spec.k, spec.n, "fp32", range(spec.L))
    assert np.array_equal(S, tr[-1])
    # without teacher forcing: the oracle's own whole step agrees as well
    o_out, o_S, _ = O.decode_step(P.host_stack(data), spec.k, trace=True)
    P.check_out(out, o_out, "fp32", "whole step")


def test_tiny_stack_fp32_no_graph_matches_graph(lyc):
    spec = W.TINY
    data, out_g, S_g, tr_g = run_step(lyc, spec)
    _, out_n, S_n, tr_n = run_step(lyc, spec, data=data, no_graph=True)
    assert np.array_equal(out_g, out_n) and np.array_equal(S_g, S_n) and np.array_equal(tr_g, tr_n)


SMALL_BF16 = W.StackSpec("small-llama-like", L=4, B=2, Hq=32, Hkv=8, d=128, n=3001, k=256,
                         retrieval_per_layer=3, n_planted=64, seed=5)


@pytest.mark.parametrize("gather", GATHERS)
@pytest.mark.parametrize("mode", ["per_qhead", "kvgroup_mean"])
def test_small_bf16_stack(lyc, mode, gather):
    spec = SMALL_BF16
    om = O.SELECT_PER_QHEAD if mode == "per_qhead" else O.SELECT_KVGROUP_MEAN
    data, out, S, tr = run_step(lyc, spec, select_mode=mode, gather=gather)
    P.check_layers(data, out, tr, spec.k, spec.n, "bf16", range(spec.L), select_mode=om)
    assert np.array_equal(S, tr[-1])


@pytest.mark.parametrize("mode", ["per_qhead", "kvgroup_mean"])
def test_edge_shapes(lyc, mode):
    om = O.SELECT_PER_QHEAD if mode == "per_qhead" else O.SELECT_KVGROUP_MEAN
    cases = [
        W.StackSpec("n1", L=2, B=1, Hq=2, Hkv=1, d=64, n=1, k=1, dtype="fp32", roles="first-head",
                    planted="none"),
        W.StackSpec("k>n", L=3, B=2, Hq=4, Hkv=4, d=64, n=70, k=100, dtype="fp32",
                    retrieval_per_layer=1, planted="none"),
        W.StackSpec("k=n", L=2, B=1, Hq=8, Hkv=2, d=128, n=130, k=130, retrieval_per_layer=2,
                    planted="none"),
        W.StackSpec("mha-d64-bf16", L=3, B=1, Hq=6, Hkv=6, d=64, n=1000, k=65,
                    retrieval_per_layer=2, planted="none", seed=2),
        W.StackSpec("group8", L=2, B=1, Hq=16, Hkv=2, d=128, n=700, k=63, retrieval_per_layer=3,
                    planted="none", seed=4),
        W.StackSpec("fp32-d128", L=2, B=1, Hq=4, Hkv=2, d=128, n=333, k=40, dtype="fp32",
                    retrieval_per_layer=1, planted="none", seed=6),
        W.StackSpec("padded-rows", L=2, B=1, Hq=4, Hkv=2, d=64, n=200, k=32, dtype="fp32",
                    retrieval_per_layer=1, planted="none", seed=7, n_max=260),
    ]
    for spec in cases:
        data, out, S, tr = run_step(lyc, spec, select_mode=mode)
        P.check_layers(data, out, tr, spec.k, spec.n, spec.dtype, range(spec.L), select_mode=om)


def test_k_ge_n_sparse_equals_dense(lyc):
    spec = W.StackSpec("kgen", L=2, B=1, Hq=4, Hkv=2, d=64, n=90, k=90, dtype="fp32",
                       roles="first-head", planted="none", seed=3)
    data, out, S, tr = run_step(lyc, spec)
    dense = dict(data)
    dense["role"] = np.ones_like(data["role"])
    _, out_d, _, _ = run_step(lyc, spec, data=dense)
    # same rows, same order of tiles: sparse heads reproduce the dense result
    np.testing.assert_allclose(out, out_d, rtol=1e-6, atol=1e-6)
    assert np.array_equal(S[0, 1], np.arange(90))


@pytest.mark.parametrize("gather", GATHERS)
@pytest.mark.parametrize("pattern", ["blocks", "scattered"])
def test_set_input_single_layer(lyc, pattern, gather):
    """One layer with inherited sets given (the single-layer kernel sweep form)."""
    spec = W.StackSpec("one-layer", L=1, B=2, Hq=32, Hkv=8, d=128, n=16384, k=1024,
                       planted="heavy", n_planted=64, seed=8)
    data = W.make_stack(spec, "cuda")
    role = np.zeros((1, 32), dtype=np.uint8)
    role[0, [3, 17]] = 1
    data["role"] = role
    S0 = W.inherited_sets(spec.B, spec.Hq, spec.n, spec.k, pattern, seed=1, device="cuda")
    _, out, S, tr = run_step(lyc, spec, data=data, s_in=S0, gather=gather)
    P.check_layers(data, out, tr, spec.k, spec.n, "bf16", [0], S0=S0.cpu().numpy())


@pytest.mark.parametrize("mode", ["per_qhead", "kvgroup_mean"])
def test_no_retrieval_after_layer0_bf16(lyc, mode):
    """Layers with no retrieval head launch no selection: consecutive
    attention launches follow each other directly."""
    om = O.SELECT_PER_QHEAD if mode == "per_qhead" else O.SELECT_KVGROUP_MEAN
    spec = W.StackSpec("r0", L=5, B=1, Hq=16, Hkv=4, d=128, n=3000, k=300,
                       retrieval_per_layer=0, planted="heavy", n_planted=16, seed=14)
    data, out, S, tr = run_step(lyc, spec, select_mode=mode)
    P.check_layers(data, out, tr, spec.k, spec.n, "bf16", range(spec.L), select_mode=om)
    assert np.array_equal(S, tr[0])  # nothing refreshed after layer 0


@pytest.mark.parametrize("mode", ["per_qhead", "kvgroup_mean"])
def test_no_retrieval_after_layer0_launches_of_eight(lyc, mode):
    """With no selection after layer 0 an attention launch holds eight
    layers: layers 1-7 read layer 0's sets in the launch of layers 8-15
    (with its own), then layer 16 alone before the last layer's launch."""
    om = O.SELECT_PER_QHEAD if mode == "per_qhead" else O.SELECT_KVGROUP_MEAN
    spec = W.StackSpec("r0-long", L=18, B=1, Hq=32, Hkv=8, d=128, n=8192, k=1024,
                       retrieval_per_layer=0, planted="heavy", n_planted=32, seed=15)
    data, out, S, tr = run_step(lyc, spec, select_mode=mode)
    P.check_layers(data, out, tr, spec.k, spec.n, "bf16", range(spec.L), select_mode=om)
    assert np.array_equal(S, tr[0])


@pytest.mark.parametrize("gather", GATHERS)
def test_ragged_sets_bf16(lyc, gather):
    """k not a multiple of the 64-row tile nor of the four-row gather: the
    last tile of every gathered segment is partial."""
    spec = W.StackSpec("ragged", L=3, B=1, Hq=8, Hkv=2, d=128, n=2000, k=199,
                       retrieval_per_layer=2, planted="heavy", n_planted=16, seed=11)
    data, out, S, tr = run_step(lyc, spec, gather=gather)
    P.check_layers(data, out, tr, spec.k, spec.n, "bf16", range(spec.L))


def test_head_stride_not_whole_rows_falls_back(lyc):
    """A KV-head stride that is not a whole number of rows has no flattened
    row view: asked for TMA gathers, the library gathers with cp.async and the
    result is the same."""
    spec = W.StackSpec("odd-head-stride", L=2, B=1, Hq=8, Hkv=2, d=128, n=600, k=100,
                       retrieval_per_layer=2, planted="none", seed=12)
    data = W.make_stack(spec, "cuda")
    L, B, Hkv, n, d = 2, 1, 2, 600, 128
    s_token, s_head = d, n * d + 64          # 128 bytes between heads: not a whole row
    s_batch = Hkv * s_head
    s_layer = B * s_batch

    def restride(t):
        flat = torch.zeros(L * s_layer + 64, dtype=t.dtype, device="cuda")
        v = flat.as_strided((L, B, Hkv, n, d), (s_layer, s_batch, s_head, s_token, 1))
        v.copy_(t)
        return v
    odd = dict(data)
    odd["k"], odd["v"] = restride(data["k"]), restride(data["v"])
    _, out, S, tr = run_step(lyc, spec, data=odd, gather="tma")
    P.check_layers(data, out, tr, spec.k, spec.n, "bf16", range(spec.L))


@pytest.mark.parametrize("gather", GATHERS)
def test_bad_inherited_index_reported_bf16(lyc, gather):
    spec = W.StackSpec("bad16", L=1, B=1, Hq=2, Hkv=1, d=128, n=300, k=70, planted="none")
    data = W.make_stack(spec, "cuda")
    data["role"] = np.array([[1, 0]], dtype=np.uint8)
    S0 = torch.arange(70, dtype=torch.int32, device="cuda").repeat(1, 2, 1).contiguous()
    flags = {"cp_async": 0, "tma": lyc.LYC_CFG_TMA_GATHER, "tc": lyc.LYC_CFG_TCGEN05}[gather]
    ctx = lyc.Lyc(1, 1, 2, 1, 128, 300, 70, flags=flags)
    out = torch.zeros((1, 1, 2, 128), device="cuda")
    for bad in (300, -3):
        S = S0.clone()
        S[0, 1, 66] = bad
        ctx.decode_step(data["q"], data["k"], data["v"], 300, data["role"], 70, out, S, s_in=True)
        assert ctx.sync_status() == lyc.LYC_ERR_BAD_INDEX
    S = S0.clone()
    ctx.decode_step(data["q"], data["k"], data["v"], 300, data["role"], 70, out, S, s_in=True)
    assert ctx.sync_status() == 0
    ctx.close()


def test_bad_inherited_index_reported(lyc):
    """An out-of-range index handed in is skipped by the kernel's bounds check
    and reported through the status word."""
    spec = W.StackSpec("bad", L=1, B=1, Hq=2, Hkv=1, d=64, n=100, k=8, dtype="fp32",
                       planted="none")
    data = W.make_stack(spec, "cuda")
    data["role"] = np.array([[1, 0]], dtype=np.uint8)
    S0 = torch.arange(8, dtype=torch.int32, device="cuda").repeat(1, 2, 1).contiguous()
    S0[0, 1, 5] = 1000
    ctx = lyc.Lyc(1, 1, 2, 1, 64, 100, 8, dtype="fp32")
    out = torch.zeros((1, 1, 2, 64), device="cuda")
    S = S0.clone()
    ctx.decode_step(data["q"], data["k"], data["v"], 100, data["role"], 8, out, S, s_in=True)
    assert ctx.sync_status() == lyc.LYC_ERR_BAD_INDEX
    # the context stays usable
    S = S0.clone()
    S[0, 1, 5] = 5
    ctx.decode_step(data["q"], data["k"], data["v"], 100, data["role"], 8, out, S, s_in=True)
    assert ctx.sync_status() == 0
    ctx.close()


def test_host_buffer_entry_matches_device_entry(lyc):
    spec = W.TINY
    data, out, S, _ = run_step(lyc, spec)
    ctx = lyc.Lyc(spec.L, spec.B, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k, dtype="fp32")
    q_host = data["q"].cpu().pin_memory()
    out_h = torch.empty((spec.L, spec.B, spec.Hq, spec.d)).pin_memory()
    S_h = torch.empty((spec.B, ctx.Hs, spec.k), dtype=torch.int32).pin_memory()
    ctx.decode_step_host(q_host, data["k"], data["v"], spec.n, data["role"], spec.k, out_h, S_h)
    assert ctx.sync_status() == 0
    assert np.array_equal(out_h.numpy(), out) and np.array_equal(S_h.numpy(), S)
    ctx.close()


def test_repeat_is_deterministic(lyc):
    spec = SMALL_BF16.with_(L=3, B=1)
    data, out1, S1, tr1 = run_step(lyc, spec)
    _, out2, S2, tr2 = run_step(lyc, spec, data=data)
    assert np.array_equal(out1, out2) and np.array_equal(tr1, tr2)


def test_invalid_arguments_rejected(lyc):
    ctx = lyc.Lyc(1, 1, 2, 1, 64, 128, 8, dtype="fp32")
    K = torch.zeros((1, 1, 1, 128, 64), device="cuda")
    q = torch.zeros((1, 1, 2, 64), device="cuda")
    out = torch.zeros((1, 1, 2, 64), device="cuda")
    S = torch.zeros((1, 2, 8), dtype=torch.int32, device="cuda")
    role = np.ones((1, 2), dtype=np.uint8)
    with pytest.raises(lyc.LycError):
        ctx.decode_step(q, K, K, 129, role, 8, out, S)      # n > max_ctx
    with pytest.raises(lyc.LycError):
        ctx.decode_step(q, K, K, 128, role, 9, out, S)      # k > max_k
    with pytest.raises(lyc.LycError):
        ctx.decode_step(q, K, K, 0, role, 8, out, S)        # empty cache
    ctx.close()


def test_strided_rows(lyc):
    """Rows padded past d (token stride > d): the row-gather path serves the
    dense heads too."""
    spec = W.StackSpec("strided", L=2, B=1, Hq=4, Hkv=2, d=64, n=300, k=40, dtype="fp32",
                       retrieval_per_layer=1, planted="none", seed=9)
    data = W.make_stack(spec, "cuda")
    Kp = torch.full((2, 1, 2, 300, 68), 1e30, device="cuda")
    Vp = torch.full((2, 1, 2, 300, 68), -1e30, device="cuda")
    Kp[..., :64] = data["k"]
    Vp[..., :64] = data["v"]
    strided = dict(data)
    strided["k"] = Kp[..., :64]
    strided["v"] = Vp[..., :64]
    _, out, S, tr = run_step(lyc, spec, data=strided)
    P.check_layers(data, out, tr, spec.k, spec.n, "fp32", range(spec.L))


@pytest.mark.parametrize("gather", GATHERS)
def test_strided_rows_bf16(lyc, gather):
    """bf16 rows padded to 136 elements (272-byte token stride): the tensor
    maps and the row gathers follow the stride."""
    spec = W.StackSpec("strided16", L=3, B=2, Hq=8, Hkv=2, d=128, n=777, k=130,
                       retrieval_per_layer=2, planted="heavy", n_planted=8, seed=13)
    data = W.make_stack(spec, "cuda")
    pad = dict(data)
    for name, fill in (("k", 3.0), ("v", -3.0)):
        t = torch.full((3, 2, 2, 777, 136), fill, dtype=torch.bfloat16, device="cuda")
        t[..., :128] = data[name]
        pad[name] = t[..., :128]
    _, out, S, tr = run_step(lyc, spec, data=pad, gather=gather)
    P.check_layers(data, out, tr, spec.k, spec.n, "bf16", range(spec.L))


# ---------------------------------------------------------------- full-size workloads
# The whole step runs at the workload's size; the oracle checks sampled layers
# with teacher forcing (each checked layer inherits the GPU's own sets).


def _full_size(lyc, spec, layers, mode="per_qhead", gather="cp_async"):
    om = O.SELECT_PER_QHEAD if mode == "per_qhead" else O.SELECT_KVGROUP_MEAN
    data, out, S, tr = run_step(lyc, spec, select_mode=mode, gather=gather)
    assert np.isfinite(out).all()
    P.check_layers(data, out, tr, spec.k, spec.n, spec.dtype, layers, select_mode=om)
    assert np.array_equal(S, tr[-1])
    del data
    torch.cuda.empty_cache()


def bench_exact(lyc, spec, mode, layers, replays=4, batch_sel=None):
    """The whole step at the workload's full size, in the launch form the
    bench times: one context of the bench's shape, the step captured once and
    replayed `replays` times (every replay after the first runs on the other
    epoch parity of the flags and pool cursors), no trace.  Then the same
    replays with the set trace on.  The selection keys and hence the sets do
    not depend on the order in which CTAs take work, so both runs must end on
    the same sets; the trace then gives the sets each checked layer inherited
    (teacher forcing), and the oracle checks the sampled layers of the last
    replay of both runs.  batch_sel: the batch elements to check (all)."""
    om = O.SELECT_PER_QHEAD if mode == "per_qhead" else O.SELECT_KVGROUP_MEAN
    data = W.make_stack(spec, "cuda")
    ctx = lyc.Lyc(spec.L, spec.B, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k, dtype=spec.dtype,
                  select_mode=mode)
    out_u = torch.full((spec.L, spec.B, spec.Hq, spec.d), float("nan"), device="cuda")
    S_u = torch.full((spec.B, ctx.Hs, spec.k), -7, dtype=torch.int32, device="cuda")
    for _ in range(replays):
        ctx.decode_step(data["q"], data["k"], data["v"], spec.n, data["role"], spec.k, out_u, S_u)
    assert ctx.sync_status() == 0, lyc.lyc_last_error(ctx.ctx)
    out_t = torch.full_like(out_u, float("nan"))
    S_t = torch.full_like(S_u, -7)
    trace = torch.full((spec.L, spec.B, ctx.Hs, spec.k), -7, dtype=torch.int32, device="cuda")
    ctx.set_trace(trace)
    for _ in range(replays):
        ctx.decode_step(data["q"], data["k"], data["v"], spec.n, data["role"], spec.k, out_t, S_t)
    assert ctx.sync_status() == 0, lyc.lyc_last_error(ctx.ctx)
    torch.cuda.synchronize()
    ctx.close()
    out_u, out_t = out_u.cpu().numpy(), out_t.cpu().numpy()
    S_u, S_t, trace = S_u.cpu().numpy(), S_t.cpu().numpy(), trace.cpu().numpy()
    assert np.isfinite(out_u).all() and np.isfinite(out_t).all()
    assert np.array_equal(S_u, S_t), "the untraced and the traced step ended on different sets"
    assert np.array_equal(S_t, trace[-1])
    if batch_sel is not None:
        bs = list(batch_sel)
        data = {"q": data["q"][:, bs], "k": data["k"][:, bs], "v": data["v"][:, bs],
                "role": data["role"]}
        out_u, out_t, trace = out_u[:, bs], out_t[:, bs], trace[:, bs]
    P.check_layers(data, [out_u, out_t], trace, spec.k, spec.n, spec.dtype, layers, select_mode=om)
    del data
    torch.cuda.empty_cache()


def test_llama3_8b_32k_full_step(lyc):
    _full_size(lyc, W.LLAMA3_8B_32K, [0, 1, 2, 17, 31])


@pytest.mark.parametrize("mode", ["kvgroup_mean", "per_qhead"])
def test_llama3_8b_128k_bench_step(lyc, mode):
    """The bench's own workload and launch form: 32 layers at 128K, k = 4096."""
    bench_exact(lyc, W.LLAMA3_8B_128K, mode, [0, 1, 2, 15, 30, 31])


@pytest.mark.parametrize("mode", ["kvgroup_mean", "per_qhead"])
def test_llama3_8b_32k_bench_step(lyc, mode):
    # four layers per attention launch at 32K: layers 0-3 share a launch, 30 and 31 are alone
    bench_exact(lyc, W.LLAMA3_8B_32K, mode, [0, 1, 2, 3, 16, 18, 30, 31], replays=3)


@pytest.mark.parametrize("mode", ["kvgroup_mean", "per_qhead"])
def test_qwen3_8b_64k_batch4_full_step(lyc, mode):
    """The Qwen3-8B-shaped stack at its full 36 layers, batch 4."""
    bench_exact(lyc, W.QWEN3_8B_64K_B4, mode, [0, 1, 17, 35], replays=3)


@pytest.mark.parametrize("gather", ["cp_async", "tc"])
@pytest.mark.parametrize("mode", ["per_qhead", "kvgroup_mean"])
def test_llama3_8b_128k_first_layers(lyc, mode, gather):
    # the 128K stack's first 6 layers (same shapes per layer as the full 32)
    _full_size(lyc, W.LLAMA3_8B_128K.with_(L=6), [0, 1, 5], mode, gather)


@pytest.mark.parametrize("pattern", ["blocks", "scattered"])
def test_single_layer_sweep_corner(lyc, pattern):
    """The largest corner of the single-layer sweep: batch 8, n = 524288,
    k = 8192, inherited sets given, two retrieval heads.  The oracle checks
    two of the eight batch elements (elements never interact)."""
    spec = W.StackSpec("sweep-corner", L=1, B=8, Hq=32, Hkv=8, d=128, n=524288, k=8192,
                       planted="heavy", n_planted=256, seed=21)
    data = W.make_stack(spec, "cuda")
    role = np.zeros((1, 32), dtype=np.uint8)
    role[0, [5, 30]] = 1
    data["role"] = role
    S0 = W.inherited_sets(spec.B, spec.Hq, spec.n, spec.k, pattern, seed=3, device="cuda")
    _, out, S, tr = run_step(lyc, spec, data=data, s_in=S0)
    bs = [0, 7]
    sub = {"q": data["q"][:, bs], "k": data["k"][:, bs], "v": data["v"][:, bs], "role": role}
    P.check_layers(sub, out[:, bs], tr[:, bs], spec.k, spec.n, "bf16", [0],
                   S0=S0.cpu().numpy()[bs])
    assert np.isfinite(out).all()
    del data, sub
    torch.cuda.empty_cache()
