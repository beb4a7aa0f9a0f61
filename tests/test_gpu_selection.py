"""Selection rules other than a fixed k (ratio, block top-k, top-p, threshold)
through the whole step on a B200, against the fp64 oracle with the same rule
(teacher forcing per layer; set sizes and choices checked by
parity.check_set_rule, outputs with the tolerances of parity.py)."""
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


# Heavy planted keys (sinks plus 200 heavy hitters, ~94 % of the mass) over a
# ragged n: top-p and threshold sets of a few hundred rows, below the cap.
SPEC = W.StackSpec("rules-4L-8q2kv-d128-n3000-k512", L=4, B=2, Hq=8, Hkv=2, d=128, n=3000,
                   k=512, retrieval_per_layer=2, planted="heavy", n_planted=200, seed=5)

RULES = {
    "ratio-1/8": O.Selection(O.RULE_RATIO, ratio=(1, 8)),
    "ratio-1/2-capped": O.Selection(O.RULE_RATIO, ratio=(1, 2)),
    "block-64": O.Selection(O.RULE_BLOCK_TOPK, block=64),
    "block-16": O.Selection(O.RULE_BLOCK_TOPK, block=16),
    "topp-0.5": O.Selection(O.RULE_TOPP, p=0.5),
    "topp-0.9": O.Selection(O.RULE_TOPP, p=0.9),
    "topp-1.0-capped": O.Selection(O.RULE_TOPP, p=1.0),
    "threshold-1e-3": O.Selection(O.RULE_THRESHOLD, tau=1e-3),
    "threshold-above-max": O.Selection(O.RULE_THRESHOLD, tau=0.5),
}


def lib_rule(lyc, sel: O.Selection):
    code = {O.RULE_TOPK: lyc.LYC_RULE_TOPK, O.RULE_RATIO: lyc.LYC_RULE_RATIO,
            O.RULE_BLOCK_TOPK: lyc.LYC_RULE_BLOCK_TOPK, O.RULE_TOPP: lyc.LYC_RULE_TOPP,
            O.RULE_THRESHOLD: lyc.LYC_RULE_THRESHOLD}[sel.rule]
    return dict(rule=code, block=sel.block, ratio=sel.ratio, p=sel.p, tau=sel.tau)


def run_rule(lyc, spec, sel, select_mode="per_qhead", flags=0, data=None, s_in=None):
    data = data or W.make_stack(spec, "cuda")
    k = spec.k
    ctx = lyc.Lyc(spec.L, spec.B, spec.Hq, spec.Hkv, spec.d, spec.rows, k, dtype=spec.dtype,
                  select_mode=select_mode, flags=flags)
    ctx.set_selection(**lib_rule(lyc, sel))
    out = torch.full((spec.L, spec.B, spec.Hq, spec.d), float("nan"), device="cuda")
    S = torch.full((spec.B, ctx.Hs, k), -7, dtype=torch.int32, device="cuda")
    if s_in is not None:
        S.copy_(torch.from_numpy(s_in))
    trace = torch.full((spec.L, spec.B, ctx.Hs, k), -7, dtype=torch.int32, device="cuda")
    ctx.set_trace(trace)
    ctx.decode_step(data["q"], data["k"], data["v"], spec.n, data["role"], k, out, S,
                    s_in=s_in is not None, validate_s=s_in is not None)
    rc = ctx.sync_status()
    torch.cuda.synchronize()
    res = (rc, out.cpu().numpy(), S.cpu().numpy(), trace.cpu().numpy())
    ctx.close()
    return (data,) + res


def check_rule(data, spec, out, S, trace, sel, select_mode="per_qhead", layers=None):
    om = O.SELECT_PER_QHEAD if select_mode == "per_qhead" else O.SELECT_KVGROUP_MEAN
    assert np.isfinite(out).all()
    P.check_layers(data, out, trace, spec.k, spec.n, spec.dtype,
                   range(spec.L) if layers is None else layers, select_mode=om, sel=sel)
    assert np.array_equal(S, trace[-1])


@pytest.mark.parametrize("name", list(RULES))
def test_rule_bf16_per_head(lyc, name):
    sel = RULES[name]
    data, rc, out, S, tr = run_rule(lyc, SPEC, sel)
    assert rc == 0, lyc.status_string(rc)
    check_rule(data, SPEC, out, S, tr, sel)
    sizes = (tr >= 0).sum(-1)
    if name == "threshold-above-max":
        assert np.all(sizes == 1)
    if name in ("topp-1.0-capped", "ratio-1/2-capped"):
        assert np.all(sizes == SPEC.k)


@pytest.mark.parametrize("name", ["ratio-1/8", "block-64", "topp-0.9", "threshold-1e-3"])
def test_rule_bf16_kvgroup(lyc, name):
    sel = RULES[name]
    data, rc, out, S, tr = run_rule(lyc, SPEC, sel, select_mode="kvgroup_mean")
    assert rc == 0, lyc.status_string(rc)
    check_rule(data, SPEC, out, S, tr, sel, select_mode="kvgroup_mean")


@pytest.mark.parametrize("name", ["block-64", "topp-0.9", "threshold-1e-3"])
def test_rule_fp32(lyc, name):
    spec = SPEC.with_(dtype="fp32", d=64, n=1500, k=256, name="rules-fp32")
    sel = RULES[name]
    data, rc, out, S, tr = run_rule(lyc, spec, sel)
    assert rc == 0, lyc.status_string(rc)
    check_rule(data, spec, out, S, tr, sel)


@pytest.mark.parametrize("name", ["block-64", "topp-0.9"])
def test_rule_tcgen05(lyc, name):
    sel = RULES[name]
    data, rc, out, S, tr = run_rule(lyc, SPEC, sel, flags=lyc.LYC_CFG_TCGEN05)
    assert rc == 0, lyc.status_string(rc)
    check_rule(data, SPEC, out, S, tr, sel)


def test_rule_topp_uniform_keys_exact(lyc):
    """No planted keys and K = 0: every key is 0, A = 1/n exactly, and the
    running mass reaches p after exactly ceil(p n) rows, the lowest indices
    (ties to the lower index)."""
    spec = SPEC.with_(planted="none", n=2048, L=2, name="rules-uniform")
    data = W.make_stack(spec, "cuda")
    data["k"].zero_()
    for p, m in ((0.25, 512), (0.1, 205), (0.0625, 128)):
        _, rc, out, S, tr = run_rule(lyc, spec, O.Selection(O.RULE_TOPP, p=p), data=data)
        assert rc == 0
        exp = np.concatenate([np.arange(m), np.full(spec.k - m, -1)]).astype(np.int32)
        assert np.all(tr[0] == exp), f"p={p}"


def test_rule_variable_sets_as_input(lyc):
    """Shorter sets handed in by the caller (S_IN with validation) are
    accepted under a variable-size rule, and the sparse heads read only their
    valid rows."""
    sel = RULES["topp-0.9"]
    spec = SPEC
    rng = np.random.default_rng(3)
    s0 = np.full((spec.B, spec.Hq, spec.k), -1, dtype=np.int32)
    for b in range(spec.B):
        for h in range(spec.Hq):
            m = int(rng.integers(1, spec.k + 1))
            s0[b, h, :m] = np.sort(rng.choice(spec.n, size=m, replace=False))
    data = W.make_stack(spec, "cuda")
    data["role"][0] = data["role"][1]  # layer 0 obeys its role row: its sparse heads read s0
    assert 0 < data["role"][0].sum() < spec.Hq
    data, rc, out, S, tr = run_rule(lyc, spec, sel, data=data, s_in=s0)
    assert rc == 0, lyc.status_string(rc)
    om = O.SELECT_PER_QHEAD
    P.check_layers(data, out, tr, spec.k, spec.n, spec.dtype, range(spec.L), select_mode=om,
                   S0=s0, sel=sel)


@pytest.mark.parametrize("select_mode", ["per_qhead", "kvgroup_mean"])
def test_rule_short_sets_many_units(lyc, select_mode):
    """Caller sets of every length class against a capacity of four pool
    units (k = 2048): one row, a part of a tile, whole tiles, a unit and a
    row past it, up to the capacity.  Units and tiles past a set's valid
    rows are dropped on the device; the outputs must still match the oracle,
    and the sets the later layers select under the rule too."""
    sel = RULES["topp-0.9"]
    spec = SPEC.with_(n=5000, k=2048, L=3, name="rules-short-sets-k2048")
    Hs = spec.Hq if select_mode == "per_qhead" else spec.Hkv
    lengths = [1, 63, 64, 65, 511, 512, 513, 1000, 1536, 1537, 2047, 2048, 700, 129, 1025, 3]
    rng = np.random.default_rng(11)
    s0 = np.full((spec.B, Hs, spec.k), -1, dtype=np.int32)
    i = 0
    for b in range(spec.B):
        for h in range(Hs):
            m = lengths[i % len(lengths)]
            i += 1
            s0[b, h, :m] = np.sort(rng.choice(spec.n, size=m, replace=False))
    data = W.make_stack(spec, "cuda")
    data["role"][0] = data["role"][1]  # layer 0 obeys its role row: its sparse heads read s0
    assert 0 < data["role"][0].sum() < spec.Hq
    data, rc, out, S, tr = run_rule(lyc, spec, sel, select_mode=select_mode, data=data, s_in=s0)
    assert rc == 0, lyc.status_string(rc)
    om = O.SELECT_PER_QHEAD if select_mode == "per_qhead" else O.SELECT_KVGROUP_MEAN
    P.check_layers(data, out, tr, spec.k, spec.n, spec.dtype, range(spec.L), select_mode=om,
                   S0=s0, sel=sel)


def test_rule_bad_input_set_rejected(lyc):
    """A -1 inside a caller's set (valid entries after it) is still an error."""
    sel = RULES["topp-0.9"]
    s0 = np.tile(np.arange(SPEC.k, dtype=np.int32), (SPEC.B, SPEC.Hq, 1))
    s0[1, 2, 10] = -1
    _, rc, *_ = run_rule(lyc, SPEC, sel, s_in=s0)
    assert rc == lyc.LYC_ERR_BAD_INDEX


def test_rule_ratio_serving_varlen(lyc):
    """The ratio budget per batch element (its own n) in the serving form."""
    from tests.test_gpu_serving import serving_case, run_serving, check_case  # noqa: F401
    case = serving_case(3, 3, 8, 2, 128, [3000, 1500, 777], "bf16", seed=81, page_rows=64)
    sel = O.Selection(O.RULE_RATIO, ratio=(1, 4))
    L, B, Hq, d = case["q"].shape
    k = 512
    ctx = lyc.Lyc(L, B, Hq, 2, d, max(case["n"]), k)
    ctx.set_selection(**lib_rule(lyc, sel))
    out = torch.full((L, B, Hq, d), float("nan"), device="cuda")
    S = torch.full((B, ctx.Hs, k), -7, dtype=torch.int32, device="cuda")
    trace = torch.full((L, B, ctx.Hs, k), -7, dtype=torch.int32, device="cuda")
    ctx.set_trace(trace)
    ctx.decode_step_batch(case["q"], case["K"], case["V"], case["n"], case["role"], k, out, S,
                          k_new=case["k_new"], v_new=case["v_new"],
                          block_table=case["block_table"], page_rows=case["page_rows"])
    assert ctx.sync_status() == 0
    torch.cuda.synchronize()
    out, tr = out.cpu().numpy(), trace.cpu().numpy()
    ctx.close()
    P.check_layers_varlen(W.host_view(case["q"]), W.host_view(case["Kl"]), W.host_view(case["Vl"]),
                          case["role"], case["n"], out, tr, k, "bf16", range(L), sel=sel)
    for b, nb in enumerate(case["n"]):
        assert np.all((tr[:, b] >= 0).sum(-1) == min(k, -(-nb // 4)))


@pytest.mark.parametrize("name", ["block-64", "topp-0.9", "threshold-1e-3", "ratio-1/2-capped"])
def test_rule_full_size_llama3_8b_128k(lyc, name):
    """The 128K Llama3-8B stack under each rule: layers 0, 1 and the last
    checked against the oracle (teacher forcing)."""
    spec = W.LLAMA3_8B_128K
    sel = RULES[name]
    data, rc, out, S, tr = run_rule(lyc, spec, sel)
    assert rc == 0, lyc.status_string(rc)
    P.check_layers(data, out, tr, spec.k, spec.n, spec.dtype, [0, 1, spec.L - 1], sel=sel)
