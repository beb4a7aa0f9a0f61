"""The serving form of the step (lyc_decode_step_batch): a batch whose
elements have cache lengths of their own, a contiguous or paged cache, and the
current token's K/V appended by the step.  Every element is checked against
the fp64 oracle as a one-element step over its own rows of the logical cache
(after the append), with the tolerances of tests/parity.py."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from tests import parity as P
from hybrid_head_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lyc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from hybrid_head_sparse_b200 import lyc as lycmod
    lycmod.load()
    return lycmod

GARBAGE = 37.0  # cache rows past n[b], and the rows the step must append


def _role(L, Hq, per_layer, seed):
    rng = np.random.default_rng(seed)
    role = np.zeros((L, Hq), dtype=np.uint8)
    for l in range(L):
        role[l, rng.permutation(Hq)[:per_layer]] = 1
    return role


def serving_case(L, B, Hq, Hkv, d, n_list, dtype, seed, page_rows=0, extra_pages=3,
                 retrieval=2):
    """Logical cache (what attention must see after the append), the physical
    cache handed to the library (append rows and rows past n[b] garbage) and,
    when paged, the page pool and block table (pages shuffled, some unused)."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    nmax = max(n_list)
    q = torch.randn((L, B, Hq, d), generator=g, device=dev).to(dt)
    Kl = torch.randn((L, B, Hkv, nmax, d), generator=g, device=dev).to(dt)
    Vl = torch.randn((L, B, Hkv, nmax, d), generator=g, device=dev).to(dt)
    # a few keys aligned with their group's mean query, so that selection has
    # clear winners (the recipe's planted positions)
    G = Hq // Hkv
    for b, nb in enumerate(n_list):
        for gg in range(Hkv):
            qbar = q[:, b, gg * G:(gg + 1) * G].float().mean(1)  # [L][d]
            pos = torch.randperm(nb, generator=g, device=dev)[: min(8, nb)]
            Kl[:, b, gg, pos] = (2.0 * qbar[:, None, :]).to(dt)
    for b, nb in enumerate(n_list):
        Kl[:, b, :, nb:] = GARBAGE
        Vl[:, b, :, nb:] = GARBAGE
    k_new = torch.stack([Kl[:, b, :, nb - 1] for b, nb in enumerate(n_list)], dim=1).contiguous()
    v_new = torch.stack([Vl[:, b, :, nb - 1] for b, nb in enumerate(n_list)], dim=1).contiguous()
    role = _role(L, Hq, retrieval, seed + 1)
    case = dict(q=q, Kl=Kl, Vl=Vl, k_new=k_new, v_new=v_new, role=role, n=list(n_list),
                page_rows=page_rows)
    if page_rows == 0:
        Kc, Vc = Kl.clone(), Vl.clone()
        for b, nb in enumerate(n_list):
            Kc[:, b, :, nb - 1] = GARBAGE
            Vc[:, b, :, nb - 1] = GARBAGE
        case.update(K=Kc, V=Vc, block_table=None)
        return case
    rng = np.random.default_rng(seed + 2)
    blocks = [(nb + page_rows - 1) // page_rows for nb in n_list]
    npages = sum(blocks) + extra_pages
    perm = rng.permutation(npages)
    max_blocks = max(blocks) + 1
    bt = np.zeros((B, max_blocks), dtype=np.int32)
    Kp = torch.full((L, npages, page_rows, Hkv, d), GARBAGE, device=dev, dtype=dt)
    Vp = torch.full((L, npages, page_rows, Hkv, d), GARBAGE, device=dev, dtype=dt)
    j = 0
    for b, nb in enumerate(n_list):
        for blk in range(blocks[b]):
            p = int(perm[j])
            j += 1
            bt[b, blk] = p
            r0, r1 = blk * page_rows, min(nb, (blk + 1) * page_rows)
            Kp[:, p, : r1 - r0] = Kl[:, b, :, r0:r1].permute(0, 2, 1, 3)
            Vp[:, p, : r1 - r0] = Vl[:, b, :, r0:r1].permute(0, 2, 1, 3)
        last = nb - 1
        p = int(bt[b, last // page_rows])
        Kp[:, p, last % page_rows] = GARBAGE
        Vp[:, p, last % page_rows] = GARBAGE
    case.update(K=Kp, V=Vp, block_table=torch.from_numpy(bt).to(dev))
    return case


def run_serving(lyc, case, k, dtype, select_mode="per_qhead", append=True, flags=0, S0=None):
    L, B, Hq, d = case["q"].shape
    Hkv = case["Kl"].shape[2]
    ctx = lyc.Lyc(L, B, Hq, Hkv, d, max(case["n"]), k, dtype=dtype, select_mode=select_mode,
                  flags=flags)
    out = torch.full((L, B, Hq, d), float("nan"), device="cuda")
    S = torch.full((B, ctx.Hs, k), -7, dtype=torch.int32, device="cuda")
    if S0 is not None:
        S.copy_(torch.from_numpy(S0))
    trace = torch.full((L, B, ctx.Hs, k), -7, dtype=torch.int32, device="cuda")
    ctx.set_trace(trace)
    ctx.decode_step_batch(case["q"], case["K"], case["V"], case["n"], case["role"], k, out, S,
                          s_in=S0 is not None, validate_s=S0 is not None,
                          k_new=case["k_new"] if append else None,
                          v_new=case["v_new"] if append else None,
                          block_table=case["block_table"], page_rows=case["page_rows"])
    rc = ctx.sync_status()
    torch.cuda.synchronize()
    res = (rc, out.cpu().numpy(), S.cpu().numpy(), trace.cpu().numpy())
    ctx.close()
    return res


def check_case(case, out, S, trace, k, dtype, select_mode="per_qhead", layers=None):
    import oracle as O
    L = out.shape[0]
    om = O.SELECT_PER_QHEAD if select_mode == "per_qhead" else O.SELECT_KVGROUP_MEAN
    assert np.isfinite(out).all()
    P.check_layers_varlen(W.host_view(case["q"]), W.host_view(case["Kl"]), W.host_view(case["Vl"]),
                          case["role"], case["n"], out, trace, k, dtype,
                          range(L) if layers is None else layers, select_mode=om)
    assert np.array_equal(S, trace[-1])


def appended_rows_ok(case):
    """After the step the cache holds the current token's rows at n[b]-1."""
    for b, nb in enumerate(case["n"]):
        if case["block_table"] is None:
            got_k = case["K"][:, b, :, nb - 1]
            got_v = case["V"][:, b, :, nb - 1]
        else:
            pr = case["page_rows"]
            p = int(case["block_table"][b, (nb - 1) // pr])
            got_k = case["K"][:, p, (nb - 1) % pr]
            got_v = case["V"][:, p, (nb - 1) % pr]
        if not (torch.equal(got_k, case["k_new"][:, b]) and torch.equal(got_v, case["v_new"][:, b])):
            return False
    return True


def test_serving_fp32_varlen_append_contiguous(lyc):
    case = serving_case(2, 3, 4, 2, 64, [512, 200, 37], "fp32", seed=11)
    rc, out, S, tr = run_serving(lyc, case, 64, "fp32")
    assert rc == 0
    check_case(case, out, S, tr, 64, "fp32")
    assert appended_rows_ok(case)


@pytest.mark.parametrize("page_rows", [64, 128])
def test_serving_bf16_varlen_append_paged(lyc, page_rows):
    case = serving_case(3, 3, 8, 2, 128, [3000, 1500, 777], "bf16", seed=21, page_rows=page_rows)
    rc, out, S, tr = run_serving(lyc, case, 256, "bf16")
    assert rc == 0
    check_case(case, out, S, tr, 256, "bf16")
    assert appended_rows_ok(case)


def test_serving_bf16_varlen_paged_kvgroup(lyc):
    case = serving_case(3, 2, 8, 2, 128, [2100, 900], "bf16", seed=31, page_rows=64)
    rc, out, S, tr = run_serving(lyc, case, 128, "bf16", select_mode="kvgroup_mean")
    assert rc == 0
    check_case(case, out, S, tr, 128, "bf16", select_mode="kvgroup_mean")


def test_serving_bf16_varlen_contiguous_tcgen05(lyc):
    case = serving_case(3, 3, 8, 2, 128, [2500, 1300, 640], "bf16", seed=41)
    rc, out, S, tr = run_serving(lyc, case, 256, "bf16", flags=lyc.LYC_CFG_TCGEN05)
    assert rc == 0
    check_case(case, out, S, tr, 256, "bf16")


def test_serving_edge_n1_and_k_above_n(lyc):
    """One element of a single row (the current token only), one shorter than
    k (sets of n[b] rows padded with -1), one longer."""
    case = serving_case(2, 3, 8, 2, 128, [1, 50, 300], "bf16", seed=51, page_rows=64)
    rc, out, S, tr = run_serving(lyc, case, 64, "bf16")
    assert rc == 0
    check_case(case, out, S, tr, 64, "bf16")
    assert np.all(S[0, :, 1:] == -1) and np.all(S[0, :, 0] == 0)
    assert np.all(S[1, :, 50:] == -1)


def test_serving_paged_equal_lengths_match_contiguous(lyc):
    """Equal lengths, no append: the paged cache gives the sets of the
    contiguous step on the same rows exactly, and its outputs up to the order
    in which a CTA's warps merge a pool unit (which CTA takes a unit, and so at
    which warp it starts, is decided at run time)."""
    n = 2048
    case = serving_case(3, 2, 8, 2, 128, [n, n], "bf16", seed=61, page_rows=128)
    # the paged cache must hold the appended row already (no append here)
    for b in range(2):
        p = int(case["block_table"][b, (n - 1) // 128])
        case["K"][:, p, (n - 1) % 128] = case["k_new"][:, b]
        case["V"][:, p, (n - 1) % 128] = case["v_new"][:, b]
    rc, out_p, S_p, tr_p = run_serving(lyc, case, 256, "bf16", append=False)
    assert rc == 0
    L, B, Hq, d = case["q"].shape
    ctx = lyc.Lyc(L, B, Hq, 2, d, n, 256)
    out = torch.full((L, B, Hq, d), float("nan"), device="cuda")
    S = torch.full((B, ctx.Hs, 256), -7, dtype=torch.int32, device="cuda")
    ctx.decode_step(case["q"], case["Kl"], case["Vl"], n, case["role"], 256, out, S)
    assert ctx.sync_status() == 0
    ctx.close()
    assert np.allclose(out.cpu().numpy(), out_p, rtol=1e-5, atol=1e-6)
    assert np.array_equal(S.cpu().numpy(), S_p)


def test_serving_bad_index_is_per_element(lyc):
    """An inherited index that is valid for one element (n = 100) but not for
    another (n = 40) is reported for the second only."""
    case = serving_case(2, 2, 8, 2, 128, [100, 40], "bf16", seed=71)
    k = 32
    S0 = np.tile(np.arange(k, dtype=np.int32), (2, 8, 1))
    S0[0, 3, -1] = 45  # fine: 45 < 100
    S0[0, 3] = np.sort(S0[0, 3])
    rc, out, S, tr = run_serving(lyc, case, k, "bf16", S0=S0)
    assert rc == 0
    S0[1, 3, -1] = 45  # not below n[1] = 40
    S0[1, 3] = np.sort(S0[1, 3])
    rc, out, S, tr = run_serving(lyc, case, k, "bf16", S0=S0)
    assert rc == lyc.LYC_ERR_BAD_INDEX
