"""Sharded step (hybrid_head_sparse_b200/shard.py) through the library on one
B200.  A rank's part of a head- or batch-sharded step is an ordinary step on
strided views of the caller's cache, so the ranks of a world of 2 (or 4) can
run one after the other on one GPU.  Their outputs and set traces, joined in
rank order, are checked against the fp64 oracle's whole step on every layer
(teacher forcing with the joined trace), and against the library's whole
step: outputs within the bf16 tolerances, sets equal (the selection keys of
a KV group do not depend on how the work is cut).  The all-gather itself runs
on CPU ranks in tests/test_shard.py.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from hybrid_head_sparse_b200 import shard, workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lyc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from hybrid_head_sparse_b200 import lyc as lycmod
    lycmod.load()
    return lycmod


@pytest.mark.parametrize("kind,world,mode", [
    ("heads", 2, "kvgroup_mean"), ("heads", 4, "per_qhead"), ("batch", 2, "kvgroup_mean"),
])
def test_shards_join_to_the_whole_step(lyc, kind, world, mode):
    B = 2 if kind == "batch" else 1
    spec = W.LLAMA3_8B_32K.with_(L=4, B=B, n=8192, k=1024, name=f"shard-{kind}")
    data = W.make_stack(spec, "cuda")
    whole = lyc.Lyc(spec.L, B, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k, select_mode=mode)
    out = torch.empty((spec.L, B, spec.Hq, spec.d), device="cuda")
    S = torch.empty((B, whole.Hs, spec.k), dtype=torch.int32, device="cuda")
    whole.decode_step(data["q"], data["k"], data["v"], spec.n, data["role"], spec.k, out, S)
    assert whole.sync_status() == 0
    outs, sets, traces = [], [], []
    for r in range(world):
        sh = shard.shard_of(kind, r, world, B, spec.Hq, spec.Hkv)
        qs, Ks, Vs, rs = shard.take(sh, data["q"], data["k"], data["v"], data["role"])
        st = shard.ShardedStep(sh, spec.L, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k,
                               select_mode=mode)
        tr = torch.full((spec.L,) + tuple(st.S.shape), -7, dtype=torch.int32, device="cuda")
        st.ctx.set_trace(tr)
        st.ctx.decode_step(qs, Ks, Vs, spec.n, rs, spec.k, st.out, st.S)
        assert st.ctx.sync_status() == 0
        torch.cuda.synchronize()
        outs.append(st.out.clone())
        sets.append(st.S.clone())
        traces.append(tr)
        st.close()
    sh0 = shard.shard_of(kind, 0, world, B, spec.Hq, spec.Hkv)
    joined = torch.cat(outs, dim=shard.out_dim(sh0)).cpu().numpy()
    joined_S = torch.cat(sets, dim=shard.sets_dim(sh0)).cpu().numpy()
    joined_tr = torch.cat(traces, dim=shard.sets_dim(sh0) + 1).cpu().numpy()
    whole.close()
    # the joined shards against the oracle, every layer, teacher-forced with
    # the joined trace (the sets each layer of each shard inherited)
    om = O.SELECT_PER_QHEAD if mode == "per_qhead" else O.SELECT_KVGROUP_MEAN
    assert np.array_equal(joined_S, joined_tr[-1])
    P.check_layers(data, joined, joined_tr, spec.k, spec.n, "bf16", range(spec.L), select_mode=om)
    # and against the library's whole step
    P.check_out(joined, out.cpu().numpy().astype(np.float64), "bf16", f"{kind} x{world} {mode}")
    assert np.array_equal(joined_S, S.cpu().numpy())


def test_sharded_step_world_one_is_the_step(lyc):
    """World 1: the sharded step is the step itself (no gather)."""
    spec = W.LLAMA3_8B_32K.with_(L=3, n=4096, k=512, name="shard-one")
    data = W.make_stack(spec, "cuda")
    sh = shard.shard_of("heads", 0, 1, 1, spec.Hq, spec.Hkv)
    st = shard.ShardedStep(sh, spec.L, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k)
    qs, Ks, Vs, rs = shard.take(sh, data["q"], data["k"], data["v"], data["role"])
    out, S = st.step(qs, Ks, Vs, spec.n, rs)
    assert st.ctx.sync_status() == 0
    whole = lyc.Lyc(spec.L, 1, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k, select_mode="kvgroup_mean")
    out2 = torch.empty_like(out)
    S2 = torch.empty_like(S)
    whole.decode_step(data["q"], data["k"], data["v"], spec.n, data["role"], spec.k, out2, S2)
    torch.cuda.synchronize()
    # outputs within the bf16 tolerances (which CTA takes which pool unit is
    # decided at run time, and with it the fp32 summation order), sets exact
    # (a tile's selection keys do not depend on who computes them)
    P.check_out(out.cpu().numpy(), out2.cpu().numpy().astype(np.float64), "bf16", "world 1")
    assert torch.equal(S, S2)
    st.close()
    whole.close()
