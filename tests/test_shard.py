"""Head and batch sharding (hybrid_head_sparse_b200/shard.py) on CPU.

Two gloo ranks stand in for two GPUs.  Each rank takes its shard of the
step's inputs with `shard.take`, runs the fp64 oracle on that shard (the
stand-in for the library's step, which needs a GPU), and the ranks' results
are joined with `shard.gather`.  The joined outputs and sets must equal the
oracle's run on the whole problem exactly: every (batch element, KV group)
chain of the step is independent of the others, so a shard computes the same
numbers as the whole.
"""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _spec(kind):
    from hybrid_head_sparse_b200 import workloads as W
    # the tiny workload over three layers, one seeded retrieval head in each
    # later layer; batch sharding needs two batch elements
    spec = W.TINY.with_(B=2) if kind == "batch" else W.TINY
    return spec.with_(roles="random", retrieval_per_layer=1, L=3)


def _oracle_step(q, K, V, role, mode, k):
    import oracle as O
    from hybrid_head_sparse_b200 import workloads as W
    st = O.Stack(W.host_view(q), W.host_view(K.contiguous()), W.host_view(V.contiguous()),
                 np.ascontiguousarray(role),
                 O.SELECT_KVGROUP_MEAN if mode == "kvgroup_mean" else O.SELECT_PER_QHEAD)
    out, S, _ = O.decode_step(st, k)
    return out, S


def _rank_main(rank, world, port, kind, mode, q):
    import torch
    import torch.distributed as dist
    from hybrid_head_sparse_b200 import shard, workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        spec = _spec(kind)
        data = W.make_stack(spec, "cpu")
        sh = shard.shard_of(kind, rank, world, spec.B, spec.Hq, spec.Hkv)
        qs, Ks, Vs, rs = shard.take(sh, data["q"], data["k"], data["v"], data["role"])
        out, S = _oracle_step(qs, Ks, Vs, rs, mode, spec.k)
        out_full = shard.gather(sh, torch.from_numpy(out), shard.out_dim(sh))
        S_full = shard.gather(sh, torch.from_numpy(S), shard.sets_dim(sh))
        q.put((rank, out_full.numpy(), S_full.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kind", ["heads", "batch"])
@pytest.mark.parametrize("mode", ["per_qhead", "kvgroup_mean"])
def test_sharded_step_equals_whole_gloo_two_ranks(kind, mode):
    from hybrid_head_sparse_b200 import workloads as W
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, kind, mode, qu)) for r in range(2)]
    for p in procs:
        p.start()
    got = [qu.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    spec = _spec(kind)
    data = W.make_stack(spec, "cpu")
    assert data["role"][1:].sum() > 0
    out, S = _oracle_step(data["q"], data["k"], data["v"], data["role"], mode, spec.k)
    for rank, o, s in got:
        assert o.shape == out.shape and s.shape == S.shape
        assert np.array_equal(o, out), f"rank {rank}: outputs differ from the whole step"
        assert np.array_equal(s, S), f"rank {rank}: sets differ from the whole step"


def test_shard_ranges_partition_the_problem():
    from hybrid_head_sparse_b200 import shard
    for world in (1, 2, 4, 8):
        hs = [shard.shard_of("heads", r, world, 1, 32, 8) for r in range(world)]
        assert [(s.g0, s.g1) for s in hs] == [(r * 8 // world, (r + 1) * 8 // world) for r in range(world)]
        assert all(s.h0 == 4 * s.g0 and s.h1 == 4 * s.g1 and (s.b0, s.b1) == (0, 1) for s in hs)
        assert all(s.slots(True) == (s.g0, s.g1) and s.slots(False) == (s.h0, s.h1) for s in hs)
    for world in (1, 2, 4):
        bs = [shard.shard_of("batch", r, world, 4, 32, 8) for r in range(world)]
        assert [(s.b0, s.b1) for s in bs] == [(r * 4 // world, (r + 1) * 4 // world) for r in range(world)]
        assert all((s.g0, s.g1, s.h0, s.h1) == (0, 8, 0, 32) for s in bs)
    with pytest.raises(ValueError):
        shard.shard_of("heads", 0, 3, 1, 32, 8)   # 8 KV groups do not split 3 ways
    with pytest.raises(ValueError):
        shard.shard_of("batch", 0, 2, 1, 32, 8)   # one batch element
    with pytest.raises(ValueError):
        shard.shard_of("rows", 0, 2, 2, 32, 8)
    with pytest.raises(ValueError):
        shard.shard_of("heads", 2, 2, 1, 32, 8)


def test_take_views_and_gather_single_rank():
    import torch
    from hybrid_head_sparse_b200 import shard
    L, B, Hq, Hkv, n, d = 2, 2, 8, 2, 16, 4
    q = torch.arange(L * B * Hq * d, dtype=torch.float32).reshape(L, B, Hq, d)
    K = torch.randn(L, B, Hkv, n, d)
    role = np.zeros((L, Hq), dtype=np.uint8)
    sh = shard.shard_of("heads", 1, 2, B, Hq, Hkv)
    qs, Ks, Vs, rs = shard.take(sh, q, K, K, role)
    assert qs.is_contiguous() and torch.equal(qs, q[:, :, 4:8])
    assert Ks.data_ptr() == K[:, :, 1:2].data_ptr() and Ks.stride() == K.stride()  # a view
    assert rs.shape == (L, 4)
    one = shard.shard_of("heads", 0, 1, B, Hq, Hkv)
    assert shard.gather(one, q, 2) is q
