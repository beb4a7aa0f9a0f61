"""Head and batch sharding of the decode step over several GPUs.

Why it needs no exchange inside the stack (page "LycheeDecode: Accelerating
Long-Context LLM Inference via Hybrid-Head Sparse Decoding", paper-graph-ui
summary, section 3.4, Eq. 1-3, and the GQA handling of the hyperparameter
summary): a head's token set is chosen from its own scores (or, with the
queries of a KV group pooled, from its group's) and is passed on only to
later layers of the same head (or group).  Roles are per head and frozen.  So
every (batch element, KV group) chain of the L-layer step is independent of
every other one.  A rank can run the whole step on a contiguous range of KV
groups with their query heads ("heads"), or on a contiguous range of batch
elements ("batch"), on its own GPU.  The only collective is one all-gather
of the outputs (and of the outgoing sets) per step.

This module holds the plumbing around the library's step: which part of the
problem a rank owns, the views of the caller's tensors it passes to
`lyc_decode_step`, and the gather that puts the ranks' results back in the
full layouts.  Every step of the attention itself runs in the library's
kernels.  Splits are even (an all-gather takes equal parts): Hkv or B must be
a multiple of the world size.
"""
from __future__ import annotations

from dataclasses import dataclass

KINDS = ("heads", "batch")


@dataclass(frozen=True)
class Shard:
    """The part of one step that rank `rank` of `world` owns: KV groups
    [g0, g1) with query heads [h0, h1), batch elements [b0, b1)."""
    kind: str
    rank: int
    world: int
    g0: int
    g1: int
    h0: int
    h1: int
    b0: int
    b1: int

    @property
    def Hq(self) -> int:
        return self.h1 - self.h0

    @property
    def Hkv(self) -> int:
        return self.g1 - self.g0

    @property
    def B(self) -> int:
        return self.b1 - self.b0

    def slots(self, kvgroup: bool) -> tuple[int, int]:
        """Set slots [s0, s1) of this shard: one per query head (per-head
        selection) or one per KV group (KV-group selection)."""
        return (self.g0, self.g1) if kvgroup else (self.h0, self.h1)


def shard_of(kind: str, rank: int, world: int, B: int, Hq: int, Hkv: int) -> Shard:
    """Rank `rank`'s shard.  heads: Hkv / world consecutive KV groups and
    their G = Hq / Hkv query heads each (GQA groups are contiguous: query head
    h reads KV head h // G).  batch: B / world consecutive batch elements."""
    if kind not in KINDS:
        raise ValueError(f"shard kind {kind!r}: expected one of {KINDS}")
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if Hq % Hkv:
        raise ValueError(f"Hq={Hq} is not a multiple of Hkv={Hkv}")
    G = Hq // Hkv
    if kind == "heads":
        if Hkv % world:
            raise ValueError(f"head sharding needs Hkv={Hkv} to be a multiple of the world size {world}")
        per = Hkv // world
        g0, g1 = rank * per, (rank + 1) * per
        return Shard(kind, rank, world, g0, g1, g0 * G, g1 * G, 0, B)
    if B % world:
        raise ValueError(f"batch sharding needs B={B} to be a multiple of the world size {world}")
    per = B // world
    return Shard(kind, rank, world, 0, Hkv, 0, Hq, rank * per, (rank + 1) * per)


def take(sh: Shard, q, K, V, role):
    """This shard's inputs from the full ones: q [L][B][Hq][d] (a contiguous
    copy: the library reads q densely), K/V [L][B][Hkv][rows][d] (views: the
    library takes the cache by strides), role [L][Hq] (numpy, a copy).  Works
    on torch tensors on any device."""
    qs = q[:, sh.b0:sh.b1, sh.h0:sh.h1].contiguous()
    Ks = K[:, sh.b0:sh.b1, sh.g0:sh.g1]
    Vs = V[:, sh.b0:sh.b1, sh.g0:sh.g1]
    rs = role[:, sh.h0:sh.h1].copy()
    return qs, Ks, Vs, rs


def out_dim(sh: Shard) -> int:
    """Dimension of out [L][B][Hq][d] along which the ranks' parts join."""
    return 2 if sh.kind == "heads" else 1


def sets_dim(sh: Shard) -> int:
    """Dimension of S [B][Hs][k] along which the ranks' parts join."""
    return 1 if sh.kind == "heads" else 0


def gather(sh: Shard, part, dim: int, group=None):
    """All ranks' parts (equal shapes), joined along `dim` in rank order: one
    all-gather (NCCL on GPUs, gloo on CPU)."""
    import torch
    import torch.distributed as dist
    if sh.world == 1:
        return part
    part = part.contiguous()
    bufs = [torch.empty_like(part) for _ in range(sh.world)]
    dist.all_gather(bufs, part, group=group)
    return torch.cat(bufs, dim=dim)


class ShardedStep:
    """One rank's part of a sharded decode step on its own GPU.

    A library context for the shard's shapes (`lyc.Lyc`), the shard's views
    of the caller's inputs, and the gather of the results.  `step()` runs the
    rank's L-layer step (one CUDA graph replay) and all-gathers the outputs
    and the outgoing sets into full-size tensors on every rank."""

    def __init__(self, sh: Shard, L: int, Hq: int, Hkv: int, d: int, n_max: int, k: int,
                 dtype: str = "bf16", select_mode: str = "kvgroup_mean", device: int = 0,
                 flags: int = 0):
        import torch
        from hybrid_head_sparse_b200 import lyc
        self.sh = sh
        self.kvgroup = select_mode == "kvgroup_mean"
        self.ctx = lyc.Lyc(L, sh.B, sh.Hq, sh.Hkv, d, n_max, k, dtype=dtype,
                           select_mode=select_mode, device=device, flags=flags)
        dev = torch.device("cuda", device)
        self.out = torch.empty((L, sh.B, sh.Hq, d), device=dev)
        self.S = torch.empty((sh.B, self.ctx.Hs, k), dtype=torch.int32, device=dev)
        self.k = k

    def step(self, q, K, V, n: int, role, stream=None, group=None):
        """q, K, V, role: the shard's inputs (`take`).  Returns the full
        out [L][B][Hq][d] and S [B][Hs][k], gathered over the ranks."""
        self.ctx.decode_step(q, K, V, n, role, self.k, self.out, self.S, stream=stream)
        return (gather(self.sh, self.out, out_dim(self.sh), group),
                gather(self.sh, self.S, sets_dim(self.sh), group))

    def close(self):
        self.ctx.close()
