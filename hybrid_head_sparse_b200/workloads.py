"""Seeded synthetic inputs for the hybrid-head sparse decode step.

This module only draws numbers: queries, the KV cache, role masks and
inherited token sets, with the shapes and value distributions of the
workloads the LycheeDecode pages evaluate (Llama3-8B- and Qwen3-8B-class GQA
attention stacks, 16K-128K context, token budget k up to 4096, batch 1-4; page
"LycheeDecode ..." paper-graph-ui summary, section 4 setup and Figure 4).  It
holds none of the method's arithmetic.  Both the CUDA path's tests and the
oracle's tests take their inputs from here, so the two sides always see the
same bytes.

Layouts (what the library expects):
  q     [L][B][Hq][d]         bf16 or fp32
  K, V  [L][B][Hkv][n][d]     same dtype, d contiguous
  role  [L][Hq] uint8         1 = retrieval head
  S     [B][Hs][k] int32      Hs = Hq (per-head selection) or Hkv (group mode)
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class StackSpec:
    name: str
    L: int
    B: int
    Hq: int
    Hkv: int
    d: int
    n: int
    k: int
    dtype: str = "bf16"            # "bf16" | "fp32"
    roles: str = "random"          # "first-head" | "random" | "all"
    retrieval_per_layer: int = 2   # for roles == "random"
    planted: str = "heavy"         # "normalised" | "heavy" | "none"
    n_planted: int = 256
    seed: int = 0
    n_max: int | None = None       # allocated cache rows (>= n); default n

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def rows(self) -> int:
        return self.n if self.n_max is None else self.n_max

    def with_(self, **kw) -> "StackSpec":
        return replace(self, **kw)


# The workloads, by what they are.
TINY = StackSpec("tiny-2L-4q2kv-d64-fp32-n512-k64", L=2, B=1, Hq=4, Hkv=2, d=64, n=512,
                 k=64, dtype="fp32", roles="first-head", planted="normalised",
                 n_planted=8, seed=0)
LLAMA3_8B_32K = StackSpec("llama3-8b-attn-stack-n32768-k4096", L=32, B=1, Hq=32, Hkv=8,
                          d=128, n=32768, k=4096, retrieval_per_layer=2)
LLAMA3_8B_128K = StackSpec("llama3-8b-attn-stack-n131072-k4096", L=32, B=1, Hq=32, Hkv=8,
                           d=128, n=131072, k=4096, retrieval_per_layer=2)
QWEN3_8B_64K_B4 = StackSpec("qwen3-8b-attn-stack-b4-n65536-k2048", L=36, B=4, Hq=32,
                            Hkv=8, d=128, n=65536, k=2048, retrieval_per_layer=3)

WORKLOADS = {s.name: s for s in (TINY, LLAMA3_8B_32K, LLAMA3_8B_128K, QWEN3_8B_64K_B4)}


def role_mask(spec: StackSpec) -> np.ndarray:
    """[L][Hq] uint8.  Layer 0 is all ones (every head of layer 0 retrieves)."""
    L, Hq = spec.L, spec.Hq
    role = np.zeros((L, Hq), dtype=np.uint8)
    role[0, :] = 1
    if spec.roles == "all":
        role[:, :] = 1
    elif spec.roles == "first-head":
        role[1:, 0] = 1
    elif spec.roles == "random":
        g = torch.Generator(device="cpu")
        g.manual_seed(10_000 + spec.seed)
        for l in range(1, L):
            pick = torch.randperm(Hq, generator=g)[: spec.retrieval_per_layer]
            role[l, pick.numpy()] = 1
    else:
        raise ValueError(spec.roles)
    return role


def _torch_dtype(spec: StackSpec):
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[spec.dtype]


def make_stack(spec: StackSpec, device: str | torch.device = "cpu") -> dict:
    """Draw q, K, V for one step.  Returns torch tensors on `device` plus the
    role mask (numpy).  Draw order: q, then K layer by layer, then V layer by
    layer, then the planted positions; everything from one generator seeded
    with spec.seed on `device`."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(spec.seed)
    dt = _torch_dtype(spec)
    L, B, Hq, Hkv, d, rows = spec.L, spec.B, spec.Hq, spec.Hkv, spec.d, spec.rows
    q = torch.randn((L, B, Hq, d), generator=gen, device=device, dtype=torch.float32).to(dt)
    K = torch.empty((L, B, Hkv, rows, d), device=device, dtype=dt)
    V = torch.empty((L, B, Hkv, rows, d), device=device, dtype=dt)
    for l in range(L):
        K[l] = torch.randn((B, Hkv, rows, d), generator=gen, device=device,
                           dtype=torch.float32).to(dt)
    for l in range(L):
        V[l] = torch.randn((B, Hkv, rows, d), generator=gen, device=device,
                           dtype=torch.float32).to(dt)
    G = spec.G
    n = spec.n
    if spec.planted != "none":
        for l in range(L):
            for b in range(B):
                for g in range(Hkv):
                    qbar = q[l, b, g * G:(g + 1) * G].float().mean(dim=0)
                    if spec.planted == "normalised":
                        # keys = 3 x the normalised mean query of the group
                        pos = torch.randperm(n, generator=gen, device=device)[: spec.n_planted]
                        key = 3.0 * qbar / qbar.norm()
                    elif spec.planted == "heavy":
                        # sinks 0-3 plus n_planted heavy hitters, keys = 2 x mean query
                        extra = torch.randperm(max(n - 4, 0), generator=gen,
                                               device=device)[: spec.n_planted] + 4
                        sinks = torch.arange(min(4, n), device=device)
                        pos = torch.cat([sinks, extra])
                        key = 2.0 * qbar
                    else:
                        raise ValueError(spec.planted)
                    K[l, b, g, pos] = key.to(dt)
    return {"q": q, "k": K, "v": V, "role": role_mask(spec), "spec": spec}


def inherited_sets(B: int, Hs: int, n: int, k: int, pattern: str, seed: int,
                   device: str | torch.device = "cpu") -> torch.Tensor:
    """[B][Hs][k] int32 ascending, distinct.  pattern "blocks": k/64 distinct
    64-token blocks; "scattered": k distinct uniform indices.  k <= n."""
    assert k <= n
    gen = torch.Generator(device="cpu")
    gen.manual_seed(20_000 + seed)
    out = torch.empty((B, Hs, k), dtype=torch.int32)
    for b in range(B):
        for s in range(Hs):
            if pattern == "blocks":
                assert k % 64 == 0 and n >= k
                nblk = n // 64
                blk = torch.randperm(nblk, generator=gen)[: k // 64].sort().values
                idx = (blk[:, None] * 64 + torch.arange(64)[None, :]).reshape(-1)
            elif pattern == "scattered":
                idx = torch.randperm(n, generator=gen)[:k].sort().values
            else:
                raise ValueError(pattern)
            out[b, s] = idx.to(torch.int32)
    return out.to(device)


def host_view(t: torch.Tensor) -> np.ndarray:
    """Contiguous host numpy copy; bf16 becomes its uint16 bit patterns."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
