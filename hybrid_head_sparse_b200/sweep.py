"""Single-layer kernel sweep: retrieval (dense) and gather (sparse) attention
GB/s, measured separately on one B200.

One layer of 32 query / 8 KV heads, d = 128, bf16, batch B in {1, 8}, context
n in {4K, 16K, 64K, 256K, 512K}, budget k in {256, 1024, 4096, 8192}.
- "dense" runs every head as a retrieval head (the layer-0 form): the pooled
  attention kernel streams all n rows of every KV group, then the selection
  kernel runs.  Bytes = B * Hkv * n * d * 2 (K and V) * 2.
- "gather" hands every head an inherited set (LYC_STEP_S_IN, no retrieval
  head): the kernel reads only the k rows of each set.  Sets are k/64 whole
  64-token blocks ("blocks") or k scattered tokens ("scattered"), seeded and
  sorted.  Bytes = the K and V rows of every pass: one pass per query head in
  per-head selection mode, one per KV group in group mode.

Each case is timed with CUDA events around the attention launches (the
library's timing mode: the layer's launch and the small launch that combines
its split rows) over R replays of the captured step, with the L2 flushed (a
256 MiB write) before every replay.  One JSON line per case goes to stdout.

Usage: python -m hybrid_head_sparse_b200.sweep [--quick] [--gather cp_async|tma]
       [--select-mode per_qhead|kvgroup_mean] [--reps R]
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np
import torch

from . import lyc
from . import workloads as W

HQ, HKV, D = 32, 8, 128
FULL = dict(B=(1, 8), n=(4096, 16384, 65536, 262144, 524288), k=(256, 1024, 4096, 8192))
QUICK = dict(B=(1,), n=(16384, 131072), k=(1024, 4096))


def measured_hbm_gbs() -> float | None:
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"])
    except (OSError, KeyError, ValueError):
        return None


def attn_ms(ctx, run, flush, reps: int):
    """CUDA-event time per replay of the attention launches (the layer's, plus
    the launch that combines its split rows) and of the selection launch, if
    any, over `reps` replays, L2 flushed before each."""
    ctx.set_timing(True)
    run()
    torch.cuda.synchronize()
    ctx.kernel_times()
    for _ in range(reps):
        flush.zero_()
        run()
    torch.cuda.synchronize()
    t = ctx.kernel_times()
    ctx.set_timing(False)
    a = sum(x[2] for x in t if x[0] == 0) / reps
    s = [x[2] for x in t if x[0] == 1]
    return float(a), (float(sum(s) / reps) if s else None)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--quick", action="store_true", help="a few cases only")
    ap.add_argument("--gather", choices=["tma", "cp_async"], default="cp_async")
    ap.add_argument("--select-mode", choices=["per_qhead", "kvgroup_mean"], default="per_qhead")
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--patterns", default="blocks,scattered")
    args = ap.parse_args(argv)
    grid = QUICK if args.quick else FULL
    peak = measured_hbm_gbs()
    lyc.load()
    dev = torch.device("cuda", torch.cuda.current_device())
    Bmax, nmax = max(grid["B"]), max(grid["n"])
    kmax = max(grid["k"])
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    K = torch.randn((1, Bmax, HKV, nmax, D), generator=gen, device=dev).to(torch.bfloat16)
    V = torch.randn((1, Bmax, HKV, nmax, D), generator=gen, device=dev).to(torch.bfloat16)
    q = torch.randn((1, Bmax, HQ, D), generator=gen, device=dev).to(torch.bfloat16)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flags = lyc.LYC_CFG_TMA_GATHER if args.gather == "tma" else 0
    for B in grid["B"]:
        ctx = lyc.Lyc(1, B, HQ, HKV, D, nmax, kmax, select_mode=args.select_mode, flags=flags)
        Hs = ctx.Hs
        qB = q[:, :B].contiguous()
        KB, VB = K[:, :B], V[:, :B]
        out = torch.empty((1, B, HQ, D), device=dev)
        for n in grid["n"]:
            # retrieval kernel: every head dense
            kk = min(kmax, n)
            S = torch.empty((B, Hs, kk), dtype=torch.int32, device=dev)
            ones = np.ones((1, HQ), dtype=np.uint8)
            ms, sel_ms = attn_ms(ctx, lambda: ctx.decode_step(qB, KB, VB, n, ones, kk, out, S),
                                 flush, args.reps)
            nbytes = B * HKV * n * D * 2 * 2
            line = {"kernel": "dense", "B": B, "n": n, "k": kk, "select_mode": args.select_mode,
                    "attn_us": ms * 1e3, "bytes": nbytes, "gbs": nbytes / (ms / 1e3) / 1e9,
                    "selection_us": None if sel_ms is None else sel_ms * 1e3}
            if peak:
                line["frac_of_measured_peak"] = line["gbs"] / peak
            print(json.dumps(line), flush=True)
            # gather kernel: every head sparse over an inherited set
            zeros = np.zeros((1, HQ), dtype=np.uint8)
            for k in grid["k"]:
                if k > n:
                    continue
                for pattern in args.patterns.split(","):
                    if pattern == "blocks" and k % 64:
                        continue
                    S0 = W.inherited_sets(B, Hs, n, k, pattern, seed=n + k, device=dev)
                    S = torch.empty_like(S0)

                    def run():
                        S.copy_(S0)
                        ctx.decode_step(qB, KB, VB, n, zeros, k, out, S, s_in=True)
                    ms, _ = attn_ms(ctx, run, flush, args.reps)
                    nbytes = B * Hs * k * D * 2 * 2
                    line = {"kernel": "gather", "B": B, "n": n, "k": k, "pattern": pattern,
                            "select_mode": args.select_mode, "gather": args.gather,
                            "attn_us": ms * 1e3, "bytes": nbytes,
                            "gbs": nbytes / (ms / 1e3) / 1e9}
                    if peak:
                        line["frac_of_measured_peak"] = line["gbs"] / peak
                    print(json.dumps(line), flush=True)
                    rc = ctx.sync_status()
                    if rc != 0:
                        raise RuntimeError(f"device status: {lyc.lyc_status_string(rc)}")
        ctx.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
