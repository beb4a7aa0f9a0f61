"""Throughput of the hybrid-head sparse decode step (attention stack) on B200.

Default workload: the Llama3-8B-shaped attention stack (32 layers, 32 query /
8 KV heads, d=128, bf16) at n = 131072 tokens with token budget k = 4096,
batch 1, layer 0 all retrieval and 2 retrieval query heads per later layer at
seeded positions; synthetic seeded data.  One step = one pass of the whole
L-layer stack (dense retrieval heads + top-k selection + sparse gathered
heads, every layer), launched as one CUDA graph.

Prints one JSON line on rank 0.  `--impl reference` times the fp64 CPU
oracle instead: whole L-layer steps of the same workload on the host cores.
`--workload` picks the Llama3-8B-shaped stack at 128K (default) or 32K, or the
Qwen3-8B-shaped stack (36 layers, batch 4, 64K, k=2048).
Multi-GPU (torchrun): every rank runs its own replica of the step (the path
has no exchange step); value = all ranks' steps / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attn-stack decode steps/s at 128K ctx, k=4096; HBM GB/s vs peak"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
# the sources that decide what an attention launch reads: the kernel and the
# plan that cuts the rows into pieces
ATTN_SOURCES = ["attn_mma_kernel.cu", "lyc_plan.h", "lyc_device.cuh", "lyc_api.cu"]


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["lyc", "reference"], default="lyc")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama3-8b-128k",
                    help="llama3-8b-128k (32 layers, n=131072, k=4096, 2 retrieval heads per "
                         "layer: the headline), llama3-8b-32k (n=32768), qwen3-8b-64k-b4 (36 "
                         "layers, batch 4, n=65536, k=2048, 3 retrieval heads per layer)")
    ap.add_argument("--n", type=int, default=None, help="context length (default: the workload's)")
    ap.add_argument("--k", type=int, default=None, help="token budget (default: the workload's)")
    ap.add_argument("--layers", type=int, default=None, help="layers (default: the workload's)")
    ap.add_argument("--retrieval-heads", type=int, default=None,
                    help="retrieval query heads per layer after layer 0 (default: the "
                         "workload's); -1 = all (the all-retrieval dense baseline)")
    ap.add_argument("--select-mode", choices=["per_qhead", "kvgroup_mean"], default="kvgroup_mean",
                    help="kvgroup_mean: one set per KV group, keyed by the group's mean query (the "
                         "pages' GQA handling, whose bytes are the analytic floor); per_qhead: one "
                         "set per query head (the line also times the mode not chosen)")
    ap.add_argument("--attn-kernel", choices=["mma", "tcgen05"], default="mma",
                    help="bf16 attention kernel: mma.sync (default) or tcgen05/TMEM")
    ap.add_argument("--serving", action="store_true",
                    help="the serving form instead: lyc_decode_step_batch on a batch of four "
                         "cache lengths, paged cache (64-row pages), current token appended")
    ap.add_argument("--selection", choices=["topk", "ratio", "block", "topp", "threshold"],
                    default="topk",
                    help="selection rule; anything but topk prints the rule's own line instead of "
                         "the default one")
    ap.add_argument("--ratio", default="1/64", help="ratio rule: theta as num/den")
    ap.add_argument("--block", type=int, default=64, help="block rule: rows per block")
    ap.add_argument("--p", type=float, default=0.5, help="top-p rule: probability mass")
    ap.add_argument("--tau", type=float, default=1e-4, help="threshold rule: smallest probability")
    ap.add_argument("--correction", action="store_true",
                    help="Cache Correction instead: dense causal attention of the T most recent "
                         "positions over the cache (lyc_cache_correction), one line")
    ap.add_argument("--T", type=int, default=32, help="Cache Correction: positions refreshed")
    ap.add_argument("--noalloc", action="store_true",
                    help="the allocation-free entry point instead: one layer of sparse heads "
                         "over given sets (lyc_sparse_attention_noalloc), every head sparse, "
                         "batch 8 unless --batch, one line")
    ap.add_argument("--shard", choices=["heads", "batch"], default=None,
                    help="under torchrun: split one step over the ranks (KV groups with their "
                         "query heads, or batch elements), all-gather the outputs and sets every "
                         "step; strong scaling.  Default: every rank runs its own replica")
    ap.add_argument("--batch", type=int, default=None, help="batch elements (default: the workload's)")
    ap.add_argument("--traffic-from", default=None, metavar="CSV",
                    help="print the traffic record of an ncu capture (dram__bytes_read.sum and "
                         "dram__bytes_write.sum, --csv) of this command line's attention "
                         "launches: one whole step's launches, summed and divided by the layers, "
                         "stamped with the hash of the sources here; no GPU work")
    ap.add_argument("--launches-per-step", type=int, default=0,
                    help="with --traffic-from: the attention launches of one step (the capture's "
                         "count must match; the bench line's attention launch count)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-other-mode", action="store_true",
                    help="skip timing the selection mode not chosen")
    ap.add_argument("--sustained-ms", type=float, default=500.0,
                    help="after the K timed steps, replay for at least this long with the clock "
                         "sampler still running (a longer sample of the same step; reported "
                         "apart from the timed value)")
    return ap.parse_args(argv)


# workload choice -> (spec name in workloads.py, family prefix of the line's name)
WORKLOADS = {"llama3-8b-128k": ("LLAMA3_8B_128K", "llama3-8b"),
             "llama3-8b-32k": ("LLAMA3_8B_32K", "llama3-8b"),
             "qwen3-8b-64k-b4": ("QWEN3_8B_64K_B4", "qwen3-8b")}


def workload_spec(args):
    """The chosen workload with the command line's overrides; its name spells
    out the shape that differs from nothing: batch (when > 1), n, k, layers
    (when not the workload's), retrieval heads per layer (or dense)."""
    from hybrid_head_sparse_b200 import workloads as W
    attr, family = WORKLOADS[args.workload]
    base = getattr(W, attr)
    over = {}
    for key, val in (("n", args.n), ("k", args.k), ("L", args.layers), ("B", args.batch)):
        if val is not None:
            over[key] = val
    spec = base.with_(**over)
    r = base.retrieval_per_layer if args.retrieval_heads is None else args.retrieval_heads
    name = f"{family}-attn-stack" + (f"-b{spec.B}" if spec.B != 1 else "") + f"-n{spec.n}-k{spec.k}"
    if spec.L != base.L:
        name += f"-L{spec.L}"
    if r < 0:
        return spec.with_(roles="all", name=name + "-dense")
    return spec.with_(retrieval_per_layer=r, name=name + f"-r{r}")


def retrieval_heads(spec) -> int:
    return -1 if spec.roles == "all" else spec.retrieval_per_layer


def line_config(spec, args, world: int, kv_bytes: int) -> dict:
    """The `config` of a line: the same for the library arm and the oracle arm."""
    return {"workload": spec.name, "L": spec.L, "B": spec.B, "Hq": spec.Hq, "Hkv": spec.Hkv,
            "d": spec.d, "n": spec.n, "k": spec.k,
            "retrieval_heads_per_layer": retrieval_heads(spec),
            "select_mode": args.select_mode, "attn_kernel": args.attn_kernel,
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (KV cache %.1f GB per GPU)" % (kv_bytes / 1e9)}


def kv_cache_bytes(spec) -> int:
    es = 2 if spec.dtype == "bf16" else 4
    return 2 * spec.L * spec.B * spec.Hkv * spec.rows * spec.d * es


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_tflops() -> float:
    """Burst cuBLAS bf16 throughput of this GPU (the correction kernel is timed
    alone), else the fallback figure."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def attn_source_hash() -> str:
    h = hashlib.sha256()
    for f in ATTN_SOURCES:
        with open(os.path.join(ROOT, "hybrid_head_sparse_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, select_mode: str):
    """DRAM bytes per attention launch from the committed ncu summary, if it
    was taken on the current kernel source, workload and selection mode."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    want = attn_source_hash()
    for name in sorted(os.listdir(pdir)):
        if not name.startswith("attn_mma_layer_kernel") or not name.endswith(".md"):
            continue
        for line in open(os.path.join(pdir, name)):
            if line.startswith("traffic-record:"):
                try:
                    rec = json.loads(line.split(":", 1)[1])
                except ValueError:
                    continue
                if (rec.get("source_sha") == want and rec.get("workload") == workload
                        and rec.get("select_mode", "per_qhead") == select_mode):
                    return rec.get("bytes_per_launch")
    return None


def max_over_ranks(x: float, device=None) -> float:
    """The largest x over the ranks of the default process group (x itself
    without one).  Every rank must call it at the same point."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_steps_per_s(world: int, steps: int, ms_slowest: float) -> float:
    """Whole-job throughput of replicas: every rank ran `steps` steps and the
    job took as long as its slowest rank."""
    return world * steps / (ms_slowest / 1e3)


def percentiles(xs):
    xs = sorted(xs)

    def q(f):
        i = min(len(xs) - 1, max(0, int(round(f * (len(xs) - 1)))))
        return xs[i]
    return {"p10": q(0.10), "p50": q(0.50), "p90": q(0.90)}


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].isdigit():
                    rows.append(parts)
        except OSError:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [int(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": int(rows[0][2]),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None}


# ---------------------------------------------------------------- oracle timing


def oracle_step_seconds(spec, host_stack) -> float:
    """Wall time of one whole L-layer step of the oracle (every layer, every
    head, full n) on the host cores."""
    import oracle as O
    t0 = time.perf_counter()
    O.decode_step(host_stack, spec.k, n=spec.n)
    return time.perf_counter() - t0


def cpu_cores() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    if n and n.isdigit():
        return int(n)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def host_stack(spec, data, select_mode: str):
    """Host copy of the whole step's inputs for the oracle."""
    import oracle as O
    from hybrid_head_sparse_b200 import workloads as W
    mode = O.SELECT_KVGROUP_MEAN if select_mode == "kvgroup_mean" else O.SELECT_PER_QHEAD
    return O.Stack(W.host_view(data["q"]), W.host_view(data["k"]), W.host_view(data["v"]),
                   data["role"].copy(), mode)


def sample_text(spec, steps: int):
    return (f"oracle (fp64 C, OpenMP over heads) on {steps} whole step(s) of the same workload: "
            f"all {spec.L} layers, every head, n={spec.n}, k={spec.k}, same seeded inputs")


def oracle_baseline(spec, hs, budget_s: float, single_core: bool, max_steps: int = 5) -> dict:
    """cpu_baseline object: whole oracle steps on every host core, as many as
    fit in about budget_s seconds (at least one, at most max_steps), and
    (single_core) one more whole step on one core."""
    import oracle as O
    cores = O.max_threads()
    secs = [oracle_step_seconds(spec, hs)]
    while len(secs) < max_steps and sum(secs) + secs[0] <= budget_s:
        secs.append(oracle_step_seconds(spec, hs))
    sec = sum(secs) / len(secs)
    res = {"value": 1.0 / sec, "unit": "steps/s", "cores": cores, "kind": "oracle",
           "sample": sample_text(spec, len(secs)), "step_seconds": [round(t, 3) for t in secs]}
    if single_core:
        O.set_threads(1)
        try:
            s1 = oracle_step_seconds(spec, hs)
        finally:
            O.set_threads(cores)
        res["single_core"] = {"value": 1.0 / s1, "unit": "steps/s", "cores": 1,
                              "step_seconds": round(s1, 3)}
    return res


def union_ms(iv) -> float:
    """Length (ms) of the union of (start ns, end ns) intervals."""
    tot = 0
    cur_s = cur_e = None
    for a, b in sorted(iv):
        if cur_e is None or a > cur_e:
            if cur_e is not None:
                tot += cur_e - cur_s
            cur_s, cur_e = a, b
        else:
            cur_e = max(cur_e, b)
    if cur_e is not None:
        tot += cur_e - cur_s
    return tot / 1e6


# ---------------------------------------------------------------- reference arm


def run_reference(args):
    """The oracle arm: whole L-layer steps of the fp64 oracle on the host
    cores, on the library arm's workload, metric and config.  Rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch

    import oracle as O
    from hybrid_head_sparse_b200 import workloads as W
    O.build()
    spec = workload_spec(args)
    # the same seeded recipe as the library arm (drawn on the GPU when there
    # is one, as the library arm does, then copied to the host)
    data = W.make_stack(spec, "cuda" if torch.cuda.is_available() else "cpu")
    hs = host_stack(spec, data, args.select_mode)
    del data
    for _ in range(args.warmup):
        oracle_step_seconds(spec, hs)
    secs = [oracle_step_seconds(spec, hs) for _ in range(args.steps)]
    sec = sum(secs) / len(secs)
    value = 1.0 / sec
    cores = O.max_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": line_config(spec, args, args.gpus, kv_cache_bytes(spec)),
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle",
                         "sample": sample_text(spec, args.steps)},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- library arm


def run_lyc(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from hybrid_head_sparse_b200 import build as Bld
    from hybrid_head_sparse_b200 import lyc, workloads as W

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    Bld.build()
    lyc.load()

    def barrier():
        if world > 1:
            dist.barrier()

    spec = workload_spec(args)
    data = W.make_stack(spec, dev)
    torch.cuda.synchronize()
    kflags = lyc.LYC_CFG_TCGEN05 if args.attn_kernel == "tcgen05" else 0
    ctx = lyc.Lyc(spec.L, spec.B, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k, dtype=spec.dtype,
                  select_mode=args.select_mode, device=local, flags=kflags)
    out = torch.empty((spec.L, spec.B, spec.Hq, spec.d), device=dev)
    S = torch.empty((spec.B, ctx.Hs, spec.k), dtype=torch.int32, device=dev)
    role = data["role"]
    stream = torch.cuda.current_stream(dev)

    def step():
        ctx.decode_step(data["q"], data["k"], data["v"], spec.n, role, spec.k, out, S, stream=stream)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    rc = ctx.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {lyc.lyc_status_string(rc)}")

    # ---- timed region: K graph replays, device-timed, max over ranks.  The
    # clock sampler keeps running through a longer window of the same replays
    # right after it (reported apart), so that the clock record is not three
    # samples of a 20 ms region.
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local) as clk:
        evs[0].record(stream)
        for i in range(args.steps):
            step()
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_total_local = evs[0].elapsed_time(evs[-1])
        n_sus = max(args.steps, int(args.sustained_ms / max(ms_total_local / args.steps, 1e-3)) + 1)
        ev0.record(stream)
        for _ in range(n_sus):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    clocks = clk.summary()
    ms_total = max_over_ranks(ms_total_local, dev)
    ms_sus = max_over_ranks(ev0.elapsed_time(ev1), dev)
    step_ms = percentiles([evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)])
    ms_step = ms_total / args.steps
    value = job_steps_per_s(world, args.steps, ms_total)
    sustained = {"replays": n_sus, "ms_per_step": ms_sus / n_sus,
                 "value": job_steps_per_s(world, n_sus, ms_sus), "unit": "steps/s",
                 "note": "the same step replayed right after the timed region, clocks sampled "
                         "through both"}
    rc = ctx.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status after timing: {lyc.lyc_status_string(rc)}")

    analytic, distinct = ctx.step_bytes(role, spec.n, spec.k)
    peak, peak_kind = measured_peaks()
    per_layer = spec.L

    # ---- where the step's time goes: the same K replays with the device
    # timeline on (every CTA of the attention and selection launches records
    # its start and end on the GPU's global timer).  The attention kernel's
    # share of the step is the union of its CTAs' busy intervals over the
    # span; its time per step is that share of the timed ms_per_step, so it
    # can never exceed the step.
    cap = args.steps * (spec.L + 1) * (2 * 148 + 64)
    tl = torch.zeros(1 + 3 * cap, dtype=torch.int64, device=dev)
    ctx.set_timeline(tl, cap)
    step()
    torch.cuda.synchronize()
    tl.zero_()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    ms_step_tl = ev0.elapsed_time(ev1) / args.steps
    ctx.set_timeline(None, 0)
    rec = tl.cpu().numpy()
    nrec = int(min(rec[0], cap))
    r3 = rec[1:1 + 3 * nrec].reshape(-1, 3)
    kinds = (r3[:, 2] >> 32) & 0xffff
    att = [(int(a), int(b)) for a, b, kd in zip(r3[:, 0], r3[:, 1], kinds) if kd == 0]
    sel = [(int(a), int(b)) for a, b, kd in zip(r3[:, 0], r3[:, 1], kinds) if kd == 1]
    span_ms = (r3[:, 1].max() - r3[:, 0].min()) / 1e6 if nrec else float("nan")
    attn_share = union_ms(att) / span_ms if nrec else float("nan")
    sel_share = union_ms(sel) / span_ms if nrec else float("nan")
    attn_ms_step = attn_share * ms_step
    achieved = distinct / (attn_ms_step / 1e3) / 1e9
    traffic = profiled_traffic(spec.name, args.select_mode)

    # ---- the same launches one at a time: event nodes retargeted into the
    # graph serialise them, so each one is timed alone (no overlap)
    ctx.set_timing(True)
    step()
    torch.cuda.synchronize()
    ctx.kernel_times()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    ktimes = ctx.kernel_times()
    ctx.set_timing(False)
    iso_attn_ms = sum(t[2] for t in ktimes if t[0] == 0) / args.steps
    iso_topk_ms = sum(t[2] for t in ktimes if t[0] == 1) / args.steps
    # launches per step: attention launches (each of two, four or eight layers, the
    # last layer's own, and a merge launch) and selection launches (one per
    # layer)
    attn_launches, topk_launches, other_launches = ctx.step_launches()

    roofline = {
        "bound": "hbm",
        "kernel": ("attn_tc_layer_kernel" if args.attn_kernel == "tcgen05" else "attn_mma_layer_kernel")
                  + " (pooled dense + sparse attention of two, four or eight layers per launch)",
        "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs), burst figure",
        "traffic": traffic,
        "algorithmic_bytes_per_launch": distinct / per_layer,
        "avg_launch_ms": attn_ms_step / per_layer,
        "attn_share_of_step": round(attn_share, 4),
        "selection_share_of_step": round(sel_share, 4),
        "note": ("achieved = K+V bytes the attention kernel must read per step (dense groups: n "
                 "rows; each sparse pass: k rows) / its time per step; its time per step = the "
                 "union of its CTAs' busy intervals on the device timeline (same K replays), as "
                 "a share of the span, times the timed ms_per_step.  Launches overlap and each "
                 "runs several layers, so bytes and time 'per launch' are both per layer "
                 "(divided by L), like the traffic record"),
        "isolated_launches": ({
            "attn_ms_per_step": iso_attn_ms, "topk_ms_per_step": iso_topk_ms,
            "attn_gbs": round(distinct / (iso_attn_ms / 1e3) / 1e9, 1),
            "note": "each launch timed alone by event nodes in the graph, which serialise the "
                    "launches (no overlap between layers): an upper bound on launch time"}
            if iso_attn_ms > 0 else
            {"note": "not measured"}),
        "timeline_ms_per_step": ms_step_tl,
    }
    step_gbs = analytic / (ms_step / 1e3) / 1e9

    # ---- end to end through the host-buffer entry point
    e2e = None
    if not args.no_e2e:
        q_h = data["q"].cpu().pin_memory()
        out_h = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        S_h = torch.empty(S.shape, dtype=torch.int32).pin_memory()

        def hstep():
            ctx.decode_step_host(q_h, data["k"], data["v"], spec.n, role, spec.k, out_h, S_h,
                                 stream=stream)

        for _ in range(2):
            hstep()
        torch.cuda.synchronize()
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            hstep()
        ev1.record(stream)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), dev)
        e2e = {"value": job_steps_per_s(world, args.steps, ms_e2e), "unit": "steps/s",
               "h2d_bytes_per_step": q_h.numel() * q_h.element_size(),
               "d2h_bytes_per_step": out_h.numel() * 4 + S_h.numel() * 4,
               "note": "lyc_decode_step_host: q from pinned host memory in, outputs and sets back "
                       "to pinned host memory, every step; KV cache resident on the device"}
        rc = ctx.sync_status()
        if rc != 0:
            raise RuntimeError(f"device status after e2e: {lyc.lyc_status_string(rc)}")

    # ---- the other selection mode on the same inputs (its steps/s and byte rates)
    other = None
    if not args.no_other_mode:
        omode = "per_qhead" if args.select_mode == "kvgroup_mean" else "kvgroup_mean"
        octx = lyc.Lyc(spec.L, spec.B, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k, dtype=spec.dtype,
                       select_mode=omode, device=local, flags=kflags)
        oS = torch.empty((spec.B, octx.Hs, spec.k), dtype=torch.int32, device=dev)

        def ostep():
            octx.decode_step(data["q"], data["k"], data["v"], spec.n, role, spec.k, out, oS,
                             stream=stream)

        for _ in range(max(args.warmup, 1)):
            ostep()
        torch.cuda.synchronize()
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            ostep()
        ev1.record(stream)
        torch.cuda.synchronize()
        oms = max_over_ranks(ev0.elapsed_time(ev1), dev)
        rc = octx.sync_status()
        if rc != 0:
            raise RuntimeError(f"device status ({omode}): {lyc.lyc_status_string(rc)}")
        oan, odi = octx.step_bytes(role, spec.n, spec.k)
        octx.close()
        oms_step = oms / args.steps
        other = {"select_mode": omode, "value": job_steps_per_s(world, args.steps, oms),
                 "unit": "steps/s", "ms_per_step": oms_step,
                 "analytic_frac_of_measured_peak": round(oan / (oms_step / 1e3) / 1e9 / peak, 4),
                 "kernel_bytes_per_step": odi,
                 "kernel_gbs": round(odi / (oms_step / 1e3) / 1e9, 1)}

    # ---- the oracle on the host cores (rank 0, one GPU only): whole steps
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle as O
        O.build()
        hs = host_stack(spec, data, args.select_mode)
        cpu = oracle_baseline(spec, hs, budget_s=8.0, single_core=True)
        del hs

    launches_per_step = attn_launches + topk_launches + other_launches
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "step_ms_distribution": {k: round(v, 4) for k, v in step_ms.items()},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if spec.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) q/K/V, sinks + 256 planted heavy hitters per KV head)",
        "config": line_config(spec, args, world, kv_cache_bytes(spec)),
        "hbm": {"analytic_bytes_per_step": analytic, "kernel_bytes_per_step": distinct,
                "analytic_gbs": round(step_gbs, 1),
                "frac_of_measured_peak": round(step_gbs / peak, 4),
                "frac_of_8tbs": round(step_gbs / NOMINAL_HBM_GBS, 4),
                "kernel_gbs": round(distinct / (ms_step / 1e3) / 1e9, 1)},
        "roofline": roofline,
        "sustained": sustained,
        "other_select_mode": other,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "launches_per_step": {"attention": attn_launches, "selection": topk_launches,
                              "other": other_launches},
        "clocks": clocks,
    }
    ctx.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


SERVING_N = (131072, 98304, 65536, 32768)


def serving_analytic_bytes(role, n_list, k, L, Hq, Hkv, d, select_mode):
    """The step's byte floor for per-element lengths: per layer and element,
    n[b] rows of K and V for every KV group with a retrieval head (all groups
    at layer 0), min(k, n[b]) rows for every other group."""
    G = Hq // Hkv
    total = 0
    for l in range(L):
        ret = [True] * Hkv if l == 0 else [bool(role[l, g * G:(g + 1) * G].any()) for g in range(Hkv)]
        for nb in n_list:
            for g in range(Hkv):
                total += (nb if ret[g] else min(k, nb)) * d * 2 * 2
    return total


def run_serving(args):
    """The serving form on one GPU: Llama3-8B-shaped stack, a batch of four
    cache lengths, a paged cache of 64-row pages (shuffled), the current
    token's K/V appended by the step; steps/s and the byte-floor rate."""
    import numpy as np
    import torch

    from hybrid_head_sparse_b200 import build as Bld
    from hybrid_head_sparse_b200 import lyc, workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    Bld.build()
    lyc.load()
    base = workload_spec(args)
    L, Hq, Hkv, d, k = base.L, base.Hq, base.Hkv, base.d, base.k
    n_list = list(SERVING_N)
    B = len(n_list)
    page_rows = 64
    blocks = [(nb + page_rows - 1) // page_rows for nb in n_list]
    npages = sum(blocks)
    rng = np.random.default_rng(7)
    perm = rng.permutation(npages)
    max_blocks = max(blocks)
    bt = np.zeros((B, max_blocks), dtype=np.int32)
    j = 0
    for b in range(B):
        for blk in range(blocks[b]):
            bt[b, blk] = perm[j]
            j += 1
    gen = torch.Generator(device=dev)
    gen.manual_seed(base.seed)
    Kp = torch.empty((L, npages, page_rows, Hkv, d), device=dev, dtype=torch.bfloat16)
    Vp = torch.empty_like(Kp)
    for l in range(L):  # layer by layer: bounded float32 staging
        Kp[l] = torch.randn((npages, page_rows, Hkv, d), generator=gen, device=dev).to(torch.bfloat16)
        Vp[l] = torch.randn((npages, page_rows, Hkv, d), generator=gen, device=dev).to(torch.bfloat16)
    q = torch.randn((L, B, Hq, d), generator=gen, device=dev).to(torch.bfloat16)
    k_new = torch.randn((L, B, Hkv, d), generator=gen, device=dev).to(torch.bfloat16)
    v_new = torch.randn((L, B, Hkv, d), generator=gen, device=dev).to(torch.bfloat16)
    role = W.role_mask(base.with_(B=B))
    bt_dev = torch.from_numpy(bt).to(dev)
    ctx = lyc.Lyc(L, B, Hq, Hkv, d, max(n_list), k, select_mode=args.select_mode)
    out = torch.empty((L, B, Hq, d), device=dev)
    S = torch.empty((B, ctx.Hs, k), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ctx.decode_step_batch(q, Kp, Vp, n_list, role, k, out, S, stream=stream, k_new=k_new,
                              v_new=v_new, block_table=bt_dev, page_rows=page_rows)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    rc = ctx.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {lyc.lyc_status_string(rc)}")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        evs[0].record(stream)
        for i in range(args.steps):
            step()
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
    ms_total = evs[0].elapsed_time(evs[-1])
    step_ms = percentiles([evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)])
    rc = ctx.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status after timing: {lyc.lyc_status_string(rc)}")
    ms_step = ms_total / args.steps
    analytic = serving_analytic_bytes(role, n_list, k, L, Hq, Hkv, d, args.select_mode)
    peak, _ = measured_peaks()
    gbs = analytic / (ms_step / 1e3) / 1e9
    line = {
        "metric": "serving decode steps/s (batch of 4 lengths, paged cache, current token appended)",
        "value": args.steps / (ms_total / 1e3), "unit": "steps/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "step_ms_distribution": {kk: round(v, 4) for kk, v in step_ms.items()},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) pages, q and appended rows; shuffled 64-row pages)",
        "config": {"workload": "llama3-8b-serving-b4-paged64", "L": L, "B": B, "Hq": Hq,
                   "Hkv": Hkv, "d": d, "n": n_list, "k": k, "page_rows": page_rows,
                   "retrieval_heads_per_layer": retrieval_heads(base),
                   "select_mode": args.select_mode, "append": True, "parallelism": "replicas x1",
                   "l2": "inputs larger than L2 (KV pages %.1f GB)" % (
                       2 * Kp.numel() * Kp.element_size() / 1e9)},
        "hbm": {"analytic_bytes_per_step": analytic, "analytic_gbs": round(gbs, 1),
                "frac_of_measured_peak": round(gbs / peak, 4),
                "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4)},
        "clocks": clk.summary(),
    }
    ctx.close()
    print(json.dumps(line), flush=True)
    return 0


def run_sharded(args):
    """One step split over the ranks (hybrid_head_sparse_b200/shard.py): each
    rank runs the L-layer step on its KV groups (or batch elements) and the
    outputs and sets are all-gathered every step (NCCL).  Total work is fixed
    as the rank count grows (strong scaling)."""
    import torch
    import torch.distributed as dist

    from hybrid_head_sparse_b200 import build as Bld
    from hybrid_head_sparse_b200 import lyc, shard, workloads as W

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    Bld.build()
    lyc.load()

    def barrier():
        if world > 1:
            dist.barrier()

    spec = workload_spec(args)
    data = W.make_stack(spec, dev)
    sh = shard.shard_of(args.shard, rank, world, spec.B, spec.Hq, spec.Hkv)
    qs, Ks, Vs, rs = shard.take(sh, data["q"], data["k"], data["v"], data["role"])
    ss = shard.ShardedStep(sh, spec.L, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k,
                           select_mode=args.select_mode, device=local)
    stream = torch.cuda.current_stream(dev)

    def step():
        return ss.step(qs, Ks, Vs, spec.n, rs, stream=stream)

    for _ in range(max(args.warmup, 1)):
        out, S = step()
    torch.cuda.synchronize()
    rc = ss.ctx.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {lyc.lyc_status_string(rc)}")
    barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            out, S = step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    rc = ss.ctx.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status after timing: {lyc.lyc_status_string(rc)}")
    cfg_role = data["role"]
    full = lyc.Lyc(spec.L, spec.B, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k,
                   select_mode=args.select_mode, device=local)
    analytic, _ = full.step_bytes(cfg_role, spec.n, spec.k)
    full.close()
    ss.close()
    ms_step = ms / args.steps
    peak, _ = measured_peaks()
    gbs = analytic / (ms_step / 1e3) / 1e9
    line = {
        "metric": METRIC + f" ({args.shard}-sharded step)", "value": args.steps / (ms / 1e3),
        "unit": "steps/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/K/V, sinks + 256 planted heavy hitters per KV head)",
        "config": {"workload": spec.name, "L": spec.L, "B": spec.B, "Hq": spec.Hq,
                   "Hkv": spec.Hkv, "d": spec.d, "n": spec.n, "k": spec.k,
                   "select_mode": args.select_mode, "parallelism": f"{args.shard}-shard x{world}",
                   "per_rank": {"kv_groups": sh.Hkv, "q_heads": sh.Hq, "batch": sh.B},
                   "collective": "all-gather of outputs and sets per step (NCCL)"},
        "hbm": {"analytic_bytes_per_step": analytic, "analytic_gbs_all_ranks": round(gbs, 1),
                "frac_of_measured_peak_x_ranks": round(gbs / (peak * world), 4)},
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_correction(args):
    """Cache Correction on one GPU: the T most recent positions of the
    Llama3-8B-shaped stack at n tokens are attended again, densely and
    causally, over the whole cache, every layer, with their refreshed K/V rows
    written first.  One pass = one lyc_cache_correction call (the row append,
    the attention launch and the launch that merges split rows)."""
    import numpy as np
    import torch

    from hybrid_head_sparse_b200 import build as Bld
    from hybrid_head_sparse_b200 import lyc, workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    Bld.build()
    lyc.load()
    spec = workload_spec(args)
    L, B, Hq, Hkv, d, n, T = spec.L, spec.B, spec.Hq, spec.Hkv, spec.d, spec.n, args.T
    data = W.make_stack(spec, dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(spec.seed + 1)
    q = torch.randn((L, B, Hq, T, d), generator=gen, device=dev).to(torch.bfloat16)
    k_new = torch.randn((L, B, Hkv, T, d), generator=gen, device=dev).to(torch.bfloat16)
    v_new = torch.randn((L, B, Hkv, T, d), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty((L, B, Hq, T, d), device=dev)
    ctx = lyc.Lyc(L, B, Hq, Hkv, d, n, spec.k)
    stream = torch.cuda.current_stream(dev)

    def step():
        ctx.cache_correction(q, data["k"], data["v"], n, out, k_new=k_new, v_new=v_new,
                             stream=stream)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    rc = ctx.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {lyc.lyc_status_string(rc)}")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        evs[0].record(stream)
        for i in range(args.steps):
            step()
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
    ms_total = evs[0].elapsed_time(evs[-1])
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    rc = ctx.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status after timing: {lyc.lyc_status_string(rc)}")
    ms_pass = ms_total / args.steps
    # algorithmic bytes: every (l, b, g) group's n K and V rows read once (the
    # causal mask only drops rows past each query's position, all inside the
    # last tile); q read, out written and the T refreshed rows written are
    # counted apart
    kv_bytes = L * B * Hkv * n * d * 2 * 2
    io_bytes = L * B * Hq * T * d * (2 + 4) + L * B * Hkv * T * d * 2 * 2
    flops = 0
    for t in range(T):  # QK and PV, 2 flops per multiply-add, causal rows
        flops += 4 * L * B * Hq * (n - T + t + 1) * d
    peak, peak_kind = measured_peaks()
    gbs = kv_bytes / (ms_pass / 1e3) / 1e9
    tflops = flops / (ms_pass / 1e3) / 1e12
    line = {
        "metric": f"Cache Correction passes/s at {n // 1024}K ctx (T={T} positions, every layer)",
        "value": args.steps / (ms_total / 1e3), "unit": "passes/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_pass,
        "step_ms_distribution": {kk: round(v, 4) for kk, v in percentiles(per).items()},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/K/V with sinks and planted heavy hitters; "
                "seeded N(0,1) refreshed rows)",
        "config": {"workload": f"llama3-8b-cache-correction-n{n}-T{T}", "L": L, "B": B,
                   "Hq": Hq, "Hkv": Hkv, "d": d, "n": n, "T": T, "append": True,
                   "parallelism": "replicas x1",
                   "l2": "inputs larger than L2 (KV cache %.1f GB)" % (
                       2 * data["k"].numel() * data["k"].element_size() / 1e9)},
        "roofline": {
            "bound": "hbm", "kernel": "correction_tc_kernel (tcgen05, one launch for all layers)"
                                      " + its split-merge launch + the row append",
            "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
            "frac": round(gbs / peak, 4),
            "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
            "traffic": None, "algorithmic_bytes_per_launch": kv_bytes,
            "avg_launch_ms": ms_pass,
            "note": "achieved = K+V bytes of every (layer, KV group) / CUDA-event time of the "
                    "whole call; q, out and refreshed rows (%d bytes) not counted" % io_bytes},
        "tensor": {"tflops": round(tflops, 1), "flops_per_pass": flops,
                   "frac_of_measured_bf16": round(tflops / measured_bf16_tflops(), 4)},
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline:
        import oracle as O
        idx = torch.tensor([0], device=dev)
        Kh = W.host_view(data["k"].index_select(0, idx)[:, :, :, :n]).copy()
        Vh = W.host_view(data["v"].index_select(0, idx)[:, :, :, :n]).copy()
        Kh[:, :, :, n - T:n] = W.host_view(k_new.index_select(0, idx))
        Vh[:, :, :, n - T:n] = W.host_view(v_new.index_select(0, idx))
        st = O.Stack(W.host_view(data["q"].index_select(0, idx)), Kh, Vh,
                     np.ones((1, Hq), dtype=np.uint8))
        t0 = time.perf_counter()
        O.correction(st, W.host_view(q.index_select(0, idx)))
        sec = (time.perf_counter() - t0) * L
        line["cpu_baseline"] = {
            "value": 1.0 / sec, "unit": "passes/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"oracle (fp64 C, OpenMP) on layer 0 of one pass at full size (n={n}, "
                      f"T={T}, all {Hq} heads); pass time = {L} x that layer"}
    ctx.close()
    print(json.dumps(line), flush=True)
    return 0


def rule_kernel_bytes(role, trace, n, L, Hq, Hkv, d, select_mode):
    """K+V bytes the attention kernels read in one step under a selection
    rule: n rows for every KV group with a retrieval head (all at layer 0),
    and for every sparse pass (a sparse head in per-head mode, a group's
    sparse heads in group mode) the valid rows of the set it inherits."""
    import numpy as np
    G = Hq // Hkv
    row = d * 2 * 2
    sizes = (trace >= 0).sum(-1)  # [L][B][Hs]
    total = 0
    for l in range(L):
        ret = np.ones(Hq, dtype=bool) if l == 0 else role[l].astype(bool)
        for b in range(trace.shape[1]):
            for g in range(Hkv):
                heads = range(g * G, (g + 1) * G)
                if any(ret[h] for h in heads):
                    total += n * row
                if l == 0:
                    continue
                if select_mode == "kvgroup_mean":
                    if not all(ret[h] for h in heads):
                        total += int(sizes[l - 1, b, g]) * row
                else:
                    total += sum(int(sizes[l - 1, b, h]) * row for h in heads if not ret[h])
    return total


def run_rule(args):
    """The default workload under a selection rule other than a fixed k:
    steps/s, the observed set sizes and the rate on the bytes the kernels
    must read for those sets."""
    import numpy as np
    import torch

    from hybrid_head_sparse_b200 import build as Bld
    from hybrid_head_sparse_b200 import lyc, workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    Bld.build()
    lyc.load()
    spec = workload_spec(args)
    data = W.make_stack(spec, dev)
    ctx = lyc.Lyc(spec.L, spec.B, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k, dtype=spec.dtype,
                  select_mode=args.select_mode)
    num, den = (int(x) for x in args.ratio.split("/"))
    rule = {"ratio": lyc.LYC_RULE_RATIO, "block": lyc.LYC_RULE_BLOCK_TOPK, "topp": lyc.LYC_RULE_TOPP,
            "threshold": lyc.LYC_RULE_THRESHOLD}[args.selection]
    ctx.set_selection(rule, block=args.block, ratio=(num, den), p=args.p, tau=args.tau)
    out = torch.empty((spec.L, spec.B, spec.Hq, spec.d), device=dev)
    S = torch.empty((spec.B, ctx.Hs, spec.k), dtype=torch.int32, device=dev)
    role = data["role"]
    stream = torch.cuda.current_stream(dev)
    # one untimed step with the set trace: the sizes the rule chose
    trace = torch.empty((spec.L, spec.B, ctx.Hs, spec.k), dtype=torch.int32, device=dev)
    ctx.set_trace(trace)
    ctx.decode_step(data["q"], data["k"], data["v"], spec.n, role, spec.k, out, S, stream=stream)
    torch.cuda.synchronize()
    tr = trace.cpu().numpy()
    ctx.set_trace(None)
    sizes = (tr >= 0).sum(-1)

    def step():
        ctx.decode_step(data["q"], data["k"], data["v"], spec.n, role, spec.k, out, S, stream=stream)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    rc = ctx.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {lyc.lyc_status_string(rc)}")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(0) as clk:
        evs[0].record(stream)
        for i in range(args.steps):
            step()
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
    rc = ctx.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status after timing: {lyc.lyc_status_string(rc)}")
    ms_total = evs[0].elapsed_time(evs[-1])
    ms_step = ms_total / args.steps
    kbytes = rule_kernel_bytes(role, tr, spec.n, spec.L, spec.Hq, spec.Hkv, spec.d, args.select_mode)
    peak, _ = measured_peaks()
    gbs = kbytes / (ms_step / 1e3) / 1e9
    params = {"ratio": {"theta": args.ratio}, "block": {"block": args.block}, "topp": {"p": args.p},
              "threshold": {"tau": args.tau}}[args.selection]
    line = {
        "metric": f"decode steps/s at 128K ctx, selection rule {args.selection}",
        "value": args.steps / (ms_total / 1e3), "unit": "steps/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "step_ms_distribution": {kk: round(v, 4) for kk, v in percentiles(
            [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]).items()},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/K/V, sinks + 256 planted heavy hitters per KV head)",
        "config": {"workload": spec.name, "L": spec.L, "B": spec.B, "Hq": spec.Hq, "Hkv": spec.Hkv,
                   "d": spec.d, "n": spec.n, "k_capacity": spec.k, "selection": args.selection,
                   **params, "retrieval_heads_per_layer": retrieval_heads(spec),
                   "select_mode": args.select_mode, "parallelism": "replicas x1",
                   "l2": "inputs larger than L2 (KV cache %.1f GB)" % (
                       2 * data["k"].numel() * data["k"].element_size() / 1e9)},
        "sets": {"rows_min": int(sizes.min()), "rows_mean": round(float(sizes.mean()), 1),
                 "rows_max": int(sizes.max())},
        "hbm": {"kernel_bytes_per_step": kbytes, "kernel_gbs": round(gbs, 1),
                "frac_of_measured_peak": round(gbs / peak, 4)},
        "clocks": clk.summary(),
    }
    ctx.close()
    print(json.dumps(line), flush=True)
    return 0


def run_noalloc(args):
    """lyc_sparse_attention_noalloc on one GPU: one layer of the Llama3-8B
    shapes with every query head sparse, each over its own set of k scattered
    rows (ascending, seeded), B*Hq sets per call.  The timed region is K calls
    on resident inputs; the rate counts the K/V rows the sets name."""
    import numpy as np
    import torch

    from hybrid_head_sparse_b200 import build as Bld
    from hybrid_head_sparse_b200 import lyc, workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    Bld.build()
    lyc.load()
    base = workload_spec(args)
    spec = base.with_(L=1, B=args.batch or 8, planted="none")
    B, Hq, Hkv, d, n, k = spec.B, spec.Hq, spec.Hkv, spec.d, spec.n, spec.k
    data = W.make_stack(spec, dev)
    rng = np.random.default_rng(spec.seed + 7)
    S = np.empty((B, Hq, k), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            S[b, h] = np.sort(rng.choice(n, size=k, replace=False))
    S = torch.from_numpy(S).to(dev)
    out = torch.empty((B, Hq, d), device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    kv = lyc.lyc_kv_cache(data["k"].data_ptr(), data["v"].data_ptr(), n, 0, *data["k"].stride()[1:4])
    stream = torch.cuda.current_stream(dev)

    def call():
        rc = lyc.lyc_sparse_attention_noalloc(data["q"].data_ptr(), kv, B, Hq, Hkv, d, S.data_ptr(),
                                              k, out.data_ptr(), status.data_ptr(),
                                              stream.cuda_stream)
        if rc != lyc.LYC_OK:
            raise RuntimeError(lyc.lyc_status_string(rc))

    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(0) as clk:
        evs[0].record(stream)
        for i in range(args.steps):
            call()
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
    ms_total = evs[0].elapsed_time(evs[-1])
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    ms_call = ms_total / args.steps
    kv_bytes = B * Hq * k * d * 2 * 2
    peak, peak_kind = measured_peaks()
    gbs = kv_bytes / (ms_call / 1e3) / 1e9
    line = {
        "metric": f"allocation-free sparse attention calls/s ({B * Hq} sets of {k} rows, {n // 1024}K ctx)",
        "value": args.steps / (ms_total / 1e3), "unit": "calls/s", "n_gpus": 1,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_call,
        "step_ms_distribution": {kk: round(v, 4) for kk, v in percentiles(per).items()},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/K/V; seeded scattered ascending sets)",
        "config": {"workload": f"llama3-8b-noalloc-b{B}-n{n}-k{k}", "B": B, "Hq": Hq, "Hkv": Hkv,
                   "d": d, "n": n, "k": k, "parallelism": "replicas x1",
                   "l2": "inputs larger than L2 (%.2f GB of K/V rows per call)" % (kv_bytes / 1e9)},
        "roofline": {"bound": "hbm", "kernel": "attn_mma_layer_kernel (gathered segments only) "
                                               "+ its work-list and combine launches",
                     "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4),
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                     "traffic": None, "algorithmic_bytes_per_launch": kv_bytes,
                     "avg_launch_ms": ms_call,
                     "note": "achieved = K+V bytes of the rows the sets name / CUDA-event time of "
                             "the whole call (work-list kernel, attention, combine, status copy)"},
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def traffic_record(args) -> int:
    """The traffic record line of an ncu capture of this command's attention
    launches (`ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum -k
    regex:attn_mma -s S -c N --csv`, N the step's attention launches, the
    combine launch of the last layer included): one whole step of the graph.
    Its DRAM bytes are summed and divided by the layers, the same unit as the
    roofline's algorithmic bytes per launch.  The source hash is taken from
    the files next to this script, so run it where the capture ran."""
    import csv
    spec = workload_spec(args)
    per = {}
    with open(args.traffic_from) as f:
        for r in csv.DictReader(line for line in f if line.startswith('"')):
            if "attn_mma" not in r["Kernel Name"]:
                continue
            scale = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}[r["Metric Unit"]]
            per.setdefault(int(r["ID"]), {})[r["Metric Name"]] = float(r["Metric Value"]) * scale
    launches = [v for _, v in sorted(per.items())
                if "dram__bytes_read.sum" in v and "dram__bytes_write.sum" in v]
    want = args.launches_per_step
    if want and len(launches) != want:
        print(f"expected {want} attention launches (one step), found {len(launches)}",
              file=sys.stderr)
        return 2
    rd = sum(v["dram__bytes_read.sum"] for v in launches)
    wr = sum(v["dram__bytes_write.sum"] for v in launches)
    rec = {"workload": spec.name, "select_mode": args.select_mode, "source_sha": attn_source_hash(),
           "bytes_per_launch": round((rd + wr) / spec.L), "step_read_bytes": round(rd),
           "step_write_bytes": round(wr), "launches": len(launches),
           "note": "one step's attention launches of the bench command at full size, summed, / L"}
    print("traffic-record: " + json.dumps(rec))
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.traffic_from:
        return traffic_record(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.serving:
        return run_serving(args)
    if args.correction:
        return run_correction(args)
    if args.noalloc:
        return run_noalloc(args)
    if args.shard:
        return run_sharded(args)
    if args.selection != "topk":
        return run_rule(args)
    return run_lyc(args)


if __name__ == "__main__":
    sys.exit(main())
