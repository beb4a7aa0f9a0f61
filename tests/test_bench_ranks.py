"""Multi-rank logic of bench.py on CPU: two gloo ranks stand in for two GPUs.

The step has no exchange between replicas, so the only cross-rank work is the
timing reduction: every rank times its own K steps, the job time is the
slowest rank's, and the whole-job value counts every rank's steps.
"""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms, steps, q):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        slow = bench.max_over_ranks(ms[rank])
        q.put((rank, slow, bench.job_steps_per_s(world, steps, slow)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ms = [12.5, 20.0]
    steps = 10
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, ms, steps, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slow, value in got:
        assert slow == 20.0                       # the slowest rank's time, on every rank
        assert value == pytest.approx(2 * steps / 0.020)  # all ranks' steps / that time


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.job_steps_per_s(1, 50, 100.0) == pytest.approx(500.0)


def test_reference_arm_only_rank0_works(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = bench.parse_args(["--impl", "reference", "--gpus", "2"])
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""          # ranks other than 0 print nothing


def test_percentiles():
    import bench
    p = bench.percentiles([5.0, 1.0, 3.0, 2.0, 4.0])
    assert (p["p10"], p["p50"], p["p90"]) == (1.0, 3.0, 5.0)


def test_traffic_record_lookup(tmp_path, monkeypatch):
    """The bench takes DRAM traffic from a committed ncu summary only when the
    summary was taken on the current attention-kernel source, workload and
    selection mode."""
    import bench
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "attn_mma_layer_kernel_some-workload.md").write_text(
        "summary\n"
        'traffic-record: {"workload": "w1", "source_sha": "abc", "bytes_per_launch": 123}\n')
    (prof / "attn_mma_layer_kernel_other.md").write_text(
        'traffic-record: {"workload": "w1", "select_mode": "kvgroup_mean", "source_sha": "abc", '
        '"bytes_per_launch": 456}\n')
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "attn_source_hash", lambda: "abc")
    # a record without a selection mode was taken per head
    assert bench.profiled_traffic("w1", "per_qhead") == 123
    assert bench.profiled_traffic("w1", "kvgroup_mean") == 456
    assert bench.profiled_traffic("w2", "per_qhead") is None
    monkeypatch.setattr(bench, "attn_source_hash", lambda: "def")
    assert bench.profiled_traffic("w1", "per_qhead") is None
    assert bench.profiled_traffic("w1", "kvgroup_mean") is None


def test_traffic_record_from_capture(tmp_path, monkeypatch, capsys):
    """--traffic-from sums one step's attention launches of an ncu capture
    (read + write, any byte unit), divides by the layers and stamps the
    record with the source hash; a capture of the wrong length is refused."""
    import json

    import bench
    head = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream",'
            '"Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit",'
            '"Metric Value"\n')
    rows = []
    vals = [(100.0, "Mbyte", 1.5, "Mbyte"), (200.0, "Mbyte", 2.5, "Mbyte"), (1024.0, "byte", 0.0, "byte")]
    for i, (r, ru, w, wu) in enumerate(vals):
        k = '"void attn_mma_layer_kernel<128, 6, 8, 6, 0, 0>(AttnMmaParams)"'
        base = f'"{i}","1","python","h",{k},"1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","m",'
        rows.append(base + f'"dram__bytes_read.sum","{ru}","{r}"\n')
        rows.append(base + f'"dram__bytes_write.sum","{wu}","{w}"\n')
    csvf = tmp_path / "t.csv"
    csvf.write_text("==PROF== noise\n" + head + "".join(rows))
    monkeypatch.setattr(bench, "attn_source_hash", lambda: "feed")
    assert bench.main(["--traffic-from", str(csvf), "--layers", "2", "--launches-per-step", "3"]) == 0
    line = capsys.readouterr().out.strip()
    assert line.startswith("traffic-record: ")
    rec = json.loads(line.split(":", 1)[1])
    assert rec["source_sha"] == "feed" and rec["launches"] == 3
    assert rec["workload"] == "llama3-8b-attn-stack-n131072-k4096-L2-r2"
    assert rec["bytes_per_launch"] == round((300e6 + 4e6 + 1024) / 2)
    assert bench.main(["--traffic-from", str(csvf), "--layers", "3", "--launches-per-step", "4"]) == 2


def test_reference_arm_times_whole_steps_on_the_library_arms_config(capsys):
    """The oracle arm runs whole L-layer steps of the chosen workload and
    reports the same config as the library arm (a small override of the
    Llama3-8B shape, drawn on the host)."""
    import json

    import bench
    args = bench.parse_args(["--impl", "reference", "--n", "256", "--k", "32", "--layers", "2",
                             "--steps", "2", "--warmup", "0"])
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    spec = bench.workload_spec(args)
    assert line["impl"] == "reference"
    assert line["config"] == bench.line_config(spec, args, 1, bench.kv_cache_bytes(spec))
    assert line["config"]["workload"] == "llama3-8b-attn-stack-n256-k32-L2-r2"
    assert line["steps"] == 2 and line["ms_per_step"] > 0
    assert line["cpu_baseline"]["sample"].startswith("oracle (fp64 C, OpenMP over heads) on 2 whole")


def test_workload_names():
    import bench
    spec = bench.workload_spec(bench.parse_args([]))
    assert spec.name == "llama3-8b-attn-stack-n131072-k4096-r2"
    spec = bench.workload_spec(bench.parse_args(["--workload", "qwen3-8b-64k-b4"]))
    assert spec.name == "qwen3-8b-attn-stack-b4-n65536-k2048-r3" and spec.L == 36 and spec.B == 4
    spec = bench.workload_spec(bench.parse_args(["--retrieval-heads", "-1"]))
    assert spec.name.endswith("-dense") and spec.roles == "all"
    spec = bench.workload_spec(bench.parse_args(["--workload", "llama3-8b-32k", "--retrieval-heads", "8"]))
    assert spec.name == "llama3-8b-attn-stack-n32768-k4096-r8" and spec.retrieval_per_layer == 8


def test_union_ms():
    import bench
    assert bench.union_ms([]) == 0
    assert bench.union_ms([(0, 1_000_000), (500_000, 2_000_000), (3_000_000, 4_000_000)]) == pytest.approx(3.0)
