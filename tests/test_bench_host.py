"""Host-side logic of bench.py that needs no GPU: the multi-process plumbing
(two gloo ranks on the CPU: barrier and the max of the ranks' times), and the
reference arm (the CPU oracle), including its rank-0-only rule under a
multi-process launch."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench

    d = bench.Dist(world, backend="gloo")
    d.barrier()
    # every rank reports its own time; the job's time is the slowest rank's
    m = d.max(10.0 + rank)
    d.barrier()
    d.close()
    q.put((rank, m))


def test_dist_two_gloo_ranks_take_the_max():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 11.0), (1, 11.0)]


def test_dist_rejects_a_gpu_count_without_the_processes(monkeypatch):
    import bench

    monkeypatch.delenv("WORLD_SIZE", raising=False)
    with pytest.raises(SystemExit):
        bench.Dist(2)


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        env.pop(k, None)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True, timeout=600)


def test_reference_arm_prints_the_contract_line():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "3", "--reference-seconds", "0.2"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    import bench

    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is True and line["value"] > 0
    assert line["steps"] == 1 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_zero_only():
    r = _run_bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--reference-seconds", "0.2"],
                   {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "2"])
    assert r.returncode != 0


def test_traffic_comes_only_from_a_capture_of_the_current_kernel_source(monkeypatch):
    """roofline.traffic is the committed ncu figure while the capture's
    source fingerprint equals the kernel sources' one, and null otherwise
    (the figure no longer describes the kernel that runs)."""
    import re

    sys.path.insert(0, ROOT)
    import bench

    text = open(os.path.join(ROOT, "profiles", "gemv_q4_traffic.md")).read()
    sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text).group(1)
    per = int(re.search(r"dram_bytes_per_full_launch:\s*([0-9]+)", text).group(1))
    assert per >= 13_745_029_120  # DRAM traffic cannot be below the weight bytes the launch streams
    assert re.fullmatch(r"[0-9a-f]{16}", bench.kernel_source_sha())
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: sha)
    assert bench.profiled_traffic() == per
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "f" * 16 if sha != "f" * 16 else "0" * 16)
    assert bench.profiled_traffic() is None


def test_oracle_timing_per_configuration_on_one_core():
    """The CPU baseline's per-configuration oracle timing, as the bench runs
    it for its one-core figures: a fresh process whose OpenMP runtime has one
    thread, every configuration (1-4 and the decode stream) with its rate,
    the implied time for the whole configuration and the sample it timed."""
    r = _run_bench(["--oracle-configs", "--cpu-seconds", "0.1"], {"OMP_NUM_THREADS": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["threads"] == 1
    names = {"q4_4096x4096_M1", "layer_q4_M1", "layer_q4_M4", "head.mapped_q8_65536x5120_M1",
             "head.full_q8_248320x5120_M1", "decode_stream_M1"}
    assert names <= set(out)
    for name in names:
        c = out[name]
        assert c["GBps"] > 0 and c["us"] > 0 and c["seconds"] > 0, name
        assert c["sample"] == "whole" or " of " in c["sample"], name
