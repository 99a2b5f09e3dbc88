"""Host-side logic of bench.py without a GPU: the multi-rank aggregation
(world size 2 over gloo on CPU), the whole-job throughput formula and the
reference arm's rank handling."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms_per_rank, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        m = bench.reduce_max(ms_per_rank[rank], world)
        out[rank] = (m, bench.whole_job_gbs(1_000_000, world, m))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        ms = [0.25, 0.75]
        mp.start_processes(_rank_main, args=(2, port, ms, out), nprocs=2, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 0.75
    # both ranks' replicas (2 x 1 MB) over the slowest rank's time
    assert res[0][1] == pytest.approx(2 * 1_000_000 / 0.75e-3 / 1e9)


def test_single_rank_is_identity():
    assert bench.reduce_max(1.5, 1) == 1.5
    assert bench.whole_job_gbs(5_000_000_000, 1, 1000.0) == pytest.approx(5.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_json_line():
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_ncu_traffic_only_for_captured_sources(monkeypatch):
    import bench
    traffic = dict(bench.NCU_TRAFFIC)
    monkeypatch.setattr(bench, "NCU_TRAFFIC", dict(traffic, sources_sha256=bench.kernel_sources_sha256()))
    bwd = traffic["backward"]
    assert bench.ncu_traffic("backward") == bwd["read"] + bwd["write"]
    assert bench.ncu_dram("backward") == bwd
    monkeypatch.setattr(bench, "NCU_TRAFFIC", dict(traffic, sources_sha256="0" * 64))
    assert bench.ncu_traffic("backward") is None
    assert bench.ncu_dram("backward") is None
