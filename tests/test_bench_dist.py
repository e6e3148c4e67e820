"""CPU (gloo) tests of the multi-rank logic of bench.py: the max-over-ranks timing, the whole-job
throughput, and that the reference arm runs on rank 0 only."""
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        t = bench.max_over_ranks(10.0 + 5.0 * rank, ws)  # each rank's elapsed ms
        bench.barrier(ws)
        q.put((rank, t, bench.job_throughput(1000, ws, t)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2])
def test_max_over_ranks_and_throughput(ws):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(ws))
    slowest = 10.0 + 5.0 * (ws - 1)
    for rank, t, thr in res:
        assert t == slowest  # every rank sees the max
        assert abs(thr - ws * 1000 / (slowest * 1e-3)) < 1e-6


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_recorded_traffic_tracks_the_timed_kernels_sources(tmp_path, monkeypatch):
    """The committed DRAM figure is reported only while the timed kernels' own source files are unchanged:
    a change to another kernel's file keeps it, a change to one of them drops it to None."""
    import shutil
    sys.path.insert(0, ROOT)
    import bench
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(ROOT, "gated_delta_rule_105_b200", "csrc"), root / "gated_delta_rule_105_b200" / "csrc")
    (root / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    kernel = "gdn_tc_wy_kernel+gdn_tc_fwd_kernel"
    line = (f"kernel={kernel} workload=w sources={bench.kernel_source_hash(kernel)} bytes_per_launch=123 "
            f"source=x\n")
    (root / "profiles" / "dram_traffic.txt").write_text(line)
    assert bench.recorded_traffic(kernel, "w") == 123.0
    assert bench.recorded_traffic(kernel, "other") is None
    csrc = root / "gated_delta_rule_105_b200" / "csrc"
    (csrc / "gdn_simt.cuh").write_text((csrc / "gdn_simt.cuh").read_text() + "\n// edit\n")
    assert bench.recorded_traffic(kernel, "w") == 123.0  # not one of this kernel's files
    (csrc / "gdn_tc.cuh").write_text((csrc / "gdn_tc.cuh").read_text() + "\n// edit\n")
    assert bench.recorded_traffic(kernel, "w") is None

