"""The multi-GPU bench path is replicas only: each rank times its own replica and
rank 0 reports the max over ranks.  This runs that plumbing with two gloo ranks on
CPU (no GPU), including a rank that is slower than the other."""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import os, sys, time
sys.path.insert(0, %r)
import bench
dist = bench.init_dist("gloo")
rank, _, world = bench.dist_env()
assert world == 2
bench.barrier(dist)
t0 = time.perf_counter()
time.sleep(0.05 * (rank + 1))
ms = (time.perf_counter() - t0) * 1e3
m = bench.max_over_ranks(ms, dist)
bench.barrier(dist)
print(f"rank {rank} local {ms:.1f} max {m:.1f}", flush=True)
assert m >= ms - 1e-9
if rank == 1:
    assert abs(m - ms) < 1e-9
dist.destroy_process_group()
"""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_two_rank_max_over_ranks(tmp_path):
    script = tmp_path / "dist_probe.py"
    script.write_text(SCRIPT % ROOT)
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = []
    for p in procs:
        try:
            out, _ = p.communicate(timeout=120)
        except subprocess.TimeoutExpired:
            p.kill()
            pytest.fail("gloo ranks did not finish")
        outs.append(out)
        assert p.returncode == 0, out
    m0 = float(outs[0].split("max ")[1])
    m1 = float(outs[1].split("max ")[1])
    assert m0 == m1 and m0 >= 100.0


def test_algorithmic_bytes_headline():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.algorithmic_bytes(64, 128, 8192, 128) == 630_259_968
    assert bench.algorithmic_flops(64, 128, 8192) == 146_028_888_064


def test_reference_arm_two_ranks_rank0_reports():
    # Under torchrun with N > 1 the reference arm (the fp64 oracle) runs on rank 0 only:
    # rank 0 prints one JSON line, every other rank exits 0 without output.
    import json
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(_free_port()))
        procs.append(subprocess.Popen([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                                       "--gpus", "2", "--steps", "1", "--warmup", "3"], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True, cwd=ROOT))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=300)
        except subprocess.TimeoutExpired:
            p.kill()
            pytest.fail("reference arm did not finish")
        assert p.returncode == 0, err
        outs.append(out)
    lines0 = [l for l in outs[0].splitlines() if l.startswith("{")]
    assert len(lines0) == 1
    rec = json.loads(lines0[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
    # both arms describe the workload with the same config object
    sys.path.insert(0, ROOT)
    import bench
    assert rec["config"] == bench.workload_config(2)
    assert not [l for l in outs[1].splitlines() if l.startswith("{")]
