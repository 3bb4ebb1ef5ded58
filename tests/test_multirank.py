"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

bench.py runs N independent replicas of the layer (one per GPU); the only
cross-rank steps are the max-over-ranks reductions of the timed totals and
of the device status, and the final barrier.  These run here with the gloo
backend (no GPU).
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import os, sys, datetime
import torch.distributed as dist
sys.path.insert(0, sys.argv[1])
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
# rank r timed 10 + 5r ms in total and saw device status r (nonzero on rank 1)
mx = bench.max_over_ranks(10.0 + 5.0 * rank, world)
st = bench.max_over_ranks(rank, world)
v = bench.replica_throughput(world, 4, 20480, mx)
dist.barrier()
dist.destroy_process_group()
print(f"rank={rank} max={mx} status={st} value={v:.6f}", flush=True)
'''


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.timeout(180)
def test_two_gloo_ranks_take_the_slowest_rank():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD, ROOT], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=150) for p in procs]
    for p, (out, err) in zip(procs, outs):
        assert p.returncode == 0, err[-2000:]
    expect_value = 2 * 4 * 20480 / (15.0e-3)
    for rank, (out, _) in enumerate(outs):
        line = out.strip().splitlines()[-1]
        assert line.startswith(f"rank={rank} max=15.0 status=1.0 value=")
        assert abs(float(line.split("value=")[1]) - expect_value) < 1e-6 * expect_value


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3, 1) == 3.0
    assert bench.replica_throughput(1, 2, 100, 4.0) == 2 * 100 / 4e-3


@pytest.mark.timeout(300)
def test_reference_arm_other_ranks_exit_without_work():
    # rank 1 of a two-rank launch of the reference arm returns at once
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny"],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=280)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
