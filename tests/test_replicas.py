"""Host logic of `bench.py --gpus N` (replicas, weak scaling), run as world-size-2 gloo ranks on CPU.

The scan has no exchange step: every rank runs its own copy of the workload, the step time is the
max over ranks, and the whole-job value counts every rank's tokens.
"""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, ms_by_rank, out):
    import torch.distributed as td
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    td.init_process_group("gloo", rank=rank, world_size=world)
    try:
        slowest = bench.max_over_ranks(ms_by_rank[rank], td, "cpu")
        out.put((rank, slowest, bench.replica_throughput(1000, slowest, world)))
    finally:
        td.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_replicas_take_the_slowest_rank_and_count_every_rank():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    ms_by_rank = [2.0, 5.0]
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, ms_by_rank, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in procs)
    for rank, slowest, value in res:
        assert slowest == 5.0                         # both ranks see the max
        assert value == pytest.approx(2 * 1000 / 5e-3)  # 2 replicas x 1000 tokens / slowest step


def test_single_process_is_its_own_max():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.replica_throughput(4096, 2.0, 1) == pytest.approx(4096 / 2e-3)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
