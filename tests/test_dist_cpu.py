"""Multi-process (gloo, CPU) checks of the benchmark's data-parallel plumbing: every rank
draws its own token batch, the step time is the maximum over ranks, and the whole-job
value counts the work of every rank.  The path itself has no exchange step, so the
only collective is the timing reduction."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

pytestmark = pytest.mark.cpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    from ternary_weight_bit_absmean_b200 import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 20.0][rank]
        mx = bench.max_over_ranks(local_ms)
        X = synth.activations(4, 64, seed=bench.rank_seed(2, 4, rank))
        xs = [torch.zeros_like(X.float()) for _ in range(world)]
        dist.all_gather(xs, X.float())
        out[rank] = (mx, bench.whole_job_tops(1e12, 10, world, mx), bool(torch.equal(xs[0], xs[1])))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_aggregation():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        mx, tops, same_tokens = res[rank]
        assert mx == 20.0                      # the slowest rank's time
        assert tops == pytest.approx(1e12 * 10 * 2 / 20e-3 / 1e12)
        assert not same_tokens                 # ranks hold different token batches


def test_single_process_aggregation_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_tops(2e12, 5, 1, 1000.0) == pytest.approx(10.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
