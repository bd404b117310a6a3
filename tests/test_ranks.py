"""Multi-rank plumbing of the benchmark on the CPU: two gloo ranks.

Every rank runs its own batch (weak scaling, no collective on the data path);
the only collectives are the barrier around the timed region and the
reductions of its time (maximum) and of the units processed (sum).
"""
import json
import os
import socket
import subprocess
import sys
import time

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int) -> None:
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    _env(rank, world, port)
    from speculative_verification_isd_b200 import inputs as I
    from speculative_verification_isd_b200 import ranks as RK
    R = RK.setup(use_cuda=False, timeout_s=30)
    t_ms = 10.0 + 5.0 * rank            # this rank's timed region
    steps = 100 + rank                  # steps this rank ran
    R.barrier()
    res = dict(rank=R.rank, world=R.world, t_max=R.max(t_ms), steps_sum=R.sum(steps),
               rate=RK.job_throughput(steps, R, R.max(t_ms)))
    inp = I.make_step_inputs(I.CONFIGS["ragged_small"], seed=RK.rank_seed(0, rank))
    res["kv_len"] = inp["kv_len"].tolist()
    R.barrier()
    R.close()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks_reduce_and_run_independent_batches(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{k}.json")) for k in range(2)]
    for k in range(2):
        assert r[k]["rank"] == k and r[k]["world"] == 2
        assert r[k]["t_max"] == 15.0            # the job ends with its slowest rank
        assert r[k]["steps_sum"] == 201.0       # units of the whole job
        assert r[k]["rate"] == pytest.approx(201.0 / 0.015)
    assert r[0]["kv_len"] != r[1]["kv_len"]     # independent batches per rank


def _leaver(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    _env(rank, world, port)
    from speculative_verification_isd_b200 import ranks as RK
    R = RK.setup(use_cuda=False, timeout_s=5)
    R.barrier()
    if rank == 1:
        return                              # leaves between steps, no collective in flight
    t0 = time.time()
    err = None
    try:
        R.max(1.0)
    except Exception as e:                  # the missing peer ends the collective
        err = type(e).__name__
    with open(os.path.join(out_dir, "rank0.json"), "w") as f:
        json.dump(dict(err=err, seconds=time.time() - t0), f)


def test_a_rank_that_leaves_ends_the_next_collective_with_an_error(tmp_path):
    port = _free_port()
    ctx = mp.start_processes(_leaver, args=(2, port, str(tmp_path)), nprocs=2, join=False,
                             start_method="spawn")
    deadline = time.time() + 120
    while not ctx.join(timeout=5):
        assert time.time() < deadline, "ranks did not finish"
    res = json.load(open(tmp_path / "rank0.json"))
    assert res["err"] is not None
    assert res["seconds"] < 60


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""
