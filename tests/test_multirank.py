"""The benchmark's multi-rank logic on CPU (gloo, two ranks): each rank verifies its own batch,
there is no collective on the data path, and the job's time is the slowest rank's."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 100.0 + 25.0 * rank  # rank 1 is the slower one
        ms = bench.max_over_ranks(my_ms, world, "cpu")
        rate = bench.whole_job_rate(world, 8, 3, 10, ms)
        out[rank] = (ms, rate)
    finally:
        dist.destroy_process_group()


def test_time_is_the_slowest_rank_and_rate_counts_every_rank():
    world = 2
    out = mp.get_context("spawn").Manager().dict()  # no fork after threads have started
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        ms, rate = out[rank]
        assert ms == 125.0
        assert rate == pytest.approx(world * 8 * 3 * 10 / 0.125)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.whole_job_rate(1, 8, 3, 10, 1000.0) == pytest.approx(240.0)


def test_ranks_verify_distinct_batches():
    import synthetic as S
    seeds = [bench.rank_seed(r) for r in range(4)]
    assert len(set(seeds)) == 4
    w = [S.Workload("g", 2, 64, 2, 4, 1, [S.AttnLayer(64)], 64, 1024, seed=sd) for sd in seeds[:2]]
    q0 = S.make_step_qkv(w[0], 0, 3)["q"]
    q1 = S.make_step_qkv(w[1], 0, 3)["q"]
    assert not torch.equal(q0, q1)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    """Under torchrun the oracle arm prints from rank 0; the other ranks exit without work."""
    import sys
    saved = sys.argv
    sys.argv = ["bench.py", "--impl", "reference"]
    try:
        args = bench.parse()
    finally:
        sys.argv = saved
    assert bench.run_reference(args, 1, 2) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_covers_the_drafter_layer_mode(capsys):
    """The oracle arm of the drafter-layer workload: one step of one sequence through the
    drafter's dense layers, printed as one JSON line naming that workload."""
    import json
    import sys
    saved = sys.argv
    sys.argv = ["bench.py", "--impl", "reference", "--drafter-layers", "--steps", "1",
                "--warmup", "0"]
    try:
        args = bench.parse()
    finally:
        sys.argv = saved
    bench.run_reference(args, 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"]["workload"] == "spec_step_b8_ctx16384_k2_drafter_layers"
