"""The multi-rank host logic of bench.py, on CPU with two gloo ranks.

The layer has no cross-GPU exchange, so N GPUs run N replicas (weak
scaling); what the ranks share is the timing: the slowest rank's span is the
job's, every rank takes part in each reduction in the same order, and only
rank 0 prints.  These run as two spawned processes over gloo on 127.0.0.1."""
import contextlib
import io
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        from tile_sparse_video_b200.inputs import TINY, make_inputs
        res = {}
        # rank r's "span" is 10 + 5 r ms: the job's span is the largest
        res["span_max"] = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        # a second reduction in the same order on every rank
        res["e2e_max"] = bench.max_over_ranks(100.0 - rank, world, "cpu")
        res["ms_layer"] = bench.job_ms_per_layer(res["span_max"], 4, world)
        w = bench.rank_workload(TINY, rank)
        res["seed"] = w.seed_base
        res["q_sum"] = float(make_inputs(w)["q"].float().sum())
        # the reference arm: rank 0 alone prints its one line
        class A:
            steps, warmup = 1, 3
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            if rank != 0:
                bench.run_reference(A, rank)
        res["ref_stdout"] = buf.getvalue()
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    out = tmp_path_factory.mktemp("ranks")
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(out)), nprocs=world,
                       join=True, start_method="spawn")
    return [json.load(open(out / f"rank{r}.json")) for r in range(world)]


def test_max_over_ranks_is_the_slowest_rank(two_ranks):
    for r in two_ranks:
        assert r["span_max"] == 15.0
        assert r["e2e_max"] == 100.0


def test_job_time_divides_by_all_layers(two_ranks):
    # 2 ranks x 4 layers each in a 15 ms span
    assert all(r["ms_layer"] == 15.0 / 8 for r in two_ranks)


def test_replicas_get_their_own_batch(two_ranks):
    from tile_sparse_video_b200.inputs import TINY
    assert two_ranks[0]["seed"] == TINY.seed_base
    assert two_ranks[1]["seed"] != TINY.seed_base
    assert two_ranks[0]["q_sum"] != two_ranks[1]["q_sum"]


def test_reference_arm_prints_on_rank0_only(two_ranks):
    assert two_ranks[1]["ref_stdout"] == ""


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.job_ms_per_layer(30.0, 10, 1) == 3.0
