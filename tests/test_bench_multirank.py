"""bench.py's multi-rank logic on CPU: two gloo ranks (no GPU).

Each rank reports its own timings; the benchmark must take the max over
ranks (the slowest replica bounds the job) and report whole-job throughput
as world_size x per-rank units / that time.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    # rank r "took" 100 + 50 r ms for 10 steps and 40 + 5 r ms for its end-to-end leg
    vals = bench.max_over_ranks([100.0 + 50 * rank, 40.0 + 5 * rank], world, "cpu")
    out[rank] = (vals, bench.whole_job_rate(world, 10, vals[0]))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        vals, rate = res[rank]
        assert vals == [150.0, 45.0]                      # max over ranks, element-wise
        assert rate == pytest.approx(2 * 10 / 0.150)      # both replicas' frames / slowest time


def test_single_rank_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0], 1, "cpu") == [3.0, 4.0]
    assert bench.whole_job_rate(1, 925, 20000.0) == pytest.approx(46.25)


def test_timed_window_is_centred_in_the_stream():
    """The timed frames of the 24-block stream sit in the middle of its 1000
    frames (after the 72-frame steady-state pre-fill and the warm-up); the
    defaults time frames 75..999; other workloads keep their pre-fill."""
    sys.path.insert(0, ROOT)
    import bench
    for warmup, steps in ((3, 925), (5, 20), (3, 2), (3, 200), (5, 1000)):
        p = bench.prefill_frames("vitl_stream24", warmup, steps)
        first, last = p + warmup, p + warmup + steps - 1
        assert p >= bench.PREFILL["vitl_stream24"]
        if steps <= 925:
            assert last <= 999
            before = first - (bench.PREFILL["vitl_stream24"] + warmup)
            assert abs(before - (999 - last)) <= 1
    assert bench.prefill_frames("vitl_stream24", 3, 925) == 72
    assert bench.prefill_frames("vitl_step", 5, 20) == bench.PREFILL["vitl_step"]


def test_secondary_workloads_use_defined_shapes():
    sys.path.insert(0, ROOT)
    import bench
    from streaming_video_transformer_b200.inputs import WORKLOADS
    assert set(bench.PREFILL) <= set(WORKLOADS)
    for name, base in bench.SECONDARY.items():
        assert base in WORKLOADS, name
    # the rows of the scope table each have a measurement line
    assert {"first_pass8", "skip_append", "nocross_step", "tiny_stream"} <= set(bench.SECONDARY)
