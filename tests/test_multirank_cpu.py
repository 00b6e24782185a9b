"""The benchmark's multi-rank host logic on CPU: two gloo ranks on 127.0.0.1.

With N GPUs bench.py runs one independent layer replica per rank (weak
scaling, no collective on the data path) and reduces only its timings: each
time is the maximum over ranks, and the whole-job throughput counts every
rank's tokens over the slowest rank's time."""
import importlib.util
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench = _bench()
        # rank r's timed region took (r + 1) seconds, its kernel 10 - r microseconds
        secs, kern = bench.max_over_ranks([rank + 1.0, 10.0 - rank], "cpu")
        value = bench.job_tokens_per_s(world, 100, 4, secs)
        out[rank] = (secs, kern, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_with_two_gloo_ranks():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank in range(world):
        secs, kern, value = res[rank]
        assert secs == 2.0 and kern == 10.0          # the slowest rank's time, on every rank
        assert value == world * 100 * 4 / 2.0        # all ranks' tokens over that time


def test_single_process_reduction_is_the_identity():
    bench = _bench()
    assert bench.max_over_ranks([1.5, 2.5], "cpu") == [1.5, 2.5]
    assert bench.job_tokens_per_s(1, 10, 8, 2.0) == 40.0
