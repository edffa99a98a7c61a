"""bench.py's multi-rank host logic on CPU: two gloo ranks, as torchrun would start them.
The job time is the maximum over ranks, throughput counts every rank's tokens, and the ranks
draw disjoint token streams."""
import importlib.util
import os
import socket

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        b = _bench()
        local = 10.0 + 5.0 * rank  # rank 1 is the slower one
        job = b.job_time_ms(local, world, "cpu")
        out[rank] = (job, b.job_throughput(world, 16, 30, job))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] == res[1][1] == world * 16 * 30 / 0.015


def test_ranks_draw_disjoint_token_streams():
    b = _bench()
    streams = [{b.token_stream(r, i) for i in range(32)} for r in range(8)]
    for r in range(8):
        for q in range(r):
            assert not streams[r] & streams[q]


def test_single_rank_needs_no_process_group():
    b = _bench()
    assert b.job_time_ms(12.5, 1, "cpu") == 12.5
