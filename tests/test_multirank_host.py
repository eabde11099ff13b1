"""The multi-rank host logic of bench.py on CPU: two gloo ranks, no GPU.

The path shards by independent (batch, head) work with no data-path collective; the
only cross-rank steps are the barrier and the max-over-ranks timing that turns the
per-rank spans into one whole-job number.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, spans, out_q):
    import datetime
    import importlib.util

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    dist.barrier()
    span, value = bench.weak_scaling_value(spans[rank], 2.0e12, 10, dist, device="cpu")
    out_q.put((rank, span, value))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("spans", [(100.0, 250.0), (300.0, 300.0)])
def test_weak_scaling_takes_the_slowest_rank(spans):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, spans, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = max(spans)
    for _, span, value in res:
        assert span == slowest                          # every rank reports the max
        assert abs(value - 2 * 2.0e12 * 10 / (slowest / 1e3) / 1e12) < 1e-9


def test_single_process_needs_no_group():
    import importlib.util
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_mod1", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    span, value = bench.weak_scaling_value(50.0, 1.0e12, 5, None)
    assert span == 50.0 and abs(value - 1.0e12 * 5 / 0.05 / 1e12) < 1e-9
