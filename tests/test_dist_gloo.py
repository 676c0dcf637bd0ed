"""World-size-2 checks of the multi-rank host logic on CPU (gloo): the timed
region's barrier, max-over-ranks timing, whole-job aggregation and the layer
partition that the benchmark uses under torchrun."""

import os
import socket

import pytest
import torch.multiprocessing as mp

from h2o_kv_cache_attn_b200 import dist as hd


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    ws, r, _ = hd.init("gloo", timeout_s=60)
    assert (ws, r) == (world, rank)
    hd.barrier()
    # rank r "processed" 1000 * (r + 1) tokens in 10 * (r + 1) ms
    tps, ms = hd.job_throughput(1000.0 * (rank + 1), 10.0 * (rank + 1))
    layers = hd.layers_for_rank(36, world, rank)
    out.put((rank, tps, ms, layers))
    hd.barrier()
    hd.shutdown()


def test_two_ranks_timing_and_partition():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, tps, ms, layers in res:
        assert ms == 20.0                      # the slowest rank's time
        assert tps == pytest.approx(3000.0 / 0.020)  # all tokens over that time
    all_layers = sorted(l for _, _, _, layers in res for l in layers)
    assert all_layers == list(range(36))


def test_single_process_defaults():
    assert hd.layers_for_rank(5, 1, 0) == [0, 1, 2, 3, 4]
    assert hd.max_over_ranks(3.5) == 3.5
    tps, ms = hd.job_throughput(100.0, 50.0)
    assert ms == 50.0 and tps == pytest.approx(2000.0)
