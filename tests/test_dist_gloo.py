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


class _WallClock:
    """Host stand-in for the device clock of the stack driver."""

    def mark(self):
        import time
        return time.perf_counter()

    def sync(self):
        pass

    @staticmethod
    def ms(a, b):
        return (b - a) * 1e3


def _stack_worker(rank, world, port, out):
    """Each rank runs its share of a 36-layer stack through the stack driver with a
    CPU stand-in step (a tiny matrix product per layer and chunk)."""
    import numpy as np

    from h2o_kv_cache_attn_b200.stack import run_stack

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    ws, r, _ = hd.init("gloo", timeout_s=60)
    layers = hd.layers_for_rank(36, ws, r)
    seen = {"evict": [], "attend": [], "finish": 0}
    state = {L: np.zeros(4) for L in layers}

    def make_inputs(L, c):
        return np.full(4, L * 100 + c, dtype=np.float64)

    def evict(c, inputs):
        assert sorted(inputs) == layers  # one batched call over this rank's layers
        seen["evict"].append(c)

    def attend(L, c, x):
        state[L] += x @ np.eye(4)
        seen["attend"].append((L, c))

    def finish():
        seen["finish"] += 1

    n_chunks = 5
    times = run_stack(layers, n_chunks, lambda c: 128, make_inputs, evict, attend, finish, _WallClock())
    ms = hd.max_over_ranks(times.total_ms)
    layer_sum = hd.sum_over_ranks(float(len(layers)))
    out.put((r, layers, seen["evict"], sorted(seen["attend"]), seen["finish"], len(times.evict_ms),
             times.total_ms <= ms, layer_sum, {L: float(state[L][0]) for L in layers}))
    hd.barrier()
    hd.shutdown()


def test_two_ranks_run_the_stack_driver():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_stack_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    all_layers = []
    for rank, layers, ev, att, fin, n_times, slower_or_equal, layer_sum, state in res:
        assert layers == list(range(rank, 36, world))
        assert ev == list(range(5))                       # one eviction call per chunk
        assert att == sorted((L, c) for L in layers for c in range(5))
        assert fin == 1 and n_times == 5 and slower_or_equal
        assert layer_sum == 36.0
        for L, v in state.items():                        # each layer saw its own chunks only
            assert v == sum(L * 100 + c for c in range(5))
        all_layers += layers
    assert sorted(all_layers) == list(range(36))
