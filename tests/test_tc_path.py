"""Tensor-core path (head_dim 128, bf16 / int8 / int4 cache): parity with the oracle on every
chunk of small workloads whose shapes exercise the tiling -- several 128-slot
and 128-row tiles, ragged slot and row tails, chunks shorter than a row tile,
one-token chunks, a chunk as large as the cache, MHA and GQA, batch > 1."""

import pytest

from h2o_kv_cache_attn_b200.configs import Workload

from .harness import run_and_check

pytestmark = pytest.mark.gpu


def tc(name, **kw):
    base = dict(name=name, B=1, Hq=8, Hk=2, d=128, capacity=2048, seq_len=4096, chunk=512,
                q_dtype="bf16", kv_dtype="bf16", heavy_hitters=True, seed=11)
    base.update(kw)
    return Workload(**base)


CASES = [
    tc("tc_q4_c2048_s512"),
    tc("tc_b2_q4_c1000_s300", B=2, Hq=4, Hk=1, capacity=1000, chunk=300, seq_len=2100),
    tc("tc_s1", Hq=4, Hk=2, capacity=130, chunk=1, seq_len=150),
    tc("tc_s_eq_capacity", capacity=256, chunk=256, seq_len=768),
    tc("tc_mha_c384_s128", Hq=2, Hk=2, capacity=384, chunk=128, seq_len=1024),
    tc("tc_s100_c700", Hq=4, Hk=1, capacity=700, chunk=100, seq_len=1200, heavy_hitters=False),
    tc("tc_mha_s300_odd_tiles", Hq=2, Hk=2, capacity=640, chunk=300, seq_len=1500),
]


# int8 / int4 caches: the loader warps dequantize while they load (exact integer
# keys with the key scale on the logits, values multiplied by their scale)
QCASES = [
    tc("tc_i8_q4_c2048_s512", kv_dtype="i8"),
    tc("tc_i4_q4_c2048_s512", kv_dtype="i4", seed=12),
    tc("tc_i4_b2_q4_c1000_s300", kv_dtype="i4", B=2, Hq=4, Hk=1, capacity=1000, chunk=300,
       seq_len=2100),
    tc("tc_i8_s1", kv_dtype="i8", Hq=4, Hk=2, capacity=130, chunk=1, seq_len=150),
    tc("tc_i8_s_eq_capacity", kv_dtype="i8", capacity=256, chunk=256, seq_len=768),
    tc("tc_i4_mha_s300_odd_tiles", kv_dtype="i4", Hq=2, Hk=2, capacity=640, chunk=300,
       seq_len=1500),
    tc("tc_i8_s100_c700", kv_dtype="i8", Hq=4, Hk=1, capacity=700, chunk=100, seq_len=1200,
       heavy_hitters=False),
]


# Shapes whose one-CTA-per-pair grid would leave most SMs idle: the kernels run over
# equal shares of (pair, K/V tile) units, most pairs split over several CTAs (partial
# maxima, sums and outputs combined).
SPLIT_CASES = [
    tc("tc_split_c8192_s512", capacity=8192, chunk=512, seq_len=9216),
    tc("tc_split_c8000_s300_ragged", capacity=8000, chunk=300, seq_len=8600),
]
# an odd number of query tiles per KV group: the last pair of each group has no second
# tile, so some segments run one tile (split attention pass, score sums, combination)
SPLIT_ODD_CASES = [
    tc("tc_split_mha_c8192_s300_odd_tiles", Hq=2, Hk=2, capacity=8192, chunk=300, seq_len=8900),
]


@pytest.mark.parametrize("wl", SPLIT_CASES + SPLIT_ODD_CASES, ids=[w.name for w in SPLIT_CASES + SPLIT_ODD_CASES])
def test_split_schedule(wl, cuda_device):
    last = wl.n_chunks - 1
    run, n = run_and_check(wl, cuda_device, check_chunks={0, last - 1, last})
    assert n == 3


@pytest.mark.parametrize("wl", SPLIT_CASES, ids=[w.name for w in SPLIT_CASES])
def test_split_schedule_fused_kernel(wl, cuda_device, monkeypatch):
    """The fused kernel's own split schedule (phase A / phase B persistent kernels)."""
    monkeypatch.setenv("H2OKV_TC_FUSED", "1")
    last = wl.n_chunks - 1
    run, n = run_and_check(wl, cuda_device, check_chunks={0, last - 1, last})
    assert n == 3


@pytest.mark.parametrize("wl", CASES + QCASES, ids=[w.name for w in CASES + QCASES])
def test_tc_workload_every_chunk(wl, cuda_device):
    run, n = run_and_check(wl, cuda_device)
    assert n == wl.n_chunks


# bf16 caches run two passes (attention with an online softmax, then the score sums
# against the final LSE); H2OKV_TC_FUSED=1 selects the single kernel that runs both
# phases per CTA.  Both stay at parity.
FUSED_CASES = [CASES[0], CASES[1], CASES[2], CASES[6]]


@pytest.mark.parametrize("wl", FUSED_CASES, ids=[w.name for w in FUSED_CASES])
def test_tc_fused_kernel(wl, cuda_device, monkeypatch):
    monkeypatch.setenv("H2OKV_TC_FUSED", "1")
    run, n = run_and_check(wl, cuda_device)
    assert n == wl.n_chunks


def test_forced_wait_timeout_reports_status_and_recovers(cuda_device):
    """Every device-side wait of the tensor-core kernel is bounded.  With the
    limit set to 0 the first wait that is not already complete gives up: the
    kernel drains its own copies and matrix operations, frees its tensor memory
    and records H2OKV_ERR_TIMEOUT.  The context stays usable and the next call
    with the default limit is correct again."""
    import torch

    from h2o_kv_cache_attn_b200 import binding as hb
    from h2o_kv_cache_attn_b200.runner import LayerRunner
    from h2o_kv_cache_attn_b200.synth import ChunkSource

    from .harness import check_attend, snapshot, to_np

    wl = tc("timeout", capacity=512, chunk=256, seq_len=512)
    run = LayerRunner(wl, cuda_device, with_wq=True)
    q, k, v = (t.to(cuda_device) for t in ChunkSource(wl).chunk(0))
    run.cache.evict_insert(None, k, v, 256, 0)
    torch.cuda.synchronize()
    h = run.cache.handle
    assert hb.kv_cache_device_status(h) == 0
    hb.kv_cache_set_wait_timeout(h, 0)
    hb.attn_chunk_with_scoresum(h, q, 256, 0, run.y, run.lse, run.w[0], run.wq)
    assert hb.kv_cache_device_status(h) == hb.ERR_TIMEOUT
    hb.kv_cache_set_wait_timeout(h, 2_000_000_000)
    hb.attn_chunk_with_scoresum(h, q, 256, 0, run.y, run.lse, run.w[0], run.wq)
    assert hb.kv_cache_device_status(h) == 0
    after = snapshot(run.cache)
    check_attend(wl, after, to_np(q), 256, 0, to_np(run.y), to_np(run.lse), to_np(run.w[0]),
                 to_np(run.wq), [(0, 0), (0, 1)])


def test_rows_without_visible_slot(cuda_device):
    """Attention over a cache that holds none of the chunk's tokens: every row
    sees nothing, so y = 0, lse = -inf and no weight (the convention of the
    C ABI), on the tensor-core path."""
    import numpy as np
    import torch

    from h2o_kv_cache_attn_b200.runner import LayerRunner
    from h2o_kv_cache_attn_b200.synth import ChunkSource

    from .harness import to_np

    wl = tc("empty_rows", capacity=384, chunk=200, seq_len=400)
    run = LayerRunner(wl, cuda_device, with_wq=True)
    q, _, _ = (t.to(cuda_device) for t in ChunkSource(wl).chunk(0))
    y = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=cuda_device)
    run.cache.attend(q, 200, 0, y, lse, run.w[0], run.wq)
    torch.cuda.synchronize()
    assert np.all(to_np(y) == 0) and np.all(np.isneginf(to_np(lse)))
    assert np.all(to_np(run.w[0]) == 0) and np.all(to_np(run.wq) == 0)


def test_create_clears_nonfinite_rows(cuda_device):
    """The tensor-core kernels read every slot and mask empty ones
    arithmetically, so kv_cache_create zero-fills the rows: a cache created over
    buffers full of NaN gives bit for bit the outputs of one created over zeros."""
    import numpy as np
    import torch

    from h2o_kv_cache_attn_b200 import binding as hb
    from h2o_kv_cache_attn_b200.runner import LayerRunner
    from h2o_kv_cache_attn_b200.synth import ChunkSource

    from .harness import to_np

    wl = tc("nan_rows", capacity=384, chunk=128, seq_len=256)
    src = ChunkSource(wl)
    outs = []
    for poison in (False, True):
        run = LayerRunner(wl, cuda_device, with_wq=True)
        if poison:
            c = run.cache
            c.keys.fill_(float("nan"))
            c.values.fill_(float("nan"))
            old = c.handle
            c.handle = hb.kv_cache_create(c._desc, c._bufs, None)
            hb.kv_cache_destroy(old)
        res = []
        for ci in range(wl.n_chunks):
            q, k, v = (t.to(cuda_device) for t in src.chunk(ci))
            y, _, w, wq, _ = run.step(q, k, v)
            torch.cuda.synchronize()
            res.append((to_np(y).copy(), to_np(w).copy(), to_np(wq).copy()))
        outs.append(res)
    for a, b in zip(*outs):
        assert np.all(np.isfinite(b[0])) and np.all(np.isfinite(b[1]))
        for x, z in zip(a, b):
            assert np.array_equal(x, z)
