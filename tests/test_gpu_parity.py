"""Parity of the CUDA path with the CPU oracle (needs a B200).

Every call goes through the C ABI.  Small workloads (the oracle finishes in
seconds) are compared on every chunk and every (b, h_k); they span several
128-slot tiles with ragged tails, a partially filling chunk, GQA and MHA, and
all four cache dtypes.  The full-size workloads are compared on sampled chunks
and KV heads, with the oracle re-seeded from the GPU cache state each time.
"""

import numpy as np
import pytest
import torch

import oracle
from h2o_kv_cache_attn_b200 import binding as hb
from h2o_kv_cache_attn_b200.configs import QWEN_64K, QWEN_128K, QWEN_INT8, STACK_INT4, TINY_F32, Workload
from h2o_kv_cache_attn_b200.synth import ChunkSource

from .harness import assert_w_close, run_and_check, to_np

pytestmark = pytest.mark.gpu


def small(name, **kw):
    base = dict(name=name, B=2, Hq=4, Hk=2, d=64, capacity=300, seq_len=1000, chunk=128,
                q_dtype="bf16", kv_dtype="bf16", heavy_hitters=True, seed=77)
    base.update(kw)
    return Workload(**base)


SMALL = [
    small("bf16_d64_ragged"),
    small("bf16_d128_ragged", d=128, capacity=700, chunk=200, seq_len=1800, B=1, Hq=8, Hk=2),
    small("i8_d128", d=128, kv_dtype="i8", capacity=384, chunk=96, seq_len=900),
    small("i4_d128", d=128, kv_dtype="i4", capacity=330, chunk=130, seq_len=1000),
    small("f32_tiny_shape", q_dtype="f32", kv_dtype="f32", capacity=256, chunk=128, seq_len=1024,
          heavy_hitters=False),
    small("mha_d256", Hq=2, Hk=2, d=256, capacity=160, chunk=50, seq_len=400),
    small("chunk1", B=1, Hq=4, Hk=1, capacity=20, chunk=1, seq_len=60),
    small("chunk_eq_capacity", capacity=64, chunk=64, seq_len=320),
    small("i4_d64_q8", Hq=8, Hk=1, kv_dtype="i4", capacity=200, chunk=64, seq_len=500),
]


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_small_workload_every_chunk(wl, cuda_device):
    run, n = run_and_check(wl, cuda_device)
    assert n == wl.n_chunks


def test_tiny_fp32_workload_every_chunk(cuda_device):
    run, n = run_and_check(TINY_F32, cuda_device)
    assert n == TINY_F32.n_chunks == 8


def test_four_slot_toy_on_gpu(cuda_device):
    # The hand-derived toy (q = 0): uniform attention over the visible slots.
    wl = Workload("toy", B=1, Hq=2, Hk=1, d=8, capacity=4, seq_len=8, chunk=2, q_dtype="f32",
                  kv_dtype="f32")
    from h2o_kv_cache_attn_b200.runner import LayerRunner
    run = LayerRunner(wl, cuda_device, with_wq=True)
    expect_w = [[1.5, 0.5, 0, 0], [7 / 12, 7 / 12, 7 / 12, 0.25], [7 / 12, 7 / 12, 7 / 12, 0.25],
                [7 / 12, 7 / 12, 7 / 12, 0.25]]
    expect_slots = [[0, 1], [2, 3], [2, 3], [2, 3]]
    for c in range(4):
        P = 2 * c
        toks = torch.tensor([P, P + 1], dtype=torch.float32)
        v = torch.zeros((1, 1, 2, 8))
        v[0, 0, :, 0] = toks
        v[0, 0, :, 1] = 10 - toks
        k = torch.randn((1, 1, 2, 8))
        q = torch.zeros((1, 2, 2, 8))
        y, lse, w, wq, slots = run.step(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device))
        torch.cuda.synchronize()
        assert to_np(slots)[0, 0].tolist() == expect_slots[c]
        np.testing.assert_allclose(to_np(w)[0, 0], 2 * np.array(expect_w[c]), rtol=1e-6)
        np.testing.assert_allclose(to_np(wq)[0, 0], expect_w[c], rtol=1e-6)


# ---------------------------------------------------------------------------
# Quantizer: bit-exact against the oracle's float32 rules.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("kind", ["i8", "i4"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_quantize_bit_exact(kind, d, cuda_device):
    g = torch.Generator().manual_seed(5)
    n = 4096
    x = torch.randn((n, d), generator=g) * torch.exp(torch.randn((n, 1), generator=g) * 3)
    x[0] = 0
    x[1] = 1e-30  # scale underflows to a zero fp16
    x[2] = 3e-6   # subnormal fp16 scale
    x[3] = 1e7    # saturated scale
    x[4, : d // 2] = 2.0 ** -3 * torch.arange(d // 2) % 15 - 7
    x[5] = torch.linspace(-1, 1, d)  # many exact halves
    xb = x.to(torch.bfloat16)
    row = d // 2 if kind == "i4" else d
    codes = torch.empty((n, row), dtype=torch.int8 if kind == "i8" else torch.uint8, device=cuda_device)
    scales = torch.empty((n,), dtype=torch.float16, device=cuda_device)
    hb.kv_cache_quantize(kind, xb.to(cuda_device), codes, scales)
    torch.cuda.synchronize()
    rc, rs = oracle.quantize_rows(xb.float().numpy(), kind)
    if kind == "i4":
        rc = oracle.pack_int4(rc)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    np.testing.assert_array_equal(codes.cpu().numpy().view(np.uint8), rc.view(np.uint8))


def _bf16_rows_up_to(anchors, d, seed):
    """Rows of d bf16 values: element 0 is +-A (it sets the row's absmax, hence its
    scale), the other d - 1 run through every finite bf16 value with |x| <= A."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    allv = (bits.astype(np.uint32) << 16).view(np.float32)
    allv = allv[np.isfinite(allv)]
    rng = np.random.default_rng(seed)
    rows = []
    for a in anchors:
        a = float(np.float32(torch.tensor(a).to(torch.bfloat16).float()))
        vals = allv[np.abs(allv) <= a]
        n = -(-len(vals) // (d - 1))
        pad = np.resize(vals, n * (d - 1))
        block = np.empty((n, d), np.float32)
        block[:, 0] = a * rng.choice([-1.0, 1.0], size=n)
        block[:, 1:] = pad.reshape(n, d - 1)
        rows.append(block)
    return np.concatenate(rows)


@pytest.mark.parametrize("kind", ["i8", "i4"])
def test_quantize_every_bf16_value(kind, cuda_device):
    """Every finite bf16 value x, quantized in rows whose scale ranges over fp16
    normals, subnormals, the 65504 clamp and rounding ties of x / scale: codes and
    scales equal the oracle's (IEEE float32 division), bit for bit."""
    anchors = [2.0 ** e * m for e in range(-20, 21, 3) for m in (1.0, 1.015625, 1.5, 1.9921875)]
    anchors += [7.0, 127.0, 3.5, 63.5, 6.5e-6, 1e-7, 4.0e6, 1e9, 1e30, 3e38]
    x = _bf16_rows_up_to(anchors, 128, seed=11)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    n, d = x.shape
    row = d // 2 if kind == "i4" else d
    codes = torch.empty((n, row), dtype=torch.int8 if kind == "i8" else torch.uint8, device=cuda_device)
    scales = torch.empty((n,), dtype=torch.float16, device=cuda_device)
    hb.kv_cache_quantize(kind, xb.to(cuda_device), codes, scales)
    torch.cuda.synchronize()
    rc, rs = oracle.quantize_rows(xb.float().numpy(), kind)
    if kind == "i4":
        rc = oracle.pack_int4(rc)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    np.testing.assert_array_equal(codes.cpu().numpy().view(np.uint8), rc.view(np.uint8))


# ---------------------------------------------------------------------------
# Eviction: bit-exact on tie-heavy score arrays, every capacity regime.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("capacity,S", [(10, 3), (1000, 100), (32768, 1024), (53248, 2048),
                                        (60000, 512), (65536, 4096)])
def test_eviction_bit_exact_ties(capacity, S, cuda_device):
    wl = Workload("ev", B=2, Hq=2, Hk=2, d=8, capacity=capacity, seq_len=capacity + S, chunk=S,
                  q_dtype="bf16", kv_dtype="bf16")
    from h2o_kv_cache_attn_b200.runner import LayerRunner
    from .harness import check_insert, snapshot
    run = LayerRunner(wl, cuda_device)
    cache = run.cache
    g = torch.Generator().manual_seed(capacity)
    # a full cache with integer (tie-heavy) scores, plus exact zeros and negative zeros
    cache.token_pos.copy_(torch.arange(capacity, dtype=torch.int32).repeat(2, 2, 1))
    sc = torch.randint(0, 4, (2, 2, capacity), generator=g).float()
    sc[0, 0, ::5] = -0.0
    cache.scores.copy_(sc)
    cache.set_fill(capacity)
    w_prev = torch.randint(0, 3, (2, 2, capacity), generator=g).float() * 0.5
    w_prev[1, 1] = 0.0
    k = torch.randn((2, 2, S, 8), generator=g).to(torch.bfloat16)
    v = torch.randn((2, 2, S, 8), generator=g).to(torch.bfloat16)
    torch.cuda.synchronize()
    before = snapshot(cache)
    slots = torch.empty((2, 2, S), dtype=torch.int32, device=cuda_device)
    cache.evict_insert(w_prev.to(cuda_device), k.to(cuda_device), v.to(cuda_device), S, capacity, slots)
    torch.cuda.synchronize()
    after = snapshot(cache)
    check_insert(wl, before, after, w_prev.numpy(), k.float().numpy(), v.float().numpy(), S,
                 capacity, to_np(slots), [(0, 0), (0, 1), (1, 0), (1, 1)])


def test_partial_fill_then_evict(cuda_device):
    # 300 slots, chunks of 128: the third chunk fills 44 empty slots and evicts 84
    wl = small("partial", capacity=300, chunk=128, seq_len=640)
    run, n = run_and_check(wl, cuda_device)
    assert n == 5


def test_fold_only_call_and_reset(cuda_device):
    wl = small("fold", capacity=256, chunk=128, seq_len=512, kv_dtype="bf16")
    run, _ = run_and_check(wl, cuda_device, check_chunks=set())
    sc = to_np(run.cache.scores)
    # after folding the last w in, every group's scores sum to the weights of
    # the chunks that are still cached; each is positive
    assert np.all(sc >= 0) and np.all(np.isfinite(sc))
    run.reset()
    torch.cuda.synchronize()
    assert run.cache.n_filled == 0
    assert np.all(to_np(run.cache.token_pos) == hb.EMPTY_POS)
    assert np.all(to_np(run.cache.scores) == 0)


def test_error_paths_leave_device_usable(cuda_device):
    wl = small("err", capacity=64, chunk=32, seq_len=64)
    from h2o_kv_cache_attn_b200.runner import LayerRunner
    run = LayerRunner(wl, cuda_device)
    q, k, v = ChunkSource(wl).chunk(0)
    q, k, v = q.to(cuda_device), k.to(cuda_device), v.to(cuda_device)
    with pytest.raises(hb.H2OKVError):
        hb.h2o_evict_insert(run.cache.handle, None, k, v, 65, 0)  # S > capacity
    with pytest.raises(hb.H2OKVError):
        hb.h2o_evict_insert(run.cache.handle, None, k, v, 32, 2**31 - 10)  # P overflow
    with pytest.raises(hb.H2OKVError):
        hb.attn_chunk_with_scoresum(run.cache.handle, q, 0, 0, run.y, None, run.w[0])
    with pytest.raises(hb.H2OKVError):
        hb.attn_chunk_with_scoresum(run.cache.handle, q, 33, 0, run.y, None, run.w[0])
    y, lse, w, wq, slots = run.step(q, k, v)
    torch.cuda.synchronize()
    assert abs(float(w.sum()) - 32 * wl.q_g * wl.B * wl.Hk) < 1e-2


# ---------------------------------------------------------------------------
# Full-size workloads, sampled chunks and KV heads.
# ---------------------------------------------------------------------------
def _sampled(wl, n_extra_mid=1):
    n_fill = -(-wl.capacity // wl.chunk)
    picks = {0, n_fill, wl.n_chunks - 1}
    for t in range(1, n_extra_mid + 1):
        picks.add(n_fill + t * (wl.n_chunks - n_fill) // (n_extra_mid + 1))
    return picks


@pytest.mark.parametrize("wl", [QWEN_64K, QWEN_128K, QWEN_INT8], ids=lambda w: w.name)
def test_full_size_sampled(wl, cuda_device):
    src = ChunkSource(wl, 0, cuda_device)
    run, n = run_and_check(wl, cuda_device, check_chunks=_sampled(wl),
                           groups=[(0, 0), (0, 3), (0, 5), (0, 7)], with_wq=False, source=src)
    assert n == len(_sampled(wl))


def test_full_size_128k_per_head_sums_sampled(cuda_device):
    """The per-query-head summed weights (wq) of the 128K layer at full size, as the
    bench's split and every-SM schedules produce them, on a fill and an eviction chunk."""
    wl = QWEN_128K
    src = ChunkSource(wl, 0, cuda_device)
    n_fill = -(-wl.capacity // wl.chunk)
    run, n = run_and_check(wl, cuda_device, check_chunks={n_fill - 1, n_fill + 5},
                           groups=[(0, 2), (0, 6)], with_wq=True, source=src)
    assert n == 2


def test_full_size_int4_stack_one_layer_sampled(cuda_device):
    wl = STACK_INT4.with_(layers=1)
    src = ChunkSource(wl, 7, cuda_device)
    run, n = run_and_check(wl, cuda_device, check_chunks={0, 16, 63}, groups=[(0, 1), (3, 6)],
                           with_wq=False, source=src)
    assert n == 3
