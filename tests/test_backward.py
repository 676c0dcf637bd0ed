"""Gradients of a chunk's SDPA over the cache (row f4 of the hot path: the
backward pass of §A.5 runs autograd over each chunk): the CUDA kernels against the
float64 oracle re-seeded from the GPU cache state, after a few chunks of
insertion and eviction.  Tolerance: |d| <= 1e-3 * max|ref| per (b, h) block for dq
and per (b, h_k) block for dk, dv (float32 math on bf16 / quantized inputs; the
forward's float32 log-sum-exp feeds the probabilities)."""

import numpy as np
import pytest

from h2o_kv_cache_attn_b200.configs import QWEN_64K, Workload

from .harness import oracle_group, snapshot, to_np

pytestmark = pytest.mark.gpu

TOL = 1e-3


def wl_(name, **kw):
    base = dict(name=name, B=1, Hq=4, Hk=2, d=128, capacity=300, seq_len=800, chunk=100,
                q_dtype="bf16", kv_dtype="bf16", heavy_hitters=True, seed=5)
    base.update(kw)
    return Workload(**base)


CASES = [
    wl_("bwd_f32_d64", d=64, q_dtype="f32", kv_dtype="f32"),
    wl_("bwd_bf16_gqa_b2", B=2),
    # tensor-core path: three row tiles and six slot tiles, both ragged; one slot tile
    wl_("bwd_bf16_tiles", Hq=8, Hk=2, capacity=700, chunk=300, seq_len=1500),
    wl_("bwd_bf16_one_tile", capacity=100, chunk=60, seq_len=300),
    # an odd number of packed row tiles (MHA, three tiles): the last D-kernel CTA has one
    wl_("bwd_bf16_mha_odd_tiles", Hq=2, Hk=2, capacity=500, chunk=300, seq_len=900),
    wl_("bwd_i8", kv_dtype="i8"),
    wl_("bwd_i4_mha", Hq=2, Hk=2, kv_dtype="i4", capacity=260, chunk=90, seq_len=700),
]


def _close(got, ref, what):
    scale = np.max(np.abs(ref)) + 1e-30
    err = np.max(np.abs(np.asarray(got, np.float64) - ref))
    assert err <= TOL * scale, f"{what}: max |d| = {err:.3g}, max |ref| = {scale:.3g}"


def _run(wl, device, check_groups=None, n_chunks=None):
    import torch

    from h2o_kv_cache_attn_b200.runner import LayerRunner
    from h2o_kv_cache_attn_b200.synth import ChunkSource

    src = ChunkSource(wl, 0, device)
    run = LayerRunner(wl, device, with_wq=False)
    n = n_chunks or wl.n_chunks
    gen = torch.Generator(device=device)
    gen.manual_seed(99)
    checked = 0
    for c in range(n):
        q, k, v = src.chunk(c)
        S, P = q.shape[2], run.P
        y, lse, w, _, _ = run.step(q, k, v)
        if c not in (0, n // 2, n - 1):
            continue
        dy = torch.randn(q.shape, generator=gen, device=device).to(q.dtype)
        dq = torch.empty(q.shape, dtype=torch.float32, device=device)
        shape = (wl.B, wl.Hk, wl.capacity, wl.d)
        dk = torch.empty(shape, dtype=torch.float32, device=device)
        dv = torch.empty(shape, dtype=torch.float32, device=device)
        run.cache.attend_backward(q, dy, lse.contiguous(), S, P, dq, dk, dv)
        torch.cuda.synchronize()
        snap = snapshot(run.cache)
        qn, dyn = to_np(q), to_np(dy)
        groups = check_groups or [(b, g) for b in range(wl.B) for g in range(wl.Hk)]
        for (b, g) in groups:
            oc = oracle_group(wl, snap, b, g)
            hs = slice(g * wl.q_g, (g + 1) * wl.q_g)
            rq, rk, rv = oc.attend_backward(qn[b:b + 1, hs], dyn[b:b + 1, hs], S, P)
            _close(to_np(dq)[b, hs], rq[0], f"dq b={b} g={g} P={P}")
            _close(to_np(dk)[b, g], rk[0, 0], f"dk b={b} g={g} P={P}")
            _close(to_np(dv)[b, g], rv[0, 0], f"dv b={b} g={g} P={P}")
        checked += 1
    return checked


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_backward_matches_oracle(wl, cuda_device):
    assert _run(wl, cuda_device) == 3


def test_backward_full_size_sampled(cuda_device):
    """The 64K / 16384-slot layer: the first fill chunk, a middle and a late chunk of
    the first 10, one KV group checked."""
    assert _run(QWEN_64K, cuda_device, check_groups=[(0, 3)], n_chunks=10) == 3
