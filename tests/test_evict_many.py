"""Eviction over several caches in one call (h2o_evict_insert_many): independent
layers of one shape advanced chunk by chunk together.  Every cache must end each
chunk in the state the oracle gives for it (slots, positions, scores, stored rows
bit for bit), and its attention outputs must match the oracle as for a single
cache; the fold-only form and the argument checks are covered too."""

import numpy as np
import pytest
import torch

from h2o_kv_cache_attn_b200 import binding as hb
from h2o_kv_cache_attn_b200.configs import Workload
from h2o_kv_cache_attn_b200.runner import LayerRunner
from h2o_kv_cache_attn_b200.synth import ChunkSource

from .harness import check_attend, check_insert, snapshot, to_np

pytestmark = pytest.mark.gpu


def _wl(kv, **kw):
    base = dict(name=f"many_{kv}", B=2, Hq=4, Hk=2, d=128, capacity=384, seq_len=1300, chunk=160,
                q_dtype="bf16", kv_dtype=kv, heavy_hitters=True, seed=41)
    base.update(kw)
    return Workload(**base)


def _run_many(wl, device, n_layers, check_chunks=None, mode="h2o"):
    runs = [LayerRunner(wl, device, with_wq=True) for _ in range(n_layers)]
    if mode != "h2o":
        for r in runs:
            r.cache.set_score_mode(mode)
    srcs = [ChunkSource(wl, layer, "cpu") for layer in range(n_layers)]
    groups = [(b, g) for b in range(wl.B) for g in range(wl.Hk)]
    n_checked = 0
    for c in range(wl.n_chunks):
        chunks = [tuple(t.to(device) for t in s.chunk(c)) for s in srcs]
        S = chunks[0][0].shape[2]
        P = runs[0].P
        check = check_chunks is None or c in check_chunks
        if check:
            torch.cuda.synchronize()
            before = [snapshot(r.cache) for r in runs]
            w_prev = [to_np(r.w_prev()) for r in runs]
        slots = [torch.empty((wl.B, wl.Hk, S), dtype=torch.int32, device=device) for _ in runs]
        hb.h2o_evict_insert_many([r.cache.handle for r in runs],
                                 None if c == 0 else [r.w_prev() for r in runs],
                                 [ch[1] for ch in chunks], [ch[2] for ch in chunks], S, P, slots)
        outs = []
        for r, (q, _, _) in zip(runs, chunks):
            y = torch.empty_like(q)
            lse = torch.empty(q.shape[:3], dtype=torch.float32, device=device)
            r.cache.attend(q, S, P, y, lse, r.w_cur(), r.wq)
            outs.append((y, lse, r.w_cur(), r.wq))
            r.chunk_index += 1
            r.P += S
        if check:
            torch.cuda.synchronize()
            for i, r in enumerate(runs):
                after = snapshot(r.cache)
                q, k, v = (to_np(t) for t in chunks[i])
                check_insert(wl, before[i], after, w_prev[i], k, v, S, P, to_np(slots[i]), groups,
                             mode=mode)
                y, lse, w, wq = (to_np(t) for t in outs[i])
                check_attend(wl, after, q, S, P, y, lse, w, wq, groups)
            n_checked += 1
    # the last chunk's weights folded in for every cache at once
    torch.cuda.synchronize()
    before = [to_np(r.cache.scores).copy() for r in runs]
    w_last = [to_np(r.w_prev()) for r in runs]
    hb.h2o_evict_insert_many([r.cache.handle for r in runs], [r.w_prev() for r in runs],
                             None, None, 0, runs[0].P, None)
    torch.cuda.synchronize()
    for i, r in enumerate(runs):
        want = (before[i] + w_last[i]).astype(np.float32)
        np.testing.assert_array_equal(to_np(r.cache.scores).view(np.uint32), want.view(np.uint32))
    return n_checked


@pytest.mark.parametrize("kv", ["bf16", "i4", "i8"])
def test_many_caches_every_chunk(kv, cuda_device):
    wl = _wl(kv)
    assert _run_many(wl, cuda_device, 3) == wl.n_chunks


def test_many_caches_h2o_orig(cuda_device):
    wl = _wl("bf16", B=3, capacity=300, chunk=100, seq_len=700)
    assert _run_many(wl, cuda_device, 2, mode="h2o_orig") == wl.n_chunks


def test_many_caches_match_single_calls_at_full_width(cuda_device):
    """36 caches of the int4 layer shape at a small capacity: the state after each
    chunk equals that of caches driven one by one with h2o_evict_insert."""
    wl = Workload("many36", B=4, Hq=32, Hk=8, d=128, capacity=2048, seq_len=4096 + 512,
                  chunk=512, q_dtype="bf16", kv_dtype="i4", seed=5)
    n = 36
    a = [LayerRunner(wl, cuda_device, with_lse=False) for _ in range(n)]
    b = [LayerRunner(wl, cuda_device, with_lse=False) for _ in range(n)]
    srcs = [ChunkSource(wl, layer, cuda_device) for layer in range(n)]
    g = torch.Generator(device=cuda_device)
    g.manual_seed(9)
    for c in range(wl.n_chunks):
        ch = [s.chunk(c) for s in srcs]
        S = ch[0][0].shape[2]
        P = a[0].P
        # random weights stand in for the attention's (the choice only sees the scores)
        w = [torch.rand((wl.B, wl.Hk, wl.capacity), generator=g, device=cuda_device) for _ in range(n)]
        sa = [torch.empty((wl.B, wl.Hk, S), dtype=torch.int32, device=cuda_device) for _ in range(n)]
        sb = [torch.empty_like(x) for x in sa]
        hb.h2o_evict_insert_many([r.cache.handle for r in a], None if c == 0 else w,
                                 [x[1] for x in ch], [x[2] for x in ch], S, P, sa)
        for i, r in enumerate(b):
            r.cache.evict_insert(None if c == 0 else w[i], ch[i][1], ch[i][2], S, P, sb[i])
        for r in a + b:
            r.P += S
        torch.cuda.synchronize()
        for i in range(n):
            assert torch.equal(sa[i], sb[i]), f"slots layer {i} chunk {c}"
            for name in ("token_pos", "scores", "keys", "values", "k_scales", "v_scales"):
                assert torch.equal(getattr(a[i].cache, name), getattr(b[i].cache, name)), (name, i, c)


def test_many_caches_argument_checks(cuda_device):
    wl = _wl("bf16")
    r1 = LayerRunner(wl, cuda_device)
    r2 = LayerRunner(wl.with_(capacity=256), cuda_device)
    q, k, v = (t.to(cuda_device) for t in ChunkSource(wl).chunk(0))
    with pytest.raises(hb.H2OKVError) as e:
        hb.h2o_evict_insert_many([r1.cache.handle, r2.cache.handle], None, [k, k], [v, v], 160, 0)
    assert e.value.code == hb.ERR_INVALID_ARG and "differs" in hb.h2okv_last_error()
    with pytest.raises(hb.H2OKVError) as e:
        hb.h2o_evict_insert_many([r1.cache.handle, r1.cache.handle], None, [k, k], [v, v], 160, 0)
    assert "twice" in hb.h2okv_last_error()
    with pytest.raises(hb.H2OKVError):
        hb.h2o_evict_insert_many([r1.cache.handle], None, [k], [None], 160, 0)
    assert r1.cache.n_filled == 0  # nothing was enqueued
