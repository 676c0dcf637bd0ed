"""Score variants, replay of logged decisions and the delta encoding of cache
updates ("Learning how to Forget", §3.1.1, §3.2 / §A.5, §A.5.3) on the GPU,
against the oracle and against the GPU's own cache states, bit for bit."""

import numpy as np
import pytest

from h2o_kv_cache_attn_b200.configs import Workload

from .harness import check_insert, run_and_check, snapshot, to_np

pytestmark = pytest.mark.gpu


def wl_(name, **kw):
    base = dict(name=name, B=2, Hq=4, Hk=2, d=128, capacity=384, seq_len=1300, chunk=160,
                q_dtype="bf16", kv_dtype="bf16", heavy_hitters=True, seed=31)
    base.update(kw)
    return Workload(**base)


VARIANT_CASES = [
    ("h2o_norm", wl_("norm_bf16_tc")),
    ("h2o_norm", wl_("norm_f32_d64", d=64, q_dtype="f32", kv_dtype="f32", capacity=200, chunk=64,
                     seq_len=700)),
    ("h2o_norm", wl_("norm_i8_tc", kv_dtype="i8")),
    ("h2o_orig", wl_("orig_bf16_tc_b3", B=3)),
    ("h2o_orig", wl_("orig_i4_tc", kv_dtype="i4", capacity=300, chunk=100, seq_len=900)),
    ("h2o_orig", wl_("orig_f32_b2_s1", d=64, q_dtype="f32", kv_dtype="f32", capacity=40, chunk=1,
                     seq_len=60)),
]


@pytest.mark.parametrize("mode,wl", VARIANT_CASES, ids=[f"{m}-{w.name}" for m, w in VARIANT_CASES])
def test_score_variant_every_chunk(mode, wl, cuda_device):
    run, n = run_and_check(wl, cuda_device, mode=mode)
    assert n == wl.n_chunks


def _same_state(a, b, skip=()):
    for k, v in a.items():
        if k in skip or k == "n_filled":
            continue
        x, y = np.asarray(v), np.asarray(b[k])
        assert np.array_equal(x.view(np.uint8) if x.dtype.kind == "f" else x,
                              y.view(np.uint8) if y.dtype.kind == "f" else y), k


@pytest.mark.parametrize("kv", ["bf16", "i4"])
def test_replay_reproduces_the_cache(kv, cuda_device):
    """A replay cache fed the slots a cache chose ends every chunk in the same
    state and returns the same outputs, bit for bit."""
    import torch

    from h2o_kv_cache_attn_b200.runner import LayerRunner
    from h2o_kv_cache_attn_b200.synth import ChunkSource

    wl = wl_(f"replay_{kv}", kv_dtype=kv)
    src = ChunkSource(wl)
    a = LayerRunner(wl, cuda_device, with_wq=True)
    a.cache.set_score_mode("h2o_norm")
    r = LayerRunner(wl, cuda_device, with_wq=True)
    for c in range(wl.n_chunks):
        q, k, v = (t.to(cuda_device) for t in src.chunk(c))
        ya, _, wa, _, slots = a.step(q, k, v)
        ya, wa, slots = ya.clone(), wa.clone(), slots.clone()
        yr, _, wr, _, _ = r.step(q, k, v, slots_in=slots)
        torch.cuda.synchronize()
        _same_state(snapshot(a.cache), snapshot(r.cache))
        assert torch.equal(ya, yr) and torch.equal(wa, wr)
    assert r.cache.n_filled == a.cache.n_filled


@pytest.mark.parametrize("kv", ["bf16", "f32", "i8", "i4"])
def test_delta_encoding_round_trip(kv, cuda_device):
    """evict_insert_delta writes the overwritten rows (gather before scatter);
    restore brings the previous rows and positions back; inserting the chunk at
    the same slots again gives the updated state, bit for bit."""
    import torch

    from h2o_kv_cache_attn_b200 import binding as hb
    from h2o_kv_cache_attn_b200.runner import LayerRunner
    from h2o_kv_cache_attn_b200.synth import ChunkSource

    d = 64 if kv == "f32" else 128
    wl = wl_(f"delta_{kv}", kv_dtype=kv, q_dtype="f32" if kv == "f32" else "bf16", d=d)
    src = ChunkSource(wl)
    run = LayerRunner(wl, cuda_device)
    for c in range(wl.n_chunks):
        q, k, v = (t.to(cuda_device) for t in src.chunk(c))
        S, P = q.shape[2], run.P
        if c < 3:  # fill and the first eviction chunk through the plain path
            run.step(q, k, v)
            continue
        torch.cuda.synchronize()
        before = snapshot(run.cache)
        w_prev = run.w_prev()
        w_np = to_np(w_prev)
        delta = run.cache.delta_buffers(S)
        slots = torch.empty((wl.B, wl.Hk, S), dtype=torch.int32, device=cuda_device)
        run.cache.evict_insert_delta(w_prev, k, v, S, P, slots, delta)
        torch.cuda.synchronize()
        after = snapshot(run.cache)
        sl = to_np(slots).astype(np.int64)
        groups = [(b, g) for b in range(wl.B) for g in range(wl.Hk)]
        check_insert(wl, before, after, w_np, to_np(k), to_np(v), S, P, sl, groups)
        raw_k = "k_raw" if kv in ("i8", "i4") else "keys"
        raw_v = "v_raw" if kv in ("i8", "i4") else "values"
        for b, g in groups:
            assert np.array_equal(to_np(delta["keys"])[b, g], before[raw_k][b, g, sl[b, g]])
            assert np.array_equal(to_np(delta["values"])[b, g], before[raw_v][b, g, sl[b, g]])
            assert np.array_equal(to_np(delta["token_pos"])[b, g], before["token_pos"][b, g, sl[b, g]])
            if kv in ("i8", "i4"):
                assert np.array_equal(to_np(delta["k_scales"])[b, g].view(np.uint16),
                                      before["k_scales"][b, g, sl[b, g]].view(np.uint16))
        run.cache.restore(slots, S, delta)
        torch.cuda.synchronize()
        _same_state(before, snapshot(run.cache), skip=("scores",))
        run.cache.insert_at(None, k, v, S, P, slots)
        torch.cuda.synchronize()
        _same_state(after, snapshot(run.cache))
        assert hb.kv_cache_device_status(run.cache.handle) == 0
        # continue the sequence from the updated state
        run.cache.attend(q, S, P, run.y if S == wl.chunk else torch.empty_like(q), None, run.w_cur())
        run.chunk_index += 1
        run.P += S


def test_replay_slot_outside_the_cache_is_reported(cuda_device):
    import torch

    from h2o_kv_cache_attn_b200 import binding as hb
    from h2o_kv_cache_attn_b200.runner import LayerRunner
    from h2o_kv_cache_attn_b200.synth import ChunkSource

    wl = wl_("replay_bad", B=1, Hk=1, Hq=2, capacity=64, chunk=16, seq_len=32)
    run = LayerRunner(wl, cuda_device)
    q, k, v = (t.to(cuda_device) for t in ChunkSource(wl).chunk(0))
    slots = torch.arange(16, dtype=torch.int32, device=cuda_device).reshape(1, 1, 16).clone()
    slots[0, 0, 5] = 64  # outside [0, N_C)
    run.cache.insert_at(None, k, v, 16, 0, slots)
    assert hb.kv_cache_device_status(run.cache.handle) == hb.ERR_INVALID_ARG
    tp = to_np(run.cache.token_pos)[0, 0]
    assert tp[5] == hb.EMPTY_POS and tp[4] == 4 and tp[6] == 6
