"""The allocation-free entry point, for callers that cannot allocate device
memory (every byte they use belongs to another allocator, so they cannot hand
the library a workspace).  On two calls in a row it must give what the oracle
gives, within the stated tolerances, and what the regular entry point gives,
although its scratch is one array shared by every call.  Its cases cover every
cache dtype it serves (f32, bf16, int8, int4), a head dimension of 64 and chunks
that are not a multiple of the kernel's 32-row tiles.

This file is collected last on purpose: it runs after every other test when
the whole suite runs, and also passes on its own in a fresh process."""

import pytest
import torch

from h2o_kv_cache_attn_b200 import binding as hb
from h2o_kv_cache_attn_b200.configs import Workload
from h2o_kv_cache_attn_b200.runner import LayerRunner
from h2o_kv_cache_attn_b200.synth import ChunkSource

from .harness import (assert_lse_close, assert_w_close, assert_y_close, check_attend, snapshot,
                      to_np)

pytestmark = pytest.mark.gpu


def _wl(kv, d=128, chunk=256, capacity=384, seq_len=512, q="bf16"):
    # two calls: the second fills the free slots and evicts the rest
    return Workload(f"noalloc_{kv}_d{d}_s{chunk}", B=1, Hq=8, Hk=2, d=d, capacity=capacity,
                    seq_len=seq_len, chunk=chunk, q_dtype=q, kv_dtype=kv, heavy_hitters=True,
                    seed=21)


CASES = [
    _wl("bf16"),
    _wl("i8"),
    _wl("i4", chunk=200, capacity=300, seq_len=400),
    _wl("f32", d=64, chunk=100, capacity=150, seq_len=200, q="f32"),
]


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_noalloc_matches_oracle_on_two_calls(wl, cuda_device):
    run = LayerRunner(wl, cuda_device, with_wq=True)
    cache = run.cache
    src = ChunkSource(wl, 0, "cpu")
    groups = [(b, g) for b in range(wl.B) for g in range(wl.Hk)]
    for c in range(2):
        q, k, v = (t.to(cuda_device) for t in src.chunk(c))
        P, S = run.P, q.shape[2]
        y, lse, w, wq, _ = run.step(q, k, v)  # regular entry point (after the insert)
        y2 = torch.full_like(y, float("nan"))
        lse2 = torch.full_like(lse, float("nan"))
        w2 = torch.full_like(w, float("nan"))
        wq2 = torch.full_like(wq, float("nan"))
        hb.attn_chunk_with_scoresum_noalloc(
            cache._desc, cache.keys, cache.values, cache.k_scales, cache.v_scales,
            cache.token_pos, q, S, P, y2, lse2, w2, wq2)
        torch.cuda.synchronize()
        # against the oracle, at the stated tolerances
        check_attend(wl, snapshot(cache), to_np(q), S, P, to_np(y2), to_np(lse2), to_np(w2),
                     to_np(wq2), groups)
        # and against the regular entry point
        assert_y_close(to_np(y2), to_np(y), f"y call {c}")
        assert_lse_close(to_np(lse2), to_np(lse), f"lse call {c}")
        assert_w_close(to_np(w2), to_np(w), f"w call {c}")
        assert_w_close(to_np(wq2), to_np(wq), f"wq call {c}")


def test_noalloc_rejects_too_many_rows(cuda_device):
    desc = hb.CacheDesc(4, 32, 8, 128, 1024, 4096, hb.BF16, hb.BF16)
    t = torch.zeros(16, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(hb.H2OKVError) as e:
        hb.attn_chunk_with_scoresum_noalloc(desc, t, t, None, None, t, t, 4096, 0, t, None, t)
    assert e.value.code == hb.ERR_INVALID_ARG
    assert "static scratch" in hb.h2okv_last_error()


def test_noalloc_rejects_a_grid_too_tall_before_touching_outputs(cuda_device):
    # batch * n_kv_heads above the launch limit: refused on the host, w_out untouched
    desc = hb.CacheDesc(65536, 4, 4, 8, 1, 1, hb.BF16, hb.BF16)
    t = torch.zeros(16, dtype=torch.uint8, device=cuda_device)
    w = torch.full((4,), 7.0, device=cuda_device)
    with pytest.raises(hb.H2OKVError) as e:
        hb.attn_chunk_with_scoresum_noalloc(desc, t, t, None, None, t, t, 1, 0, t, None, w)
    assert e.value.code == hb.ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.all(w == 7.0)
