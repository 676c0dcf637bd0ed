"""The allocation-free entry point, for callers that cannot allocate device
memory (every byte they use belongs to another allocator, so they cannot hand
the library a workspace).  It must give what the regular entry point gives,
call after call, although its scratch is one array shared by every call.

This file is collected last on purpose: it runs after every other test when
the whole suite runs, and also passes on its own in a fresh process."""

import numpy as np
import pytest
import torch

from h2o_kv_cache_attn_b200 import binding as hb
from h2o_kv_cache_attn_b200.configs import Workload
from h2o_kv_cache_attn_b200.runner import LayerRunner
from h2o_kv_cache_attn_b200.synth import ChunkSource

from .harness import assert_lse_close, assert_w_close, assert_y_close, to_np

pytestmark = pytest.mark.gpu


def _wl(kv):
    # 384 slots, chunks of 256: the second call fills 128 free slots and evicts 128
    return Workload(f"noalloc_{kv}", B=1, Hq=8, Hk=2, d=128, capacity=384, seq_len=512,
                    chunk=256, q_dtype="bf16", kv_dtype=kv, heavy_hitters=True, seed=21)


@pytest.mark.parametrize("kv", ["bf16", "i8"])
def test_noalloc_matches_regular_entry_point_on_two_calls(kv, cuda_device):
    wl = _wl(kv)
    run = LayerRunner(wl, cuda_device, with_wq=True)
    cache = run.cache
    src = ChunkSource(wl, 0, "cpu")
    for c in range(2):
        q, k, v = (t.to(cuda_device) for t in src.chunk(c))
        P = run.P
        y, lse, w, wq, _ = run.step(q, k, v)  # regular entry point (after the insert)
        y2 = torch.full_like(y, float("nan"))
        lse2 = torch.full_like(lse, float("nan"))
        w2 = torch.full_like(w, float("nan"))
        wq2 = torch.full_like(wq, float("nan"))
        hb.attn_chunk_with_scoresum_noalloc(
            cache._desc, cache.keys, cache.values, cache.k_scales, cache.v_scales,
            cache.token_pos, q, q.shape[2], P, y2, lse2, w2, wq2)
        torch.cuda.synchronize()
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
