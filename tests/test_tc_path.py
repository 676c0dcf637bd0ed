"""Tensor-core path (head_dim 128, bf16 cache): parity with the oracle on every
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
]


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_tc_workload_every_chunk(wl, cuda_device):
    run, n = run_and_check(wl, cuda_device)
    assert n == wl.n_chunks
