"""A short, steady-state run of the hot path for profiler captures.

``python -m h2o_kv_cache_attn_b200.profile_case [--config 128k] [--iters 3] [--backward | --many N]``

Fills one layer's cache directly (every slot occupied, random keys, values and
scores), then runs ``--iters`` eviction chunks (h2o_evict_insert followed by
attn_chunk_with_scoresum), or with ``--backward`` one attention call (for the
row log-sum-exp) and ``--iters`` calls of attn_chunk_backward on that chunk, or
with ``--many N`` N such caches and ``--iters`` batched eviction calls
(h2o_evict_insert_many over all N, as a model's layers are advanced together).
Only a handful of launches precede the measured ones, so a profiler can capture
e.g. the second attention launch of a full 128K-token / 32768-slot layer with
the cache larger than L2.
"""

from __future__ import annotations

import argparse

import torch

from .configs import SHORT
from .runner import LayerRunner


def _fill(run, wl, g, dev):
    """Every slot occupied: random keys / values (codes and scales), positions and scores."""
    c = run.cache
    if wl.kv_dtype in ("bf16", "f32"):
        c.keys.copy_(torch.randn(c.keys.shape, generator=g, device=dev))
        c.values.copy_(torch.randn(c.values.shape, generator=g, device=dev))
    else:
        c.keys.copy_(torch.randint(-100, 100, c.keys.shape, generator=g, device=dev).to(c.keys.dtype))
        c.values.copy_(torch.randint(-100, 100, c.values.shape, generator=g, device=dev).to(c.values.dtype))
        c.k_scales.fill_(0.01)
        c.v_scales.fill_(0.01)
    c.token_pos.copy_(torch.arange(wl.capacity, dtype=torch.int32, device=dev).expand_as(c.token_pos))
    c.scores.copy_(torch.rand(c.scores.shape, generator=g, device=dev))
    c.set_fill(wl.capacity)


def _many(wl, n, iters, g, dev):
    """Batched eviction over n full caches of the workload's shape."""
    from . import binding as hb

    runs = [LayerRunner(wl, dev, with_wq=False, with_lse=False) for _ in range(n)]
    for r in runs:
        _fill(r, wl, g, dev)
    kvt = torch.float32 if wl.kv_dtype == "f32" else torch.bfloat16
    S, P = wl.chunk, wl.capacity
    w = [torch.rand((wl.B, wl.Hk, wl.capacity), generator=g, device=dev) * 0.01 for _ in runs]
    k = [torch.randn((wl.B, wl.Hk, S, wl.d), generator=g, device=dev).to(kvt) for _ in runs]
    v = [torch.randn((wl.B, wl.Hk, S, wl.d), generator=g, device=dev).to(kvt) for _ in runs]
    for _ in range(iters):
        hb.h2o_evict_insert_many([r.cache.handle for r in runs], w, k, v, S, P)
        P += S
    torch.cuda.synchronize()
    p_last = P - S  # every (b, h) holds the last call's S tokens, once each
    filled = all(int((r.cache.token_pos >= p_last).sum()) == wl.B * wl.Hk * S for r in runs)
    print(f"profile_case {wl.name}: {iters} batched evictions over {n} caches, "
          f"last chunk's tokens placed: {filled}")
    if not filled:
        raise SystemExit("batched eviction did not place the chunk")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="128k", choices=sorted(SHORT))
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--backward", action="store_true")
    ap.add_argument("--many", type=int, default=0)
    args = ap.parse_args()
    wl = SHORT[args.config]
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(wl.seed)
    if args.many > 0:
        _many(wl, args.many, args.iters, g, dev)
        return
    run = LayerRunner(wl, dev, with_wq=False, with_lse=False)
    _fill(run, wl, g, dev)
    c = run.cache
    qt = torch.float32 if wl.q_dtype == "f32" else torch.bfloat16
    kvt = torch.float32 if wl.kv_dtype == "f32" else torch.bfloat16
    S = wl.chunk
    q = torch.randn((wl.B, wl.Hq, S, wl.d), generator=g, device=dev).to(qt)
    k = torch.randn((wl.B, wl.Hk, S, wl.d), generator=g, device=dev).to(kvt)
    v = torch.randn((wl.B, wl.Hk, S, wl.d), generator=g, device=dev).to(kvt)
    run.P = wl.capacity
    run.chunk_index = 1  # the cache is full: the first w_prev is the zero buffer
    if args.backward:
        y = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        run.cache.attend(q, S, run.P, y, lse, run.w[0], None)
        dy = torch.randn(q.shape, generator=g, device=dev).to(qt)
        dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
        dk = torch.empty((wl.B, wl.Hk, wl.capacity, wl.d), dtype=torch.float32, device=dev)
        dv = torch.empty_like(dk)
        for _ in range(args.iters):
            run.cache.attend_backward(q, dy, lse, S, run.P, dq, dk, dv)
        torch.cuda.synchronize()
        ok = bool(torch.isfinite(dq).all() and torch.isfinite(dk).all() and torch.isfinite(dv).all())
        print(f"profile_case {wl.name}: {args.iters} backward calls, finite gradients: {ok}")
        if not ok:
            raise SystemExit("non-finite gradients")
        return
    for _ in range(args.iters):
        run.step(q, k, v)
    torch.cuda.synchronize()
    w = run.last[2]
    total = float(w.sum())
    expect = wl.B * wl.Hk * S * wl.q_g
    print(f"profile_case {wl.name}: {args.iters} chunks, sum(w) = {total:.1f} (expect {expect})")
    if abs(total - expect) > 1e-3 * expect:
        raise SystemExit("summed weights do not add up")


if __name__ == "__main__":
    main()
