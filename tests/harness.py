"""Test harness: run the CUDA path chunk by chunk and compare each checked
chunk with the CPU oracle re-seeded from the GPU cache state.

Tolerances (written here, used by every parity test):
  * y: |dy| <= 2e-2 * max|y_ref| per (b, h_q) block (bf16 output, fp32 math);
  * w, wq: |dw_j| <= 1e-3 * max(|w_j|, 1e-3 * max_j w_j) per (b, h) row;
  * lse: |dlse| <= 2e-4 + 1e-5 * |lse_ref|;
  * slots, token_pos, scores, stored key/value bytes and scales: bit-exact.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from h2o_kv_cache_attn_b200.configs import Workload
from h2o_kv_cache_attn_b200.runner import LayerRunner
from h2o_kv_cache_attn_b200.synth import ChunkSource

Y_TOL = 2e-2
W_TOL = 1e-3
LSE_ABS, LSE_REL = 2e-4, 1e-5


def to_np(t):
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def snapshot(cache):
    s = {"token_pos": to_np(cache.token_pos).astype(np.int64), "scores": to_np(cache.scores).copy(),
         "n_filled": cache.n_filled}
    kv = cache.shape.kv_dtype
    if kv in ("i8", "i4"):
        if kv == "i8":
            s["k_codes"], s["v_codes"] = to_np(cache.keys).copy(), to_np(cache.values).copy()
        else:
            s["k_codes"] = oracle.unpack_int4(to_np(cache.keys))
            s["v_codes"] = oracle.unpack_int4(to_np(cache.values))
        s["k_raw"], s["v_raw"] = to_np(cache.keys).copy(), to_np(cache.values).copy()
        s["k_scales"], s["v_scales"] = to_np(cache.k_scales).copy(), to_np(cache.v_scales).copy()
    else:
        s["keys"], s["values"] = to_np(cache.keys).copy(), to_np(cache.values).copy()
    return s


def oracle_group(wl: Workload, snap, b: int, g: int):
    """An oracle cache for one (b, h_k) group (B = 1, H_k = 1, H_q = q_g)."""
    oc = oracle.OracleCache(1, wl.q_g, 1, wl.d, wl.capacity, wl.kv_dtype)
    sl = (slice(b, b + 1), slice(g, g + 1))
    kw = dict(token_pos=snap["token_pos"][sl], scores=snap["scores"][sl], n_filled=snap["n_filled"])
    if wl.kv_dtype in ("i8", "i4"):
        kw.update(k_codes=snap["k_codes"][sl], v_codes=snap["v_codes"][sl],
                  k_scales=snap["k_scales"][sl], v_scales=snap["v_scales"][sl])
    else:
        kw.update(keys=snap["keys"][sl], values=snap["values"][sl])
    oc.load_state(**kw)
    return oc


def assert_w_close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    floor = W_TOL * np.max(np.abs(ref), axis=-1, keepdims=True)
    tol = W_TOL * np.maximum(np.abs(ref), floor)
    bad = np.abs(got - ref) > tol
    if np.any(bad):
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} slots outside tolerance, e.g. "
                             + ", ".join(f"{tuple(i)} got {got[tuple(i)]:.7g} ref {ref[tuple(i)]:.7g}"
                                         for i in idx))


def assert_y_close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.max(np.abs(ref), axis=(-2, -1), keepdims=True)
    err = np.abs(got - ref)
    bad = err > Y_TOL * scale
    if np.any(bad):
        raise AssertionError(f"{what}: max |dy|/max|y| = {np.max(err / np.maximum(scale, 1e-30)):.3g}")


def assert_lse_close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(got)), f"{what}: -inf pattern differs"
    err = np.abs(got[fin] - ref[fin])
    tol = LSE_ABS + LSE_REL * np.abs(ref[fin])
    assert np.all(err <= tol), f"{what}: max lse error {err.max():.3g}"


def oracle_head(wl: Workload, snap, g: int):
    """An oracle cache for KV head g over every batch row (B = wl.B, H_k = 1)."""
    oc = oracle.OracleCache(wl.B, wl.q_g, 1, wl.d, wl.capacity, wl.kv_dtype)
    sl = (slice(None), slice(g, g + 1))
    kw = dict(token_pos=snap["token_pos"][sl], scores=snap["scores"][sl], n_filled=snap["n_filled"])
    if wl.kv_dtype in ("i8", "i4"):
        kw.update(k_codes=snap["k_codes"][sl], v_codes=snap["v_codes"][sl],
                  k_scales=snap["k_scales"][sl], v_scales=snap["v_scales"][sl])
    else:
        kw.update(keys=snap["keys"][sl], values=snap["values"][sl])
    oc.load_state(**kw)
    return oc


def check_insert(wl, before, after, w_prev, k, v, S, P, slots_gpu, groups, mode="h2o"):
    """Bit-exact check of the evict/insert step for the given (b, g) groups.
    h2o_orig chooses for all batch rows of a KV head together: its oracle holds
    every batch row of the head."""
    for (b, g) in groups:
        if mode == "h2o_orig":
            oc = oracle_head(wl, before, g)
            wp = None if w_prev is None else w_prev[:, g:g + 1]
            slots = oc.evict_insert(wp, k[:, g:g + 1], v[:, g:g + 1], S, P, mode=mode)
            oc = _row_of(oc, b)
            slots = slots[b:b + 1]
        else:
            oc = oracle_group(wl, before, b, g)
            wp = None if w_prev is None else w_prev[b:b + 1, g:g + 1]
            slots = oc.evict_insert(wp, k[b:b + 1, g:g + 1], v[b:b + 1, g:g + 1], S, P, mode=mode)
        np.testing.assert_array_equal(slots_gpu[b, g], slots[0, 0], err_msg=f"slots b={b} g={g}")
        np.testing.assert_array_equal(after["token_pos"][b, g], oc.token_pos[0, 0])
        np.testing.assert_array_equal(after["scores"][b, g].view(np.uint32),
                                      oc.scores[0, 0].view(np.uint32), err_msg="scores")
        if wl.kv_dtype in ("i8", "i4"):
            np.testing.assert_array_equal(after["k_codes"][b, g], oc.k_codes[0, 0])
            np.testing.assert_array_equal(after["v_codes"][b, g], oc.v_codes[0, 0])
            np.testing.assert_array_equal(after["k_scales"][b, g].view(np.uint16),
                                          oc.k_scales[0, 0].view(np.uint16))
            np.testing.assert_array_equal(after["v_scales"][b, g].view(np.uint16),
                                          oc.v_scales[0, 0].view(np.uint16))
        else:
            np.testing.assert_array_equal(after["keys"][b, g], oc.k_store[0, 0])
            np.testing.assert_array_equal(after["values"][b, g], oc.v_store[0, 0])
    return True


class _Row:
    """Batch row b of an oracle cache, as attributes shaped like a one-row cache."""

    def __init__(self, oc, b):
        for name in ("token_pos", "scores", "k_codes", "v_codes", "k_scales", "v_scales",
                     "k_store", "v_store"):
            if hasattr(oc, name):
                setattr(self, name, getattr(oc, name)[b:b + 1])


def _row_of(oc, b):
    return _Row(oc, b)


def check_attend(wl, after, q, S, P, y, lse, w, wq, groups):
    for (b, g) in groups:
        oc = oracle_group(wl, after, b, g)
        hs = slice(g * wl.q_g, (g + 1) * wl.q_g)
        yr, lr, wr, wqr = oc.attend(q[b:b + 1, hs], S, P)
        assert_y_close(y[b, hs], yr[0], f"y b={b} g={g} P={P}")
        if lse is not None:
            assert_lse_close(lse[b, hs], lr[0], f"lse b={b} g={g} P={P}")
        assert_w_close(w[b, g], wr[0, 0], f"w b={b} g={g} P={P}")
        if wq is not None:
            assert_w_close(wq[b, hs], wqr[0], f"wq b={b} g={g} P={P}")
        # invariant: each chunk's weights add up to S * q_g per group
        np.testing.assert_allclose(np.sum(w[b, g], dtype=np.float64), S * wl.q_g, rtol=2e-4)


def run_and_check(wl: Workload, device, check_chunks=None, groups=None, with_wq=True,
                  source=None, on_chunk=None, mode="h2o"):
    """Run all chunks of one layer on the GPU; compare the chunks in
    ``check_chunks`` (None = all) for the (b, g) pairs in ``groups`` (None =
    all) against the oracle re-seeded from the GPU state before each of them.
    ``mode``: the score variant of the eviction."""
    src = source or ChunkSource(wl, 0, "cpu")
    run = LayerRunner(wl, device, with_wq=with_wq)
    if mode != "h2o":
        run.cache.set_score_mode(mode)
    if groups is None:
        groups = [(b, g) for b in range(wl.B) for g in range(wl.Hk)]
    n_checked = 0
    for c in range(wl.n_chunks):
        q, k, v = src.chunk(c)
        q, k, v = q.to(device), k.to(device), v.to(device)
        check = check_chunks is None or c in check_chunks
        if check:
            torch.cuda.synchronize()
            before = snapshot(run.cache)
            w_prev = to_np(run.w_prev())
        P = run.P
        S = q.shape[2]
        y, lse, w, wq, slots = run.step(q, k, v)
        if check:
            torch.cuda.synchronize()
            after = snapshot(run.cache)
            qn, kn, vn = to_np(q), to_np(k), to_np(v)
            check_insert(wl, before, after, w_prev, kn, vn, S, P, to_np(slots), groups, mode=mode)
            check_attend(wl, after, qn, S, P, to_np(y), to_np(lse), to_np(w), to_np(wq), groups)
            n_checked += 1
        if on_chunk:
            on_chunk(c, run)
    run.finish()
    torch.cuda.synchronize()
    return run, n_checked
