"""Pins of the CPU oracle to things other than itself (runs without a GPU).

* T1  capacity >= sequence length reduces to exact causal attention (the paper,
      §A.5.2: "for N <= N_C our method reduces to standard training"), checked
      against an independently written dense softmax from scipy, including the
      accumulated H2O scores = column sums of the full causal weight matrix.
* T2  invariants: each softmax row sums to one, so the summed weights of a chunk
      add up to S * q_g per KV head; weights are >= 0; a new slot gets no
      weight from rows before its own token (the mask of §A.1).
* T3  slot selection vs brute force over all subsets on tiny caches, tie-heavy.
* T4  the hand-derived four-slot toy in tests/golden/h2o_toy_4slot.json.
* T5  quantization closed forms: exact round trips, error <= scale / 2,
      hand-packed int4 bytes.
* T6  attention closed forms: one visible slot gives y = v and lse = logit;
      zero queries give the mean of the visible values.
* planted mistakes: altered copies of oracle functions must fail the pins.
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
from oracle import (EMPTY_POS, OracleCache, attend_head, attend_head_backward, quantize_rows,
                    select_slots, selection_keys)
from oracle import h2o_oracle as ho

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _frac(s):
    return float(Fraction(s))


# ----------------------------------------------------------------------------
# Independent textbook attention (T1).
# ----------------------------------------------------------------------------
def textbook_causal(Q, K, V):
    """Q: [Hq, N, d], K/V: [Hk, N, d] float64; plain causal softmax attention.
    Returns Y [Hq, N, d], LSE [Hq, N], M [Hq, N, N] (rows i, columns j)."""
    Hq, N, d = Q.shape
    q_g = Hq // K.shape[0]
    Y = np.zeros_like(Q)
    L = np.zeros((Hq, N))
    M = np.zeros((Hq, N, N))
    tri = np.triu(np.ones((N, N), bool), k=1)  # j > i is in the future
    for h in range(Hq):
        g = h // q_g
        logits = np.einsum("id,jd->ij", Q[h], K[g]) / np.sqrt(d)
        logits[tri] = -np.inf
        M[h] = softmax(logits, axis=1)
        L[h] = logsumexp(logits, axis=1)
        Y[h] = np.einsum("ij,jd->id", M[h], V[g])
    return Y, L, M


def run_chunks(cache, Q, K, V, sizes):
    """Feed [B,H,N,d] arrays through the oracle in chunks of the given sizes.
    Returns per-chunk (P, S, y, lse, w, wq, slots) and folds the last w in."""
    out = []
    P = 0
    w_prev = None
    for S in sizes:
        slots = cache.evict_insert(w_prev, K[:, :, P:P + S], V[:, :, P:P + S], S, P)
        y, lse, w, wq = cache.attend(Q[:, :, P:P + S], S, P)
        out.append((P, S, y, lse, w, wq, slots))
        w_prev = w
        P += S
    cache.evict_insert(w_prev, None, None, 0, P)
    return out


def _rand(rng, shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


# ----------------------------------------------------------------------------
# T1
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("sizes,capacity", [([8, 8, 5, 13, 6], 48), ([40], 40), ([1] * 12, 12)])
def test_t1_no_eviction_equals_textbook_causal(sizes, capacity):
    rng = np.random.default_rng(7)
    B, Hq, Hk, d = 2, 4, 2, 16
    N = sum(sizes)
    Q = _rand(rng, (B, Hq, N, d))
    K = _rand(rng, (B, Hk, N, d))
    V = _rand(rng, (B, Hk, N, d))
    cache = OracleCache(B, Hq, Hk, d, capacity, "f32")
    res = run_chunks(cache, Q, K, V, sizes)
    for b in range(B):
        Yt, Lt, Mt = textbook_causal(Q[b].astype(np.float64), K[b].astype(np.float64),
                                     V[b].astype(np.float64))
        for (P, S, y, lse, w, wq, slots) in res:
            np.testing.assert_allclose(y[b], Yt[:, P:P + S], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse[b], Lt[:, P:P + S], rtol=1e-12, atol=1e-12)
            # slots fill left to right: token t sits in slot t
            np.testing.assert_array_equal(slots[b], np.broadcast_to(np.arange(P, P + S), slots[b].shape))
            # per-head summed weights over this chunk's rows = column sums of M
            colsum = Mt[:, P:P + S, :].sum(axis=1)  # [Hq, N]
            np.testing.assert_allclose(wq[b][:, :N], colsum, rtol=1e-12, atol=1e-13)
        # cumulative H2O score = full-sequence column sums summed over each group
        full = Mt.sum(axis=1).reshape(Hk, Hq // Hk, N).sum(axis=1)
        np.testing.assert_allclose(cache.scores[b][:, :N], full, rtol=2e-6, atol=1e-6)
        assert np.all(cache.scores[b][:, N:] == 0)


# ----------------------------------------------------------------------------
# T2
# ----------------------------------------------------------------------------
def _evicting_run(kv="f32", seed=3, d=32, capacity=24, sizes=(8, 8, 8, 8, 5, 8, 3, 8)):
    rng = np.random.default_rng(seed)
    B, Hq, Hk = 2, 6, 2
    N = sum(sizes)
    Q = _rand(rng, (B, Hq, N, d))
    K = _rand(rng, (B, Hk, N, d))
    K[:, :, ::7] *= 4  # a few heavy hitters
    V = _rand(rng, (B, Hk, N, d))
    cache = OracleCache(B, Hq, Hk, d, capacity, kv)
    return cache, run_chunks(cache, Q, K, V, list(sizes)), (Q, K, V)


def test_t2_weight_invariants():
    cache, res, (Q, K, V) = _evicting_run()
    q_g = cache.q_g
    for (P, S, y, lse, w, wq, slots) in res:
        assert np.all(w >= 0) and np.all(wq >= 0)
        np.testing.assert_allclose(w.sum(axis=-1), S * q_g, rtol=1e-12)
        np.testing.assert_allclose(wq.sum(axis=-1), S, rtol=1e-12)
        np.testing.assert_allclose(
            w, wq.reshape(w.shape[0], w.shape[1], q_g, -1).sum(axis=2), rtol=1e-12, atol=1e-15)


def test_t2_new_slot_invisible_to_earlier_rows():
    # With the chunk's keys written, rows 0..k-1 must put zero weight on the
    # slot that holds token P+k.
    rng = np.random.default_rng(11)
    B, Hq, Hk, d, cap, S = 1, 2, 1, 8, 10, 4
    cache = OracleCache(B, Hq, Hk, d, cap, "f32")
    P = 0
    w_prev = None
    for c in range(5):
        k = _rand(rng, (B, Hk, S, d))
        v = _rand(rng, (B, Hk, S, d))
        q = _rand(rng, (B, Hq, S, d))
        slots = cache.evict_insert(w_prev, k, v, S, P)
        y, lse, w, wq = cache.attend(q, S, P)
        for kk in range(1, S):
            _, _, w_trunc, _ = cache.attend(q[:, :, :kk], kk, P)
            assert w_trunc[0, 0, slots[0, 0, kk]] == 0.0
        assert w[0, 0, slots[0, 0, S - 1]] > 0
        w_prev = w
        P += S


# ----------------------------------------------------------------------------
# T3
# ----------------------------------------------------------------------------
def brute_force_select(scores, token_pos, n_new):
    """Search every subset of size n_new for the one whose members all rank
    before every non-member under (occupied?, score, slot)."""
    n = len(scores)

    def key(j):
        occ = token_pos[j] != EMPTY_POS
        return (occ, float(scores[j]) if occ else 0.0, j)

    hits = []
    for sub in itertools.combinations(range(n), n_new):
        rest = [j for j in range(n) if j not in sub]
        if all(key(a) < key(b) for a in sub for b in rest):
            hits.append(list(sub))
    assert len(hits) == 1
    return np.array(hits[0])


def test_t3_selection_brute_force():
    rng = np.random.default_rng(5)
    for trial in range(400):
        n = int(rng.integers(1, 9))
        s = int(rng.integers(0, n + 1))
        scores = rng.integers(0, 3, n).astype(np.float32)  # many ties
        if trial % 3 == 0:
            scores = scores + rng.random(n).astype(np.float32)
        tp = np.arange(n, dtype=np.int64)
        n_empty = int(rng.integers(0, n + 1)) if trial % 4 == 0 else 0
        if n_empty:
            tp[n - n_empty:] = EMPTY_POS
        got = select_slots(scores, tp, s)
        np.testing.assert_array_equal(got, brute_force_select(scores, tp, s))


def test_t3_documented_example():
    scores = np.array([2, 1, 1, 1, 3], np.float32)
    np.testing.assert_array_equal(select_slots(scores, np.arange(5), 2), [1, 2])


# ----------------------------------------------------------------------------
# T4
# ----------------------------------------------------------------------------
def _toy_run(Hq):
    with open(os.path.join(GOLDEN, "h2o_toy_4slot.json")) as f:
        toy = json.load(f)
    cache = OracleCache(1, Hq, 1, 2, 4, "f32")
    rng = np.random.default_rng(0)
    w_prev = None
    results = []
    for ch in toy["chunks"]:
        P = ch["P"]
        toks = np.array([P, P + 1])
        v = np.stack([toks, 10 - toks], axis=-1).astype(np.float32)[None, None]
        k = _rand(rng, (1, 1, 2, 2))
        if w_prev is not None:
            pre = (cache.scores + w_prev.astype(np.float32))[0, 0]
        else:
            pre = cache.scores[0, 0].copy()
        slots = cache.evict_insert(w_prev, k, v, 2, P)
        y, lse, w, wq = cache.attend(np.zeros((1, Hq, 2, 2), np.float32), 2, P)
        results.append((ch, pre, slots, y, lse, w))
        w_prev = w
    return results


def test_t4_hand_derived_toy():
    for ch, pre, slots, y, lse, w in _toy_run(1):
        np.testing.assert_allclose(pre, [_frac(s) for s in ch["scores_before_select"]], rtol=1e-6)
        np.testing.assert_array_equal(slots[0, 0], ch["slots"])
        np.testing.assert_allclose(w[0, 0], [_frac(s) for s in ch["w"]], rtol=1e-14, atol=1e-15)
        exp_lse = [math.log(int(s[4:-1])) for s in ch["lse"]]
        np.testing.assert_allclose(lse[0, 0], exp_lse, rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(y[0, 0], [[_frac(a) for a in r] for r in ch["y"]], rtol=1e-14)


def test_t4_gqa_copy_doubles_weights():
    one = _toy_run(1)
    two = _toy_run(2)
    for (ch, _, s1, _, _, w1), (_, _, s2, y2, _, w2) in zip(one, two):
        np.testing.assert_array_equal(s1, s2)
        np.testing.assert_allclose(w2, 2 * w1, rtol=1e-15)
        np.testing.assert_allclose(y2[0, 0], y2[0, 1])


# ----------------------------------------------------------------------------
# T5
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("kind", ["i8", "i4"])
def test_t5_exact_round_trip(kind):
    qmax = oracle.QMAX[kind]
    rng = np.random.default_rng(2)
    for sigma in [2.0 ** -3, 2.0 ** -7, 0.5, 2.0 ** 4]:
        k = rng.integers(-qmax, qmax + 1, size=(16, 8))
        k[:, 0] = qmax * np.where(rng.random(16) < 0.5, -1, 1)  # max |k| = qmax
        x = (k * sigma).astype(np.float32)
        codes, scales = quantize_rows(x, kind)
        np.testing.assert_array_equal(scales.astype(np.float64), sigma)
        np.testing.assert_array_equal(codes, k)
        np.testing.assert_array_equal(oracle.dequantize_rows(codes, scales), x)


@pytest.mark.parametrize("kind", ["i8", "i4"])
def test_t5_error_bound_and_zero_rows(kind):
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((200, 128)) * rng.choice([0.01, 1, 40], (200, 1))).astype(np.float32)
    x[5] = 0.0
    codes, scales = quantize_rows(x, kind)
    assert np.all(codes[5] == 0) and scales[5] == 0
    err = np.abs(oracle.dequantize_rows(codes, scales) - x)
    assert np.all(err <= scales.astype(np.float64)[:, None] / 2 * (1 + 1e-3) + 1e-30)
    assert np.all(np.abs(codes) <= oracle.QMAX[kind])


def test_t5_int4_packing_by_hand():
    codes = np.array([[1, -1, 7, -8, 0, 3]], np.int8)
    packed = oracle.pack_int4(codes)
    # low nibble = even element: (1 | 0xF<<4), (7 | 0x8<<4), (0 | 3<<4)
    np.testing.assert_array_equal(packed, [[0xF1, 0x87, 0x30]])
    np.testing.assert_array_equal(oracle.unpack_int4(packed), codes)


def test_t5_scale_rounding_by_hand():
    # absmax 1.0 over qmax 127: float32(1/127) rounded to fp16 is 0x2008
    x = np.array([[1.0, -0.5, 0.25, 0.0]], np.float32)
    codes, scales = quantize_rows(x, "i8")
    assert scales.view(np.uint16)[0] == 0x2008
    s = float(np.float16(scales[0]))
    np.testing.assert_array_equal(codes[0], [round(1.0 / s), round(-0.5 / s), round(0.25 / s), 0])


# ----------------------------------------------------------------------------
# T6
# ----------------------------------------------------------------------------
def test_t6_single_visible_slot_and_uniform_queries():
    rng = np.random.default_rng(9)
    d, n = 8, 6
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    tp = np.array([3, 50, 51, EMPTY_POS, 52, 53])
    q = rng.standard_normal((1, d))
    y, lse, m = attend_head(q, K, V, tp, 3)  # only slot 0 (token 3) visible
    np.testing.assert_allclose(y[0], V[0], rtol=1e-15)
    np.testing.assert_allclose(lse[0], q[0] @ K[0] / np.sqrt(d), rtol=1e-14)
    np.testing.assert_array_equal(m[0], [1, 0, 0, 0, 0, 0])
    # zero queries: mean of the visible values, lse = log(#visible)
    y, lse, m = attend_head(np.zeros((3, d)), K, V, tp, 50)
    np.testing.assert_allclose(y[0], V[:2].mean(0), rtol=1e-14)
    np.testing.assert_allclose(y[1], V[:3].mean(0), rtol=1e-14)
    np.testing.assert_allclose(y[2], V[[0, 1, 2, 4]].mean(0), rtol=1e-14)
    np.testing.assert_allclose(lse, np.log([2, 3, 4]), rtol=1e-14)


def test_row_without_visible_slot_convention():
    d = 4
    K = np.ones((3, d))
    V = np.ones((3, d))
    y, lse, m = attend_head(np.ones((2, d)), K, V, np.array([5, EMPTY_POS, 9]), 4)
    assert lse[0] == -np.inf and np.all(y[0] == 0) and np.all(m[0] == 0)
    assert lse[1] == 2.0 and m[1, 0] == 1.0  # q.k / sqrt(d) = 4 / 2


def test_t6_lse_matches_library_logsumexp():
    rng = np.random.default_rng(4)
    d, n, S, P = 16, 40, 7, 30
    K = rng.standard_normal((n, d)) * 3
    V = rng.standard_normal((n, d))
    tp = rng.permutation(n) + 2
    q = rng.standard_normal((S, d))
    y, lse, m = attend_head(q, K, V, tp, P)
    for i in range(S):
        vis = tp <= P + i
        a = q[i] @ K[vis].T / np.sqrt(d)
        np.testing.assert_allclose(lse[i], logsumexp(a), rtol=1e-13)
        np.testing.assert_allclose(m[i, vis], softmax(a), rtol=1e-12)


# ----------------------------------------------------------------------------
# Planted mistakes must fail the pins.
# ----------------------------------------------------------------------------
def _t1_passes():
    try:
        test_t1_no_eviction_equals_textbook_causal([8, 8, 5, 13, 6], 48)
        test_t4_hand_derived_toy()
        test_t6_single_visible_slot_and_uniform_queries()
        return True
    except AssertionError:
        return False


def test_planted_mistakes_are_caught(monkeypatch):
    assert _t1_passes()
    good = ho.attend_head

    def off_by_one_mask(q, keys, values, token_pos, P):
        return good(q, keys, values, token_pos - 1, P)

    def no_scale(q, keys, values, token_pos, P):
        return good(np.asarray(q) * np.sqrt(q.shape[-1]), keys, values, token_pos, P)

    for bad in (off_by_one_mask, no_scale):
        monkeypatch.setattr(ho, "attend_head", bad)
        assert not _t1_passes(), bad.__name__
        monkeypatch.setattr(ho, "attend_head", good)

    good_sel = ho.select_slots

    def ties_to_highest(scores, token_pos, n_new):
        r = good_sel(scores[::-1].copy(), token_pos[::-1].copy(), n_new)
        return np.sort(len(scores) - 1 - r)

    monkeypatch.setattr(ho, "select_slots", ties_to_highest)
    with pytest.raises(AssertionError):
        test_t3_selection_brute_force_with(ho.select_slots)


def test_t3_selection_brute_force_with(sel=select_slots):
    rng = np.random.default_rng(8)
    for _ in range(200):
        n = int(rng.integers(2, 8))
        s = int(rng.integers(1, n))
        scores = rng.integers(0, 2, n).astype(np.float32)
        tp = np.arange(n)
        np.testing.assert_array_equal(sel(scores, tp, s), brute_force_select(scores, tp, s))


# --------------------------------------------------------------------------- #
# Score variants (§3.1.1), replay of logged decisions and the delta encoding of
# an update (§A.5.3).
# --------------------------------------------------------------------------- #
def _golden_modes():
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "h2o_score_modes.json")) as f:
        return json.load(f)


def _tp(vals):
    return np.array([EMPTY_POS if v == "empty" else v for v in vals], np.int64)


def _select_mode(mode, scores, token_pos, P, S):
    """Slots chosen by the oracle's cache for one chunk of a given variant."""
    scores = np.asarray(scores, np.float32)
    B = scores.shape[0]
    n_c = scores.shape[-1]
    c = OracleCache(B, 1, 1, 2, n_c, "f32")
    c.load_state(token_pos=np.broadcast_to(token_pos, (B, 1, n_c)).copy(),
                 scores=scores.reshape(B, 1, n_c), n_filled=n_c,
                 keys=np.zeros((B, 1, n_c, 2), np.float32), values=np.zeros((B, 1, n_c, 2), np.float32))
    kn = np.zeros((B, 1, S, 2), np.float32)
    return c.evict_insert(None, kn, kn, S, P, mode=mode)[:, 0]


def test_t7_score_variants_hand_derived():
    g = _golden_modes()
    for ex in g["h2o_norm"]:
        tp = _tp(ex["token_pos"])
        sc = np.array([ex["scores"]], np.float32)
        keys = selection_keys("h2o_norm", sc[:, None], tp[None, None], ex["P"])[0, 0]
        for j, k in enumerate(ex["keys"]):
            if k != "empty":
                assert keys[j] == np.float32(float(_frac(k)))
        assert _select_mode("h2o_norm", sc, tp, ex["P"], ex["S"])[0].tolist() == ex["slots"]
        assert _select_mode("h2o", sc, tp, ex["P"], ex["S"])[0].tolist() == ex["slots_h2o"]
    for ex in g["h2o_orig"]:
        tp = _tp(ex["token_pos"])
        sc = np.array(ex["scores"], np.float32)
        got = _select_mode("h2o_orig", sc, tp, 100, ex["S"])
        for b in range(sc.shape[0]):
            assert got[b].tolist() == ex["slots"]
        per_b = _select_mode("h2o", sc, tp, 100, ex["S"])
        assert [r.tolist() for r in per_b] == ex["slots_h2o"]


def test_t7_score_variants_special_cases():
    rng = np.random.default_rng(17)
    for _ in range(50):
        n_c, S = 12, 4
        sc = rng.permutation(n_c).astype(np.float32)[None] + 1.0  # distinct scores
        # every entry of the same age (a power of two): h2o_norm orders like h2o
        tp = np.full(n_c, 3, np.int64)
        a = _select_mode("h2o_norm", sc, tp, 3 + 8, S)
        b = _select_mode("h2o", sc, tp, 3 + 8, S)
        assert np.array_equal(a, b)
        # one batch position, or identical rows: h2o_orig orders like h2o
        assert np.array_equal(_select_mode("h2o_orig", sc, np.arange(n_c), 50, S),
                              _select_mode("h2o", sc, np.arange(n_c), 50, S))
        two = np.concatenate([sc, sc])
        assert np.array_equal(_select_mode("h2o_orig", two, np.arange(n_c), 50, S)[0],
                              _select_mode("h2o", sc, np.arange(n_c), 50, S)[0])


def _brute(keys64, token_pos, S):
    best = None
    for sub in itertools.combinations(range(len(keys64)), S):
        lst = sorted(((0, 0.0, j) if token_pos[j] == EMPTY_POS else (1, keys64[j], j)) for j in sub)
        if best is None or lst < best[0]:
            best = (lst, sub)
    return sorted(best[1])


def test_t7_score_variants_brute_force():
    rng = np.random.default_rng(5)
    for _ in range(200):
        n_c, P = int(rng.integers(3, 9)), 40
        S = int(rng.integers(1, n_c + 1))
        tp = rng.integers(0, P, n_c).astype(np.int64)
        tp[rng.random(n_c) < 0.2] = EMPTY_POS
        # small integer scores: float32 sums are exact, quotients are compared in float64
        sc = rng.integers(0, 6, (2, n_c)).astype(np.float32)
        occ = tp != EMPTY_POS
        norm64 = np.where(occ, sc[0].astype(np.float64) / np.where(occ, P - tp, 1), 0.0)
        # compare where float32 rounding merges no two distinct float64 keys
        if len(set(norm64[occ].tolist())) == len(set(np.float32(norm64[occ]).tolist())):
            assert _select_mode("h2o_norm", sc[:1], tp, P, S)[0].tolist() == _brute(norm64, tp, S)
        orig64 = sc[0].astype(np.float64) + sc[1]
        got = _select_mode("h2o_orig", sc, tp, P, S)
        assert got[0].tolist() == got[1].tolist() == _brute(orig64, tp, S)


def test_t8_replay_reproduces_the_cache():
    rng = np.random.default_rng(9)
    for kv in ("f32", "i8", "i4"):
        B, Hq, Hk, d, n_c = 2, 4, 2, 16, 20
        a = OracleCache(B, Hq, Hk, d, n_c, kv)
        r = OracleCache(B, Hq, Hk, d, n_c, kv)
        P = 0
        w = None
        for S in (8, 8, 6, 8, 5, 8):
            kn = _rand(rng, (B, Hk, S, d))
            vn = _rand(rng, (B, Hk, S, d))
            q = _rand(rng, (B, Hq, S, d))
            slots = a.evict_insert(w, kn, vn, S, P, mode="h2o_norm" if P else "h2o")
            r.evict_insert(w, kn, vn, S, P, slots=slots)
            for name in ("token_pos", "scores") + (("k_codes", "v_codes", "k_scales", "v_scales")
                                                    if kv != "f32" else ("k_store", "v_store")):
                assert np.array_equal(getattr(a, name), getattr(r, name)), name
            _, _, w, _ = a.attend(q, S, P)
            w = w.astype(np.float32)
            P += S


def test_t9_delta_encoding_round_trip():
    rng = np.random.default_rng(21)
    for kv in ("f32", "bf16", "i8", "i4"):
        B, Hq, Hk, d, n_c = 2, 2, 2, 8, 12
        c = OracleCache(B, Hq, Hk, d, n_c, kv)
        P = 0
        w = None
        for S in (6, 6, 5, 6, 6):
            names = ("token_pos",) + (("k_codes", "v_codes", "k_scales", "v_scales")
                                      if kv in ("i8", "i4") else ("k_store", "v_store"))
            before = {n: getattr(c, n).copy() for n in names}
            kn = _rand(rng, (B, Hk, S, d))
            vn = _rand(rng, (B, Hk, S, d))
            slots, dl = c.evict_insert(w, kn, vn, S, P, delta=True)
            # the delta rows are the overwritten rows: gather(keys, index)
            for b in range(B):
                for g in range(Hk):
                    src = "k_codes" if kv in ("i8", "i4") else "k_store"
                    assert np.array_equal(dl["keys"][b, g], before[src][b, g, slots[b, g]])
                    assert np.array_equal(dl["token_pos"][b, g], before["token_pos"][b, g, slots[b, g]])
            after = {n: getattr(c, n).copy() for n in names}
            c.restore(slots, dl)
            for n in names:
                assert np.array_equal(getattr(c, n), before[n]), n
            # redo the update (the cache moves on)
            c.restore(slots, {"keys": after[names[1]][np.arange(B)[:, None, None], np.arange(Hk)[None, :, None], slots],
                              "values": after[names[2]][np.arange(B)[:, None, None], np.arange(Hk)[None, :, None], slots],
                              "token_pos": after["token_pos"][np.arange(B)[:, None, None], np.arange(Hk)[None, :, None], slots],
                              **({"k_scales": after["k_scales"][np.arange(B)[:, None, None], np.arange(Hk)[None, :, None], slots],
                                  "v_scales": after["v_scales"][np.arange(B)[:, None, None], np.arange(Hk)[None, :, None], slots]}
                                 if kv in ("i8", "i4") else {})})
            for n in names:
                assert np.array_equal(getattr(c, n), after[n]), n
            q = _rand(rng, (B, Hq, S, d))
            _, _, w, _ = c.attend(q, S, P)
            w = w.astype(np.float32)
            P += S


def test_t7_planted_age_off_by_one_is_caught(monkeypatch):
    import oracle.h2o_oracle as ho
    good = ho.selection_keys

    def age_plus_one(mode, scores, token_pos, P):
        return good(mode, scores, token_pos, P + 1)

    monkeypatch.setattr(ho, "selection_keys", age_plus_one)
    with pytest.raises(AssertionError):
        test_t7_score_variants_hand_derived()


# --------------------------------------------------------------------------- #
# Gradients of the chunk's SDPA over the cache (§A.5 autograd per chunk).
# --------------------------------------------------------------------------- #
def _loss(q, k, v, tp, P, dy):
    y, _, _ = attend_head(q, k, v, tp, P)
    return float(np.sum(y * dy))


def test_t10_backward_matches_finite_differences():
    """Central differences of L = sum(dy * y) along random directions: pins every
    term of the analytic gradient without restating its formula."""
    rng = np.random.default_rng(41)
    for P, n_c, S, d in ((0, 9, 6, 5), (7, 12, 4, 8)):
        q = rng.standard_normal((S, d))
        k = rng.standard_normal((n_c, d))
        v = rng.standard_normal((n_c, d))
        tp = rng.integers(0, P + S, n_c).astype(np.int64)
        tp[0] = 0  # every row sees at least one slot
        tp[rng.random(n_c) < 0.2] = EMPTY_POS
        tp[0] = 0
        dy = rng.standard_normal((S, d))
        dq, dk, dv = attend_head_backward(q, k, v, tp, P, dy)
        h = 1e-6
        for grad, which in ((dq, 0), (dk, 1), (dv, 2)):
            for _ in range(3):
                dirn = rng.standard_normal(grad.shape)
                args = [q, k, v]
                plus = [a.copy() for a in args]
                minus = [a.copy() for a in args]
                plus[which] = plus[which] + h * dirn
                minus[which] = minus[which] - h * dirn
                fd = (_loss(*plus, tp, P, dy) - _loss(*minus, tp, P, dy)) / (2 * h)
                assert abs(fd - float(np.sum(grad * dirn))) <= 1e-6 * max(1.0, abs(fd))


def test_t10_backward_closed_forms():
    rng = np.random.default_rng(43)
    d = 6
    # one visible slot: y = v_0, so dv_0 = sum of dy, dq = 0, dk = 0
    q = rng.standard_normal((3, d))
    k = rng.standard_normal((4, d))
    v = rng.standard_normal((4, d))
    tp = np.array([0, EMPTY_POS, EMPTY_POS, EMPTY_POS])
    dy = rng.standard_normal((3, d))
    dq, dk, dv = attend_head_backward(q, k, v, tp, 5, dy)
    assert np.allclose(dv[0], dy.sum(axis=0)) and np.allclose(dv[1:], 0)
    assert np.allclose(dq, 0) and np.allclose(dk, 0)
    # q = 0 (uniform weights over the visible slots): dk = 0, dv_j = sum_i dy_i / n_i
    tp = np.array([0, 1, 2, 3])
    q0 = np.zeros((4, d))
    dq, dk, dv = attend_head_backward(q0, k, v, tp, 0, dy := rng.standard_normal((4, d)))
    assert np.allclose(dk, 0)
    want = np.zeros((4, d))
    for i in range(4):
        for j in range(i + 1):
            want[j] += dy[i] / (i + 1)
    assert np.allclose(dv, want)
    # identical keys: every row's weights are uniform whatever q is, so dq = 0
    kk = np.tile(rng.standard_normal((1, d)), (4, 1))
    dq, _, _ = attend_head_backward(rng.standard_normal((4, d)), kk, v, tp, 0, dy)
    assert np.allclose(dq, 0)


def test_t10_cache_backward_sums_group_heads():
    rng = np.random.default_rng(47)
    c = OracleCache(1, 2, 1, 4, 6, "f32")
    c.evict_insert(None, _rand(rng, (1, 1, 6, 4)), _rand(rng, (1, 1, 6, 4)), 6, 0)
    q = _rand(rng, (1, 1, 6, 4))
    dy = _rand(rng, (1, 1, 6, 4))
    q2 = np.concatenate([q, q], axis=1)
    dy2 = np.concatenate([dy, dy], axis=1)
    dq, dk, dv = c.attend_backward(q2, dy2, 6, 0)
    a, bk, bv = attend_head_backward(q[0, 0], c.keys(0, 0), c.values(0, 0), c.token_pos[0, 0], 0, dy[0, 0])
    assert np.allclose(dk[0, 0], 2 * bk) and np.allclose(dv[0, 0], 2 * bv)
    assert np.allclose(dq[0, 0], a) and np.allclose(dq[0, 1], a)
