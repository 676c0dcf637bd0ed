"""Float64 CPU oracle for chunked KV-cache attention with H2O scoring and eviction.

TEST INFRASTRUCTURE.  Only tests, the smoke check and the benchmark's CPU-baseline
leg use this module; the CUDA library never does.  It shares no code, header or
table with the CUDA path.

Source: "Learning how to Forget: Fine-tuning for Long-Context Sparse Attention"
(the paper of the KeysAndValues library).  Section references below are to that
paper:

* §3.1 "Sparse Attention. Key-Value Caching": cache buffers ``keys, values`` of
  shape (B, H_k, N_C, d_h) and ``token_pos`` of shape (B, H_k, N_C); filled left
  to right up to N_C, then a per-(b, h) policy chooses the slots that new tokens
  overwrite; a sequence is processed in chunks of S tokens; GQA maps q_g
  consecutive query heads to one KV head (H_q = H_k * q_g).
* §A.1 "SDPA Kernels for Sparse Attention": the causal mask for a call that
  processes tokens P..P+N_q-1 is -inf where P + i < token_pos[b, h, j]; the new
  keys/values are written into the cache before SDPA runs.
* §A.7 "Computing Summed Attention Weights in SDPA": SDPA is
  softmax(mask(d_h^{-1/2} Q K^T)) V (the paper's eq. (2), lost in extraction, is
  read as this); the summed attention weights sum_i m[b,h,i,j] have shape
  (B, H_q, N_k); the log-sum-exp of a row is log(sum_j exp(a_ij)).
* §3.1.1 "Variants of Heavy-Hitter Oracle": the H2O score of an entry is the
  cumulative sum of its attention weights while it sits in the cache (the
  paper's eq. (3), read as this); the entry with the lowest score is evicted.
* §A.5.3: the buffer update is keys' = scatter(keys, index, key_new) (eq. (4));
  the delta encoding of an update is delta_key = gather(keys, index), from which
  keys is rebuilt as scatter(keys', index, delta_key).
* §3.1.1 also defines two score variants: h2o_orig selects the same slots for
  every batch position by the score summed over b, and h2o_norm divides an
  entry's score by its age t - t(b, h, j).
* §3.2 / §A.5: eviction decisions are written to a replay log in the forward
  pass and replayed by replay caches (insertion at given slots).
* §2 "Related Work" and the library's feature list in §A.10: cache buffers may
  be quantized to 8 or 4 bits.  The paper gives no scheme; the oracle uses a
  symmetric per-(token, KV-head) absmax scheme with an fp16 scale (see
  ``quantize_rows``).

Readings where the pages are silent (each one is listed again in the design
notes): h2o_norm's time t (undefined in the pages) is P, the position of the
chunk's first token, so an entry's age P - t(b, h, j) >= 1 counts the query
positions that could attend to it; the normalised key is the float32 quotient
float32(score) / float32(age), the same precision the kernel decides in;
h2o_orig's summed score is accumulated in float32 in batch order; the GQA reduction of the summed weights is a SUM over the group's query
heads; ties between equal scores go to the lowest slot index; chosen slots are
filled in ascending slot order with the chunk's tokens in order; a new slot
starts with score 0 and then accumulates its own chunk's weights; empty slots
are taken before any occupied slot; scores are stored in float32 and updated as
float32(score + float32(w)).
"""

from __future__ import annotations

import math

import numpy as np

#: token position stored in a slot that holds no token (masked for every query).
EMPTY_POS = np.iinfo(np.int32).max

#: largest code magnitude of the symmetric 8-bit and 4-bit cache formats.
QMAX = {"i8": 127, "i4": 7}

_F16_MAX = 65504.0


# --------------------------------------------------------------------------- #
# Quantization of cache rows (8/4-bit; the paper gives only the bit widths).
# --------------------------------------------------------------------------- #
def quantize_rows(x: np.ndarray, kind: str):
    """Quantize rows of ``x`` (float32 values of bf16 inputs), one scale per row.

    Scheme (the paper states only "8 or 4 bits", §2 / §A.10; this reading is the
    plainest symmetric absmax one):

    * absmax = max_e |x_e| over the row (the head dimension), exact in float32;
    * scale = fp16 round-to-nearest-even of float32(absmax / qmax), saturated to
      the largest finite fp16 value (65504);
    * code_e = clamp(round-half-even(float32(x_e / float32(scale))), -qmax, qmax);
      a zero scale gives all-zero codes.

    Returns ``(codes int8 [..., d], scales float16 [...])``.
    """
    qmax = QMAX[kind]
    x = np.asarray(x, dtype=np.float32)
    absmax = np.max(np.abs(x), axis=-1)
    ratio = absmax / np.float32(qmax)  # float32 IEEE division
    ratio = np.minimum(ratio, np.float32(_F16_MAX))
    scales = ratio.astype(np.float16)  # round to nearest even
    s32 = scales.astype(np.float32)
    codes = np.zeros(x.shape, dtype=np.int8)
    nz = s32 > 0
    if np.any(nz):
        q = x[nz] / s32[nz][..., None]  # float32 IEEE division
        q = np.rint(q)  # round half to even
        q = np.clip(q, -qmax, qmax)
        codes[nz] = q.astype(np.int8)
    return codes, scales


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Exact float64 value of stored codes: code * scale."""
    return codes.astype(np.float64) * scales.astype(np.float64)[..., None]


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Pack 4-bit two's-complement codes two per byte: element 2e in the low
    nibble, element 2e+1 in the high nibble."""
    c = codes.astype(np.int16) & 0xF
    lo = c[..., 0::2]
    hi = c[..., 1::2]
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """Inverse of ``pack_int4``; returns int8 codes in [-8, 7]."""
    p = packed.astype(np.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


# --------------------------------------------------------------------------- #
# H2O slot selection (§3.1, §3.1.1).
# --------------------------------------------------------------------------- #
def select_slots(scores: np.ndarray, token_pos: np.ndarray, n_new: int) -> np.ndarray:
    """Slots that the ``n_new`` tokens of a chunk overwrite, for one (b, h).

    Empty slots first, lowest index first (the cache fills left to right, §3.1);
    then the occupied slots with the smallest (score, slot index) pairs, i.e. the
    lowest H2O score, ties to the lowest slot (§3.1.1; the tie rule is a
    reading).  The result is sorted ascending: chunk token k goes to the k-th
    smallest chosen slot.
    """
    n_c = scores.shape[0]
    if n_new > n_c:
        raise ValueError("chunk larger than the cache")

    def key(j):
        empty = token_pos[j] == EMPTY_POS
        return (0 if empty else 1, 0.0 if empty else float(scores[j]), j)

    chosen = sorted(range(n_c), key=key)[:n_new]
    return np.array(sorted(chosen), dtype=np.int64)


SCORE_MODES = ("h2o", "h2o_norm", "h2o_orig")


def selection_keys(mode: str, scores: np.ndarray, token_pos: np.ndarray, P: int) -> np.ndarray:
    """Per-slot selection key [B, H_k, N_C] (float32) of a score variant (§3.1.1).

    h2o:      the cumulative score itself.
    h2o_norm: score / (t - t(b, h, j)) with t = P (a reading), in float32; empty
              slots are taken first whatever their key, so their key is 0.
    h2o_orig: sum over batch positions b of the scores (float32, b in order); the
              same key, hence the same slots, for every b.
    """
    scores = np.asarray(scores, np.float32)
    if mode == "h2o":
        return scores.copy()
    if mode == "h2o_norm":
        occupied = token_pos != EMPTY_POS
        age = np.where(occupied, P - np.asarray(token_pos, np.int64), 1).astype(np.float32)
        if np.any(age[occupied] < 1):
            raise ValueError("an occupied slot holds a token at or after the chunk start")
        return np.where(occupied, scores / age, np.float32(0)).astype(np.float32)
    if mode == "h2o_orig":
        total = np.zeros(scores.shape[1:], np.float32)
        for b in range(scores.shape[0]):
            total = (total + scores[b]).astype(np.float32)
        return np.broadcast_to(total, scores.shape).copy()
    raise ValueError(f"unknown score mode {mode!r}")


# --------------------------------------------------------------------------- #
# SDPA with the token-position mask and summed weights (§A.1, §A.7).
# --------------------------------------------------------------------------- #
def attend_head(q: np.ndarray, keys: np.ndarray, values: np.ndarray,
                token_pos: np.ndarray, P: int):
    """One query head against one cache head, float64.

    q: [S, d] queries for tokens P..P+S-1; keys, values: [N_C, d] (already
    dequantized); token_pos: [N_C].
    Returns (y [S, d], lse [S], m [S, N_C]) where m is the attention-weight
    matrix: a_ij = q_i . k_j / sqrt(d), -inf where P + i < token_pos[j];
    m = softmax over j; y = m V; lse_i = log sum_j exp(a_ij).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(keys, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    S, d = q.shape
    a = (q @ k.T) / math.sqrt(d)
    rows = P + np.arange(S, dtype=np.int64)[:, None]
    masked = rows < token_pos.astype(np.int64)[None, :]
    a = np.where(masked, -np.inf, a)
    seen = ~np.all(masked, axis=1)
    amax = np.max(a, axis=1, keepdims=True)
    amax = np.where(seen[:, None], amax, 0.0)
    e = np.exp(a - amax)
    total = np.sum(e, axis=1, keepdims=True)
    # A row with no visible slot (only possible if the chunk's own keys were not
    # inserted first) has an empty softmax: by convention it gets zero weights,
    # y = 0 and lse = -inf.
    m = e / np.where(seen[:, None], total, 1.0)
    y = m @ v
    with np.errstate(divide="ignore"):
        lse = (amax + np.log(total))[:, 0]
    return y, lse, m


def attend_head_backward(q: np.ndarray, keys: np.ndarray, values: np.ndarray,
                         token_pos: np.ndarray, P: int, dy: np.ndarray):
    """Gradients of one head's SDPA over the cache (§A.5: autograd through the
    attention of each chunk; the cache policy itself is not differentiated).

    For L = sum(dy * y) with y = m V, m = softmax_j(a), a_ij = q_i . k_j / sqrt(d)
    (masked entries fixed at -inf): dV = m^T dy; dm = dy V^T;
    da = m * (dm - rowsum(m * dm)); dq = da K / sqrt(d); dK = da^T q / sqrt(d).
    Returns (dq [S, d], dk [N_C, d], dv [N_C, d]) in float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(keys, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    d = q.shape[1]
    _, _, m = attend_head(q, k, v, token_pos, P)
    dv = m.T @ dy
    dm = dy @ v.T
    da = m * (dm - np.sum(m * dm, axis=1, keepdims=True))
    dq = (da @ k) / math.sqrt(d)
    dk = (da.T @ q) / math.sqrt(d)
    return dq, dk, dv


# --------------------------------------------------------------------------- #
# One attention layer's cache, processed chunk by chunk (§3.1, §A.1, §A.5.3).
# --------------------------------------------------------------------------- #
class OracleCache:
    """State of one layer's fixed-capacity cache and its H2O scores.

    kv_dtype: "f32" or "bf16" (values stored as given: the caller passes values
    already rounded to the storage type), "i8" or "i4" (stored as codes and fp16
    scales, read back exactly as code * scale).
    """

    def __init__(self, B, Hq, Hk, d, capacity, kv_dtype="bf16"):
        if Hq % Hk:
            raise ValueError("H_q must be a multiple of H_k")
        self.B, self.Hq, self.Hk, self.d, self.N_C = B, Hq, Hk, d, capacity
        self.q_g = Hq // Hk
        self.kv_dtype = kv_dtype
        self.quantized = kv_dtype in QMAX
        shape = (B, Hk, capacity, d)
        if self.quantized:
            self.k_codes = np.zeros(shape, np.int8)
            self.v_codes = np.zeros(shape, np.int8)
            self.k_scales = np.zeros(shape[:3], np.float16)
            self.v_scales = np.zeros(shape[:3], np.float16)
        else:
            self.k_store = np.zeros(shape, np.float32)
            self.v_store = np.zeros(shape, np.float32)
        self.token_pos = np.full((B, Hk, capacity), EMPTY_POS, np.int64)
        self.scores = np.zeros((B, Hk, capacity), np.float32)
        self.n_filled = 0

    # -- buffers as float64 values -------------------------------------------
    def keys(self, b, g):
        if self.quantized:
            return dequantize_rows(self.k_codes[b, g], self.k_scales[b, g])
        return self.k_store[b, g].astype(np.float64)

    def values(self, b, g):
        if self.quantized:
            return dequantize_rows(self.v_codes[b, g], self.v_scales[b, g])
        return self.v_store[b, g].astype(np.float64)

    # -- H2O score update, selection and overwrite ---------------------------
    def evict_insert(self, w_prev, k_new, v_new, S, P, mode="h2o", slots=None, delta=False):
        """Fold the previous chunk's summed weights into the scores, choose S
        slots per (b, h_k) and overwrite them with the chunk's keys/values.

        w_prev: [B, H_k, N_C] or None.  k_new, v_new: [B, H_k, S, d] float32
        values of the storage type (bf16-rounded for bf16/i8/i4 caches).
        mode: the score variant that ranks occupied slots (``SCORE_MODES``).
        slots: [B, H_k, S] slots to write instead of choosing them (replay of a
        logged decision, §A.5); each (b, h_k) row must hold distinct slots.
        delta: also return the rows the update overwrites (§A.5.3's
        delta_key = gather(keys, index)), as a dict of arrays indexed like the
        chunk: "keys", "values" (stored values, or codes and "k_scales",
        "v_scales" for quantized caches) and "token_pos".
        Returns the slots [B, H_k, S] (ascending per (b, h_k) when chosen here),
        and the delta dict when ``delta`` is set.
        """
        if w_prev is not None:
            self.scores = (self.scores + np.asarray(w_prev, np.float32)).astype(np.float32)
        out = np.zeros((self.B, self.Hk, S), np.int64)
        d = None
        if delta:
            shape = (self.B, self.Hk, S)
            if self.quantized:
                d = {"keys": np.zeros(shape + (self.d,), np.int8),
                     "values": np.zeros(shape + (self.d,), np.int8),
                     "k_scales": np.zeros(shape, np.float16), "v_scales": np.zeros(shape, np.float16)}
            else:
                d = {"keys": np.zeros(shape + (self.d,), np.float32),
                     "values": np.zeros(shape + (self.d,), np.float32)}
            d["token_pos"] = np.zeros(shape, np.int64)
        if S == 0:
            return (out, d) if delta else out
        if slots is None:
            keys = selection_keys(mode, self.scores, self.token_pos, P)
        for b in range(self.B):
            for g in range(self.Hk):
                if slots is None:
                    chosen = select_slots(keys[b, g], self.token_pos[b, g], S)
                else:
                    chosen = np.asarray(slots[b, g], np.int64)
                    if len(set(chosen.tolist())) != S or chosen.min() < 0 or chosen.max() >= self.N_C:
                        raise ValueError("replayed slots must be distinct and inside the cache")
                out[b, g] = chosen
                if delta:
                    if self.quantized:
                        d["keys"][b, g] = self.k_codes[b, g, chosen]
                        d["values"][b, g] = self.v_codes[b, g, chosen]
                        d["k_scales"][b, g] = self.k_scales[b, g, chosen]
                        d["v_scales"][b, g] = self.v_scales[b, g, chosen]
                    else:
                        d["keys"][b, g] = self.k_store[b, g, chosen]
                        d["values"][b, g] = self.v_store[b, g, chosen]
                    d["token_pos"][b, g] = self.token_pos[b, g, chosen]
                kk = np.asarray(k_new[b, g], np.float32)
                vv = np.asarray(v_new[b, g], np.float32)
                if self.quantized:
                    kc, ks = quantize_rows(kk, self.kv_dtype)
                    vc, vs = quantize_rows(vv, self.kv_dtype)
                    self.k_codes[b, g, chosen] = kc
                    self.k_scales[b, g, chosen] = ks
                    self.v_codes[b, g, chosen] = vc
                    self.v_scales[b, g, chosen] = vs
                else:
                    self.k_store[b, g, chosen] = kk
                    self.v_store[b, g, chosen] = vv
                self.token_pos[b, g, chosen] = P + np.arange(S)
                self.scores[b, g, chosen] = 0.0
        self.n_filled = min(self.N_C, self.n_filled + S)
        return (out, d) if delta else out

    def restore(self, slots, d):
        """Undo an update from its delta encoding: scatter the overwritten rows and
        token positions back into ``slots`` (the recurrence of §A.5.3 played
        backwards).  Scores are not restored."""
        for b in range(self.B):
            for g in range(self.Hk):
                chosen = np.asarray(slots[b, g], np.int64)
                if self.quantized:
                    self.k_codes[b, g, chosen] = d["keys"][b, g]
                    self.v_codes[b, g, chosen] = d["values"][b, g]
                    self.k_scales[b, g, chosen] = d["k_scales"][b, g]
                    self.v_scales[b, g, chosen] = d["v_scales"][b, g]
                else:
                    self.k_store[b, g, chosen] = d["keys"][b, g]
                    self.v_store[b, g, chosen] = d["values"][b, g]
                self.token_pos[b, g, chosen] = d["token_pos"][b, g]

    # -- SDPA over the cache with summed weights -----------------------------
    def attend(self, q, S, P):
        """q: [B, H_q, S, d].  Returns y [B,H_q,S,d], lse [B,H_q,S],
        w [B,H_k,N_C] (summed over rows and the group's query heads) and
        wq [B,H_q,N_C] (summed over rows only), all float64."""
        B, Hq, Hk, d, N_C = self.B, self.Hq, self.Hk, self.d, self.N_C
        y = np.zeros((B, Hq, S, d))
        lse = np.zeros((B, Hq, S))
        wq = np.zeros((B, Hq, N_C))
        w = np.zeros((B, Hk, N_C))
        for b in range(B):
            for g in range(Hk):
                K = self.keys(b, g)
                V = self.values(b, g)
                tp = self.token_pos[b, g]
                for r in range(self.q_g):
                    h = g * self.q_g + r
                    yh, lh, m = attend_head(q[b, h], K, V, tp, P)
                    y[b, h] = yh
                    lse[b, h] = lh
                    wq[b, h] = m.sum(axis=0)
                    w[b, g] += wq[b, h]
        return y, lse, w, wq

    # -- gradients of the chunk's SDPA over the cache -------------------------
    def attend_backward(self, q, dy, S, P):
        """q, dy: [B, H_q, S, d].  Returns dq [B, H_q, S, d] and dk, dv
        [B, H_k, N_C, d] (summed over the group's query heads), float64, with
        respect to the stored (dequantized) keys and values."""
        B, Hq, Hk, d, N_C = self.B, self.Hq, self.Hk, self.d, self.N_C
        dq = np.zeros((B, Hq, S, d))
        dk = np.zeros((B, Hk, N_C, d))
        dv = np.zeros((B, Hk, N_C, d))
        for b in range(B):
            for g in range(Hk):
                K, V = self.keys(b, g), self.values(b, g)
                for r in range(self.q_g):
                    h = g * self.q_g + r
                    a, bk, bv = attend_head_backward(q[b, h], K, V, self.token_pos[b, g], P, dy[b, h])
                    dq[b, h] = a
                    dk[b, g] += bk
                    dv[b, g] += bv
        return dq, dk, dv

    # -- state transfer (re-seeding from another implementation) -------------
    def load_state(self, *, token_pos, scores, n_filled, keys=None, values=None,
                   k_codes=None, v_codes=None, k_scales=None, v_scales=None):
        """Replace the whole cache state (used to re-seed from a captured state)."""
        self.token_pos = np.asarray(token_pos, np.int64).copy()
        self.scores = np.asarray(scores, np.float32).copy()
        self.n_filled = int(n_filled)
        if self.quantized:
            self.k_codes = np.asarray(k_codes, np.int8).copy()
            self.v_codes = np.asarray(v_codes, np.int8).copy()
            self.k_scales = np.asarray(k_scales, np.float16).copy()
            self.v_scales = np.asarray(v_scales, np.float16).copy()
        else:
            self.k_store = np.asarray(keys, np.float32).copy()
            self.v_store = np.asarray(values, np.float32).copy()
