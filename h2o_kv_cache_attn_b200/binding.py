"""Python binding of the C ABI in ``include/h2okv.h`` (ctypes).

Argument marshalling only: every step of the computation runs in the CUDA
library.  The functions keep the C names; tensors are torch tensors on the
library's device (dtype, shape and contiguity are checked here, sizes and
values again in C).  If ``libh2okv.so`` cannot be loaded, every call raises:
there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libh2okv.so")

F32, BF16, I8, I4 = 0, 1, 2, 3
DTYPE_CODE = {"f32": F32, "bf16": BF16, "i8": I8, "i4": I4}
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, -1, -2, -3, -4
EMPTY_POS = 2**31 - 1
BUF_NAMES = ("keys", "values", "k_scales", "v_scales", "token_pos", "scores", "workspace")
EXPORTED = ("kv_cache_query_sizes", "kv_cache_create", "kv_cache_reset", "kv_cache_destroy",
            "kv_cache_get_fill", "kv_cache_set_fill", "kv_cache_quantize", "h2o_evict_insert",
            "attn_chunk_with_scoresum", "kv_cache_device_status", "kv_cache_set_wait_timeout",
            "attn_chunk_with_scoresum_noalloc", "h2okv_last_error", "h2okv_abi_version",
            "kv_cache_set_score_mode", "h2o_evict_insert_delta", "h2o_insert_at",
            "kv_cache_restore", "attn_chunk_backward", "h2o_evict_insert_many")
SCORE_MODE = {"h2o": 0, "h2o_norm": 1, "h2o_orig": 2}


class H2OKVError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"h2okv error {code}: {msg}")
        self.code = code


class CacheDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("max_chunk", ctypes.c_int32),
                ("q_dtype", ctypes.c_int32), ("kv_dtype", ctypes.c_int32)]


class Delta(ctypes.Structure):
    _fields_ = [("keys", ctypes.c_void_p), ("values", ctypes.c_void_p),
                ("k_scales", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("token_pos", ctypes.c_void_p)]


class CacheBuffers(ctypes.Structure):
    _fields_ = [("keys", ctypes.c_void_p), ("values", ctypes.c_void_p),
                ("k_scales", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("token_pos", ctypes.c_void_p), ("scores", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p)]


_lib = None


def lib_path() -> str:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Load the library (once).  Raises if it is missing or incomplete."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {_LIB_PATH} (run "
                           "`python -m h2o_kv_cache_attn_b200.build`)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "kv_cache_query_sizes": (ctypes.c_int, [ctypes.POINTER(CacheDesc), ctypes.POINTER(sz)]),
        "kv_cache_create": (ctypes.c_int, [ctypes.POINTER(CacheDesc), ctypes.POINTER(CacheBuffers),
                                           vp, ctypes.POINTER(vp)]),
        "kv_cache_reset": (ctypes.c_int, [vp, vp]),
        "kv_cache_destroy": (ctypes.c_int, [vp]),
        "kv_cache_get_fill": (ctypes.c_int, [vp, ctypes.POINTER(i32)]),
        "kv_cache_set_fill": (ctypes.c_int, [vp, i32]),
        "kv_cache_quantize": (ctypes.c_int, [i32, vp, i64, i32, vp, vp, vp]),
        "h2o_evict_insert": (ctypes.c_int, [vp, vp, vp, vp, i32, i64, vp, vp]),
        "attn_chunk_with_scoresum": (ctypes.c_int, [vp, vp, i32, i64, vp, vp, vp, vp, vp]),
        "kv_cache_device_status": (ctypes.c_int, [vp, ctypes.POINTER(i32), vp]),
        "kv_cache_set_wait_timeout": (ctypes.c_int, [vp, ctypes.c_uint64]),
        "attn_chunk_with_scoresum_noalloc": (ctypes.c_int, [ctypes.POINTER(CacheDesc), vp, vp, vp, vp,
                                                            vp, vp, i32, i64, vp, vp, vp, vp, vp]),
        "kv_cache_set_score_mode": (ctypes.c_int, [vp, i32]),
        "h2o_evict_insert_delta": (ctypes.c_int, [vp, vp, vp, vp, i32, i64, vp,
                                                  ctypes.POINTER(Delta), vp]),
        "h2o_insert_at": (ctypes.c_int, [vp, vp, vp, vp, i32, i64, vp, ctypes.POINTER(Delta), vp]),
        "kv_cache_restore": (ctypes.c_int, [vp, vp, i32, ctypes.POINTER(Delta), vp]),
        "attn_chunk_backward": (ctypes.c_int, [vp, vp, vp, vp, i32, i64, vp, vp, vp, vp]),
        "h2o_evict_insert_many": (ctypes.c_int, [ctypes.POINTER(vp), i32, ctypes.POINTER(vp),
                                                 ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i64,
                                                 ctypes.POINTER(vp), vp]),
        "h2okv_last_error": (ctypes.c_char_p, []),
        "h2okv_abi_version": (i32, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)  # AttributeError if a symbol is missing
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(rc: int):
    if rc != OK:
        raise H2OKVError(rc, load().h2okv_last_error().decode())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ---- thin wrappers with the C names ------------------------------------------
def kv_cache_query_sizes(desc: CacheDesc) -> dict:
    arr = (ctypes.c_size_t * len(BUF_NAMES))()
    _check(load().kv_cache_query_sizes(ctypes.byref(desc), arr))
    return dict(zip(BUF_NAMES, list(arr)))


def kv_cache_create(desc: CacheDesc, bufs: CacheBuffers, stream=None) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(load().kv_cache_create(ctypes.byref(desc), ctypes.byref(bufs), _stream(stream),
                                  ctypes.byref(h)))
    return h


def kv_cache_reset(handle, stream=None):
    _check(load().kv_cache_reset(handle, _stream(stream)))


def kv_cache_destroy(handle):
    _check(load().kv_cache_destroy(handle))


def kv_cache_get_fill(handle) -> int:
    n = ctypes.c_int32()
    _check(load().kv_cache_get_fill(handle, ctypes.byref(n)))
    return n.value


def kv_cache_set_fill(handle, n_filled: int):
    _check(load().kv_cache_set_fill(handle, int(n_filled)))


def kv_cache_quantize(kv_dtype: str, x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                      stream=None):
    if x.dtype != torch.bfloat16 or scales.dtype != torch.float16:
        raise ValueError("x must be bf16 and scales fp16")
    d = x.shape[-1]
    n_rows = x.numel() // d if d else 0
    _check(load().kv_cache_quantize(DTYPE_CODE[kv_dtype], _ptr(x), n_rows, d, _ptr(codes),
                                    _ptr(scales), _stream(stream)))


def h2o_evict_insert(handle, w_prev, k_new, v_new, S: int, P: int, slots_out=None, stream=None):
    _check(load().h2o_evict_insert(handle, _ptr(w_prev), _ptr(k_new), _ptr(v_new), int(S), int(P),
                                   _ptr(slots_out), _stream(stream)))


def _ptr_array(items):
    """A C array of void* from handles / tensors / None (None stays NULL), or NULL for None."""
    if items is None:
        return None
    vals = []
    for x in items:
        if x is None:
            vals.append(None)
        elif isinstance(x, torch.Tensor):
            vals.append(_ptr(x).value)
        elif isinstance(x, ctypes.c_void_p):
            vals.append(x.value)
        else:
            vals.append(int(x))
    return (ctypes.c_void_p * len(vals))(*vals)


def h2o_evict_insert_many(handles, w_prev, k_new, v_new, S: int, P: int, slots_out=None,
                          stream=None):
    """h2o_evict_insert on several caches of one shape in one call (lists of the
    per-cache arguments; w_prev / slots_out may be None)."""
    _check(load().h2o_evict_insert_many(_ptr_array(handles), len(handles), _ptr_array(w_prev),
                                        _ptr_array(k_new), _ptr_array(v_new), int(S), int(P),
                                        _ptr_array(slots_out), _stream(stream)))


def kv_cache_set_score_mode(handle, mode: str):
    _check(load().kv_cache_set_score_mode(handle, SCORE_MODE[mode]))


def _delta(d):
    """A Delta struct from a dict of tensors (keys, values, token_pos[, k_scales, v_scales])."""
    if d is None:
        return None
    return ctypes.byref(Delta(_ptr(d["keys"]), _ptr(d["values"]), _ptr(d.get("k_scales")),
                              _ptr(d.get("v_scales")), _ptr(d["token_pos"])))


def h2o_evict_insert_delta(handle, w_prev, k_new, v_new, S: int, P: int, slots_out, delta,
                           stream=None):
    _check(load().h2o_evict_insert_delta(handle, _ptr(w_prev), _ptr(k_new), _ptr(v_new), int(S),
                                         int(P), _ptr(slots_out), _delta(delta), _stream(stream)))


def h2o_insert_at(handle, w_prev, k_new, v_new, S: int, P: int, slots_in, delta=None, stream=None):
    _check(load().h2o_insert_at(handle, _ptr(w_prev), _ptr(k_new), _ptr(v_new), int(S), int(P),
                                _ptr(slots_in), _delta(delta), _stream(stream)))


def kv_cache_restore(handle, slots, S: int, delta, stream=None):
    _check(load().kv_cache_restore(handle, _ptr(slots), int(S), _delta(delta), _stream(stream)))


def attn_chunk_backward(handle, q, dy, lse, S: int, P: int, dq_out, dk_out, dv_out, stream=None):
    _check(load().attn_chunk_backward(handle, _ptr(q), _ptr(dy), _ptr(lse), int(S), int(P),
                                      _ptr(dq_out), _ptr(dk_out), _ptr(dv_out), _stream(stream)))


def attn_chunk_with_scoresum(handle, q, S: int, P: int, y_out, lse_out, w_out, wq_out=None,
                             stream=None):
    _check(load().attn_chunk_with_scoresum(handle, _ptr(q), int(S), int(P), _ptr(y_out),
                                           _ptr(lse_out), _ptr(w_out), _ptr(wq_out),
                                           _stream(stream)))


def kv_cache_device_status(handle, stream=None) -> int:
    """Read and clear the device status word (0 = ok, else an error code)."""
    v = ctypes.c_int32()
    _check(load().kv_cache_device_status(handle, ctypes.byref(v), _stream(stream)))
    return v.value


def kv_cache_set_wait_timeout(handle, timeout_ns: int):
    _check(load().kv_cache_set_wait_timeout(handle, int(timeout_ns)))


def attn_chunk_with_scoresum_noalloc(desc: CacheDesc, keys, values, k_scales, v_scales, token_pos,
                                     q, S: int, P: int, y_out, lse_out, w_out, wq_out=None,
                                     stream=None):
    """Allocation-free attention over caller-owned cache buffers (no handle, no
    workspace); its scratch is a fixed array inside the library."""
    _check(load().attn_chunk_with_scoresum_noalloc(
        ctypes.byref(desc), _ptr(keys), _ptr(values), _ptr(k_scales), _ptr(v_scales),
        _ptr(token_pos), _ptr(q), int(S), int(P), _ptr(y_out), _ptr(lse_out), _ptr(w_out),
        _ptr(wq_out), _stream(stream)))


def h2okv_last_error() -> str:
    return load().h2okv_last_error().decode()


def h2okv_abi_version() -> int:
    return int(load().h2okv_abi_version())


# ---- a cache whose buffers torch allocates -----------------------------------
_TORCH_KV = {"f32": torch.float32, "bf16": torch.bfloat16, "i8": torch.int8, "i4": torch.uint8}
_TORCH_Q = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class CacheShape:
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    capacity: int
    max_chunk: int
    q_dtype: str = "bf16"
    kv_dtype: str = "bf16"

    def desc(self) -> CacheDesc:
        return CacheDesc(self.batch, self.n_q_heads, self.n_kv_heads, self.head_dim,
                         self.capacity, self.max_chunk, DTYPE_CODE[self.q_dtype],
                         DTYPE_CODE[self.kv_dtype])


class KVCache:
    """One layer's cache: torch owns the device buffers, the library the rest.

    Buffers (torch tensors): keys, values [B, H_k, N_C, d] (int4: d/2 bytes),
    k_scales, v_scales [B, H_k, N_C] fp16 (quantized caches), token_pos,
    scores [B, H_k, N_C], workspace (bytes).
    """

    def __init__(self, shape: CacheShape, device="cuda", stream=None):
        self.shape = shape
        self.device = torch.device(device)
        s = shape
        desc = s.desc()
        sizes = kv_cache_query_sizes(desc)
        B, Hk, NC, d = s.batch, s.n_kv_heads, s.capacity, s.head_dim
        row = d // 2 if s.kv_dtype == "i4" else d
        kvt = _TORCH_KV[s.kv_dtype]
        self.keys = torch.zeros((B, Hk, NC, row), dtype=kvt, device=self.device)
        self.values = torch.zeros_like(self.keys)
        quant = s.kv_dtype in ("i8", "i4")
        self.k_scales = torch.zeros((B, Hk, NC), dtype=torch.float16, device=self.device) if quant else None
        self.v_scales = torch.zeros_like(self.k_scales) if quant else None
        self.token_pos = torch.empty((B, Hk, NC), dtype=torch.int32, device=self.device)
        self.scores = torch.empty((B, Hk, NC), dtype=torch.float32, device=self.device)
        self.workspace = torch.empty(max(sizes["workspace"], 256), dtype=torch.uint8, device=self.device)
        for name in ("keys", "values", "k_scales", "v_scales", "token_pos", "scores"):
            t = getattr(self, name)
            if t is not None and t.numel() * t.element_size() != sizes[name]:
                raise AssertionError(f"size mismatch for {name}")
        self._bufs = CacheBuffers(*(_ptr(getattr(self, n)) for n in BUF_NAMES))
        self._desc = desc
        self.handle = kv_cache_create(desc, self._bufs, stream)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _lib is not None:
            _lib.kv_cache_destroy(h)
            self.handle = None

    @property
    def q_g(self):
        return self.shape.n_q_heads // self.shape.n_kv_heads

    @property
    def n_filled(self) -> int:
        return kv_cache_get_fill(self.handle)

    def set_fill(self, n: int):
        kv_cache_set_fill(self.handle, n)

    def reset(self, stream=None):
        kv_cache_reset(self.handle, stream)

    def evict_insert(self, w_prev, k_new, v_new, S, P, slots_out=None, stream=None):
        if S > 0:
            want = (self.shape.batch, self.shape.n_kv_heads, S, self.shape.head_dim)
            for t in (k_new, v_new):
                if tuple(t.shape) != want or t.dtype != _TORCH_Q[self.shape.q_dtype] or t.device != self.device:
                    raise ValueError(f"k_new/v_new must be {want} {self.shape.q_dtype} on {self.device}")
        self._check_w(w_prev, allow_none=True)
        h2o_evict_insert(self.handle, w_prev, k_new, v_new, S, P, slots_out, stream)

    def attend_backward(self, q, dy, lse, S, P, dq_out, dk_out, dv_out, stream=None):
        """Gradients of the chunk's SDPA (dq [B,H_q,S,d], dk/dv [B,H_k,N_C,d] float32)."""
        s = self.shape
        if tuple(dk_out.shape) != (s.batch, s.n_kv_heads, s.capacity, s.head_dim) or \
                dk_out.dtype != torch.float32 or dv_out.shape != dk_out.shape or dv_out.dtype != torch.float32:
            raise ValueError("dk_out/dv_out must be [B, H_k, N_C, d] float32")
        if tuple(dq_out.shape) != (s.batch, s.n_q_heads, S, s.head_dim) or dq_out.dtype != torch.float32:
            raise ValueError("dq_out must be [B, H_q, S, d] float32")
        attn_chunk_backward(self.handle, q, dy, lse, S, P, dq_out, dk_out, dv_out, stream)

    def set_score_mode(self, mode: str):
        kv_cache_set_score_mode(self.handle, mode)

    def delta_buffers(self, S):
        """Device buffers for the delta encoding of one chunk of S rows."""
        s = self.shape
        B, Hk = s.batch, s.n_kv_heads
        row = self.keys.shape[-1]
        d = {"keys": torch.empty((B, Hk, S, row), dtype=self.keys.dtype, device=self.device),
             "values": torch.empty((B, Hk, S, row), dtype=self.keys.dtype, device=self.device),
             "token_pos": torch.empty((B, Hk, S), dtype=torch.int32, device=self.device)}
        if self.k_scales is not None:
            d["k_scales"] = torch.empty((B, Hk, S), dtype=torch.float16, device=self.device)
            d["v_scales"] = torch.empty((B, Hk, S), dtype=torch.float16, device=self.device)
        return d

    def evict_insert_delta(self, w_prev, k_new, v_new, S, P, slots_out, delta, stream=None):
        self._check_kv(k_new, v_new, S)
        self._check_w(w_prev, allow_none=True)
        h2o_evict_insert_delta(self.handle, w_prev, k_new, v_new, S, P, slots_out, delta, stream)

    def insert_at(self, w_prev, k_new, v_new, S, P, slots_in, delta=None, stream=None):
        self._check_kv(k_new, v_new, S)
        self._check_w(w_prev, allow_none=True)
        if slots_in.dtype != torch.int32 or tuple(slots_in.shape) != (self.shape.batch, self.shape.n_kv_heads, S):
            raise ValueError("slots_in must be int32 [B, H_k, S]")
        h2o_insert_at(self.handle, w_prev, k_new, v_new, S, P, slots_in, delta, stream)

    def restore(self, slots, S, delta, stream=None):
        kv_cache_restore(self.handle, slots, S, delta, stream)

    def _check_kv(self, k_new, v_new, S):
        want = (self.shape.batch, self.shape.n_kv_heads, S, self.shape.head_dim)
        for t in (k_new, v_new):
            if tuple(t.shape) != want or t.dtype != _TORCH_Q[self.shape.q_dtype] or t.device != self.device:
                raise ValueError(f"k_new/v_new must be {want} {self.shape.q_dtype} on {self.device}")

    def attend(self, q, S, P, y_out, lse_out, w_out, wq_out=None, stream=None):
        s = self.shape
        want = (s.batch, s.n_q_heads, S, s.head_dim)
        for t in (q, y_out):
            if tuple(t.shape) != want or t.dtype != _TORCH_Q[s.q_dtype] or t.device != self.device:
                raise ValueError(f"q/y_out must be {want} {s.q_dtype} on {self.device}")
        self._check_w(w_out, allow_none=False)
        if lse_out is not None and (tuple(lse_out.shape) != want[:3] or lse_out.dtype != torch.float32):
            raise ValueError("lse_out must be [B, H_q, S] float32")
        if wq_out is not None and (tuple(wq_out.shape) != (s.batch, s.n_q_heads, s.capacity)
                                   or wq_out.dtype != torch.float32):
            raise ValueError("wq_out must be [B, H_q, N_C] float32")
        attn_chunk_with_scoresum(self.handle, q, S, P, y_out, lse_out, w_out, wq_out, stream)

    def _check_w(self, w, allow_none):
        if w is None:
            if allow_none:
                return
            raise ValueError("w_out is required")
        s = self.shape
        if tuple(w.shape) != (s.batch, s.n_kv_heads, s.capacity) or w.dtype != torch.float32 \
                or w.device != self.device:
            raise ValueError("w must be [B, H_k, N_C] float32 on the cache device")
