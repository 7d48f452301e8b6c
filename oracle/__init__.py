"""f64 CPU oracle for states-form KV-cache attention.

TEST INFRASTRUCTURE ONLY.  Only `tests/`, `__graft_entry__.smoke()` and the
CPU-baseline leg of `bench.py` may import this package.  It shares no code
with the CUDA library and never imports it.

`attention()` is a ctypes front end to the plain C definition in
attn_oracle.c (the states-form attention of the Karume v0.8.0 / v0.12.0
release notes: softmax(q k^T * scale + causal/window mask) v, NaN-preserving
row max, fully masked row = 0).  `brute` holds an independent
Python-`decimal` implementation used to pin it.

Arrays are numpy arrays in their stored format: float32, float16, or bf16
carried as uint16 bit patterns together with dtype="bf16".
"""
import ctypes

import numpy as np

from . import build as _build

F32, F16, BF16, F64 = 0, 1, 2, 3
_DTYPES = {"f32": F32, "f16": F16, "bf16": BF16, "f64": F64}
_lib = None


def bind(path: str):
    """ctypes handle for an oracle library at `path` (the tests also bind
    deliberately broken copies to check that the pins catch them)."""
    lib = ctypes.CDLL(path)
    lib.oracle_attention.restype = ctypes.c_int
    lib.oracle_attention.argtypes = [
        ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_void_p]
    lib.oracle_decode_element.restype = ctypes.c_double
    lib.oracle_decode_element.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64]
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(_build.build())
    return _lib


def dtype_code(arr: np.ndarray, dtype: str | None) -> int:
    if dtype is None:
        dtype = {np.dtype(np.float32): "f32", np.dtype(np.float16): "f16",
                 np.dtype(np.float64): "f64"}[arr.dtype]
    code = _DTYPES[dtype]
    want = {F32: np.float32, F16: np.float16, BF16: np.uint16, F64: np.float64}[code]
    if arr.dtype != want:
        raise TypeError(f"array of {arr.dtype} does not carry {dtype}")
    return code


def num_threads() -> int:
    return _load().oracle_max_threads()


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def attention(q, k, v, pos, kv_base=None, *, window=0, scale=1.0 / 16.0,
              n_kv_heads=1, q_dtype=None, kv_dtype=None, lib=None) -> np.ndarray:
    """Plain f64 attention of each query row over its visible cached rows.

    q       : [n_query, n_q_heads, head_dim]
    k, v    : [rows, n_kv_heads, head_dim] (or [rows, head_dim] when n_kv_heads == 1)
    pos     : [n_query] absolute positions (pos < 0 sees no key -> output 0)
    kv_base : [n_query] first row of each query's sequence in k/v (default 0)
    Returns float64 [n_query, n_q_heads, head_dim].
    """
    lib = lib or _load()
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    if q.ndim != 3:
        raise ValueError("q must be [n_query, n_q_heads, head_dim]")
    n_query, n_q_heads, head_dim = q.shape
    if k.shape != v.shape or k.shape[-1] != head_dim:
        raise ValueError("k/v shape mismatch")
    qc = dtype_code(q, q_dtype)
    kc = dtype_code(k, kv_dtype)
    if dtype_code(v, kv_dtype) != kc:
        raise TypeError("k and v must share a dtype")
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(n_query))
    if kv_base is None:
        kv_base = np.zeros(n_query, dtype=np.int64)
    kv_base = np.ascontiguousarray(np.asarray(kv_base, dtype=np.int64).reshape(n_query))
    out = np.empty((n_query, n_q_heads, head_dim), dtype=np.float64)
    rc = lib.oracle_attention(q.ctypes.data, qc, k.ctypes.data, v.ctypes.data, kc,
                              kv_base.ctypes.data, pos.ctypes.data, n_query, n_q_heads,
                              int(n_kv_heads), head_dim, int(window), float(scale),
                              out.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle_attention rejected its arguments")
    return out


def decode_elements(arr: np.ndarray, dtype: str | None = None, lib=None) -> np.ndarray:
    """Widen stored elements to float64 with the oracle's own decoders."""
    lib = lib or _load()
    arr = np.ascontiguousarray(arr)
    code = dtype_code(arr, dtype)
    flat = arr.reshape(-1)
    return np.array([lib.oracle_decode_element(flat.ctypes.data, code, i)
                     for i in range(flat.size)], dtype=np.float64).reshape(arr.shape)


def visible_range(pos: int, window: int) -> tuple[int, int]:
    """[lo, hi] of the keys a query at `pos` sees (empty when hi < lo)."""
    lo = max(0, pos - window + 1) if window > 0 else 0
    return lo, pos
