"""B200-native states-form KV-cache attention (chunked causal prefill and
split-context decode, 8 query heads sharing one KV head, head_dim 256).

Thin ctypes binding over libkca.so, whose C ABI is declared in
include/kca.h.  The functions keep the C names and only marshal arguments:
torch tensors become device pointers, dtypes become codes, the current torch
stream becomes the cudaStream_t.  Every step of the attention runs in the
library's CUDA kernels; there is no fallback, and a missing or unloadable
library raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import synth  # noqa: F401  (seeded inputs; no attention arithmetic)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkca.so")

F32, F16, BF16, I8 = 0, 1, 2, 3
I8_ROW_BYTES = 272        # packed int8 K row: 256 codes, f32 scale, 12 zero bytes
N_Q_HEADS, N_KV_HEADS, HEAD_DIM = 8, 1, 256
MAX_CHUNK_ROWS, MAX_POSITION, MAX_BATCH, MAX_BATCH_ROWS = 768, 131072, 256, 15
WORKSPACE_HEADER = 24832  # status word + per-(row, head) merge counters
STATUS = {0: "KCA_OK", -1: "KCA_ERR_NULL", -2: "KCA_ERR_GEOMETRY", -3: "KCA_ERR_DTYPE",
          -4: "KCA_ERR_RANGE", -5: "KCA_ERR_WORKSPACE", -6: "KCA_ERR_ALIGN", -7: "KCA_ERR_CUDA",
          -8: "KCA_ERR_DEVICE"}

_lib = None


class KcaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({status_string(status)})")


LIB_CHECKED_PATH = os.path.join(_HERE, "libkca_checked.so")


def lib() -> ctypes.CDLL:
    """The loaded libkca.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        _lib = load_library(LIB_PATH)
    return _lib


def load_library(path: str) -> ctypes.CDLL:
    """A libkca build at `path` with its C signatures declared (the binding
    itself uses lib(); tests load the bounds-checked build with this)."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m kv_cache_attention_states_b200.build`")
    L = ctypes.CDLL(path)
    vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)
    p64 = ctypes.POINTER(ctypes.c_int64)
    p32 = ctypes.POINTER(ctypes.c_int32)
    L.attn_prefill.argtypes = [vp, i32, vp, vp, i32, i32, i32, i32, i64, i64, i32, i64, i32,
                               f32, vp, vp, sz, vp]
    L.attn_prefill.restype = ctypes.c_int
    L.attn_decode.argtypes = [vp, i32, vp, vp, i32, i32, i32, i32, i64, i32, p64, i32, f32, vp,
                              vp, sz, vp]
    L.attn_decode.restype = ctypes.c_int
    L.attn_prefill_batch.argtypes = [vp, i32, vp, vp, i32, i32, i32, i32, i64, i32, i32, p64, i32, f32,
                                     vp, vp, sz, vp]
    L.attn_prefill_batch.restype = ctypes.c_int
    L.attn_prefill_batch_workspace_bytes.argtypes = [i32, i32, p64, i32]
    L.attn_prefill_batch_workspace_bytes.restype = sz
    L.attn_decode_dev.argtypes = [vp, i32, vp, vp, i32, i32, i32, i32, i64, i32, vp, i64, i32, f32,
                                  vp, vp, sz, vp]
    L.attn_decode_dev.restype = ctypes.c_int
    L.attn_append_kv.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp, i32, i64, vp, i64, vp, vp]
    L.attn_append_kv.restype = ctypes.c_int
    L.attn_decode_static.argtypes = [vp, i32, vp, vp, i32, i32, i32, i32, i64, i32, p64, i32,
                                     f32, vp, vp]
    L.attn_decode_static.restype = ctypes.c_int
    L.attn_decode_partial.argtypes = [vp, i32, vp, vp, i32, i32, i32, i32, i64, i32, p64, i64, i32,
                                      f32, vp, vp, sz, vp]
    L.attn_decode_partial.restype = ctypes.c_int
    L.attn_merge_partials.argtypes = [i32, i32, vp, i64, vp, vp]
    L.attn_merge_partials.restype = ctypes.c_int
    L.attn_decode_partial_workspace_bytes.argtypes = [i32, p64, i64, i64, i32]
    L.attn_decode_partial_workspace_bytes.restype = sz
    L.attn_prefill_workspace_bytes.argtypes = [i32, i32, i64, i32, i32]
    L.attn_prefill_workspace_bytes.restype = sz
    L.attn_decode_workspace_bytes.argtypes = [i32, p64, i32]
    L.attn_decode_workspace_bytes.restype = sz
    L.attn_workspace_init.argtypes = [vp, sz, vp]
    L.attn_workspace_init.restype = ctypes.c_int
    L.attn_device_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    L.attn_device_status.restype = ctypes.c_int
    L.attn_prefill_plan.argtypes = [i32, i32, i64, i32, i32, i32, p32, p64, i32, p32, p32]
    L.attn_prefill_plan.restype = ctypes.c_int
    L.attn_decode_plan.argtypes = [i32, p64, i32, i32, i32, p32, p64, i32, p32, p32]
    L.attn_decode_plan.restype = ctypes.c_int
    L.attn_decode_static_scratch.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(sz)]
    L.attn_decode_static_scratch.restype = ctypes.c_int
    L.attn_quantize_k.argtypes = [vp, i32, i64, vp, vp]
    L.attn_quantize_k.restype = ctypes.c_int
    L.attn_decode_q8.argtypes = [vp, i32, vp, vp, i32, i32, i32, i32, i64, i32, p64, i32, f32, vp, vp, sz, vp]
    L.attn_decode_q8.restype = ctypes.c_int
    L.attn_decode_q8_workspace_bytes.argtypes = [i32, p64, i32]
    L.attn_decode_q8_workspace_bytes.restype = sz
    L.attn_dot_canary.argtypes = [vp, p32]
    L.attn_dot_canary.restype = ctypes.c_int
    L.attn_decode_cluster_capacity.argtypes = [p32]
    L.attn_decode_cluster_capacity.restype = ctypes.c_int
    L.attn_force_path.argtypes = [i32, i32]
    L.attn_force_path.restype = ctypes.c_int
    L.attn_status_string.argtypes = [ctypes.c_int]
    L.attn_status_string.restype = ctypes.c_char_p
    return L


def status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


_CODES = None


def dtype_code(t) -> int:
    global _CODES
    if _CODES is None:
        import torch
        _CODES = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}
    code = _CODES.get(t.dtype)
    if code is None:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return code


def _stream_ptr(stream, device=None):
    """cudaStream_t of `stream`, else of torch's current stream on `device`
    (a torch.device, an index, or None for the current device).  The current
    stream is read through torch's raw-stream query, which costs a fraction
    of building a torch.cuda.Stream object per call."""
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    import torch
    idx = device.index if isinstance(device, torch.device) else device
    if idx is None:
        idx = torch.cuda.current_device()
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    if raw is not None:
        return ctypes.c_void_p(raw(idx))
    return ctypes.c_void_p(torch.cuda.current_stream(idx).cuda_stream)


_I64P = ctypes.POINTER(ctypes.c_int64)


def _i64_array(vals):
    """(n, pointer) of host int64 values; the pointer object keeps them alive.
    Short lists and tuples become a ctypes array directly (no numpy round
    trip), anything else goes through numpy."""
    if isinstance(vals, (list, tuple)) and len(vals) <= 64:
        return len(vals), (ctypes.c_int64 * len(vals))(*vals)
    arr = np.ascontiguousarray(np.asarray(vals, dtype=np.int64).reshape(-1))
    return arr.size, arr.ctypes.data_as(_I64P)


def _check(status: int, what: str):
    if status != 0:
        raise KcaError(status, what)


# ----------------------------------------------------------------- workspace

def attn_prefill_workspace_bytes(q_dtype: int, kv_dtype: int, chunk_start: int, chunk_rows: int,
                                 window: int = 0) -> int:
    n = lib().attn_prefill_workspace_bytes(q_dtype, kv_dtype, chunk_start, chunk_rows, window)
    if n == 0:
        raise KcaError(-4, "attn_prefill_workspace_bytes")
    return int(n)


def attn_decode_workspace_bytes(ctx_len, window: int = 0) -> int:
    nctx, ptr = _i64_array(ctx_len)
    n = lib().attn_decode_workspace_bytes(nctx, ptr, window)
    if n == 0:
        raise KcaError(-4, "attn_decode_workspace_bytes")
    return int(n)


def new_workspace(nbytes: int, device="cuda", stream=None):
    """A zero-status workspace of at least nbytes (torch uint8, 256-aligned)."""
    import torch
    ws = torch.empty(max(int(nbytes), WORKSPACE_HEADER), dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    _check(lib().attn_workspace_init(ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream_ptr(stream)),
           "attn_workspace_init")
    return ws


def attn_device_status(workspace, stream=None) -> tuple[int, int]:
    """(status, detail) of the workspace's device status word; clears it."""
    detail = ctypes.c_uint32(0)
    st = lib().attn_device_status(ctypes.c_void_p(workspace.data_ptr()), _stream_ptr(stream),
                                  ctypes.byref(detail))
    return int(st), int(detail.value)


# --------------------------------------------------------------------- calls

def attn_prefill(q_chunk, k_cache, v_cache, chunk_start: int, window: int = 0,
                 scale: float = 1.0 / 16.0, out=None, workspace=None, stream=None):
    """Chunked causal prefill of one sequence.

    q_chunk: [rows, 8, 256]; k_cache / v_cache: the sequence's [capacity, 256]
    (or [capacity, 1, 256]) rows with the chunk's own rows already written;
    returns out [rows, 8, 256] float32.
    """
    import torch
    rows = q_chunk.shape[0]
    capacity = k_cache.shape[0]
    for t in (q_chunk, k_cache, v_cache):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    if k_cache.dtype != v_cache.dtype:
        raise TypeError("k_cache and v_cache must share a dtype")
    if out is None:
        out = torch.empty((rows, N_Q_HEADS, HEAD_DIM), dtype=torch.float32, device=q_chunk.device)
    qd, kd = dtype_code(q_chunk), dtype_code(k_cache)
    if workspace is None:
        workspace = new_workspace(attn_prefill_workspace_bytes(qd, kd, chunk_start, rows, window),
                                  q_chunk.device, stream)
    st = lib().attn_prefill(ctypes.c_void_p(q_chunk.data_ptr()), qd, ctypes.c_void_p(k_cache.data_ptr()),
                            ctypes.c_void_p(v_cache.data_ptr()), kd, N_Q_HEADS, N_KV_HEADS, HEAD_DIM,
                            capacity, chunk_start, rows, chunk_start + rows, window, scale,
                            ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
                            workspace.numel(), _stream_ptr(stream))
    _check(st, "attn_prefill")
    return out


def attn_decode(q, k_cache, v_cache, ctx_len, window: int = 0, scale: float = 1.0 / 16.0,
                out=None, workspace=None, stream=None):
    """One query row per sequence at position ctx_len[b]-1.

    q: [batch, 8, 256]; k_cache / v_cache: [batch, capacity, 256] (or with a
    KV-head axis of 1); ctx_len: host sequence of ints; returns out
    [batch, 8, 256] float32.
    """
    import torch
    batch = q.shape[0]
    capacity = k_cache.shape[1]
    for t in (q, k_cache, v_cache):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    if k_cache.shape[0] != batch:
        raise ValueError("k_cache batch does not match q")
    nctx, ptr = _i64_array(ctx_len)
    if nctx != batch:
        raise ValueError("ctx_len must have one entry per sequence")
    if out is None:
        out = torch.empty((batch, N_Q_HEADS, HEAD_DIM), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(attn_decode_workspace_bytes(ctx_len, window), q.device, stream)
    st = lib().attn_decode(ctypes.c_void_p(q.data_ptr()), dtype_code(q), ctypes.c_void_p(k_cache.data_ptr()),
                           ctypes.c_void_p(v_cache.data_ptr()), dtype_code(k_cache), N_Q_HEADS,
                           N_KV_HEADS, HEAD_DIM, capacity, batch, ptr, window, scale,
                           ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
                           workspace.numel(), _stream_ptr(stream))
    _check(st, "attn_decode")
    return out


def attn_prefill_batch_workspace_bytes(ctx_len, rows: int, window: int = 0) -> int:
    nctx, ptr = _i64_array(ctx_len)
    n = lib().attn_prefill_batch_workspace_bytes(nctx, rows, ptr, window)
    if n == 0:
        raise KcaError(-4, "attn_prefill_batch_workspace_bytes")
    return int(n)


def attn_prefill_batch(q, k_cache, v_cache, ctx_len, window: int = 0, scale: float = 1.0 / 16.0,
                       out=None, workspace=None, stream=None):
    """Short chunks of several sequences in one call.

    q: [batch, rows, 8, 256] (rows 1..15); k_cache / v_cache: [batch,
    capacity, 256]; ctx_len: host ints, row i of sequence b sits at position
    ctx_len[b] - rows + i; returns out [batch, rows, 8, 256] float32.
    """
    import torch
    batch, rows = q.shape[0], q.shape[1]
    capacity = k_cache.shape[1]
    for t in (q, k_cache, v_cache):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    if k_cache.shape[0] != batch:
        raise ValueError("k_cache batch does not match q")
    nctx, ptr = _i64_array(ctx_len)
    if nctx != batch:
        raise ValueError("ctx_len must have one entry per sequence")
    if out is None:
        out = torch.empty((batch, rows, N_Q_HEADS, HEAD_DIM), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(attn_prefill_batch_workspace_bytes(ctx_len, rows, window), q.device, stream)
    vp = ctypes.c_void_p
    st = lib().attn_prefill_batch(vp(q.data_ptr()), dtype_code(q), vp(k_cache.data_ptr()), vp(v_cache.data_ptr()),
                                  dtype_code(k_cache), N_Q_HEADS, N_KV_HEADS, HEAD_DIM, capacity, batch, rows, ptr,
                                  window, scale, vp(out.data_ptr()), vp(workspace.data_ptr()), workspace.numel(),
                                  _stream_ptr(stream))
    _check(st, "attn_prefill_batch")
    return out


def attn_decode_dev(q, k_cache, v_cache, ctx_len_dev, ctx_bound: int, window: int = 0,
                    scale: float = 1.0 / 16.0, out=None, workspace=None, stream=None):
    """attn_decode with the context lengths in device memory.

    ctx_len_dev: int64 CUDA tensor [batch], each value in 0..ctx_bound, read
    by the kernels when they run (so a captured CUDA graph of this call can be
    replayed after updating it in place); ctx_bound: host upper bound that
    the launch is planned for.
    """
    import torch
    batch = q.shape[0]
    capacity = k_cache.shape[1]
    for t in (q, k_cache, v_cache, ctx_len_dev):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    if ctx_len_dev.dtype != torch.int64 or ctx_len_dev.numel() != batch or k_cache.shape[0] != batch:
        raise ValueError("ctx_len_dev must be int64 with one entry per sequence")
    if out is None:
        out = torch.empty((batch, N_Q_HEADS, HEAD_DIM), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(attn_decode_workspace_bytes([ctx_bound] * batch, window), q.device, stream)
    st = lib().attn_decode_dev(ctypes.c_void_p(q.data_ptr()), dtype_code(q), ctypes.c_void_p(k_cache.data_ptr()),
                               ctypes.c_void_p(v_cache.data_ptr()), dtype_code(k_cache), N_Q_HEADS,
                               N_KV_HEADS, HEAD_DIM, capacity, batch, ctypes.c_void_p(ctx_len_dev.data_ptr()),
                               int(ctx_bound), window, scale, ctypes.c_void_p(out.data_ptr()),
                               ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream))
    _check(st, "attn_decode_dev")
    return out


def partial_floats(batch: int) -> int:
    """Floats of one partial record of `batch` sequences: (m, l) pairs
    [batch][8][2], then acc [batch][8][256]."""
    return batch * N_Q_HEADS * (2 + HEAD_DIM)


def split_partial(part, batch: int):
    """Views (ml [batch, 8, 2], acc [batch, 8, 256]) of a partial record."""
    n = batch * N_Q_HEADS * 2
    return (part[..., :n].reshape(*part.shape[:-1], batch, N_Q_HEADS, 2),
            part[..., n:n + batch * N_Q_HEADS * HEAD_DIM].reshape(*part.shape[:-1], batch, N_Q_HEADS, HEAD_DIM))


def attn_decode_partial_workspace_bytes(ctx_len, key_begin: int, capacity: int, window: int = 0) -> int:
    nctx, ptr = _i64_array(ctx_len)
    n = lib().attn_decode_partial_workspace_bytes(nctx, ptr, key_begin, capacity, window)
    if n == 0:
        raise KcaError(-4, "attn_decode_partial_workspace_bytes")
    return int(n)


def attn_decode_partial(q, k_shard, v_shard, ctx_len, key_begin: int, window: int = 0,
                        scale: float = 1.0 / 16.0, part=None, workspace=None, stream=None):
    """Decode over one context shard, as a partial-softmax record.

    k_shard / v_shard: [batch, capacity, 256] holding positions
    [key_begin, key_begin + capacity) of each sequence; q: [batch, 8, 256];
    ctx_len: host ints (the whole context, which may extend past the shard).
    Returns part, float32 [partial_floats(batch)] (see split_partial).
    """
    import torch
    batch = q.shape[0]
    capacity = k_shard.shape[1]
    for t in (q, k_shard, v_shard):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    if k_shard.shape[0] != batch:
        raise ValueError("k_shard batch does not match q")
    nctx, ptr = _i64_array(ctx_len)
    if nctx != batch:
        raise ValueError("ctx_len must have one entry per sequence")
    if part is None:
        part = torch.empty(partial_floats(batch), dtype=torch.float32, device=q.device)
    if part.dtype != torch.float32 or not part.is_contiguous() or part.numel() < partial_floats(batch):
        raise ValueError("part must be a contiguous float32 tensor of partial_floats(batch) elements")
    if workspace is None:
        workspace = new_workspace(attn_decode_partial_workspace_bytes(ctx_len, key_begin, capacity, window),
                                  q.device, stream)
    vp = ctypes.c_void_p
    st = lib().attn_decode_partial(vp(q.data_ptr()), dtype_code(q), vp(k_shard.data_ptr()),
                                   vp(v_shard.data_ptr()), dtype_code(k_shard), N_Q_HEADS, N_KV_HEADS, HEAD_DIM,
                                   capacity, batch, ptr, int(key_begin), window, scale, vp(part.data_ptr()),
                                   vp(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream))
    _check(st, "attn_decode_partial")
    return part


def attn_merge_partials(parts, batch: int, out=None, stream=None):
    """Merge partial records parts [n_parts, stride] (float32, stride >=
    partial_floats(batch), a multiple of 4) into out [batch, 8, 256]."""
    import torch
    if parts.dim() != 2 or parts.dtype != torch.float32 or not parts.is_cuda or parts.stride(1) != 1:
        raise ValueError("parts must be a float32 CUDA tensor [n_parts, stride] with unit inner stride")
    if out is None:
        out = torch.empty((batch, N_Q_HEADS, HEAD_DIM), dtype=torch.float32, device=parts.device)
    st = lib().attn_merge_partials(parts.shape[0], batch, ctypes.c_void_p(parts.data_ptr()), parts.stride(0),
                                   ctypes.c_void_p(out.data_ptr()), _stream_ptr(stream))
    _check(st, "attn_merge_partials")
    return out


def attn_append_kv(k_new, v_new, k_cache, v_cache, dst, rope_cos=None, rope_sin=None, workspace=None,
                   stream=None):
    """Write new K/V rows into the cache, K rotated by RoPE when cos/sin are given.

    k_new / v_new: [n, 256] (or [n, 1, 256]); k_cache / v_cache: contiguous with
    a last axis of 256, addressed as rows; dst: an int (rows dst .. dst+n-1) or
    an int64 CUDA tensor [n] of destination rows; rope_cos / rope_sin: float32
    CUDA tensors [n, 256] or None.
    """
    import torch
    n = k_new.numel() // HEAD_DIM
    for t in (k_new, v_new, k_cache, v_cache):
        if not t.is_cuda or not t.is_contiguous() or t.shape[-1] != HEAD_DIM:
            raise ValueError("tensors must be contiguous CUDA tensors with a last axis of 256")
    if v_new.numel() != k_new.numel() or v_cache.numel() != k_cache.numel():
        raise ValueError("k and v shapes differ")
    if (rope_cos is None) != (rope_sin is None):
        raise ValueError("give both rope_cos and rope_sin, or neither")
    vp = ctypes.c_void_p
    cos_p = vp(rope_cos.data_ptr()) if rope_cos is not None else None
    sin_p = vp(rope_sin.data_ptr()) if rope_sin is not None else None
    if rope_cos is not None:
        for t in (rope_cos, rope_sin):
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or t.numel() != n * HEAD_DIM:
                raise ValueError("rope_cos / rope_sin must be float32 CUDA tensors [n, 256]")
    if isinstance(dst, int):
        dst_p, dst0 = None, dst
    else:
        if dst.dtype != torch.int64 or not dst.is_cuda or dst.numel() != n:
            raise ValueError("dst must be an int or an int64 CUDA tensor [n]")
        dst_p, dst0 = vp(dst.data_ptr()), 0
    st = lib().attn_append_kv(vp(k_new.data_ptr()), vp(v_new.data_ptr()), dtype_code(k_new), n, cos_p, sin_p,
                              vp(k_cache.data_ptr()), vp(v_cache.data_ptr()), dtype_code(k_cache),
                              k_cache.numel() // HEAD_DIM, dst_p, dst0,
                              vp(workspace.data_ptr()) if workspace is not None else None,
                              _stream_ptr(stream))
    _check(st, "attn_append_kv")


# ------------------------------------------------------- quantised-dot decode

def attn_quantize_k(k, out=None, stream=None):
    """K rows [..., 256] (f32 / f16 / bf16, contiguous CUDA) -> packed int8
    rows uint8 [..., 272]: 256 codes, the row's f32 scale, 12 zero bytes."""
    import torch
    if not k.is_cuda or not k.is_contiguous() or k.shape[-1] != HEAD_DIM:
        raise ValueError("k must be a contiguous CUDA tensor with a last axis of 256")
    n = k.numel() // HEAD_DIM
    if out is None:
        out = torch.empty((*k.shape[:-1], I8_ROW_BYTES), dtype=torch.uint8, device=k.device)
    if out.dtype != torch.uint8 or not out.is_contiguous() or out.numel() != n * I8_ROW_BYTES:
        raise ValueError("out must be a contiguous uint8 tensor [..., 272]")
    st = lib().attn_quantize_k(ctypes.c_void_p(k.data_ptr()), dtype_code(k), n, ctypes.c_void_p(out.data_ptr()),
                               _stream_ptr(stream, k.device))
    _check(st, "attn_quantize_k")
    return out


def attn_dot_canary(stream=None) -> int:
    """Mask of the dot-product variants that passed the known-answer check on
    the current device: 1 the dp4a instruction, 2 its emulation, 4 the int8
    tensor-core MMA; raises when neither dp4a nor its emulation did."""
    v = ctypes.c_int32(-1)
    _check(lib().attn_dot_canary(_stream_ptr(stream), ctypes.byref(v)), "attn_dot_canary")
    return int(v.value)


def attn_decode_q8_workspace_bytes(ctx_len, window: int = 0) -> int:
    nctx, ptr = _i64_array(ctx_len)
    n = lib().attn_decode_q8_workspace_bytes(nctx, ptr, window)
    if n == 0:
        raise KcaError(-4, "attn_decode_q8_workspace_bytes")
    return int(n)


def attn_decode_q8(q, k8_cache, v_cache, ctx_len, window: int = 0, scale: float = 1.0 / 16.0, out=None,
                   workspace=None, stream=None):
    """Quantised-dot decode: q [batch, 8, 256]; k8_cache uint8 [batch, capacity,
    272] packed int8 rows (attn_quantize_k); v_cache [batch, capacity, 256];
    returns out [batch, 8, 256] float32."""
    import torch
    batch = q.shape[0]
    capacity = k8_cache.shape[1]
    for t in (q, k8_cache, v_cache):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    if k8_cache.dtype != torch.uint8 or k8_cache.shape[-1] != I8_ROW_BYTES or k8_cache.shape[0] != batch:
        raise ValueError("k8_cache must be uint8 [batch, capacity, 272]")
    if v_cache.shape[0] != batch or v_cache.shape[1] != capacity:
        raise ValueError("v_cache must be [batch, capacity, 256]")
    nctx, ptr = _i64_array(ctx_len)
    if nctx != batch:
        raise ValueError("ctx_len must have one entry per sequence")
    if out is None:
        out = torch.empty((batch, N_Q_HEADS, HEAD_DIM), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(attn_decode_q8_workspace_bytes(ctx_len, window), q.device, stream)
    vp = ctypes.c_void_p
    st = lib().attn_decode_q8(vp(q.data_ptr()), dtype_code(q), vp(k8_cache.data_ptr()), vp(v_cache.data_ptr()),
                              dtype_code(v_cache), N_Q_HEADS, N_KV_HEADS, HEAD_DIM, capacity, batch, ptr, window,
                              scale, vp(out.data_ptr()), vp(workspace.data_ptr()), workspace.numel(),
                              _stream_ptr(stream))
    _check(st, "attn_decode_q8")
    return out


def attn_decode_static(q, k_cache, v_cache, ctx_len, window: int = 0, scale: float = 1.0 / 16.0,
                       out=None, stream=None):
    """attn_decode for callers that cannot allocate device memory: the split
    partials go to the library's fixed 16 MiB device array instead of a
    workspace (see include/kca.h for the sharing rules)."""
    import torch
    batch = q.shape[0]
    nctx, ptr = _i64_array(ctx_len)
    if nctx != batch or k_cache.shape[0] != batch:
        raise ValueError("ctx_len / k_cache must have one entry per sequence")
    if out is None:
        out = torch.empty((batch, N_Q_HEADS, HEAD_DIM), dtype=torch.float32, device=q.device)
    st = lib().attn_decode_static(ctypes.c_void_p(q.data_ptr()), dtype_code(q),
                                  ctypes.c_void_p(k_cache.data_ptr()), ctypes.c_void_p(v_cache.data_ptr()),
                                  dtype_code(k_cache), N_Q_HEADS, N_KV_HEADS, HEAD_DIM, k_cache.shape[1],
                                  batch, ptr, window, scale, ctypes.c_void_p(out.data_ptr()),
                                  _stream_ptr(stream))
    _check(st, "attn_decode_static")
    return out


# ------------------------------------------------------------ path control

OP_PREFILL, OP_ROWS, OP_BATCH = 0, 1, 2           # attn_force_path operations
PATH_AUTO, PATH_ROWS, PATH_TENSOR_CORE = -1, 0, 1
PATH_CUDA_CORE = 0                               # OP_ROWS: the CUDA-core kernel
PATH_MMA_SYNC, PATH_TCGEN05 = 0, 1               # OP_BATCH: the multi-row kernels
PATH_MULTI_ROW = 2                               # OP_PREFILL: multi-row units (short chunks, 16-bit cache)


def attn_force_path(op: int, path: int) -> None:
    """Pin the kernel family of later calls, process-wide (see include/kca.h):
    op OP_PREFILL with PATH_ROWS / PATH_TENSOR_CORE / PATH_MULTI_ROW, op OP_ROWS with
    PATH_CUDA_CORE / PATH_TENSOR_CORE, op OP_BATCH with PATH_MMA_SYNC /
    PATH_TCGEN05; PATH_AUTO restores the automatic choice."""
    _check(lib().attn_force_path(int(op), int(path)), "attn_force_path")


class forced_path:
    """Context manager: attn_force_path(op, path) inside, PATH_AUTO after."""

    def __init__(self, op: int, path: int):
        self.op, self.path = op, path

    def __enter__(self):
        attn_force_path(self.op, self.path)
        return self

    def __exit__(self, *exc):
        attn_force_path(self.op, PATH_AUTO)
        return False


# --------------------------------------------------------------------- plans

def _num_sms(num_sms):
    """num_sms as given, else the current CUDA device's SM count (the count
    the calls plan for); without a device it has to be given."""
    if num_sms is not None:
        return int(num_sms)
    import torch
    if not torch.cuda.is_available():
        raise ValueError("no CUDA device: pass num_sms to plan for a given SM count")
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


def attn_prefill_path(q_dtype: int, kv_dtype: int, chunk_start: int, chunk_rows: int,
                      window: int = 0) -> int:
    """The path a prefill call takes: 1 tensor-core, 2 multi-row units, 0 rows
    (host only; no device needed)."""
    n = ctypes.c_int32(0)
    path = ctypes.c_int32(-1)
    # the path does not depend on the SM count; any positive count serves
    st = lib().attn_prefill_plan(q_dtype, kv_dtype, chunk_start, chunk_rows, window, 1, None, None, 0,
                                 ctypes.byref(n), ctypes.byref(path))
    if path.value < 0:
        raise KcaError(st, "attn_prefill_plan")
    return int(path.value)


def attn_decode_cluster_capacity() -> tuple[int, int, int]:
    """Resident clusters of 2, 4 and 8 CTAs of the tensor-core rows kernel on
    the current device (what the device plans use)."""
    cap = (ctypes.c_int32 * 3)()
    _check(lib().attn_decode_cluster_capacity(cap), "attn_decode_cluster_capacity")
    return int(cap[0]), int(cap[1]), int(cap[2])


def _capacity(cluster_capacity):
    """int32[3] of resident clusters of 2, 4, 8 CTAs, or None (the device's)."""
    if cluster_capacity is None:
        return None
    return (ctypes.c_int32 * 3)(*[int(x) for x in cluster_capacity])


def attn_prefill_plan(q_dtype: int, kv_dtype: int, chunk_start: int, chunk_rows: int,
                      window: int = 0, num_sms: int | None = None, cluster_capacity=None):
    """(path, items[n, 4]) -- see include/kca.h.  num_sms defaults to the
    current device's SM count.  Host only, except the rows plan of 16-bit
    caches without cluster_capacity (resident clusters of 2, 4, 8 CTAs),
    which is the tensor-core kernel's cluster plan on the current device."""
    if cluster_capacity is None and num_sms is None:
        num_sms = _num_sms(None)
    num_sms = int(num_sms)
    cap = _capacity(cluster_capacity)
    n = ctypes.c_int32(0)
    path = ctypes.c_int32(0)
    st = lib().attn_prefill_plan(q_dtype, kv_dtype, chunk_start, chunk_rows, window, num_sms, cap, None,
                                 0, ctypes.byref(n), ctypes.byref(path))
    if st not in (0, -4) or (st == -4 and n.value == 0):
        raise KcaError(st, "attn_prefill_plan")
    items = np.zeros((max(n.value, 1), 4), dtype=np.int64)
    st = lib().attn_prefill_plan(q_dtype, kv_dtype, chunk_start, chunk_rows, window, num_sms, cap,
                                 items.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n.value,
                                 ctypes.byref(n), ctypes.byref(path))
    _check(st, "attn_prefill_plan")
    return int(path.value), items[:n.value]


def attn_decode_plan(ctx_len, window: int = 0, num_sms: int | None = None, kv_dtype: int = F32,
                     cluster_capacity=None, with_cluster: bool = False):
    """items[n, 4] of a decode call -- see include/kca.h -- and, with
    with_cluster, the cluster size (items, cluster).  kv_dtype F32: the
    CUDA-core kernel's plan for num_sms SMs (default: the current device's
    count); F16 / BF16: the tensor-core kernel's cluster plan for num_sms SMs
    holding cluster_capacity = (clusters of 2, 4, 8 CTAs) at once, host only,
    or without cluster_capacity for the current device."""
    if kv_dtype in (F16, BF16) and cluster_capacity is None and num_sms is None:
        num_sms = 1          # not used: the plan asks the device itself
    num_sms = _num_sms(num_sms)
    cap = _capacity(cluster_capacity)
    nctx, ptr = _i64_array(ctx_len)
    n = ctypes.c_int32(0)
    cl = ctypes.c_int32(0)
    st = lib().attn_decode_plan(nctx, ptr, window, kv_dtype, num_sms, cap, None, 0, ctypes.byref(n), None)
    if st not in (0, -4) or (st == -4 and n.value == 0):
        raise KcaError(st, "attn_decode_plan")
    items = np.zeros((max(n.value, 1), 4), dtype=np.int64)
    st = lib().attn_decode_plan(nctx, ptr, window, kv_dtype, num_sms, cap,
                                items.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n.value,
                                ctypes.byref(n), ctypes.byref(cl))
    _check(st, "attn_decode_plan")
    return (items[:n.value], int(cl.value)) if with_cluster else items[:n.value]
