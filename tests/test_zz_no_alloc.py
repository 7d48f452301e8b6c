"""attn_decode_static: decode for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc at the point where they decode (a host
callback, an allocator's own code path, a memory pool that admits no new
allocations, a runtime that only hands out the tensors it owns), so they
cannot provide the workspace that attn_decode writes its per-split partials
to.  attn_decode_static takes that scratch from a fixed device array inside
the library instead.  These tests call it through the C ABI (ctypes, raw
pointers) and check it against attn_decode on the same inputs, three times
in a row with different shapes so that the array's leftover contents from
one call cannot leak into the next, and once after the array's header (the
status word and the merge counters) was filled with garbage, which the
call must clear before its kernel runs.  The status of each call is read
back through the array's address (attn_decode_static_scratch).  This file
is collected last, and it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth

pytestmark = pytest.mark.gpu

STATIC_BYTES = 16 * 1024 * 1024


def _static_call(q, k, v, ctx, window, out):
    arr = np.ascontiguousarray(np.asarray(ctx, dtype=np.int64))
    vp = ctypes.c_void_p
    return kca.lib().attn_decode_static(
        vp(q.data_ptr()), kca.dtype_code(q), vp(k.data_ptr()), vp(v.data_ptr()), kca.dtype_code(k),
        8, 1, 256, k.shape[1], q.shape[0], arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        window, 1.0 / 16.0, vp(out.data_ptr()), vp(torch.cuda.current_stream().cuda_stream))


def _scratch():
    ptr = ctypes.c_void_p(0)
    size = ctypes.c_size_t(0)
    assert kca.lib().attn_decode_static_scratch(ctypes.byref(ptr), ctypes.byref(size)) == 0
    assert ptr.value and ptr.value % 256 == 0 and size.value == STATIC_BYTES
    return ptr.value


def _static_status():
    detail = ctypes.c_uint32(0)
    st = kca.lib().attn_device_status(ctypes.c_void_p(_scratch()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                      ctypes.byref(detail))
    return st, detail.value


class _DeviceBytes:
    """A torch view of n bytes of device memory at a raw address (CUDA array
    interface); used to scribble over the array's header."""

    def __init__(self, ptr, n):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "|u1", "data": (ptr, False),
                                         "version": 3, "strides": None}


def _inputs(seed, batch, cap, q_dtype, kv_dtype):
    k = synth.as_torch(synth.draw(seed, "k", (batch, cap, 256), kv_dtype), kv_dtype).cuda()
    v = synth.as_torch(synth.draw(seed, "v", (batch, cap, 256), kv_dtype), kv_dtype).cuda()
    q = synth.as_torch(synth.draw(seed, "q", (batch, 8, 256), q_dtype), q_dtype).cuda()
    return q, k, v


def test_static_scratch_decode_matches_attn_decode_three_times(cuda_ok):
    cases = [
        (1, 16448, [16384], 0, "f32", "f16"),               # one long sequence: 100+ splits
        (4, 9000, [8999, 1, 4500, 7777], 300, "bf16", "bf16"),  # ragged batch with a window
        (1, 16448, [16384], 0, "f32", "f16"),               # the first case again, after the second
    ]
    for i, (batch, cap, ctx, window, qd, kd) in enumerate(cases):
        q, k, v = _inputs(10 + i, batch, cap, qd, kd)
        want = kca.attn_decode(q, k, v, ctx, window)
        got = torch.full((batch, 8, 256), float("nan"), dtype=torch.float32, device="cuda")
        assert _static_call(q, k, v, ctx, window, got) == 0
        torch.cuda.synchronize()
        err = (got - want).abs().max().item()
        tol = 2e-6 if (qd, kd) == ("f32", "f32") else 4e-3
        assert err <= tol, (i, err)
        assert torch.isfinite(got).all()
        assert _static_status() == (0, 0), i


def test_static_scratch_decode_clears_a_garbage_header(cuda_ok):
    # Nonzero status word and merge counters left by an imagined failed
    # call: the next call clears them before its kernel runs, so its output
    # and status are those of a clean start.
    header = kca.WORKSPACE_HEADER
    view = torch.as_tensor(_DeviceBytes(_scratch(), header), device="cuda")
    q, k, v = _inputs(20, 1, 16448, "f32", "f16")
    want = kca.attn_decode(q, k, v, [16384])
    for fill in (0xFF, 0x01):
        view.fill_(fill)
        torch.cuda.synchronize()
        got = torch.full((1, 8, 256), float("nan"), dtype=torch.float32, device="cuda")
        assert _static_call(q, k, v, [16384], 0, got) == 0
        torch.cuda.synchronize()
        assert (got - want).abs().max().item() <= 4e-3, fill
        assert _static_status() == (0, 0), fill


def test_static_scratch_rejects_plans_beyond_its_size(cuda_ok):
    # 100 sequences beside one at 131072 positions: the one-wave plan needs
    # 100 x 49 partial slots of 8 KiB, more than the 16 MiB array.
    batch, cap = 100, 131072
    ctx = [131072] + [1] * (batch - 1)
    need = kca.attn_decode_workspace_bytes(ctx)
    assert need > STATIC_BYTES
    q = torch.zeros((batch, 8, 256), dtype=torch.float32, device="cuda")
    k = torch.empty((batch, cap, 256), dtype=torch.float16, device="cuda")
    v = torch.empty((batch, cap, 256), dtype=torch.float16, device="cuda")
    out = torch.zeros((batch, 8, 256), dtype=torch.float32, device="cuda")
    assert _static_call(q, k, v, ctx, 0, out) == -5   # KCA_ERR_WORKSPACE, nothing launched
    del k, v
    torch.cuda.empty_cache()
