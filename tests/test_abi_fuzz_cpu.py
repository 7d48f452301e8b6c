"""Host-side argument validation under random input (CPU only): every entry
point that takes sizes, positions, dtypes and pointers from the caller must
return one of the documented status codes for any combination -- extreme
integers, NaN and infinite scales, NULL and misaligned pointers -- and never
crash.  The pointers are fake device addresses, so the test runs only where
no GPU is present: a call whose arguments all pass validation then stops at
its first CUDA call (KCA_ERR_CUDA) and nothing is ever dereferenced."""
import ctypes

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import kv_cache_attention_states_b200 as kca


@pytest.fixture(scope="module", autouse=True)
def _no_gpu():
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake device pointers: CPU-only test")


CODES = {-1, -2, -3, -4, -5, -6, -7}
I32 = st.one_of(st.integers(-3, 3), st.integers(-(2**31), 2**31 - 1), st.sampled_from([8, 1, 256, 768, 769, 255]))
I64 = st.one_of(st.integers(-3, 3), st.integers(-(2**63), 2**63 - 1),
                st.sampled_from([131071, 131072, 131073, 16384, 2**31, 2**32 + 5]))
PTR = st.sampled_from([0, 0x10000, 0x10008, 0x10004, 0x10100, 0x7fff0000])
DT = st.one_of(st.integers(-2, 4), st.sampled_from([kca.F32, kca.F16, kca.BF16]))
SCALE = st.one_of(st.floats(allow_nan=True, allow_infinity=True, width=32), st.just(0.0625))
CTX = st.lists(st.one_of(st.integers(-2, 20000), st.integers(-(2**63), 2**63 - 1)), min_size=0, max_size=300)
WSB = st.one_of(st.integers(0, 2**20), st.just(1 << 40), st.just(2**64 - 1))


def _arr(ctx):
    a = np.asarray(ctx if ctx else [0], dtype=np.int64)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


vp = ctypes.c_void_p


@settings(max_examples=400, deadline=None, derandomize=True)
@given(q=PTR, qd=DT, k=PTR, v=PTR, kd=DT, hq=I32, hkv=I32, d=I32, cap=I64, cs=I64, rows=I32, ctx=I64,
       window=I32, scale=SCALE, out=PTR, ws=PTR, wsb=WSB)
def test_prefill_returns_a_status_for_any_arguments(q, qd, k, v, kd, hq, hkv, d, cap, cs, rows, ctx, window, scale,
                                                     out, ws, wsb):
    st_ = kca.lib().attn_prefill(vp(q), qd, vp(k), vp(v), kd, hq, hkv, d, cap, cs, rows, ctx, window, scale, vp(out),
                                 vp(ws), wsb, None)
    assert st_ in CODES


@settings(max_examples=400, deadline=None, derandomize=True)
@given(q=PTR, qd=DT, k=PTR, v=PTR, kd=DT, hq=I32, hkv=I32, d=I32, cap=I64, ctx=CTX, batch=I32, window=I32,
       scale=SCALE, out=PTR, ws=PTR, wsb=WSB, rows=I32)
def test_decode_and_batch_return_a_status_for_any_arguments(q, qd, k, v, kd, hq, hkv, d, cap, ctx, batch, window,
                                                            scale, out, ws, wsb, rows):
    arr, ptr = _arr(ctx)
    n = min(batch, len(arr)) if batch > 0 else batch      # never more entries than the array holds
    lib = kca.lib()
    assert lib.attn_decode(vp(q), qd, vp(k), vp(v), kd, hq, hkv, d, cap, n, ptr, window, scale, vp(out), vp(ws),
                           wsb, None) in CODES
    assert lib.attn_prefill_batch(vp(q), qd, vp(k), vp(v), kd, hq, hkv, d, cap, n, rows, ptr, window, scale,
                                  vp(out), vp(ws), wsb, None) in CODES
    assert lib.attn_decode_q8(vp(q), qd, vp(k), vp(v), kd, hq, hkv, d, cap, n, ptr, window, scale, vp(out), vp(ws),
                              wsb, None) in CODES


@settings(max_examples=400, deadline=None, derandomize=True)
@given(ctx=CTX, batch=I32, rows=I32, window=I32, qd=DT, kd=DT, cs=I64, key_begin=I64, cap=I64)
def test_workspace_queries_return_a_size_or_zero_for_any_arguments(ctx, batch, rows, window, qd, kd, cs, key_begin,
                                                                   cap):
    arr, ptr = _arr(ctx)
    n = min(batch, len(arr)) if batch > 0 else batch
    lib = kca.lib()
    for got in (lib.attn_decode_workspace_bytes(n, ptr, window),
                lib.attn_prefill_batch_workspace_bytes(n, rows, ptr, window),
                lib.attn_decode_q8_workspace_bytes(n, ptr, window),
                lib.attn_decode_partial_workspace_bytes(n, ptr, key_begin, cap, window)):
        assert got == 0 or got >= kca.WORKSPACE_HEADER
    got = lib.attn_prefill_workspace_bytes(qd, kd, cs, rows, window)
    assert got == 0 or got >= kca.WORKSPACE_HEADER


@settings(max_examples=300, deadline=None, derandomize=True)
@given(q=PTR, qd=DT, k=PTR, v=PTR, kd=DT, hq=I32, hkv=I32, d=I32, cap=I64, ctx=CTX, batch=I32, window=I32,
       scale=SCALE, out=PTR, ws=PTR, wsb=WSB, bound=I64, key_begin=I64, ctx_dev=PTR)
def test_device_context_static_and_partial_decode_return_a_status(q, qd, k, v, kd, hq, hkv, d, cap, ctx, batch,
                                                                   window, scale, out, ws, wsb, bound, key_begin,
                                                                   ctx_dev):
    arr, ptr = _arr(ctx)
    n = min(batch, len(arr)) if batch > 0 else batch
    lib = kca.lib()
    assert lib.attn_decode_dev(vp(q), qd, vp(k), vp(v), kd, hq, hkv, d, cap, batch, vp(ctx_dev), bound, window,
                               scale, vp(out), vp(ws), wsb, None) in CODES
    assert lib.attn_decode_static(vp(q), qd, vp(k), vp(v), kd, hq, hkv, d, cap, n, ptr, window, scale, vp(out),
                                  None) in CODES
    assert lib.attn_decode_partial(vp(q), qd, vp(k), vp(v), kd, hq, hkv, d, cap, n, ptr, key_begin, window, scale,
                                   vp(out), vp(ws), wsb, None) in CODES


@settings(max_examples=300, deadline=None, derandomize=True)
@given(kn=PTR, vn=PTR, ind=DT, n_rows=I32, cos=PTR, sin=PTR, kc=PTR, vc=PTR, kd=DT, cache_rows=I64, dst=PTR,
       dst0=I64, ws=PTR, n_parts=I32, batch=I32, parts=PTR, stride=I64, out=PTR)
def test_append_and_merge_return_a_status(kn, vn, ind, n_rows, cos, sin, kc, vc, kd, cache_rows, dst, dst0, ws,
                                          n_parts, batch, parts, stride, out):
    lib = kca.lib()
    assert lib.attn_append_kv(vp(kn), vp(vn), ind, n_rows, vp(cos), vp(sin), vp(kc), vp(vc), kd, cache_rows,
                              vp(dst), dst0, vp(ws), None) in CODES
    assert lib.attn_merge_partials(n_parts, batch, vp(parts), stride, vp(out), None) in CODES
