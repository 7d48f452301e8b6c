"""The bounds-checked build (libkca_checked.so, -DKCA_BOUNDS_CHECK): every
index a kernel computes into the caches, the workspace's partial slots and
its merge counters is checked against the extents the host planned, and a
failure is recorded in the status word (error bit 8) instead of making the
access -- the library's stand-in for a memory sanitizer.  Each call below
runs through both builds on the same inputs: the checked build must record
nothing and give the same bits as the normal one (the checks change no
arithmetic)."""
import numpy as np
import pytest
import torch

import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth
from tests.helpers import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def checked(cuda_ok):
    normal = kca.lib()
    chk = kca.load_library(kca.LIB_CHECKED_PATH)
    return normal, chk


def _both(libs, fn):
    """fn() under the normal build, then under the checked one; returns both
    outputs and the checked run's device status."""
    normal, chk = libs
    a = fn()
    torch.cuda.synchronize()
    saved = kca._lib
    kca._lib = chk
    try:
        b = fn()
        torch.cuda.synchronize()
    finally:
        kca._lib = saved
    return a, b


def _ws(n):
    return kca.new_workspace(n)


def _check(libs, fn, ws_list):
    a, b = _both(libs, fn)
    assert torch.equal(a[0] if isinstance(a, tuple) else a, b[0] if isinstance(b, tuple) else b)
    normal, chk = libs
    saved = kca._lib
    kca._lib = chk
    try:
        for ws in ws_list:
            st, detail = kca.attn_device_status(ws)
            assert st == 0, hex(detail)
    finally:
        kca._lib = saved


def _cache(seed, batch, cap, dtype):
    k = dev(synth.draw(seed, "k", (batch, cap, 256), dtype), dtype)
    v = dev(synth.draw(seed, "v", (batch, cap, 256), dtype), dtype)
    return k, v


@pytest.mark.parametrize("dtype,cs,rows,window", [("bf16", 2048, 768, 0), ("bf16", 5000, 300, 300),
                                                  ("f32", 1000, 200, 0), ("bf16", 13000, 7, 0),
                                                  ("f16", 100, 5, 0)])
def test_prefill_through_the_checked_build(checked, dtype, cs, rows, window):
    k, v = _cache(80, 1, cs + rows, dtype)
    q = dev(synth.draw(80, "q", (rows, 8, 256), dtype), dtype)
    code = {"f32": kca.F32, "f16": kca.F16, "bf16": kca.BF16}[dtype]
    ws = _ws(kca.attn_prefill_workspace_bytes(code, code, cs, rows, window))
    _check(checked, lambda: kca.attn_prefill(q, k[0], v[0], cs, window, workspace=ws), [ws])


@pytest.mark.parametrize("kv,batch,cap,window", [("f16", 8, 20000, 0), ("f32", 4, 9000, 0), ("bf16", 3, 6000, 700),
                                                 ("f16", 256, 300, 0), ("f16", 1, 16448, 0)])
def test_decode_through_the_checked_build(checked, kv, batch, cap, window):
    k, v = _cache(81, batch, cap, kv)
    q = dev(synth.draw(81, "q", (batch, 8, 256), "f32"), "f32")
    ctx = [int(c) for c in synth.integers(81, "ctx", 0, cap, batch)]
    ctx[0] = cap
    ws = _ws(kca.attn_decode_workspace_bytes(ctx, window))
    _check(checked, lambda: kca.attn_decode(q, k, v, ctx, window, workspace=ws), [ws])
    dctx = torch.tensor(ctx, dtype=torch.int64, device="cuda")
    ws2 = _ws(kca.attn_decode_workspace_bytes([cap] * batch, window))
    _check(checked, lambda: kca.attn_decode_dev(q, k, v, dctx, cap, window, workspace=ws2), [ws2])


@pytest.mark.parametrize("kv,rows", [("f16", 4), ("f16", 15), ("f32", 3)])
def test_batched_rows_through_the_checked_build(checked, kv, rows):
    batch, cap = 16, 6000
    k, v = _cache(82, batch, cap, kv)
    q = dev(synth.draw(82, "q", (batch, rows, 8, 256), "f32"), "f32")
    ctx = [int(c) for c in synth.integers(82, "ctx", rows, cap, batch)]
    ws = _ws(kca.attn_prefill_batch_workspace_bytes(ctx, rows))
    _check(checked, lambda: kca.attn_prefill_batch(q, k, v, ctx, workspace=ws), [ws])


@pytest.mark.parametrize("v_dtype", ["f16", "f32"])
def test_quantised_decode_through_the_checked_build(checked, v_dtype):
    batch, cap = 6, 20000
    kf, v = _cache(83, batch, cap, v_dtype)
    k8 = kca.attn_quantize_k(kf)
    q = dev(synth.draw(83, "q", (batch, 8, 256), "f32"), "f32")
    ctx = [20000, 1, 0, 5000, 12345, 64]
    ws = _ws(kca.attn_decode_q8_workspace_bytes(ctx))
    _check(checked, lambda: kca.attn_decode_q8(q, k8, v, ctx, workspace=ws), [ws])


def test_context_split_through_the_checked_build(checked):
    batch, cap, shards = 3, 8192, 4
    k, v = _cache(84, batch, cap * shards, "f16")
    q = dev(synth.draw(84, "q", (batch, 8, 256), "f32"), "f32")
    ctx = [cap * shards, 10000, 3]
    parts = torch.empty((shards, kca.partial_floats(batch)), dtype=torch.float32, device="cuda")
    wss = []
    for r in range(shards):
        wss.append(_ws(kca.attn_decode_partial_workspace_bytes(ctx, r * cap, cap)))

    def run():
        for r in range(shards):
            ks = k[:, r * cap:(r + 1) * cap].contiguous()
            vs = v[:, r * cap:(r + 1) * cap].contiguous()
            kca.attn_decode_partial(q, ks, vs, ctx, r * cap, part=parts[r], workspace=wss[r])
        return kca.attn_merge_partials(parts, batch)
    _check(checked, run, wss)
