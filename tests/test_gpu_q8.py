"""The quantised-dot attention on the GPU against oracle/quant.py: the packed
int8 K rows of attn_quantize_k are the oracle's bytes exactly (codes and
scale; the codes are integer decisions both sides take in float32), and
attn_decode_q8 -- the query quantised inside the kernel, QK exact on the
codes, softmax and V sum in f32 -- matches the oracle's float64 attention
over the same codes within the bar of V's dtype (2e-6 for f32 V, 4e-3 for
16-bit V), over ragged batches, windows, long contexts and NaN rows.  The
device canary must find the dp4a instruction sane on B200."""
import numpy as np
import pytest
import torch

import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth
from oracle import quant
from tests.helpers import dev, max_err

pytestmark = pytest.mark.gpu

TOL = {"f32": 2e-6, "f16": 4e-3, "bf16": 4e-3}


@pytest.fixture(scope="module", autouse=True)
def _setup(cuda_ok):
    kca.lib()


def test_canary_finds_every_variant_sane():
    # dp4a, its emulation and the int8 MMA all give the known answers on B200
    assert kca.attn_dot_canary() == 7


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_quantized_rows_are_the_oracle_bytes(dtype):
    k = synth.draw(70, "k", (1000, 256), dtype, 3.0)
    k32 = quant.widen32(k, dtype)
    if dtype == "f32":
        k[5] = 0.0
        k[6, 9] = np.nan
        k[7, 3] = np.inf
        k[8, :8] = [127.0, -126.5, 2.5, 3.5, -2.5, 0.5, 1.5, -0.5]
        k[8, 8:] = 0.0
        k32 = k
    got = kca.attn_quantize_k(dev(k, dtype)).cpu().numpy()
    codes, scales = quant.quantize_rows(k32)
    assert got.shape == (1000, quant.ROW_BYTES)
    got_codes, got_scales = quant.unpack_rows(got)
    assert np.array_equal(got_codes, codes)                       # every integer decision
    assert np.array_equal(got_scales, scales, equal_nan=True)     # bit for bit, NaN payloads aside
    assert not got[:, 260:].any()


def _case(seed, batch, cap, ctx, q_dtype, v_dtype, std=1.0):
    k = synth.normal(seed, "k", (batch * cap, 256), std)
    codes, scales = quant.quantize_rows(k)
    packed = quant.pack_rows(codes, scales)
    v = synth.draw(seed, "v", (batch, cap, 256), v_dtype)
    q = synth.draw(seed, "q", (batch, 8, 256), q_dtype)
    return codes, scales, packed.reshape(batch, cap, quant.ROW_BYTES), v, q


def _oracle(codes, scales, v, q, ctx, window, q_dtype, v_dtype):
    batch, cap = v.shape[0], v.shape[1]
    pos = np.asarray(ctx) - 1
    base = np.arange(batch) * cap
    return quant.attention_q8(q, q_dtype, codes, scales, v.reshape(-1, 256), v_dtype, pos, base, window=window,
                              scale=synth.SCALE)


@pytest.mark.parametrize("q_dtype,v_dtype,window", [("f32", "f32", 0), ("f32", "f16", 0), ("bf16", "bf16", 300),
                                                    ("f16", "f32", 1000), ("f32", "bf16", 0)])
def test_decode_q8_matches_oracle(q_dtype, v_dtype, window):
    # 16-bit V: the tensor-core kernel (int8 MMA); f32 V: the CUDA-core one (dp4a)
    batch, cap = 6, 5000
    ctx = [5000, 1, 0, 64, 4097, 2345]
    codes, scales, packed, v, q = _case(71, batch, cap, ctx, q_dtype, v_dtype)
    ws = kca.new_workspace(kca.attn_decode_q8_workspace_bytes(ctx, window))
    out = kca.attn_decode_q8(dev(q, q_dtype), torch.from_numpy(packed).cuda(), dev(v, v_dtype), ctx, window,
                             workspace=ws)
    want = _oracle(codes, scales, v, q, ctx, window, q_dtype, v_dtype)
    assert max_err(out.cpu().numpy(), want) <= TOL[v_dtype]
    assert torch.all(out[2] == 0)
    assert kca.attn_device_status(ws)[0] == 0


def test_decode_q8_long_contexts_f32():
    batch, cap = 2, 65536
    ctx = [16384, 65536]
    codes, scales, packed, v, q = _case(72, batch, cap, ctx, "f32", "f32")
    out = kca.attn_decode_q8(dev(q, "f32"), torch.from_numpy(packed).cuda(), dev(v, "f32"), ctx)
    want = _oracle(codes, scales, v, q, ctx, 0, "f32", "f32")
    assert max_err(out.cpu().numpy(), want) <= 2e-6


def test_decode_q8_on_the_library_quantizer_and_nan_rows():
    # K quantised on the GPU by attn_quantize_k, one K row NaN (its scale
    # NaN): only the sequence that sees it is NaN
    batch, cap = 3, 3000
    ctx = [3000, 1500, 2999]
    k = synth.draw(73, "k", (batch, cap, 256), "f16")
    k[0, 1700, 4] = np.nan
    v = synth.draw(73, "v", (batch, cap, 256), "f16")
    q = synth.draw(73, "q", (batch, 8, 256), "f32")
    k8 = kca.attn_quantize_k(dev(k, "f16"))
    out = kca.attn_decode_q8(dev(q, "f32"), k8, dev(v, "f16"), ctx).cpu().numpy()
    codes, scales = quant.quantize_rows(quant.widen32(k, "f16").reshape(-1, 256))
    want = _oracle(codes, scales, v, q, ctx, 0, "f32", "f16")
    assert np.isnan(out[0]).all() and np.isnan(want[0]).all()
    assert max_err(out[1:], want[1:]) <= 4e-3


def test_decode_q8_cuda_core_kernel_on_16bit_v():
    # the dp4a kernel pinned on a 16-bit V cache gives the oracle's values too
    batch, cap = 3, 4000
    ctx = [4000, 17, 2500]
    codes, scales, packed, v, q = _case(74, batch, cap, ctx, "f32", "f16")
    with kca.forced_path(kca.OP_ROWS, kca.PATH_CUDA_CORE):
        out = kca.attn_decode_q8(dev(q, "f32"), torch.from_numpy(packed).cuda(), dev(v, "f16"), ctx)
    want = _oracle(codes, scales, v, q, ctx, 0, "f32", "f16")
    assert max_err(out.cpu().numpy(), want) <= 4e-3


def test_decode_q8_at_the_maximum_batch():
    batch, cap = kca.MAX_BATCH, 700
    ctx = list(synth.integers(75, "ctx", 0, cap, batch))
    ctx[0], ctx[1] = 0, cap
    codes, scales, packed, v, q = _case(75, batch, cap, ctx, "f32", "f16")
    ws = kca.new_workspace(kca.attn_decode_q8_workspace_bytes(ctx))
    out = kca.attn_decode_q8(dev(q, "f32"), torch.from_numpy(packed).cuda(), dev(v, "f16"), ctx, workspace=ws)
    want = _oracle(codes, scales, v, q, ctx, 0, "f32", "f16")
    assert max_err(out.cpu().numpy(), want) <= 4e-3
    assert torch.all(out[0] == 0)
    assert kca.attn_device_status(ws)[0] == 0
