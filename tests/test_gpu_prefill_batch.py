"""attn_prefill_batch: short chunks (1-15 query rows) of several sequences in
one call, every row against the f64 oracle (row i of sequence b at position
ctx[b] - rows + i, its own sequence's keys), for 1, 8 and 64 sequences of
ragged contexts (the shortest exactly `rows` long, one at the capacity),
the multi-row tensor-core kernel (16-bit cache: units of up to 4 rows of a
sequence) and the CUDA-core kernel (f32 cache), with and without a window,
against attn_prefill of the same rows; and with one row per sequence it is
attn_decode, bit for bit."""
import numpy as np
import pytest
import torch

import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth
from tests.helpers import dev, max_err, oracle_threads, tol
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(cuda_ok):
    oracle_threads()
    kca.lib()


def _inputs(seed, batch, rows, cap, q_dtype, kv_dtype):
    ctx = synth.integers(seed, "ctx", rows, cap, batch)
    ctx[0] = rows
    if batch > 1:
        ctx[1] = cap
    k = synth.draw(seed, "k", (batch, cap, 256), kv_dtype)
    v = synth.draw(seed, "v", (batch, cap, 256), kv_dtype)
    q = synth.draw(seed, "q", (batch, rows, 8, 256), q_dtype)
    return [int(c) for c in ctx], q, k, v


def _oracle(q, k, v, ctx, rows, window, q_dtype, kv_dtype):
    batch, cap = k.shape[0], k.shape[1]
    pos = np.array([c - rows + i for c in ctx for i in range(rows)], dtype=np.int64)
    base = np.repeat(np.arange(batch, dtype=np.int64) * cap, rows)
    want = oracle.attention(q.reshape(batch * rows, 8, 256), k.reshape(-1, 256), v.reshape(-1, 256), pos, base,
                            window=window, scale=synth.SCALE, q_dtype=q_dtype, kv_dtype=kv_dtype)
    return want.reshape(batch, rows, 8, 256)


@pytest.mark.parametrize("batch", [1, 8, 64])
@pytest.mark.parametrize("rows", [1, 3, 15])
def test_batched_short_chunks_match_oracle(batch, rows):
    cap = 20000 if batch <= 8 else 5000
    ctx, q, k, v = _inputs(40 + rows, batch, rows, cap, "f32", "f16")
    ws = kca.new_workspace(kca.attn_prefill_batch_workspace_bytes(ctx, rows))
    out = kca.attn_prefill_batch(dev(q, "f32"), dev(k, "f16"), dev(v, "f16"), ctx, workspace=ws)
    want = _oracle(q, k, v, ctx, rows, 0, "f32", "f16")
    assert max_err(out.cpu().numpy(), want) <= 4e-3
    st, detail = kca.attn_device_status(ws)
    assert st == 0, hex(detail)


@pytest.mark.parametrize("q_dtype,kv_dtype,window", [("bf16", "bf16", 300), ("f32", "f32", 0), ("f32", "f32", 700),
                                                     ("f16", "bf16", 0)])
def test_batched_short_chunks_dtypes_and_window(q_dtype, kv_dtype, window):
    batch, rows, cap = 8, 5, 9000
    ctx, q, k, v = _inputs(50, batch, rows, cap, q_dtype, kv_dtype)
    out = kca.attn_prefill_batch(dev(q, q_dtype), dev(k, kv_dtype), dev(v, kv_dtype), ctx, window)
    want = _oracle(q, k, v, ctx, rows, window, q_dtype, kv_dtype)
    assert max_err(out.cpu().numpy(), want) <= tol(q_dtype, kv_dtype)


@pytest.mark.parametrize("kv_dtype", ["f16", "f32"])
def test_one_row_per_sequence_is_decode_bit_for_bit(kv_dtype):
    batch, cap = 8, 30000
    ctx, q, k, v = _inputs(60, batch, 1, cap, "f32", kv_dtype)
    qd, kd, vd = dev(q, "f32"), dev(k, kv_dtype), dev(v, kv_dtype)
    got = kca.attn_prefill_batch(qd, kd, vd, ctx)
    want = kca.attn_decode(qd.view(batch, 8, 256), kd, vd, ctx)
    assert torch.equal(got.view(batch, 8, 256), want)


@pytest.mark.parametrize("rows", [2, 4, 5, 7, 15])
def test_rows_of_one_sequence_match_a_prefill_chunk(rows):
    # one sequence: the batched call (multi-row units of up to 4 rows) and
    # attn_prefill of the same rows agree; both against the oracle
    cap = 3000
    ctx, q, k, v = _inputs(61, 1, rows, cap, "bf16", "bf16")
    ctx = [cap]
    qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    got = kca.attn_prefill_batch(qd, kd, vd, ctx)
    want = kca.attn_prefill(qd[0], kd[0], vd[0], cap - rows)
    assert torch.isfinite(got).all()
    assert (got[0] - want).abs().max().item() <= 4e-3
    ref = _oracle(q, k, v, ctx, rows, 0, "bf16", "bf16")
    assert max_err(got.cpu().numpy(), ref) <= 4e-3


def test_multirow_units_with_a_window_cut_inside_a_unit():
    # window 100 over 15 rows: the unit's rows see different ranges, and the
    # first rows' keys before the later rows' windows are masked per row
    batch, rows, cap = 5, 15, 6000
    ctx, q, k, v = _inputs(62, batch, rows, cap, "f32", "f16")
    out = kca.attn_prefill_batch(dev(q, "f32"), dev(k, "f16"), dev(v, "f16"), ctx, 100)
    want = _oracle(q, k, v, ctx, rows, 100, "f32", "f16")
    assert max_err(out.cpu().numpy(), want) <= 4e-3


@pytest.mark.parametrize("q_dtype,kv_dtype", [("f32", "f16"), ("f32", "f32")])
def test_batched_short_chunks_at_the_maximum_sizes(q_dtype, kv_dtype):
    # KCA_MAX_BATCH sequences x KCA_MAX_BATCH_ROWS rows (3,840 rows, 1,024
    # multi-row units on 16-bit caches), short ragged contexts
    batch, rows, cap = kca.MAX_BATCH, kca.MAX_BATCH_ROWS, 96
    ctx, q, k, v = _inputs(63, batch, rows, cap, q_dtype, kv_dtype)
    ws = kca.new_workspace(kca.attn_prefill_batch_workspace_bytes(ctx, rows))
    out = kca.attn_prefill_batch(dev(q, q_dtype), dev(k, kv_dtype), dev(v, kv_dtype), ctx, workspace=ws)
    want = _oracle(q, k, v, ctx, rows, 0, q_dtype, kv_dtype)
    assert max_err(out.cpu().numpy(), want) <= tol(q_dtype, kv_dtype)
    assert kca.attn_device_status(ws)[0] == 0
    with pytest.raises(kca.KcaError):   # one row more than the limit: rejected before any launch
        kca.attn_prefill_batch(torch.zeros((1, rows + 1, 8, 256), device="cuda"),
                               dev(k[:1], kv_dtype), dev(v[:1], kv_dtype), [rows + 1])
