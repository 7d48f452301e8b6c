"""attn_prefill_batch: short chunks (1-15 query rows) of several sequences in
one call, every row against the f64 oracle (row i of sequence b at position
ctx[b] - rows + i, its own sequence's keys), for 1, 8 and 64 sequences of
ragged contexts (the shortest exactly `rows` long, one at the capacity),
both multi-row tensor-core kernels (16-bit cache: units of up to 4 rows of
a sequence; the tcgen05 kernel and the mma.sync one, pinned with
attn_force_path) and the CUDA-core kernel (f32 cache), with and without a
window, against attn_prefill of the same rows; and with one row per
sequence it is attn_decode, bit for bit."""
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


# the multi-row kernel of 16-bit caches: tcgen05 (the automatic choice) or mma.sync
BATCH_PATHS = [kca.PATH_TCGEN05, kca.PATH_MMA_SYNC]


@pytest.fixture(params=BATCH_PATHS, ids=["tcgen05", "mma_sync"])
def batch_path(request):
    with kca.forced_path(kca.OP_BATCH, request.param):
        yield request.param


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
def test_batched_short_chunks_match_oracle(batch, rows, batch_path):
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
def test_batched_short_chunks_dtypes_and_window(q_dtype, kv_dtype, window, batch_path):
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
def test_rows_of_one_sequence_match_a_prefill_chunk(rows, batch_path):
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


def test_multirow_units_with_a_window_cut_inside_a_unit(batch_path):
    # window 100 over 15 rows: the unit's rows see different ranges, and the
    # first rows' keys before the later rows' windows are masked per row
    batch, rows, cap = 5, 15, 6000
    ctx, q, k, v = _inputs(62, batch, rows, cap, "f32", "f16")
    out = kca.attn_prefill_batch(dev(q, "f32"), dev(k, "f16"), dev(v, "f16"), ctx, 100)
    want = _oracle(q, k, v, ctx, rows, 100, "f32", "f16")
    assert max_err(out.cpu().numpy(), want) <= 4e-3


@pytest.mark.parametrize("q_dtype,kv_dtype", [("f32", "f16"), ("f32", "f32")])
def test_batched_short_chunks_at_the_maximum_sizes(q_dtype, kv_dtype, batch_path):
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


@pytest.mark.parametrize("q_dtype,kv_dtype", [("f32", "f16"), ("f32", "bf16"), ("bf16", "bf16"), ("f16", "f16")])
def test_the_two_multirow_kernels_agree(q_dtype, kv_dtype):
    # long ragged contexts (several splits per unit, a ragged last stage),
    # rows 6 (units of 4 and 2): tcgen05 and mma.sync within the tolerance of
    # the inputs' type, both within it of the oracle on sampled sequences
    batch, rows, cap = 12, 6, 40000
    ctx, q, k, v = _inputs(64, batch, rows, cap, q_dtype, kv_dtype)
    qd, kd, vd = dev(q, q_dtype), dev(k, kv_dtype), dev(v, kv_dtype)
    outs = {}
    for path in BATCH_PATHS:
        with kca.forced_path(kca.OP_BATCH, path):
            ws = kca.new_workspace(kca.attn_prefill_batch_workspace_bytes(ctx, rows))
            outs[path] = kca.attn_prefill_batch(qd, kd, vd, ctx, workspace=ws).cpu().numpy()
            assert kca.attn_device_status(ws)[0] == 0
    assert np.isfinite(outs[kca.PATH_TCGEN05]).all()
    assert np.max(np.abs(outs[kca.PATH_TCGEN05] - outs[kca.PATH_MMA_SYNC])) <= tol(q_dtype, kv_dtype)
    seqs = [0, 1, 7]
    want = _oracle(q[seqs], k[seqs], v[seqs], [ctx[s] for s in seqs], rows, 0, q_dtype, kv_dtype)
    for path in BATCH_PATHS:
        assert max_err(outs[path][seqs], want) <= tol(q_dtype, kv_dtype)


def test_tcgen05_multirow_nan_score_reaches_exactly_the_rows_that_see_it():
    # a NaN in key j of sequence 0: rows at positions >= j are NaN, the
    # others (and other sequences) finite and equal to the oracle
    batch, rows, cap = 3, 7, 5000
    ctx, q, k, v = _inputs(65, batch, rows, cap, "f32", "f16")
    ctx[0] = 4000
    j = ctx[0] - 4                      # seen by rows 3..6 of sequence 0
    k[0, j, 17] = np.float16(np.nan)
    with kca.forced_path(kca.OP_BATCH, kca.PATH_TCGEN05):
        out = kca.attn_prefill_batch(dev(q, "f32"), dev(k, "f16"), dev(v, "f16"), ctx).cpu().numpy()
    assert np.isnan(out[0, 3:]).all()
    assert np.isfinite(out[0, :3]).all() and np.isfinite(out[1:]).all()
    want = _oracle(q[1:], k[1:], v[1:], ctx[1:], rows, 0, "f32", "f16")
    assert max_err(out[1:], want) <= 4e-3


@pytest.mark.parametrize("path", BATCH_PATHS, ids=["tcgen05", "mma_sync"])
def test_nan_in_a_value_row_reaches_the_whole_multirow_unit(path):
    # include/kca.h, PRECONDITIONS: V must be finite on the union of a
    # multi-row unit's visible ranges.  A NaN V row at position ctx - 4 of
    # sequence 0 (6 rows: units of rows 0-3 and 4-5) is seen by rows 2-5;
    # rows 0-1 share unit 0 with rows that see it, so the kernels' exact-zero
    # probabilities meet the NaN there too: the whole of both units is NaN,
    # every other sequence finite and equal to the oracle.  The f32 rows path
    # (one unit per row) poisons exactly the rows that see the position.
    batch, rows, cap = 3, 6, 3000
    ctx, q, k, v = _inputs(66, batch, rows, cap, "f32", "f16")
    ctx[0] = 2000
    v[0, ctx[0] - 4, 100] = np.float16(np.nan)
    with kca.forced_path(kca.OP_BATCH, path):
        out = kca.attn_prefill_batch(dev(q, "f32"), dev(k, "f16"), dev(v, "f16"), ctx).cpu().numpy()
    assert np.isnan(out[0]).any(axis=(1, 2)).all()
    assert np.isfinite(out[1:]).all()
    want = _oracle(q[1:], k[1:], v[1:], ctx[1:], rows, 0, "f32", "f16")
    assert max_err(out[1:], want) <= 4e-3
    out32 = kca.attn_prefill_batch(dev(q, "f32"), dev(k.astype(np.float32), "f32"), dev(v.astype(np.float32), "f32"),
                                   ctx).cpu().numpy()
    assert np.isfinite(out32[0, :2]).all() and np.isnan(out32[0, 2:]).any(axis=(1, 2)).all()


@pytest.mark.parametrize("q_dtype,kv_dtype,rows,cs,window", [("f32", "bf16", 8, 20000, 0), ("f32", "f16", 15, 30000, 0),
                                                            ("bf16", "bf16", 2, 16000, 0),
                                                            ("f32", "bf16", 5, 40000, 20000)])
def test_short_prefill_chunks_on_multi_row_units(q_dtype, kv_dtype, rows, cs, window):
    # attn_prefill routes 2-15-row chunks on a 16-bit cache that the
    # tensor-core path does not take to multi-row units from 12,288 keys: every
    # row against the oracle, and the rows path (pinned) within tolerance
    from tests.helpers import oracle_prefill
    code = {"f32": kca.F32, "f16": kca.F16, "bf16": kca.BF16}
    assert kca.attn_prefill_path(code[q_dtype], code[kv_dtype], cs, rows, window) == kca.PATH_MULTI_ROW
    cap = cs + rows
    q = synth.draw(67, "q", (rows, 8, 256), q_dtype)
    k = synth.draw(67, "k", (cap, 256), kv_dtype)
    v = synth.draw(67, "v", (cap, 256), kv_dtype)
    qd, kd, vd = dev(q, q_dtype), dev(k, kv_dtype), dev(v, kv_dtype)
    ws = kca.new_workspace(kca.attn_prefill_workspace_bytes(kca.dtype_code(qd), kca.dtype_code(kd), cs, rows, window))
    got = kca.attn_prefill(qd, kd, vd, cs, window, workspace=ws).cpu().numpy()
    assert kca.attn_device_status(ws)[0] == 0
    want = oracle_prefill(q, k, v, cs, np.arange(rows), window, q_dtype, kv_dtype)
    assert max_err(got, want) <= tol(q_dtype, kv_dtype)
    with kca.forced_path(kca.OP_PREFILL, kca.PATH_ROWS):
        ref = kca.attn_prefill(qd, kd, vd, cs, window).cpu().numpy()
    assert np.max(np.abs(got - ref)) <= tol(q_dtype, kv_dtype)
