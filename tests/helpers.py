"""Shared helpers of the GPU tests: inputs come from synth (both sides see the
same bytes), expected values from the oracle only."""
import os

import numpy as np

import oracle
from kv_cache_attention_states_b200 import synth

TOL = {"f32": 2e-6, "f16": 4e-3, "bf16": 4e-3}


def tol(q_dtype: str, kv_dtype: str) -> float:
    return max(TOL[q_dtype], TOL[kv_dtype])


def dev(arr: np.ndarray, dtype: str):
    return synth.as_torch(arr, dtype).cuda()


def oracle_threads():
    oracle.set_threads(os.cpu_count() or 1)


def oracle_prefill(q, k, v, chunk_start, rows_idx, window, q_dtype, kv_dtype, scale=synth.SCALE):
    """Oracle output of chunk rows rows_idx (chunk_start + i) of a single sequence."""
    rows_idx = np.asarray(rows_idx, dtype=np.int64)
    return oracle.attention(q[rows_idx], k, v, chunk_start + rows_idx, window=window, scale=scale,
                            q_dtype=q_dtype, kv_dtype=kv_dtype)


def oracle_decode(q, k, v, ctx, window, q_dtype, kv_dtype, capacity, seqs=None, scale=synth.SCALE):
    """Oracle output of decode rows; k/v [batch, capacity, 256]."""
    batch = q.shape[0]
    seqs = np.arange(batch) if seqs is None else np.asarray(seqs)
    ctx = np.asarray(ctx, dtype=np.int64)
    kf = k.reshape(-1, k.shape[-1])
    vf = v.reshape(-1, v.shape[-1])
    return oracle.attention(q[seqs], kf, vf, ctx[seqs] - 1, seqs * capacity, window=window,
                            scale=scale, q_dtype=q_dtype, kv_dtype=kv_dtype)


def max_err(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    return float(np.max(np.abs(got - want))) if got.size else 0.0
