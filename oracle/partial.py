"""Oracle of decode over a context shard (partial-softmax states) and of the
merge of such states.

TEST INFRASTRUCTURE ONLY (same rules as the rest of `oracle/`): it shares no
code with the CUDA library and never imports it.

What it computes.  The decode of the Karume v0.12.0 release notes
("Performance", items 2-3: the softmax-weighted sum of V over a decode row's
keys, reduced in another order) restricted to the keys one shard holds.  For
a query at pos = ctx_len - 1 (head h, scaled scores s_j = scale * q_h . k_j)
and the keys J of its causal / window range that lie in the shard
[key_begin, key_end):

    m   = max_{j in J} s_j          (NaN if any s_j is NaN)
    l   = sum_{j in J} exp(s_j - m)
    acc = sum_{j in J} exp(s_j - m) v_j

and (m, l, acc) = (-inf, 0, 0) when J is empty.  The merge of states p is the
log-sum-exp identity

    M = max_p m_p,   out = sum_p e^(m_p - M) acc_p / sum_p e^(m_p - M) l_p,

with empty states weighted 0 and out = 0 when every state is empty (the
fully masked row of the v0.8.0 notes, "Breaking", softmax item).  All in
float64 from the exact stored values; plain loops over sequences and heads,
numpy for the dot products and sums.
"""
import math

import numpy as np


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored elements -> float64 exactly (bf16 as uint16 bit patterns)."""
    if dtype == "bf16":
        return (np.ascontiguousarray(x, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(x).astype(np.float64)


def shard_keys(pos: int, window: int, key_begin: int, key_end: int) -> range:
    """Absolute positions of the keys a query at pos sees inside the shard."""
    lo = max(0, pos - window + 1) if window > 0 else 0
    return range(max(lo, key_begin), min(pos + 1, key_end))


def decode_partial(q, k_shard, v_shard, ctx_len, key_begin, *, window=0, scale=1.0 / 16.0,
                   q_dtype="f32", kv_dtype="f32"):
    """States of every (sequence, head) over one shard.

    q: [batch, 8, 256]; k_shard / v_shard: [batch, capacity, 256] holding
    positions [key_begin, key_begin + capacity).  Returns (m [batch, 8],
    l [batch, 8], acc [batch, 8, 256]) in float64.
    """
    qd = widen(q, q_dtype)
    kd = widen(k_shard, kv_dtype)
    vd = widen(v_shard, kv_dtype)
    batch, heads, dim = qd.shape
    key_end = key_begin + kd.shape[1]
    m = np.full((batch, heads), -np.inf)
    l = np.zeros((batch, heads))
    acc = np.zeros((batch, heads, dim))
    for b in range(batch):
        keys = shard_keys(int(ctx_len[b]) - 1, window, key_begin, key_end)
        if len(keys) == 0:
            continue
        rows = np.arange(keys.start, keys.stop) - key_begin
        for h in range(heads):
            s = scale * (kd[b, rows] @ qd[b, h])
            mh = np.nan if np.isnan(s).any() else s.max()
            w = np.exp(s - mh)
            m[b, h] = mh
            l[b, h] = w.sum()
            acc[b, h] = w @ vd[b, rows]
    return m, l, acc


def merge_partials(ms, ls, accs):
    """Merge states in the order given: ms / ls [n, batch, 8], accs
    [n, batch, 8, 256] -> out [batch, 8, 256] float64."""
    ms = np.asarray(ms, dtype=np.float64)
    ls = np.asarray(ls, dtype=np.float64)
    accs = np.asarray(accs, dtype=np.float64)
    n, batch, heads = ms.shape
    out = np.zeros(accs.shape[1:])
    for b in range(batch):
        for h in range(heads):
            col = ms[:, b, h]
            if np.isnan(col).any():
                out[b, h] = np.nan
                continue
            M = col.max()
            if M == -math.inf:
                continue                      # every state empty: exactly 0
            w = np.where(col == -math.inf, 0.0, np.exp(col - M))
            out[b, h] = (w @ accs[:, b, h]) / (w @ ls[:, b, h])
    return out
