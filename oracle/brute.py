"""Brute-force attention in Python `decimal` arithmetic (50 significant digits).

TEST INFRASTRUCTURE ONLY: pins the C oracle on tiny inputs.  Written
independently of attn_oracle.c from the same definition -- softmax over the
visible keys of q.k*scale, applied to the value rows (Karume v0.8.0 release
notes, "Breaking Changes", softmax NaN item: NaN-preserving max, fully masked
row = 0; v0.12.0 release notes, "Performance": the f64 reference the parallel
reductions are held to).  Every input value is converted exactly
(Decimal(float) is exact for binary floating point).
"""
from decimal import Decimal, getcontext
import math

import numpy as np

PREC = 50


def _dec(x: float) -> Decimal:
    return Decimal(float(x))


def attention(q, k, v, pos, kv_base=None, *, window=0, scale=1.0 / 16.0, n_kv_heads=1):
    """q: [n, Hq, d] (any float dtype); k, v: [rows, Hkv, d] or [rows, d]; pos: [n].

    Returns a nested list [n][Hq][d] of Decimal (NaN as Decimal('NaN')).
    """
    getcontext().prec = PREC
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if k.ndim == 2:
        k = k[:, None, :]
        v = v[:, None, :]
    n, hq, d = q.shape
    hkv = n_kv_heads
    group = hq // hkv
    if kv_base is None:
        kv_base = [0] * n
    sc = _dec(scale)
    result = []
    for i in range(n):
        p = int(pos[i])
        lo = max(0, p - window + 1) if window > 0 else 0
        keys = list(range(lo, p + 1)) if p >= lo else []
        per_head = []
        for h in range(hq):
            g = h // group
            if not keys:
                per_head.append([Decimal(0)] * d)
                continue
            scores = []
            nan_seen = False
            for j in keys:
                row = int(kv_base[i]) + j
                vals = [(q[i, h, t], k[row, g, t]) for t in range(d)]
                if any(math.isnan(a) or math.isnan(b) for a, b in vals):
                    nan_seen = True
                    scores.append(None)
                    continue
                dot = sum((_dec(a) * _dec(b) for a, b in vals), Decimal(0))
                scores.append(sc * dot)
            if nan_seen:
                per_head.append([Decimal("NaN")] * d)
                continue
            m = max(scores)
            weights = [(s - m).exp() for s in scores]
            den = sum(weights, Decimal(0))
            out = []
            for t in range(d):
                num = sum((w * _dec(v[int(kv_base[i]) + j, g, t]) for w, j in zip(weights, keys)),
                          Decimal(0))
                out.append(num / den)
            per_head.append(out)
        result.append(per_head)
    return result


def to_float64(res) -> np.ndarray:
    return np.array([[[float(x) for x in row] for row in head] for head in res], dtype=np.float64)
