"""Oracle of the quantised-dot attention: int8 codes of K (per cache row) and
of q (per query row and head), the QK dot product taken exactly on the
codes, softmax and the V sum in float64.

TEST INFRASTRUCTURE ONLY (same rules as the rest of `oracle/`): it shares no
code with the CUDA library and never imports it.

What it computes (Karume v0.8.0 release notes, "Fixes": the attention dot
product on packed int8 pairs -- dp4a, or its emulation -- and the per-token
activation quantisation whose scale is amax * f32(1/127), the kernel's form
rather than amax / 127).  For a row x of 256 values, in float32:

    amax  = max_t |x_t|                      (NaN if any x_t is NaN)
    sx    = amax * f32(1/127)                (one f32 product)
    code_t = clamp(round_half_even(x_t / sx), -127, 127)   (f32 division)
             when sx is finite and > 0, else 0

These are integer decisions taken in float32, so the CUDA side takes them in
float32 too and the codes agree bit for bit.  For a query at pos (head h)
and a visible cache row j:

    s_j = scale * sq_h * sk_j * sum_t q8_h[t] k8_j[t]

(the integer sum is exact; the product in float64 here), then the plain
softmax over J(pos) and out = sum_j exp(s_j - max) v_j / sum_j exp(s_j - max)
in float64, NaN-preserving, an empty row exactly 0.  With sx = 0 (an all-zero
row) every code is 0 and the scores are 0; with sx NaN or infinite the codes
are 0 and the scores 0 * sx are NaN.

Packed K rows: the CUDA path keeps each quantised K row as 272 bytes -- the
256 codes, its f32 scale at byte 256, 12 zero bytes -- so that a row stays
16-byte aligned; `pack_rows` / `unpack_rows` write and read that format.
"""
import numpy as np

ROW_BYTES = 272
INV127 = np.float32(1.0) / np.float32(127.0)


def widen32(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored elements -> float32 exactly (bf16 as uint16 bit patterns)."""
    if dtype == "bf16":
        return (np.ascontiguousarray(x, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    return np.asarray(x).astype(np.float32)


def quantize_rows(x32: np.ndarray):
    """Codes (int8, same shape) and scales (float32, one per row of the last
    axis) of float32 rows, by the rule in the module docstring."""
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    flat = x32.reshape(-1, x32.shape[-1])
    amax = np.max(np.abs(flat), axis=1)                    # NaN propagates
    sx = (amax * INV127).astype(np.float32)
    codes = np.zeros(flat.shape, dtype=np.int8)
    ok = np.isfinite(sx) & (sx > 0)
    with np.errstate(invalid="ignore", divide="ignore"):
        q = flat[ok] / sx[ok, None]                        # float32 division, correctly rounded
    codes[ok] = np.clip(np.rint(q), -127, 127).astype(np.int8)
    return codes.reshape(x32.shape), sx.reshape(x32.shape[:-1])


def pack_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """[n, 256] int8 codes + [n] f32 scales -> [n, 272] uint8 packed rows."""
    n = codes.shape[0]
    out = np.zeros((n, ROW_BYTES), dtype=np.uint8)
    out[:, :256] = codes.view(np.uint8)
    out[:, 256:260] = np.ascontiguousarray(scales, dtype=np.float32).reshape(n, 1).view(np.uint8)
    return out


def unpack_rows(packed: np.ndarray):
    """[n, 272] uint8 packed rows -> (codes [n, 256] int8, scales [n] f32)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1, ROW_BYTES)
    codes = packed[:, :256].copy().view(np.int8)
    scales = packed[:, 256:260].copy().view(np.float32).reshape(-1)
    return codes, scales


def attention_q8(q, q_dtype, k_codes, k_scales, v, v_dtype, pos, kv_base=None, *, window=0,
                 scale=1.0 / 16.0):
    """Quantised-dot attention of each query row over its visible cache rows.

    q        : [n_query, 8, 256] stored values of q_dtype
    k_codes  : [rows, 256] int8; k_scales: [rows] float32
    v        : [rows, 256] stored values of v_dtype
    pos      : [n_query] absolute positions; kv_base: first row of each
               query's sequence (default 0)
    Returns float64 [n_query, 8, 256]."""
    from .partial import widen
    q32 = widen32(q, q_dtype)
    n_query, n_heads, d = q32.shape
    q8, sq = quantize_rows(q32)                            # [n, 8, 256], [n, 8]
    kc = np.asarray(k_codes, dtype=np.int64)
    ks = np.asarray(k_scales, dtype=np.float32).astype(np.float64)
    vv = widen(v, v_dtype).reshape(-1, d)
    pos = np.asarray(pos, dtype=np.int64).reshape(n_query)
    base = np.zeros(n_query, dtype=np.int64) if kv_base is None else np.asarray(kv_base, dtype=np.int64)
    out = np.zeros((n_query, n_heads, d), dtype=np.float64)
    for i in range(n_query):
        p = int(pos[i])
        lo = max(0, p - window + 1) if window > 0 else 0
        if p < lo:
            continue
        rows = base[i] + np.arange(lo, p + 1)
        for h in range(n_heads):
            dots = kc[rows] @ q8[i, h].astype(np.int64)     # exact integers
            with np.errstate(invalid="ignore"):
                s = scale * (float(sq[i, h]) * ks[rows]) * dots.astype(np.float64)
            if np.isnan(s).any():
                out[i, h] = np.nan
                continue
            m = s.max()
            w = np.exp(s - m)
            out[i, h] = (w[:, None] * vv[rows]).sum(axis=0) / w.sum()
    return out
