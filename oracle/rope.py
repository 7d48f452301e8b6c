"""Oracle of the K/V append with rotary position embedding (RoPE).

TEST INFRASTRUCTURE ONLY (same rules as the rest of `oracle/`): it shares no
code with the CUDA library and never imports it.

What it computes.  The pages state that rotary cos/sin rows are generated on
the host for each chunk from the model's rope parameters and handed to the
graph as inputs (Karume v0.8.0 release notes, "Features", conversation-window
item; the Gemma 4 E2B model page, "Context" item).  They do not print the
rotation itself; the plainest reading, the one Gemma models use, is the
"rotate-half" pairing of dim i with dim i + 128:

    out[i]       = x[i]       * cos[i]       - x[i + 128] * sin[i]
    out[i + 128] = x[i + 128] * cos[i + 128] + x[i]       * sin[i + 128]

for i < 128, with cos/sin rows of the full head_dim (the host duplicates the
frequencies over both halves).  Precision: every product and the sum/
difference are rounded to float32 (no fused multiply-add), then the result is
rounded to the cache's type with round-to-nearest-even; the append is a copy
of those bytes into the cache rows.  V rows are only converted.

Arrays are numpy arrays in stored form: float32, float16, or bf16 as uint16
bit patterns.
"""
import numpy as np

HALF = 128


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even; NaN stays a quiet NaN."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) & 0xFFFF
    r = np.where(nan, ((u >> 16) | 0x40) & 0xFFFF, r)
    return r.astype(np.uint16)


def f32_from_stored(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored values -> float32 (exact for every stored type)."""
    if dtype == "bf16":
        return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    return np.asarray(x).astype(np.float32)


def to_stored(x32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return x32.astype(np.float32)
    if dtype == "f16":
        return x32.astype(np.float16)
    if dtype == "bf16":
        return bf16_bits_from_f32(x32)
    raise ValueError(dtype)


def rope_rotate(x32: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE of rows x32 [n, 256] float32 with cos/sin [n, 256] float32,
    every operation rounded to float32."""
    x32 = np.asarray(x32, dtype=np.float32)
    cos = np.asarray(cos, dtype=np.float32)
    sin = np.asarray(sin, dtype=np.float32)
    x1, x2 = x32[:, :HALF], x32[:, HALF:]
    out = np.empty_like(x32)
    out[:, :HALF] = (x1 * cos[:, :HALF]).astype(np.float32) - (x2 * sin[:, :HALF]).astype(np.float32)
    out[:, HALF:] = (x2 * cos[:, HALF:]).astype(np.float32) + (x1 * sin[:, HALF:]).astype(np.float32)
    return out


def append_kv(k_new, v_new, in_dtype, cos, sin, k_cache, v_cache, kv_dtype, dst_rows):
    """Returns copies of k_cache / v_cache ([rows, 256] stored arrays) with new
    row i written at dst_rows[i]: K rotated (when cos is not None) and both
    converted to the cache type.  Rows whose destination lies outside the
    cache are skipped."""
    k_out = np.array(k_cache, copy=True)
    v_out = np.array(v_cache, copy=True)
    k32 = f32_from_stored(k_new, in_dtype)
    v32 = f32_from_stored(v_new, in_dtype)
    if cos is not None:
        k32 = rope_rotate(k32, cos, sin)
    ks = to_stored(k32, kv_dtype)
    vs = to_stored(v32, kv_dtype)
    for i, r in enumerate(np.asarray(dst_rows, dtype=np.int64)):
        if 0 <= r < k_out.shape[0]:
            k_out[r] = ks[i]
            v_out[r] = vs[i]
    return k_out, v_out


def rope_tables(positions, theta: float = 10000.0, dim: int = 256):
    """cos/sin rows [n, dim] float32 of the standard RoPE frequencies
    inv_freq[j] = theta^(-2j/dim), duplicated over both halves (what a host
    generates per chunk), computed in float64 and rounded once."""
    pos = np.asarray(positions, dtype=np.float64)[:, None]
    inv = theta ** (-np.arange(0, dim // 2, dtype=np.float64) * 2.0 / dim)
    ang = pos * inv[None, :]
    ang = np.concatenate([ang, ang], axis=1)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
