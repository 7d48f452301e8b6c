"""Pins of the quantised-dot attention oracle (oracle/quant.py), against
things other than itself:

* the per-row quantisation against a Python-decimal brute force: the scale
  is the float32 nearest to amax x f32(1/127) (the kernel form the Karume
  v0.8.0 release notes give, "Fixes", activation-quantisation item), each
  code the half-to-even rounding of the float32 nearest to x / scale, found
  with exact decimal arithmetic and an explicit nearest-float32 search;
* rounding-mode and special cases: ties go to even, the largest |x| maps to
  +-127, signs are kept, zero / NaN / infinite rows;
* the attention against the C oracle run on the dequantised inputs
  (q8 x sq and k8 x sk, exact in float64): the same scores, so the same
  output to 1e-12, over windows, batches, dtypes and NaN / zero rows;
* the packed 272-byte row format round trip.
"""
from decimal import ROUND_HALF_EVEN, Decimal, getcontext

import numpy as np
import pytest

import oracle
from oracle import quant
from kv_cache_attention_states_b200 import synth

getcontext().prec = 80


def _nearest_f32(d: Decimal) -> np.float32:
    """The float32 nearest to the decimal d (ties to even mantissa), by
    comparing exact distances to the two float32 neighbours of a guess."""
    g = np.float32(float(d))
    cands = {g, np.nextafter(g, np.float32(np.inf)), np.nextafter(g, np.float32(-np.inf))}
    best = None
    for c in cands:
        dist = abs(Decimal(float(c)) - d)
        key = (dist, int(np.array(c, dtype=np.float32).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return np.float32(best[1])


def _brute_row(x32: np.ndarray):
    inv = _nearest_f32(Decimal(1) / Decimal(127))
    amax = max(abs(Decimal(float(v))) for v in x32)
    sx = _nearest_f32(amax * Decimal(float(inv)))
    if not (np.isfinite(sx) and sx > 0):
        return np.zeros(x32.size, dtype=np.int64), sx
    codes = []
    for v in x32:
        qf = _nearest_f32(Decimal(float(v)) / Decimal(float(sx)))
        c = int(Decimal(float(qf)).quantize(Decimal(1), rounding=ROUND_HALF_EVEN))
        codes.append(max(-127, min(127, c)))
    return np.array(codes, dtype=np.int64), sx


@pytest.mark.parametrize("seed,std", [(0, 1.0), (1, 1e-3), (2, 300.0), (3, 1e-30)])
def test_quantisation_equals_decimal_brute_force(seed, std):
    x = synth.normal(seed, "qx", (6, 256), std)
    x[1, :] = np.abs(x[1, :])                      # one all-positive row
    codes, scales = quant.quantize_rows(x)
    for r in range(x.shape[0]):
        want_codes, want_scale = _brute_row(x[r])
        assert scales[r] == want_scale, r
        assert np.array_equal(codes[r].astype(np.int64), want_codes), r


def test_ties_round_to_even_and_the_extremes_map_to_127():
    # amax 127 makes the scale exactly 1.0, so x / scale = x
    x = np.zeros((1, 256), dtype=np.float32)
    x[0, :8] = [127.0, -126.5, 2.5, 3.5, -2.5, 0.5, 1.5, -0.5]
    codes, scales = quant.quantize_rows(x)
    assert scales[0] == np.float32(1.0)
    assert codes[0, :8].tolist() == [127, -126, 2, 4, -2, 0, 2, 0]
    x = synth.normal(4, "qx", (32, 256), 2.0)
    codes, scales = quant.quantize_rows(x)
    i = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(codes[np.arange(32), i]) == 127)
    assert np.all(np.sign(codes) * np.sign(x) >= 0)
    assert np.all(np.abs(x - codes * scales[:, None]) <= scales[:, None] * (0.5 + 1e-6))


def test_zero_nan_and_infinite_rows():
    x = np.ones((3, 256), dtype=np.float32)
    x[0] = 0.0
    x[1, 5] = np.nan
    x[2, 7] = -np.inf
    codes, scales = quant.quantize_rows(x)
    assert scales[0] == 0 and np.isnan(scales[1]) and scales[2] == np.inf
    assert not codes.any()


def test_packed_rows_round_trip():
    x = synth.normal(5, "qx", (9, 256), 1.0)
    codes, scales = quant.quantize_rows(x)
    packed = quant.pack_rows(codes, scales)
    assert packed.shape == (9, quant.ROW_BYTES) and not packed[:, 260:].any()
    c2, s2 = quant.unpack_rows(packed)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)


def _dequantised_oracle(q, q_dtype, kc, ks, v, v_dtype, pos, base, window):
    """The C oracle on q8 x sq, k8 x sk and V, all exact in float64."""
    from oracle.partial import widen
    q8, sq = quant.quantize_rows(quant.widen32(q, q_dtype))
    qd = q8.astype(np.float64) * sq.astype(np.float64)[..., None]
    kd = kc.astype(np.float64) * ks.astype(np.float64)[:, None]
    return oracle.attention(qd, kd, widen(v, v_dtype), pos, base, window=window, scale=synth.SCALE)


@pytest.mark.parametrize("q_dtype,v_dtype,window", [("f32", "f16", 0), ("bf16", "bf16", 37), ("f16", "f32", 0),
                                                    ("f32", "f32", 200)])
def test_attention_equals_the_c_oracle_on_dequantised_inputs(q_dtype, v_dtype, window):
    oracle.set_threads(4)
    cap, batch = 300, 3
    k = synth.normal(6, "k", (batch * cap, 256), 1.0)
    k[7] = 0.0                                     # a zero key row: scale 0, codes 0
    kc, ks = quant.quantize_rows(k)
    v = synth.draw(6, "v", (batch * cap, 256), v_dtype)
    q = synth.draw(6, "q", (5, 8, 256), q_dtype)
    pos = np.array([0, 7, 150, 299, 250])
    base = np.array([0, 0, cap, 2 * cap, 2 * cap])
    got = quant.attention_q8(q, q_dtype, kc, ks, v, v_dtype, pos, base, window=window, scale=synth.SCALE)
    want = _dequantised_oracle(q, q_dtype, kc, ks, v, v_dtype, pos, base, window)
    assert np.max(np.abs(got - want)) <= 1e-12


def test_attention_nan_rows_and_empty_rows():
    cap = 64
    k = synth.normal(7, "k", (cap, 256), 1.0)
    k[10, 3] = np.nan                              # key row 10: scale NaN
    kc, ks = quant.quantize_rows(k)
    v = synth.draw(7, "v", (cap, 256), "f32")
    q = synth.draw(7, "q", (3, 8, 256), "f32")
    q[2, 4, 0] = np.inf                            # head 4 of row 2: scores NaN
    out = quant.attention_q8(q, "f32", kc, ks, v, "f32", [9, 10, 5], scale=synth.SCALE)
    assert np.isfinite(out[0]).all()               # does not see row 10
    assert np.isnan(out[1]).all()                  # sees it
    assert np.isnan(out[2, 4]).all() and np.isfinite(np.delete(out[2], 4, axis=0)).all()
    out = quant.attention_q8(q[:1], "f32", kc, ks, v, "f32", [-1], scale=synth.SCALE)
    assert (out == 0).all()


# Random rows of random magnitude (subnormal to large) against the same
# brute force, with a few values planted at the row's extremes.
from hypothesis import given, settings, strategies as st


@settings(max_examples=25, deadline=None, derandomize=True)
@given(seed=st.integers(0, 10**6), log_std=st.floats(-40.0, 30.0), n_equal=st.integers(0, 4))
def test_random_rows_quantise_as_the_decimal_brute_force(seed, log_std, n_equal):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((1, 256)) * (10.0 ** log_std)).astype(np.float32)
    top = np.abs(x).max()
    for i in range(n_equal):                         # ties at +-amax
        x[0, 7 * i] = top if i % 2 == 0 else -top
    codes, scales = quant.quantize_rows(x)
    want_codes, want_scale = _brute_row(x[0])
    assert scales[0] == want_scale or (np.isnan(scales[0]) and np.isnan(want_scale))
    assert np.array_equal(codes[0].astype(np.int64), want_codes)
