"""Pins for the f64 oracle (CPU only).

The oracle is checked against things other than itself:
  * an independent Python-decimal brute force on tiny inputs (<= 1e-12),
  * torch's scaled_dot_product_attention in float64 with an explicit boolean
    mask (a library routine) on medium inputs,
  * closed forms (one visible key, constant V, scale 0, window 1, identical
    keys) and invariants (invisible rows, window >= context, permutations,
    equal heads, chunking),
  * the NaN / fully-masked semantics of the Karume v0.8.0 release notes
    ("Breaking Changes", softmax NaN item),
  * its f16 / bf16 decoders against numpy and torch conversions over all
    65536 bit patterns.
A plausible slip in the oracle (a dropped scale, a wrong head mapping, an
off-by-one window, a missing max subtraction that overflows, transposed
q/k) fails at least one of these.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from kv_cache_attention_states_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _tiny_case(seed, n_keys, d, hq, hkv=1, n_query=None, std=1.0):
    rng = np.random.default_rng(seed)
    rows = n_keys
    q = (rng.standard_normal((n_query or 1, hq, d)) * std).astype(np.float32)
    k = (rng.standard_normal((rows, hkv, d)) * std).astype(np.float32)
    v = rng.standard_normal((rows, hkv, d)).astype(np.float32)
    return q, k, v


@pytest.mark.parametrize("d", [1, 2, 4, 8])
@pytest.mark.parametrize("hq,hkv", [(1, 1), (2, 1), (8, 1), (4, 2)])
@pytest.mark.parametrize("window", [0, 1, 2, 3, 100])
def test_oracle_matches_decimal_brute_force(d, hq, hkv, window):
    n_keys = 6
    q, k, v = _tiny_case(1000 * d + 10 * hq + window, n_keys, d, hq, hkv, n_query=4, std=2.0)
    pos = np.array([0, 2, 5, 3], dtype=np.int64)
    got = oracle.attention(q, k, v, pos, window=window, scale=0.37, n_kv_heads=hkv)
    ref = brute.to_float64(brute.attention(q, k, v, pos, window=window, scale=0.37,
                                           n_kv_heads=hkv))
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_oracle_matches_brute_force_f16_bf16_storage():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, 8, 4)).astype(np.float32)
    kf = rng.standard_normal((5, 1, 4)).astype(np.float32)
    vf = rng.standard_normal((5, 1, 4)).astype(np.float32)
    for dt in ("f16", "bf16"):
        q = synth.to_storage(x, dt)
        k = synth.to_storage(kf, dt)
        v = synth.to_storage(vf, dt)
        qd = oracle.decode_elements(q, dt)
        kd = oracle.decode_elements(k, dt)
        vd = oracle.decode_elements(v, dt)
        pos = [4, 1, 2]
        got = oracle.attention(q, k, v, pos, q_dtype=dt, kv_dtype=dt, scale=0.5, window=3)
        ref = brute.to_float64(brute.attention(qd, kd, vd, pos, scale=0.5, window=3))
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_batched_kv_base_matches_brute_force():
    rng = np.random.default_rng(11)
    cap = 5
    k = rng.standard_normal((3 * cap, 1, 4)).astype(np.float32)
    v = rng.standard_normal((3 * cap, 1, 4)).astype(np.float32)
    q = rng.standard_normal((3, 2, 4)).astype(np.float32)
    pos = np.array([4, 0, 2])
    base = np.array([0, cap, 2 * cap])
    got = oracle.attention(q, k, v, pos, base, scale=0.8)
    ref = brute.to_float64(brute.attention(q, k, v, pos, base, scale=0.8))
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def _sdpa_reference(q, k, v, pos, window, scale):
    """torch SDPA (math backend, float64) with an explicit boolean visibility mask."""
    qt = torch.from_numpy(q.astype(np.float64)).permute(1, 0, 2)         # [H, n, d]
    kt = torch.from_numpy(k[:, 0, :].astype(np.float64))                  # [rows, d]
    vt = torch.from_numpy(v[:, 0, :].astype(np.float64))
    rows = kt.shape[0]
    j = torch.arange(rows)[None, :]
    p = torch.as_tensor(pos)[:, None]
    lo = (p - window + 1).clamp(min=0) if window > 0 else torch.zeros_like(p)
    mask = (j >= lo) & (j <= p)                                           # [n, rows]
    h = qt.shape[0]
    out = torch.nn.functional.scaled_dot_product_attention(
        qt[None], kt.expand(h, rows, -1)[None], vt.expand(h, rows, -1)[None],
        attn_mask=mask[None, None], scale=scale)
    return out[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("window", [0, 7, 64])
def test_oracle_matches_torch_sdpa_float64(window):
    rng = np.random.default_rng(3 + window)
    rows, n, d = 200, 40, 256
    q = rng.standard_normal((n, 8, d)).astype(np.float32)
    k = rng.standard_normal((rows, 1, d)).astype(np.float32)
    v = rng.standard_normal((rows, 1, d)).astype(np.float32)
    pos = np.sort(rng.integers(0, rows, size=n))
    got = oracle.attention(q, k, v, pos, window=window, scale=1 / 16)
    ref = _sdpa_reference(q, k, v, pos, window, 1 / 16)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_closed_form_single_visible_key_returns_that_value_row():
    q, k, v = _tiny_case(5, 10, 256, 8, n_query=1)
    got = oracle.attention(q, k, v, [0])
    np.testing.assert_array_equal(got[0], np.repeat(v[0, 0][None].astype(np.float64), 8, 0))


def test_closed_form_window_one_returns_own_value_row():
    q, k, v = _tiny_case(6, 10, 256, 8, n_query=3)
    pos = [3, 7, 9]
    got = oracle.attention(q, k, v, pos, window=1)
    for i, p in enumerate(pos):
        np.testing.assert_array_equal(got[i], np.repeat(v[p, 0][None].astype(np.float64), 8, 0))


def test_closed_form_constant_values():
    q, k, _ = _tiny_case(8, 50, 256, 8, n_query=2)
    v = np.full((50, 1, 256), 0.625, dtype=np.float32)
    got = oracle.attention(q, k, v, [49, 17], window=20)
    np.testing.assert_allclose(got, 0.625, rtol=0, atol=1e-15)


def test_closed_form_zero_scale_is_mean_of_visible_values():
    q, k, v = _tiny_case(9, 30, 256, 8, n_query=2)
    got = oracle.attention(q, k, v, [29, 12], window=10, scale=0.0)
    np.testing.assert_allclose(got[0], np.repeat(v[20:30, 0].astype(np.float64).mean(0)[None], 8, 0),
                               rtol=0, atol=1e-14)
    np.testing.assert_allclose(got[1], np.repeat(v[3:13, 0].astype(np.float64).mean(0)[None], 8, 0),
                               rtol=0, atol=1e-14)


def test_closed_form_identical_keys_give_uniform_mean():
    q, _, v = _tiny_case(10, 12, 256, 8, n_query=1)
    k = np.repeat(np.random.default_rng(1).standard_normal((1, 1, 256)).astype(np.float32), 12, 0)
    got = oracle.attention(q, k, v, [11])
    np.testing.assert_allclose(got[0], np.repeat(v[:, 0].astype(np.float64).mean(0)[None], 8, 0),
                               rtol=0, atol=1e-14)


def test_two_keys_closed_form_logistic():
    # d = 1, q = 1, k = (0, a): weights (1, e^{a s}) / (1 + e^{a s})
    q = np.ones((1, 1, 1), np.float32)
    k = np.array([[[0.0]], [[3.0]]], np.float32)
    v = np.array([[[1.0]], [[-2.0]]], np.float32)
    s = 0.25
    w1 = math.exp(3.0 * s)
    expect = (1.0 + w1 * -2.0) / (1.0 + w1)
    got = oracle.attention(q, k, v, [1], scale=s)
    assert abs(got[0, 0, 0] - expect) < 1e-15


def test_keys_past_position_outside_window_or_context_do_not_matter():
    q, k, v = _tiny_case(12, 64, 256, 8, n_query=3)
    pos = [40, 50, 63]
    base = oracle.attention(q, k, v, pos, window=16)
    k2, v2 = k.copy(), v.copy()
    # rows visible to nobody: < 63-16+1 = 48 except those seen by pos 40/50
    for p in range(0, 25):
        k2[p] = np.nan
        v2[p] = np.inf
    q1 = q[:1]
    only = oracle.attention(q1, k2, v2, [40], window=16)
    np.testing.assert_array_equal(only, base[:1])
    # rows after the query position
    k3, v3 = k.copy(), v.copy()
    k3[41:] = 1e30
    v3[41:] = np.nan
    np.testing.assert_array_equal(oracle.attention(q1, k3, v3, [40], window=16), base[:1])


def test_window_at_least_context_equals_no_window():
    q, k, v = _tiny_case(13, 40, 256, 8, n_query=2)
    pos = [39, 10]
    np.testing.assert_array_equal(oracle.attention(q, k, v, pos, window=40),
                                  oracle.attention(q, k, v, pos, window=0))
    np.testing.assert_array_equal(oracle.attention(q, k, v, pos, window=1000),
                                  oracle.attention(q, k, v, pos, window=0))


def test_permuting_visible_rows_of_a_decode_query():
    q, k, v = _tiny_case(14, 33, 256, 8, n_query=1)
    perm = np.random.default_rng(0).permutation(33)
    a = oracle.attention(q, k, v, [32])
    b = oracle.attention(q, k[perm], v[perm], [32])
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_equal_query_heads_give_equal_outputs():
    q, k, v = _tiny_case(15, 20, 256, 8, n_query=1)
    q[0, :, :] = q[0, 3, :]
    out = oracle.attention(q, k, v, [19])
    for h in range(8):
        np.testing.assert_array_equal(out[0, h], out[0, 0])


def test_chunked_prefill_equals_single_shot():
    rng = np.random.default_rng(16)
    rows = 90
    q = rng.standard_normal((rows, 8, 256)).astype(np.float32)
    k = rng.standard_normal((rows, 1, 256)).astype(np.float32)
    v = rng.standard_normal((rows, 1, 256)).astype(np.float32)
    whole = oracle.attention(q, k, v, np.arange(rows), window=30)
    for chunk in (1, 7, 32, 89):
        parts = [oracle.attention(q[s:s + r], k, v, np.arange(s, s + r), window=30)
                 for s, r in synth.chunks(rows, chunk)]
        np.testing.assert_array_equal(np.concatenate(parts), whole)


def test_nan_in_a_visible_key_gives_nan_and_fully_masked_row_gives_zero():
    q, k, v = _tiny_case(17, 8, 256, 8, n_query=2)
    k[3, 0, 5] = np.nan
    out = oracle.attention(q, k, v, [5, 2])
    assert np.isnan(out[0]).all()          # key 3 visible to position 5
    assert not np.isnan(out[1]).any()      # position 2 never sees key 3
    empty = oracle.attention(q[:1], k, v, [-1])
    np.testing.assert_array_equal(empty, 0.0)


def test_all_nan_scores_give_nan():
    q, k, v = _tiny_case(18, 4, 256, 8, n_query=1)
    q[0, 2, 0] = np.nan
    out = oracle.attention(q, k, v, [3])
    assert np.isnan(out[0, 2]).all()
    assert not np.isnan(out[0, 1]).any()


def test_large_scores_do_not_overflow():
    q, k, v = _tiny_case(19, 16, 256, 8, n_query=1)
    out = oracle.attention(q * 40, k * 40, v, [15], scale=1.0)
    assert np.isfinite(out).all()
    # the max-score key dominates completely: output equals its V row
    s = (q[0, 0].astype(np.float64) * 40) @ (k[:16, 0].astype(np.float64) * 40).T
    np.testing.assert_allclose(out[0, 0], v[int(np.argmax(s)), 0], rtol=0, atol=1e-12)


def test_half_decoder_matches_numpy_for_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode_elements(bits.view(np.float16), "f16")
    ref = bits.view(np.float16).astype(np.float64)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def test_bf16_decoder_matches_torch_for_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode_elements(bits, "bf16")
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def test_visible_range_definition():
    assert oracle.visible_range(10, 0) == (0, 10)
    assert oracle.visible_range(10, 4) == (7, 10)
    assert oracle.visible_range(2, 512) == (0, 2)
    assert oracle.visible_range(4159, 512) == (3648, 4159)


# Random tiny problems against the decimal brute force: shapes, head groups,
# positions, windows and scales drawn at random.
from hypothesis import given, settings, strategies as st


@settings(max_examples=60, deadline=None, derandomize=True)
@given(d=st.integers(1, 12), heads=st.sampled_from([(1, 1), (2, 1), (8, 1), (4, 2), (8, 4)]),
       n_keys=st.integers(1, 7), data=st.data(), window=st.integers(0, 9),
       scale=st.floats(0.01, 2.0), seed=st.integers(0, 2**31 - 1))
def test_random_tiny_problems_match_decimal_brute_force(d, heads, n_keys, data, window, scale, seed):
    hq, hkv = heads
    pos = np.array(data.draw(st.lists(st.integers(0, n_keys - 1), min_size=1, max_size=4)), dtype=np.int64)
    q, k, v = _tiny_case(seed, n_keys, d, hq, hkv, n_query=len(pos), std=1.5)
    got = oracle.attention(q, k, v, pos, window=window, scale=scale, n_kv_heads=hkv)
    ref = brute.to_float64(brute.attention(q, k, v, pos, window=window, scale=scale, n_kv_heads=hkv))
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
