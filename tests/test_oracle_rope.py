"""Pins of oracle/rope.py against facts that do not come from the oracle itself:
the complex-number form of a rotation (computed in float64 with Python's
complex type), the identity and composition of rotations, norm preservation,
the relative-position property RoPE exists for, and round-to-nearest-even
bf16 against torch's own conversion and hand-checked bit patterns."""
import cmath

import numpy as np
import pytest
import torch

from oracle import rope


def _rand(seed, shape, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


def test_zero_angle_is_the_identity():
    x = _rand(1, (5, 256))
    cos = np.ones((5, 256), np.float32)
    sin = np.zeros((5, 256), np.float32)
    assert np.array_equal(rope.rope_rotate(x, cos, sin), x)


def test_matches_complex_multiplication_per_pair():
    # dims (i, i + 128) as the complex number x_i + j x_{i+128}, rotated by e^{j theta}
    x = _rand(2, (3, 256))
    ang = np.random.default_rng(3).uniform(-7, 7, (3, 128))
    cos64, sin64 = np.cos(ang), np.sin(ang)
    cos = np.concatenate([cos64, cos64], 1).astype(np.float32)
    sin = np.concatenate([sin64, sin64], 1).astype(np.float32)
    got = rope.rope_rotate(x, cos, sin)
    for r in range(3):
        for i in range(128):
            z = complex(float(x[r, i]), float(x[r, i + 128])) * cmath.exp(1j * float(ang[r, i]))
            assert abs(got[r, i] - z.real) <= 1e-5 * (1 + abs(z))
            assert abs(got[r, i + 128] - z.imag) <= 1e-5 * (1 + abs(z))


def test_rotation_keeps_pair_norms_and_composes():
    x = _rand(4, (4, 256)).astype(np.float64)
    c1, s1 = rope.rope_tables([3, 50, 700, 9000])
    c2, s2 = rope.rope_tables([11, 11, 11, 11])
    c12, s12 = rope.rope_tables([14, 61, 711, 9011])
    once = rope.rope_rotate(x, c1, s1)
    twice = rope.rope_rotate(once, c2, s2)
    direct = rope.rope_rotate(x, c12, s12)
    assert np.max(np.abs(twice - direct)) <= 2e-4
    n_in = x[:, :128] ** 2 + x[:, 128:] ** 2
    n_out = once.astype(np.float64)[:, :128] ** 2 + once.astype(np.float64)[:, 128:] ** 2
    assert np.max(np.abs(n_out - n_in) / (1 + n_in)) <= 1e-5


def test_dot_products_depend_only_on_relative_position():
    q = _rand(5, (1, 256))
    k = _rand(6, (1, 256))
    dots = []
    for p, kp in [(100, 37), (1100, 1037), (5063, 5000)]:
        cq, sq = rope.rope_tables([p])
        ck, sk = rope.rope_tables([kp])
        dots.append(float(np.dot(rope.rope_rotate(q, cq, sq)[0].astype(np.float64),
                                 rope.rope_rotate(k, ck, sk)[0].astype(np.float64))))
    assert max(dots) - min(dots) <= 2e-3 * (1 + abs(dots[0]))


def test_bf16_rounding_is_round_to_nearest_even():
    vals = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e38, 1e-40, 0.0, -0.0,
                     np.inf, -np.inf], dtype=np.float32)
    bits = rope.bf16_bits_from_f32(vals)
    assert list(bits[:4]) == [0x3F80, 0x3F80, 0x3F82, 0xC020]      # ties go to the even mantissa
    x = _rand(7, (4096,), 100.0)
    x = np.concatenate([x, vals])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(rope.bf16_bits_from_f32(x), want)
    nan = rope.bf16_bits_from_f32(np.array([np.nan], np.float32))[0]
    assert (nan & 0x7F80) == 0x7F80 and (nan & 0x7F) != 0


@pytest.mark.parametrize("in_dtype,kv_dtype", [("f32", "f16"), ("bf16", "bf16"), ("f32", "f32")])
def test_append_writes_only_the_destination_rows(in_dtype, kv_dtype):
    n, rows = 3, 10
    k_new = _rand(8, (n, 256))
    v_new = _rand(9, (n, 256))
    if in_dtype == "bf16":
        k_new, v_new = rope.bf16_bits_from_f32(k_new), rope.bf16_bits_from_f32(v_new)
    zero = rope.to_stored(np.zeros((rows, 256), np.float32), kv_dtype)
    cos, sin = rope.rope_tables([4, 7, 9])
    k_out, v_out = rope.append_kv(k_new, v_new, in_dtype, cos, sin, zero, zero, kv_dtype, [4, 7, 99])
    untouched = [r for r in range(rows) if r not in (4, 7)]
    assert np.array_equal(k_out[untouched], zero[untouched])
    want_v = rope.to_stored(rope.f32_from_stored(v_new, in_dtype), kv_dtype)
    assert np.array_equal(v_out[4], want_v[0]) and np.array_equal(v_out[7], want_v[1])
    k32 = rope.f32_from_stored(k_out[[4, 7]], kv_dtype).astype(np.float64)
    src = rope.f32_from_stored(k_new[:2], in_dtype).astype(np.float64)
    norm = lambda a: a[:, :128] ** 2 + a[:, 128:] ** 2
    rel = 8e-3 if kv_dtype != "f32" else 1e-5
    assert np.max(np.abs(norm(k32) - norm(src)) / (1 + norm(src))) <= 2 * rel
    # the stored K rows are the source rows rotated: pair (i, i + 128) as the
    # complex number x_i + j x_{i+128} times e^{j angle}, angle from the tables
    ang = np.arctan2(sin[:2, :128].astype(np.float64), cos[:2, :128].astype(np.float64))
    z = (src[:, :128] + 1j * src[:, 128:]) * np.exp(1j * ang)
    want_k = np.concatenate([z.real, z.imag], 1)
    assert np.max(np.abs(k32 - want_k)) <= rel * (1 + np.max(np.abs(want_k)))


# Random rows and angles: the rotation equals the complex product of each
# (i, i + 128) pair with e^(j theta), and dot products of rotated rows depend
# only on the difference of their positions.
from hypothesis import given, settings, strategies as st


@settings(max_examples=60, deadline=None, derandomize=True)
@given(seed=st.integers(0, 10**6), scale=st.floats(1e-3, 1e3), lim=st.floats(0.0, 50.0))
def test_random_rotations_are_complex_products(seed, scale, lim):
    x = _rand(seed, (2, 256), scale)
    ang = np.random.default_rng(seed + 1).uniform(-lim, lim, (2, 128))
    cos = np.concatenate([np.cos(ang)] * 2, 1).astype(np.float32)
    sin = np.concatenate([np.sin(ang)] * 2, 1).astype(np.float32)
    got = rope.rope_rotate(x, cos, sin).astype(np.float64)
    z = (x[:, :128].astype(np.float64) + 1j * x[:, 128:].astype(np.float64)) * \
        (cos[:, :128].astype(np.float64) + 1j * sin[:, :128].astype(np.float64))
    bound = 4e-7 * (np.abs(x[:, :128]).astype(np.float64) + np.abs(x[:, 128:]).astype(np.float64))
    assert np.all(np.abs(got[:, :128] - z.real) <= bound + 1e-30)
    assert np.all(np.abs(got[:, 128:] - z.imag) <= bound + 1e-30)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(seed=st.integers(0, 10**6), p=st.integers(0, 60000), q=st.integers(0, 60000), shift=st.integers(0, 60000))
def test_random_dot_products_depend_on_relative_position(seed, p, q, shift):
    a = _rand(seed, (1, 256)).astype(np.float64)
    b = _rand(seed + 7, (1, 256)).astype(np.float64)
    c1, s1 = rope.rope_tables([p, q])
    c2, s2 = rope.rope_tables([p + shift, q + shift])
    ra = rope.rope_rotate(np.concatenate([a, b]), c1, s1).astype(np.float64)
    rb = rope.rope_rotate(np.concatenate([a, b]), c2, s2).astype(np.float64)
    d1, d2 = float(ra[0] @ ra[1]), float(rb[0] @ rb[1])
    # the tables' cos / sin are float64 values rounded once to float32, and
    # the rotation rounds each product: a few float32 ulps of |a| |b|
    assert abs(d1 - d2) <= 1e-5 * (np.linalg.norm(a) * np.linalg.norm(b))
