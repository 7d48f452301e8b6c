"""The RoPE oracle's pins catch plausible mistakes: each mutant below plants
one error in a copy of an oracle/rope.py function, and at least one pin of
tests/test_oracle_rope.py must fail with it in place."""
import numpy as np
import pytest

from oracle import rope
from tests import test_oracle_rope as pins

HALF = 128


def _pins():
    yield pins.test_zero_angle_is_the_identity
    yield pins.test_matches_complex_multiplication_per_pair
    yield pins.test_rotation_keeps_pair_norms_and_composes
    yield pins.test_dot_products_depend_only_on_relative_position
    yield pins.test_bf16_rounding_is_round_to_nearest_even
    for a, b in (("f32", "f16"), ("bf16", "bf16"), ("f32", "f32")):
        yield lambda a=a, b=b: pins.test_append_writes_only_the_destination_rows(a, b)


def _rotate(pair, sign, swap):
    def f(x32, cos, sin):
        x32 = np.asarray(x32, dtype=np.float32)
        cos = np.asarray(cos, dtype=np.float32)
        sin = np.asarray(sin, dtype=np.float32)
        if swap:
            cos, sin = sin, cos
        idx = (np.arange(256) + pair) % 256
        partner = x32[:, idx]
        out = np.empty_like(x32)
        out[:, :HALF] = (x32[:, :HALF] * cos[:, :HALF]) - sign * (partner[:, :HALF] * sin[:, :HALF])
        out[:, HALF:] = (x32[:, HALF:] * cos[:, HALF:]) + sign * (partner[:, HALF:] * sin[:, HALF:])
        return out.astype(np.float32)
    return f


def _bf16_truncating(x):
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


_ORIG_APPEND = rope.append_kv


def _append_off_by_one(k_new, v_new, in_dtype, cos, sin, k_cache, v_cache, kv_dtype, dst_rows):
    return _ORIG_APPEND(k_new, v_new, in_dtype, cos, sin, k_cache, v_cache, kv_dtype,
                        [r + 1 for r in dst_rows])


def _append_no_rotation(k_new, v_new, in_dtype, cos, sin, k_cache, v_cache, kv_dtype, dst_rows):
    # the rotation forgotten on the append path (pair norms still match)
    return _ORIG_APPEND(k_new, v_new, in_dtype, None, None, k_cache, v_cache, kv_dtype, dst_rows)


MUTANTS = {
    "pairs_i_with_i_plus_64": ("rope_rotate", _rotate(64, 1.0, False)),
    "sin_term_sign_flipped": ("rope_rotate", _rotate(128, -1.0, False)),
    "cos_and_sin_swapped": ("rope_rotate", _rotate(128, 1.0, True)),
    "bf16_truncates": ("bf16_bits_from_f32", _bf16_truncating),
    "append_row_off_by_one": ("append_kv", _append_off_by_one),
    "append_skips_the_rotation": ("append_kv", _append_no_rotation),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_mutant_fails_a_pin(monkeypatch, name):
    attr, fn = MUTANTS[name]
    # the unmutated oracle passes every pin
    for pin in _pins():
        pin()
    monkeypatch.setattr(rope, attr, fn)
    failures = 0
    for pin in _pins():
        try:
            pin()
        except AssertionError:
            failures += 1
    assert failures >= 1, f"mutant {name} passed every pin"
