"""The quantised-dot oracle's pins catch plausible mistakes: each mutant
below plants one error in a copy of oracle/quant.py (the scale as amax / 127
instead of amax x f32(1/127); codes truncated, or rounded half away from
zero; codes from the float64 quotient; the K row scale dropped from the
score; one head's q scale used for every head; no NaN propagation in amax),
and at least one pin of tests/test_oracle_quant.py must fail with it."""
import os
import types

import numpy as np
import pytest

from oracle import quant
from tests import test_oracle_quant as pins

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")
SRC = open(os.path.join(os.path.dirname(quant.__file__), "quant.py")).read()

MUTANTS = {
    "scale_by_division": ("sx = (amax * INV127).astype(np.float32)",
                          "sx = (amax / np.float32(127.0)).astype(np.float32)"),
    "truncated_codes": ("codes[ok] = np.clip(np.rint(q), -127, 127).astype(np.int8)",
                        "codes[ok] = np.clip(np.trunc(q), -127, 127).astype(np.int8)"),
    "half_away_from_zero": ("codes[ok] = np.clip(np.rint(q), -127, 127).astype(np.int8)",
                            "codes[ok] = np.clip(np.sign(q) * np.floor(np.abs(q) + 0.5), -127, 127).astype(np.int8)"),
    "float64_quotient": ("q = flat[ok] / sx[ok, None]", "q = flat[ok].astype(np.float64) / sx[ok, None].astype(np.float64)"),
    "k_scale_dropped": ("s = scale * (float(sq[i, h]) * ks[rows]) * dots.astype(np.float64)",
                        "s = scale * float(sq[i, h]) * dots.astype(np.float64)"),
    "head0_q_scale": ("s = scale * (float(sq[i, h]) * ks[rows]) * dots.astype(np.float64)",
                      "s = scale * (float(sq[i, 0]) * ks[rows]) * dots.astype(np.float64)"),
    "nan_ignoring_amax": ("amax = np.max(np.abs(flat), axis=1)", "amax = np.nanmax(np.abs(flat), axis=1)"),
}


def _mutant(name):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, name
    mod = types.ModuleType("quant_mutant")
    mod.__dict__["__package__"] = "oracle"
    exec(compile(SRC.replace(old, new), f"quant_{name}.py", "exec"), mod.__dict__)
    return mod


def _pins():
    for seed, std in ((0, 1.0), (1, 1e-3), (2, 300.0), (3, 1e-30)):
        yield lambda s=seed, d=std: pins.test_quantisation_equals_decimal_brute_force(s, d)
    yield pins.test_ties_round_to_even_and_the_extremes_map_to_127
    yield pins.test_zero_nan_and_infinite_rows
    yield pins.test_packed_rows_round_trip
    for qd, vd, w in (("f32", "f16", 0), ("bf16", "bf16", 37), ("f16", "f32", 0), ("f32", "f32", 200)):
        yield lambda a=qd, b=vd, c=w: _attention_pin_against_dequantised_reference(a, b, c)
    yield pins.test_attention_nan_rows_and_empty_rows


def _attention_pin_against_dequantised_reference(q_dtype, v_dtype, window):
    # The attention pin compares the mutant's attention with the C oracle on
    # inputs dequantised by the UNMUTATED rule, so a mistake in either the
    # codes or the scores shows.
    real = pins._dequantised_oracle
    import oracle as o
    from kv_cache_attention_states_b200 import synth
    cap, batch = 300, 3
    k = synth.normal(6, "k", (batch * cap, 256), 1.0)
    k[7] = 0.0
    kc, ks = quant.quantize_rows(k)
    v = synth.draw(6, "v", (batch * cap, 256), v_dtype)
    q = synth.draw(6, "q", (5, 8, 256), q_dtype)
    pos = np.array([0, 7, 150, 299, 250])
    base = np.array([0, 0, cap, 2 * cap, 2 * cap])
    mkc, mks = pins.quant.quantize_rows(k)
    got = pins.quant.attention_q8(q, q_dtype, mkc, mks, v, v_dtype, pos, base, window=window, scale=synth.SCALE)
    saved = pins.quant
    pins.quant = quant
    try:
        o.set_threads(4)
        want = real(q, q_dtype, kc, ks, v, v_dtype, pos, base, window)
    finally:
        pins.quant = saved
    assert np.max(np.abs(got - want)) <= 1e-12


def test_the_unmutated_oracle_passes_every_pin():
    for pin in _pins():
        pin()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_planted_mistake_fails_a_pin(monkeypatch, name):
    monkeypatch.setattr(pins, "quant", _mutant(name))
    failed = 0
    for pin in _pins():
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, name
