"""The oracle's pins must catch plausible mistakes.

Each case copies attn_oracle.c, plants one mistake in the copy (on the CPU),
compiles it with gcc, and runs a compact battery built from the same pins as
test_oracle.py against the broken copy.  The unmodified source must pass the
battery; every mutant must fail at least one check.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from oracle import brute
from tests.test_oracle import _sdpa_reference

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

MUTANTS = {
    "dropped_scale": ("s[j] = scale * dot;", "s[j] = dot;"),
    "window_off_by_one": ("lo = p - window + 1;", "lo = p - window;"),
    "wrong_head_group": ("const int g = h / group;", "const int g = h % n_kv_heads;"),
    "no_max_subtraction": ("const double w = exp(s[j] - m);", "const double w = exp(s[j]);"),
    "missing_normalisation": ("o[t] /= den;", "o[t] /= 1.0;"),
    "diagonal_key_dropped": ("const int64_t n = (p >= lo) ? p - lo + 1 : 0;",
                             "const int64_t n = (p >= lo) ? p - lo : 0;"),
    "scores_from_values": ("dot += qd[t] * orc_load(k, kv_dtype, k_off + t);",
                           "dot += qd[t] * orc_load(v, kv_dtype, k_off + t);"),
    "half_exponent_bias": ("ex - 25);", "ex - 24);"),
    # the behaviour the v0.8.0 notes retired: a NaN row silently gives 0
    "nan_row_gives_zero": ("if (any_nan) m = NAN;",
                           "if (any_nan) { free(s); free(qd); continue; }"),
}


def _compile(tmp_path, name, source):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(source)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                    "-fno-fast-math", str(c), "-o", str(so), "-lm"], check=True)
    return oracle.bind(str(so))


def _battery(lib) -> list[str]:
    """Names of the checks that fail for this oracle library."""
    failed = []
    rng = np.random.default_rng(42)
    # brute force, GQA with 2 KV heads, window 3
    q = rng.standard_normal((3, 4, 4)).astype(np.float32) * 2
    k = rng.standard_normal((6, 2, 4)).astype(np.float32) * 2
    v = rng.standard_normal((6, 2, 4)).astype(np.float32)
    pos = [5, 2, 3]
    got = oracle.attention(q, k, v, pos, window=3, scale=0.37, n_kv_heads=2, lib=lib)
    ref = brute.to_float64(brute.attention(q, k, v, pos, window=3, scale=0.37, n_kv_heads=2))
    if not np.allclose(got, ref, rtol=0, atol=1e-12, equal_nan=True):
        failed.append("brute_force")
    # library special case
    q = rng.standard_normal((20, 8, 256)).astype(np.float32)
    k = rng.standard_normal((100, 1, 256)).astype(np.float32)
    v = rng.standard_normal((100, 1, 256)).astype(np.float32)
    pos = np.sort(rng.integers(0, 100, size=20))
    got = oracle.attention(q, k, v, pos, window=9, lib=lib)
    if not np.allclose(got, _sdpa_reference(q, k, v, pos, 9, 1 / 16), rtol=0, atol=1e-12):
        failed.append("sdpa")
    # large scores stay finite
    with np.errstate(all="ignore"):
        out = oracle.attention(q[:1] * 40, k * 40, v, [99], scale=1.0, lib=lib)
    if not np.isfinite(out).all():
        failed.append("overflow")
    # NaN semantics
    k2 = k.copy()
    k2[3, 0, 0] = np.nan
    out = oracle.attention(q[:1], k2, v, [10], lib=lib)
    if not np.isnan(out).all():
        failed.append("nan")
    # half decoder over all bit patterns
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    dec = oracle.decode_elements(bits[::7], "f16", lib=lib)
    ref = bits[::7].astype(np.float64)
    if not np.array_equal(dec, ref, equal_nan=True):
        failed.append("half_decoder")
    return failed


def test_unmodified_oracle_passes_battery(tmp_path):
    lib = _compile(tmp_path, "orig", open(SRC).read())
    assert _battery(lib) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    lib = _compile(tmp_path, name, src.replace(old, new))
    assert _battery(lib), f"mutant {name} passed every pin"
