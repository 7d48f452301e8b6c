"""Pins for the partial-softmax oracle (oracle/partial.py), CPU only.

Checked against things other than itself:
  * the merged states of any cut of the context into shards equal the
    whole-context attention of the C oracle (pinned on its own in
    test_oracle.py) -- with windows, contexts that end inside or before a
    shard, and every stored dtype;
  * one shard holding the whole context: acc / l is that attention and m is
    the largest scaled score, found by a plain Python loop with math.fsum;
  * l and acc by a Python-decimal computation on a tiny case;
  * empty shards give (-inf, 0, 0), weigh nothing in a merge, and a row of
    empty states only merges to exactly 0;
  * shifting a state's reference (m + c, l e^-c, acc e^-c) changes no merge.
A slip such as a missing exp weight, a merge weighted by m instead of
e^(m - M), an off-by-one shard edge or a shard offset applied twice fails
one of these.
"""
import math
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle
from oracle import partial
from kv_cache_attention_states_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _case(seed, batch, rows, dtype, std=1.0):
    q = synth.draw(seed, "q", (batch, 8, 256), dtype if dtype != "f16" else "f32", std)
    k = synth.draw(seed, "k", (batch, rows, 256), dtype, std)
    v = synth.draw(seed, "v", (batch, rows, 256), dtype, std)
    return q, k, v, (dtype if dtype != "f16" else "f32"), dtype


def _full(q, k, v, ctx, window, qd, kd):
    batch, rows = k.shape[:2]
    kf, vf = k.reshape(-1, 256), v.reshape(-1, 256)
    return oracle.attention(q, kf, vf, np.asarray(ctx) - 1, np.arange(batch) * rows, window=window,
                            q_dtype=qd, kv_dtype=kd)


def _shards(q, k, v, ctx, cuts, window, qd, kd):
    states = []
    for kb, ke in zip(cuts[:-1], cuts[1:]):
        states.append(partial.decode_partial(q, k[:, kb:ke], v[:, kb:ke], ctx, kb, window=window,
                                             q_dtype=qd, kv_dtype=kd))
    return [np.stack(x) for x in zip(*states)]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("window", [0, 37])
def test_merged_shards_equal_whole_context_attention(dtype, window):
    q, k, v, qd, kd = _case(1, 3, 300, dtype)
    ctx = [300, 1, 173]
    want = _full(q, k, v, ctx, window, qd, kd)
    for cuts in ([0, 300], [0, 100, 200, 300], [0, 1, 172, 173, 250, 300], [0, 150, 300]):
        m, l, acc = _shards(q, k, v, ctx, cuts, window, qd, kd)
        got = partial.merge_partials(m, l, acc)
        assert np.max(np.abs(got - want)) <= 1e-12, cuts


def test_one_shard_is_the_attention_and_m_the_largest_score():
    q, k, v, qd, kd = _case(2, 2, 40, "f32")
    ctx = [40, 17]
    m, l, acc = partial.decode_partial(q, k, v, ctx, 0)
    want = _full(q, k, v, ctx, 0, qd, kd)
    assert np.max(np.abs(acc / l[..., None] - want)) <= 1e-12
    for b in range(2):
        for h in (0, 5):
            scores = [math.fsum(float(q[b, h, t]) * float(k[b, j, t]) for t in range(256)) / 16.0
                      for j in range(ctx[b])]
            assert abs(m[b, h] - max(scores)) <= 1e-12


def test_l_and_acc_against_decimal():
    getcontext().prec = 50
    q, k, v, _, _ = _case(3, 1, 6, "f32")
    kb = 2                                   # shard holds positions 2..5, query at 4
    m, l, acc = partial.decode_partial(q, k[:, kb:], v[:, kb:], [5], kb)
    for h in (0, 7):
        s = [sum(Decimal(float(q[0, h, t])) * Decimal(float(k[0, j, t])) for t in range(256)) / 16
             for j in (2, 3, 4)]
        mx = max(s)
        w = [(x - mx).exp() for x in s]
        assert abs(float(mx) - m[0, h]) <= 1e-12
        assert abs(float(sum(w)) - l[0, h]) <= 1e-12
        for d in (0, 100, 255):
            a = sum(wi * Decimal(float(v[0, j, d])) for wi, j in zip(w, (2, 3, 4)))
            assert abs(float(a) - acc[0, h, d]) <= 1e-12


def test_empty_shards_and_empty_rows():
    q, k, v, qd, kd = _case(4, 2, 64, "bf16")
    ctx = [10, 0]                            # sequence 1 has no context at all
    m, l, acc = partial.decode_partial(q, k[:, 32:], v[:, 32:], ctx, 32, q_dtype=qd, kv_dtype=kd)
    assert np.all(m == -np.inf) and np.all(l == 0) and np.all(acc == 0)
    m0, l0, a0 = partial.decode_partial(q, k[:, :32], v[:, :32], ctx, 0, q_dtype=qd, kv_dtype=kd)
    merged = partial.merge_partials(np.stack([m, m0]), np.stack([l, l0]), np.stack([acc, a0]))
    alone = partial.merge_partials(m0[None], l0[None], a0[None])
    assert np.array_equal(merged, alone)
    assert np.all(merged[1] == 0)            # fully masked row: exactly 0
    want = _full(q, k, v, ctx, 0, qd, kd)
    assert np.max(np.abs(merged - want)) <= 1e-12


def test_reference_shift_changes_no_merge():
    q, k, v, qd, kd = _case(5, 2, 90, "f32")
    ctx = [90, 61]
    m, l, acc = _shards(q, k, v, ctx, [0, 30, 90], 0, qd, kd)
    base = partial.merge_partials(m, l, acc)
    c = 3.25
    m2, l2, a2 = m.copy(), l.copy(), acc.copy()
    m2[1] += c
    l2[1] *= math.exp(-c)
    a2[1] *= math.exp(-c)
    assert np.max(np.abs(partial.merge_partials(m2, l2, a2) - base)) <= 1e-12


def test_nan_score_poisons_its_row():
    q, k, v, qd, kd = _case(6, 1, 20, "f32")
    k = k.copy()
    k[0, 3, 7] = np.nan
    m, l, acc = _shards(q, k, v, [20], [0, 10, 20], 0, qd, kd)
    out = partial.merge_partials(m, l, acc)
    assert np.all(np.isnan(out))


# Random cuts, contexts and windows: the merge of the shards' states is the
# whole-context attention.
from hypothesis import given, settings, strategies as st


@settings(max_examples=40, deadline=None, derandomize=True)
@given(data=st.data(), dtype=st.sampled_from(["f32", "f16", "bf16"]),
       window=st.one_of(st.just(0), st.integers(1, 120)), seed=st.integers(0, 10**6))
def test_random_shard_cuts_merge_to_the_whole_context(data, dtype, window, seed):
    rows = 96
    q, k, v, qd, kd = _case(seed, 2, rows, dtype)
    ctx = data.draw(st.lists(st.integers(0, rows), min_size=2, max_size=2))
    inner = data.draw(st.lists(st.integers(1, rows - 1), max_size=5, unique=True))
    cuts = [0] + sorted(inner) + [rows]
    want = _full(q, k, v, ctx, window, qd, kd)
    m, l, acc = _shards(q, k, v, ctx, cuts, window, qd, kd)
    got = partial.merge_partials(m, l, acc)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
