"""The partial-softmax oracle's pins catch plausible mistakes: each mutant
below plants one error in a copy of an oracle/partial.py function (a shard
edge off by one, a window edge off by one, a shard offset applied twice, a
missing exp weight in l, an empty state that is not (-inf, 0, 0), a merge
weighted by m instead of e^(m - M)), and at least one pin of
tests/test_oracle_partial.py must fail with it in place."""
import math

import numpy as np
import pytest

from oracle import partial
from tests import test_oracle_partial as pins

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _pins():
    for dtype in ("f32", "bf16"):
        for window in (0, 37):
            yield lambda d=dtype, w=window: pins.test_merged_shards_equal_whole_context_attention(d, w)
    yield pins.test_one_shard_is_the_attention_and_m_the_largest_score
    yield pins.test_l_and_acc_against_decimal
    yield pins.test_empty_shards_and_empty_rows
    yield pins.test_reference_shift_changes_no_merge
    yield pins.test_nan_score_poisons_its_row


def _shard_keys_drops_diagonal(pos, window, key_begin, key_end):
    lo = max(0, pos - window + 1) if window > 0 else 0
    return range(max(lo, key_begin), min(pos, key_end))


def _shard_keys_window_one_wider(pos, window, key_begin, key_end):
    lo = max(0, pos - window) if window > 0 else 0
    return range(max(lo, key_begin), min(pos + 1, key_end))


def _decode_partial(offset_twice=False, l_counts=False, empty_m=-np.inf):
    def f(q, k_shard, v_shard, ctx_len, key_begin, *, window=0, scale=1.0 / 16.0, q_dtype="f32",
          kv_dtype="f32"):
        qd = partial.widen(q, q_dtype)
        kd = partial.widen(k_shard, kv_dtype)
        vd = partial.widen(v_shard, kv_dtype)
        batch, heads, dim = qd.shape
        key_end = key_begin + kd.shape[1]
        m = np.full((batch, heads), empty_m)
        l = np.zeros((batch, heads))
        acc = np.zeros((batch, heads, dim))
        for b in range(batch):
            keys = partial.shard_keys(int(ctx_len[b]) - 1, window, key_begin, key_end)
            if len(keys) == 0:
                continue
            rows = np.arange(keys.start, keys.stop) - key_begin * (2 if offset_twice else 1)
            rows = np.clip(rows, 0, kd.shape[1] - 1)
            for h in range(heads):
                s = scale * (kd[b, rows] @ qd[b, h])
                mh = np.nan if np.isnan(s).any() else s.max()
                w = np.exp(s - mh)
                m[b, h] = mh
                l[b, h] = float(len(rows)) if l_counts else w.sum()
                acc[b, h] = w @ vd[b, rows]
        return m, l, acc
    return f


def _merge_weighted_by_m(ms, ls, accs):
    ms = np.asarray(ms, dtype=np.float64)
    ls = np.asarray(ls, dtype=np.float64)
    accs = np.asarray(accs, dtype=np.float64)
    n, batch, heads = ms.shape
    out = np.zeros(accs.shape[1:])
    for b in range(batch):
        for h in range(heads):
            col = ms[:, b, h]
            if np.isnan(col).any():
                out[b, h] = np.nan
                continue
            if col.max() == -math.inf:
                continue
            w = np.where(col == -math.inf, 0.0, col)
            out[b, h] = (w @ accs[:, b, h]) / (w @ ls[:, b, h])
    return out


MUTANTS = {
    "shard_edge_drops_the_diagonal_key": ("shard_keys", _shard_keys_drops_diagonal),
    "window_edge_one_wider": ("shard_keys", _shard_keys_window_one_wider),
    "shard_offset_applied_twice": ("decode_partial", _decode_partial(offset_twice=True)),
    "l_counts_keys_instead_of_weights": ("decode_partial", _decode_partial(l_counts=True)),
    "empty_state_m_is_zero": ("decode_partial", _decode_partial(empty_m=0.0)),
    "merge_weighted_by_m": ("merge_partials", _merge_weighted_by_m),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_mutant_fails_a_pin(monkeypatch, name):
    attr, fn = MUTANTS[name]
    for pin in _pins():                 # the unmutated oracle passes every pin
        pin()
    monkeypatch.setattr(partial, attr, fn)
    failures = 0
    for pin in _pins():
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            failures += 1
    assert failures >= 1, f"mutant {name} passed every pin"
