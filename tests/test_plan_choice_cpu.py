"""The decode planner's own choices, pinned on the CPU: for a device of a
given SM count and resident-cluster capacity (B200 at this kernel's shared
memory footprint: 148 SMs, 74 / 33 / 15 clusters of 2 / 4 / 8 CTAs), the
split length and cluster size that attn_decode_plan picks are recomputed
here from the cost model that include/kca.h documents, and the work items
it returns are compared bit-exactly with the cut they imply.  Covers the
decode configurations' contexts (one sequence at 256, 4,096 and 16,384 keys
and 63 steps later; the window-512 decode; the ragged batch) and a few
edge cases."""
import numpy as np
import pytest

import kv_cache_attention_states_b200 as kca
import oracle
from kv_cache_attention_states_b200 import synth

SMS = 148
CAPACITY = {2: 74, 4: 33, 8: 15}
STAGE = 64                 # keys per stage of the tensor-core rows kernel
MAX_CLUSTER_PARTS = 256


def _cdiv(a, b):
    return -(-a // b)


def _n_splits(nk, length):
    return 1 if nk <= 0 else _cdiv(nk, length)


def _split_len(nks, c, slots):
    """Smallest multiple of the stage whose clusters fit `slots`; one split
    per unit when even that does not fit."""
    top = _cdiv(max(max(nks), STAGE), STAGE)
    for m in range(1, top + 1):
        if sum(_cdiv(_n_splits(n, m * STAGE), c) for n in nks) <= slots:
            return m * STAGE
    return top * STAGE


def _choose(nks, sms, capacity):
    total = 0.0
    for n in nks:
        total += float(n)
    best = None
    for c in (8, 4, 2, 1):
        slots = sms if c == 1 else capacity[c]
        slots = min(slots, MAX_CLUSTER_PARTS)
        if slots <= 0:
            continue
        length = _split_len(nks, c, slots)
        mc = _cdiv(_n_splits(max(nks), length), c)
        if c == 1 and mc > 1:
            continue                  # one CTA would merge all eight heads: not a plan
        n_clusters = sum(_cdiv(_n_splits(n, length), c) for n in nks)
        waves = float(_cdiv(n_clusters, slots))
        t_hbm = total * 1024.0 / 6.5e12
        t_sm = waves * length * 1024.0 / 50e9
        t = t_hbm if t_hbm > t_sm else t_sm
        if mc > 1:
            t += 1.5e-6 + 0.6e-6 * (1 + (8 // c) * ((mc + 31) // 32))
        if best is None or t < best[0]:
            best = (t, c, length, mc)
    return best[1:]


def _items(positions, window, c, length, mc):
    rows = []
    for u, p in enumerate(positions):
        lo, hi = oracle.visible_range(int(p), window)
        n = max(0, hi - lo + 1)
        ns = _n_splits(n, length)
        nclus = _cdiv(ns, c)
        for sp in range(ns):
            kb, ke = (lo, lo) if n == 0 else (lo + sp * length, min(lo + (sp + 1) * length, hi + 1))
            rows.append((u, kb, ke, u * mc + sp // c if nclus > 1 else -1))
    return np.array(rows, dtype=np.int64)


def _cases():
    out = []
    for length in (256, 4096, 16384):
        out += [([length], 0), ([length + 63], 0)]
    out += [([4097], 512), ([4160], 512)]                       # the window-512 decode steps
    ragged = synth.ragged_f16(0).decode_ctx
    out += [(list(ragged[0]), 0), (list(ragged[-1]), 0)]          # the ragged batch, first and last step
    out += [([131072], 0), ([0, 1, 5000], 0), ([131072] * 8, 0), ([9000, 17, 70000, 4096], 300),
            ([1] * 200, 0), ([64], 0), ([65], 0)]
    return out


@pytest.mark.parametrize("kv", [kca.F16, kca.BF16])
@pytest.mark.parametrize("ctx,window", _cases())
def test_decode_planner_choice_matches_the_documented_cost_model(kv, ctx, window):
    nks = [max(0, oracle.visible_range(c - 1, window)[1] - oracle.visible_range(c - 1, window)[0] + 1)
           for c in ctx]
    c, length, mc = _choose(nks, SMS, CAPACITY)
    items, cluster = kca.attn_decode_plan(ctx, window, num_sms=SMS, kv_dtype=kv,
                                          cluster_capacity=(CAPACITY[2], CAPACITY[4], CAPACITY[8]),
                                          with_cluster=True)
    assert cluster == c
    want = _items([x - 1 for x in ctx], window, c, length, mc)
    assert items.shape == want.shape and np.array_equal(items, want)


def test_planner_choice_for_one_sequence_at_16k():
    # one sequence at 16K, with these capacities: 32 clusters of 4 CTAs, 128
    # splits of 128 keys (5.9 us estimated) beat 11 clusters of 8 with 192-key
    # splits (6.6 us)
    items, cluster = kca.attn_decode_plan([16384], 0, num_sms=SMS, kv_dtype=kca.F16,
                                          cluster_capacity=(74, 33, 15), with_cluster=True)
    assert cluster == 4 and len(items) == 128
    assert set((items[:, 2] - items[:, 1]).tolist()) == {128}
    # one cluster of 4 fewer, and clusters of 8 win
    items, cluster = kca.attn_decode_plan([16384], 0, num_sms=SMS, kv_dtype=kca.F16,
                                          cluster_capacity=(74, 31, 15), with_cluster=True)
    assert cluster == 8 and len(items) == 86


def test_planner_without_larger_clusters_and_negative_capacity():
    # a device that holds no cluster of 4 or 8 at this footprint
    items, cluster = kca.attn_decode_plan([131072] * 8, 0, num_sms=SMS, kv_dtype=kca.F16,
                                          cluster_capacity=(74, 0, 0), with_cluster=True)
    assert cluster == 2
    with pytest.raises(kca.KcaError):
        kca.attn_decode_plan([100], 0, num_sms=SMS, kv_dtype=kca.F16, cluster_capacity=(74, -1, 15))


# The same comparison on random batches, windows, SM counts and capacities.
from hypothesis import given, settings, strategies as st


@settings(max_examples=300, deadline=None, derandomize=True)
@given(ctx=st.lists(st.integers(0, 131072), min_size=1, max_size=12),
       window=st.one_of(st.just(0), st.integers(1, 40000)),
       sms=st.sampled_from([148, 132, 120, 64]),
       cap=st.tuples(st.integers(1, 74), st.integers(1, 37), st.integers(1, 18)))
def test_random_planner_choices_match_the_documented_cost_model(ctx, window, sms, cap):
    nks = [max(0, oracle.visible_range(c - 1, window)[1] - oracle.visible_range(c - 1, window)[0] + 1)
           for c in ctx]
    c, length, mc = _choose(nks, sms, {2: cap[0], 4: cap[1], 8: cap[2]})
    items, cluster = kca.attn_decode_plan(ctx, window, num_sms=sms, kv_dtype=kca.F16, cluster_capacity=cap,
                                          with_cluster=True)
    assert cluster == c
    want = _items([x - 1 for x in ctx], window, c, length, mc)
    assert items.shape == want.shape and np.array_equal(items, want)
