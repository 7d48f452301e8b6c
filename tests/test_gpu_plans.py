"""The tensor-core kernel's plans (16-bit caches), which depend on the
device's resident-cluster capacity, against an independent recomputation:
every unit's visible range J(pos) cut into equal splits of the plan's
length (a multiple of the kernel's 64-key stage) from lo, the last one
clipped at pos, and each split's cluster-partial slot
(unit * clusters-per-unit + split / cluster size, -1 for a one-cluster
unit).  Bit-exact integer comparison."""
import numpy as np
import pytest

import kv_cache_attention_states_b200 as kca
import oracle
from kv_cache_attention_states_b200 import synth

pytestmark = pytest.mark.gpu


def _expected(positions, window, split_len, cluster):
    spans = []
    for p in positions:
        lo, hi = oracle.visible_range(int(p), window)
        n = max(0, hi - lo + 1)
        ns = max(1, -(-n // split_len))
        spans.append((lo, hi, n, ns))
    max_clusters = -(-max(s[3] for s in spans) // cluster)
    rows = []
    for u, (lo, hi, n, ns) in enumerate(spans):
        nclus = -(-ns // cluster)
        for s in range(ns):
            kb, ke = (lo, lo) if n == 0 else (lo + s * split_len, min(lo + (s + 1) * split_len, hi + 1))
            rows.append((u, kb, ke, u * max_clusters + s // cluster if nclus > 1 else -1))
    return np.array(rows, dtype=np.int64)


def _check(items, positions, window):
    # The plan's split length, read off a unit with several splits (with one
    # split everywhere any length >= the longest range gives the same cut).
    multi = [u for u in range(len(positions)) if (items[:, 0] == u).sum() > 1]
    if multi:
        first = items[items[:, 0] == multi[0]][0]
        split_len = int(first[2] - first[1])
        assert split_len % 64 == 0
    else:
        split_len = max(64, int((items[:, 2] - items[:, 1]).max()))
    # The cut must be the documented one for one of the cluster sizes the
    # kernel runs (several sizes give the same items when no unit has more
    # than one cluster), and its clusters must fit one wave.
    fits = []
    for c in (1, 2, 4, 8):
        want = _expected(positions, window, split_len, c)
        if want.shape == items.shape and np.array_equal(want, items):
            fits.append(c)
    assert fits, "plan differs from the documented cut for every cluster size"
    c = fits[-1]
    n_clusters = sum(-(-int((items[:, 0] == u).sum()) // c) for u in range(len(positions)))
    assert n_clusters * c <= 148


@pytest.mark.parametrize("kv", [kca.F16, kca.BF16])
@pytest.mark.parametrize("ctx,window", [([16384], 0), ([1024], 0), ([131072], 0), ([0, 1, 5000], 0),
                                        ([4160], 512), ([131072] * 8, 0), ([9000, 17, 70000, 4096], 300)])
def test_decode_tensor_core_plan_is_the_documented_cut(cuda_ok, kv, ctx, window):
    items = kca.attn_decode_plan(ctx, window, kv_dtype=kv)
    _check(items, [c - 1 for c in ctx], window)


def test_decode_tensor_core_plan_of_the_ragged_workload(cuda_ok):
    ctx = synth.ragged_f16(0).decode_ctx[0]
    items = kca.attn_decode_plan(ctx, 0, kv_dtype=kca.F16)
    _check(items, [c - 1 for c in ctx], 0)


@pytest.mark.parametrize("cs,rows,window", [(100, 15, 0), (5000, 2, 0), (12000, 9, 0), (300, 7, 64)])
def test_short_chunk_rows_plan_on_tensor_cores_is_the_documented_cut(cuda_ok, cs, rows, window):
    path, items = kca.attn_prefill_plan(kca.BF16, kca.BF16, cs, rows, window)
    assert path == 0
    _check(items, [cs + u for u in range(rows)], window)


@pytest.mark.parametrize("ctx,window", [([16384], 0), ([16447], 0), ([4096], 0), ([256], 0), ([131072], 0),
                                        ([4160], 512), ([131072] * 8, 0)])
def test_device_plan_is_the_host_plan_for_the_device_capacity(cuda_ok, ctx, window):
    """The plan a call runs on this device equals the host-only plan for the
    device's SM count and resident-cluster capacity, which the CPU tests pin
    to the documented cost model."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cap = kca.attn_decode_cluster_capacity()
    dev_items, dev_c = kca.attn_decode_plan(ctx, window, kv_dtype=kca.F16, with_cluster=True)
    host_items, host_c = kca.attn_decode_plan(ctx, window, num_sms=sms, kv_dtype=kca.F16, cluster_capacity=cap,
                                              with_cluster=True)
    assert dev_c == host_c and np.array_equal(dev_items, host_items), (cap, dev_c, host_c)
