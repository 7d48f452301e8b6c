"""Bit-exact properties of the CUDA path (no tolerance): determinism, rows
outside every visible range are never read (NaN poison leaves the output
bitwise unchanged), guard regions around out / workspace stay intact, the
closed forms that are exact in f32, and the NaN / fully-masked semantics of
the Karume v0.8.0 release notes ("Breaking Changes", softmax NaN item)."""
import numpy as np
import pytest
import torch

import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth
from tests.helpers import dev

pytestmark = pytest.mark.gpu

NAN16 = {"bf16": np.uint16(0x7FC0), "f16": np.float16(np.nan), "f32": np.float32(np.nan)}


@pytest.fixture(scope="module", autouse=True)
def _setup(cuda_ok):
    kca.lib()


def _data(dtype, cap, rows, seed=7):
    k = synth.draw(seed, "k", (cap, 256), dtype)
    v = synth.draw(seed, "v", (cap, 256), dtype)
    q = synth.draw(seed, "q", (rows, 8, 256), dtype)
    return q, k, v


@pytest.mark.parametrize("dtype,rows", [("bf16", 200), ("f16", 64), ("f32", 40), ("bf16", 7)])
def test_prefill_is_deterministic(dtype, rows):
    cs = 900
    q, k, v = _data(dtype, cs + rows, rows)
    a = (dev(q, dtype), dev(k, dtype), dev(v, dtype), cs)
    o1 = kca.attn_prefill(*a)
    o2 = kca.attn_prefill(*a)
    assert torch.equal(o1, o2)


def test_decode_is_deterministic():
    k = dev(synth.draw(1, "k", (2, 20000, 256), "f16"), "f16")
    v = dev(synth.draw(1, "v", (2, 20000, 256), "f16"), "f16")
    q = dev(synth.draw(1, "q", (2, 8, 256), "f32"), "f32")
    o1 = kca.attn_decode(q, k, v, [20000, 12345])
    o2 = kca.attn_decode(q, k, v, [20000, 12345])
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("dtype,rows,window", [("bf16", 200, 100), ("bf16", 200, 0), ("f16", 48, 37),
                                               ("f32", 30, 20), ("bf16", 9, 50)])
def test_prefill_never_reads_rows_outside_the_visible_union(dtype, rows, window):
    cs = 1000
    cap = cs + rows + 300
    q, k, v = _data(dtype, cap, rows)
    clean = kca.attn_prefill(dev(q, dtype), dev(k, dtype), dev(v, dtype), cs, window)
    lo = max(0, cs - window + 1) if window > 0 else 0
    kp, vp = k.copy(), v.copy()
    kp[:lo] = NAN16[dtype]
    vp[:lo] = NAN16[dtype]
    kp[cs + rows:] = NAN16[dtype]
    vp[cs + rows:] = NAN16[dtype]
    poisoned = kca.attn_prefill(dev(q, dtype), dev(kp, dtype), dev(vp, dtype), cs, window)
    assert torch.isfinite(clean).all()
    assert torch.equal(clean, poisoned)


def test_decode_never_reads_invisible_rows():
    cap, ctx, window = 5000, 4321, 700
    k = synth.draw(2, "k", (1, cap, 256), "f16")
    v = synth.draw(2, "v", (1, cap, 256), "f16")
    q = dev(synth.draw(2, "q", (1, 8, 256), "f32"), "f32")
    clean = kca.attn_decode(q, dev(k, "f16"), dev(v, "f16"), [ctx], window)
    k[0, :ctx - window] = np.nan
    v[0, :ctx - window] = np.nan
    k[0, ctx:] = np.nan
    v[0, ctx:] = np.nan
    poisoned = kca.attn_decode(q, dev(k, "f16"), dev(v, "f16"), [ctx], window)
    assert torch.equal(clean, poisoned)


def test_guard_regions_untouched():
    dtype, cs, rows = "bf16", 2000, 300
    q, k, v = _data(dtype, cs + rows, rows)
    need = kca.attn_prefill_workspace_bytes(kca.BF16, kca.BF16, cs, rows)
    big = torch.full((rows * 8 * 256 + 2 * 4096,), 12345.0, dtype=torch.float32, device="cuda")
    out = big[4096:4096 + rows * 8 * 256].view(rows, 8, 256)
    ws = kca.new_workspace(need + 65536)
    ws[need:].fill_(0xAB)
    kca.attn_prefill(dev(q, dtype), dev(k, dtype), dev(v, dtype), cs, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert (big[:4096] == 12345.0).all() and (big[-4096:] == 12345.0).all()
    assert (ws[need:] == 0xAB).all()
    # decode
    kd = dev(synth.draw(3, "k", (1, 9000, 256), "f16"), "f16")
    vd = dev(synth.draw(3, "v", (1, 9000, 256), "f16"), "f16")
    qd = dev(synth.draw(3, "q", (1, 8, 256), "f32"), "f32")
    need = kca.attn_decode_workspace_bytes([9000])
    ws = kca.new_workspace(need + 4096)
    ws[need:].fill_(0xCD)
    big = torch.full((3 * 2048,), -7.0, dtype=torch.float32, device="cuda")
    kca.attn_decode(qd, kd, vd, [9000], out=big[2048:4096].view(1, 8, 256), workspace=ws)
    torch.cuda.synchronize()
    assert (big[:2048] == -7.0).all() and (big[4096:] == -7.0).all()
    assert (ws[need:] == 0xCD).all()


def test_decode_empty_context_is_exactly_zero_and_single_key_is_its_value_row():
    cap = 64
    k = synth.draw(4, "k", (3, cap, 256), "f32")
    v = synth.draw(4, "v", (3, cap, 256), "f32")
    q = dev(synth.draw(4, "q", (3, 8, 256), "f32"), "f32")
    out = kca.attn_decode(q, dev(k, "f32"), dev(v, "f32"), [0, 1, 64]).cpu().numpy()
    assert (out[0] == 0.0).all() and not np.signbit(out[0]).any()
    np.testing.assert_array_equal(out[1], np.repeat(v[1, 0][None], 8, 0))
    # window 1 at any position returns that position's value row exactly
    out = kca.attn_decode(q, dev(k, "f32"), dev(v, "f32"), [5, 30, 64], window=1).cpu().numpy()
    for b, c in enumerate([5, 30, 64]):
        np.testing.assert_array_equal(out[b], np.repeat(v[b, c - 1][None], 8, 0))


def test_prefill_equal_heads_give_equal_outputs_on_tensor_cores():
    dtype, cs, rows = "bf16", 500, 64
    q, k, v = _data(dtype, cs + rows, rows)
    q[:, :, :] = q[:, 3:4, :]
    out = kca.attn_prefill(dev(q, dtype), dev(k, dtype), dev(v, dtype), cs).cpu()
    for h in range(8):
        assert torch.equal(out[:, h], out[:, 0])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_nan_in_a_visible_key_reaches_exactly_the_rows_that_see_it(dtype):
    cs, rows = 100, 64
    q, k, v = _data(dtype, cs + rows, rows)
    k[130, 7] = NAN16[dtype]
    out = kca.attn_prefill(dev(q, dtype), dev(k, dtype), dev(v, dtype), cs).cpu().numpy()
    see = np.arange(rows) + cs >= 130
    assert np.isnan(out[see]).all()
    assert np.isfinite(out[~see]).all()


def test_decode_nan_key_gives_nan_row_only_for_that_sequence():
    k = synth.draw(5, "k", (2, 300, 256), "f16")
    v = synth.draw(5, "v", (2, 300, 256), "f16")
    k[0, 10, 0] = np.nan
    q = dev(synth.draw(5, "q", (2, 8, 256), "f32"), "f32")
    out = kca.attn_decode(q, dev(k, "f16"), dev(v, "f16"), [300, 300]).cpu().numpy()
    assert np.isnan(out[0]).all() and np.isfinite(out[1]).all()


def test_windowed_prefill_repeats_bitwise_and_matches_oracle():
    """Regression for a phase race between the softmax warps and the PV
    barrier: scores of N(0,1) data under a 512 window trigger the O rescale
    path; every repeat must give the same bits, and the oracle's values."""
    import oracle
    from tests.helpers import oracle_prefill, oracle_threads
    oracle_threads()
    cs, rows, window = 3072, 768, 512
    q, k, v = _data("bf16", cs + rows, rows, seed=11)
    args = (dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), cs, window)
    first = kca.attn_prefill(*args)
    for _ in range(20):
        assert torch.equal(kca.attn_prefill(*args), first)
    sample = np.arange(0, rows, 7)
    want = oracle_prefill(q, k, v, cs, sample, window, "bf16", "bf16")
    assert float(np.abs(first.cpu().numpy()[sample] - want).max()) <= 4e-3


def test_calls_capture_into_a_cuda_graph_and_replay_bitwise():
    cs, rows = 2048, 768
    q, k, v = _data("bf16", cs + rows, rows, seed=13)
    qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    out = torch.empty((rows, 8, 256), dtype=torch.float32, device="cuda")
    ws = kca.new_workspace(kca.attn_prefill_workspace_bytes(kca.BF16, kca.BF16, cs, rows))
    kc = dev(synth.draw(14, "k", (2, 5000, 256), "f16"), "f16")
    vc = dev(synth.draw(14, "v", (2, 5000, 256), "f16"), "f16")
    qc = dev(synth.draw(14, "q", (2, 8, 256), "f32"), "f32")
    outd = torch.empty((2, 8, 256), dtype=torch.float32, device="cuda")
    wsd = kca.new_workspace(kca.attn_decode_workspace_bytes([5000, 3333]))
    eager_p = kca.attn_prefill(qd, kd, vd, cs, out=out, workspace=ws).clone()
    eager_d = kca.attn_decode(qc, kc, vc, [5000, 3333], out=outd, workspace=wsd).clone()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        kca.attn_prefill(qd, kd, vd, cs, out=out, workspace=ws)
        kca.attn_decode(qc, kc, vc, [5000, 3333], out=outd, workspace=wsd)
    out.zero_()
    outd.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager_p) and torch.equal(outd, eager_d)
    del g


@pytest.mark.parametrize("cs,rows,window,j", [(1000, 400, 0, 350), (1000, 400, 128, 100), (64, 768, 0, 500)])
def test_nan_in_a_value_row_on_the_tensor_core_path(cs, rows, window, j):
    """A NaN in V at chunk row j (position p = cs + j) -- outside what the
    tensor-core path accepts (kca.h PRECONDITIONS: V finite on a chunk's
    visible union) -- poisons exactly the 16-row tiles whose work items
    cover p (0 x NaN in the PV product of a masked key): every row of those
    tiles is NaN, every other row is finite and equals the oracle's value.
    The rows path, on the same inputs, poisons exactly the rows that see p,
    as the definition does."""
    from tests.helpers import max_err, oracle_prefill, oracle_threads
    oracle_threads()
    dtype = "bf16"
    q, k, v = _data(dtype, cs + rows, rows, seed=17)
    p = cs + j
    v[p, :] = NAN16[dtype]
    path, items = kca.attn_prefill_plan(kca.BF16, kca.BF16, cs, rows, window)
    assert path == 1
    n_tiles = (rows + 15) // 16
    hit = np.zeros(n_tiles, dtype=bool)
    for tile, kb, ke, _ in items:
        if kb <= p < ke:
            hit[tile] = True
    tile_of_row = np.arange(rows) // 16
    poisoned = hit[tile_of_row]
    pos = cs + np.arange(rows)
    lo = np.maximum(0, pos - window + 1) if window > 0 else np.zeros(rows, dtype=np.int64)
    sees = (lo <= p) & (p <= pos)
    assert sees.any() and (~poisoned).any()
    assert not (sees & ~poisoned).any()          # every row that sees p lies in a poisoned tile
    args = (dev(q, dtype), dev(k, dtype), dev(v, dtype), cs, window)
    tc = kca.attn_prefill(*args).cpu().numpy()
    want = oracle_prefill(q, k, v, cs, np.arange(rows), window, dtype, dtype)
    assert np.isnan(want[sees]).all() and np.isfinite(want[~sees]).all()
    assert np.isnan(tc[poisoned]).all()
    assert np.isfinite(tc[~poisoned]).all()
    assert max_err(tc[~poisoned], want[~poisoned]) <= 4e-3
    with kca.forced_path(kca.OP_PREFILL, kca.PATH_ROWS):
        rw = kca.attn_prefill(*args).cpu().numpy()
    assert np.isnan(rw[sees]).all()
    assert np.isfinite(rw[~sees]).all()
    assert max_err(rw[~sees], want[~sees]) <= 4e-3
