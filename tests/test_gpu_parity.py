"""GPU parity: the CUDA path, called through the C ABI, against the f64 oracle
on the same seeded inputs (from synth).  Tolerances are the stated bars:
max |error| <= 2e-6 with f32 inputs, <= 4e-3 with f16/bf16 inputs."""
import numpy as np
import pytest
import torch

import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth
from tests.helpers import dev, max_err, oracle_decode, oracle_prefill, oracle_threads, tol

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(cuda_ok):
    oracle_threads()
    kca.lib()


def _cache(seed, capacity, rows, dtype, std=1.0, batch=None):
    shape = (capacity, 256) if batch is None else (batch, capacity, 256)
    k = np.zeros(shape, dtype=np.float32)
    v = np.zeros(shape, dtype=np.float32)
    if batch is None:
        k[:rows] = synth.normal(seed, "k", (rows, 256), std)
        v[:rows] = synth.normal(seed, "v", (rows, 256), std)
    else:
        for b in range(batch):
            r = rows[b]
            k[b, :r] = synth.normal(seed, f"k{b}", (r, 256), std)
            v[b, :r] = synth.normal(seed, f"v{b}", (r, 256), std)
    return synth.to_storage(k, dtype), synth.to_storage(v, dtype)


def _check_status(ws):
    st, detail = kca.attn_device_status(ws)
    assert st == 0, f"device status {st} detail {detail:#x}"


# ------------------------------------------------------------ tiny f32 config

def test_tiny_f32_prefill_and_decode():
    wl = synth.tiny_f32()
    seed = 0
    k, v = _cache(seed, wl.capacity, wl.capacity, "f32")
    kd, vd = dev(k, "f32"), dev(v, "f32")
    (cs, rows), = wl.prefill
    q = synth.draw(seed, "q_prefill", (rows, 8, 256), "f32")
    out = kca.attn_prefill(dev(q, "f32"), kd, vd, cs)
    want = oracle_prefill(q, k, v, cs, np.arange(rows), 0, "f32", "f32")
    assert max_err(out.cpu().numpy(), want) <= 2e-6
    qdec = synth.draw(seed, "q_decode", (len(wl.decode_ctx), 8, 256), "f32")
    for t, (ctx,) in enumerate(wl.decode_ctx):
        o = kca.attn_decode(dev(qdec[t:t + 1], "f32"), kd[None], vd[None], [ctx])
        w = oracle_decode(qdec[t:t + 1], k[None], v[None], [ctx], 0, "f32", "f32", wl.capacity)
        assert max_err(o.cpu().numpy(), w) <= 2e-6, t


# --------------------------------------------------------------- decode f16

@pytest.mark.parametrize("length", [256, 4096, 16384])
def test_decode_f16_lengths(length):
    wl = synth.decode_f16(length)
    k, v = _cache(1, wl.capacity, wl.capacity, "f16")
    kd, vd = dev(k, "f16")[None], dev(v, "f16")[None]
    q = synth.draw(1, "q", (len(wl.decode_ctx), 8, 256), "f32")
    ws = kca.new_workspace(kca.attn_decode_workspace_bytes([wl.capacity]))
    for t in (0, 1, 31, 63):
        ctx = wl.decode_ctx[t]
        o = kca.attn_decode(dev(q[t:t + 1], "f32"), kd, vd, ctx, workspace=ws)
        w = oracle_decode(q[t:t + 1], k[None], v[None], ctx, 0, "f32", "f16", wl.capacity)
        assert max_err(o.cpu().numpy(), w) <= 4e-3, (length, t)
    _check_status(ws)


@pytest.mark.parametrize("q_dtype,kv_dtype", [("f32", "f32"), ("bf16", "bf16"), ("f16", "f16"),
                                              ("f32", "bf16"), ("bf16", "f16"), ("f16", "f32")])
def test_decode_dtype_combinations(q_dtype, kv_dtype):
    cap = 3000
    ctx = [1, 17, 2999, 1500]
    k, v = _cache(2, cap, [cap] * 4, kv_dtype, batch=4)
    q = synth.draw(2, "q", (4, 8, 256), q_dtype)
    o = kca.attn_decode(dev(q, q_dtype), dev(k, kv_dtype), dev(v, kv_dtype), ctx)
    w = oracle_decode(q, k, v, ctx, 0, q_dtype, kv_dtype, cap)
    assert max_err(o.cpu().numpy(), w) <= tol(q_dtype, kv_dtype)


# -------------------------------------------------------- tensor-core prefill

@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("cs,rows,window", [(0, 768, 0), (1000, 200, 0), (3000, 17, 0),
                                            (77, 16, 0), (2048, 255, 100), (500, 300, 1),
                                            (4000, 96, 5000)])
def test_prefill_tc_matches_oracle(dtype, cs, rows, window):
    cap = cs + rows + 5
    std = 0.5
    k, v = _cache(3, cap, cs + rows, dtype, std)
    q = synth.draw(3, "q", (rows, 8, 256), dtype, std)
    code = kca.BF16 if dtype == "bf16" else kca.F16
    path, _ = kca.attn_prefill_plan(code, code, cs, rows, window)
    assert path == 1
    ws = kca.new_workspace(kca.attn_prefill_workspace_bytes(code, code, cs, rows, window))
    out = kca.attn_prefill(dev(q, dtype), dev(k, dtype), dev(v, dtype), cs, window, workspace=ws)
    want = oracle_prefill(q, k, v, cs, np.arange(rows), window, dtype, dtype)
    err = max_err(out.cpu().numpy(), want)
    assert err <= 4e-3, err
    _check_status(ws)


@pytest.mark.parametrize("rows", [1, 2, 15])
def test_prefill_short_chunks_take_rows_path(rows):
    cs = 300
    k, v = _cache(4, cs + rows, cs + rows, "bf16")
    q = synth.draw(4, "q", (rows, 8, 256), "bf16")
    out = kca.attn_prefill(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), cs)
    want = oracle_prefill(q, k, v, cs, np.arange(rows), 0, "bf16", "bf16")
    assert max_err(out.cpu().numpy(), want) <= 4e-3


@pytest.mark.parametrize("rows", [3, 9, 15])
def test_few_row_chunk_on_long_context_takes_tc_path(rows):
    # one ragged split tile: its partials keep only the chunk's rows
    cs = 16384 - rows
    k, v = _cache(6, cs + rows, cs + rows, "bf16", 0.5)
    q = synth.draw(6, "q", (rows, 8, 256), "bf16", 0.5)
    path, items = kca.attn_prefill_plan(kca.BF16, kca.BF16, cs, rows)
    assert path == 1 and len(items) > 8
    ws = kca.new_workspace(kca.attn_prefill_workspace_bytes(kca.BF16, kca.BF16, cs, rows))
    out = kca.attn_prefill(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), cs, workspace=ws)
    want = oracle_prefill(q, k, v, cs, np.arange(rows), 0, "bf16", "bf16")
    assert max_err(out.cpu().numpy(), want) <= 4e-3
    _check_status(ws)


def test_rows_and_tc_paths_agree():
    cs, rows = 640, 128
    k, v = _cache(5, cs + rows, cs + rows, "bf16")
    q = synth.draw(5, "q", (rows, 8, 256), "bf16")
    args = (dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), cs)
    tc = kca.attn_prefill(*args).cpu().numpy()
    with kca.forced_path(kca.OP_PREFILL, kca.PATH_ROWS):
        rw = kca.attn_prefill(*args).cpu().numpy()
    want = oracle_prefill(q, k, v, cs, np.arange(rows), 0, "bf16", "bf16")
    assert max_err(tc, want) <= 4e-3 and max_err(rw, want) <= 4e-3


# ------------------------------------------------------- full-size workloads

def test_prefill_16k_bf16_chunked_sampled_rows():
    wl = synth.prefill_bf16_16k()
    k, v = _cache(0, wl.capacity, wl.capacity, "bf16", wl.std)
    q = synth.draw(0, "q", (wl.capacity, 8, 256), "bf16", wl.std)
    kd, vd, qd = dev(k, "bf16"), dev(v, "bf16"), dev(q, "bf16")
    out = torch.empty((wl.capacity, 8, 256), dtype=torch.float32, device="cuda")
    ws = kca.new_workspace(max(kca.attn_prefill_workspace_bytes(2, 2, cs, r) for cs, r in wl.prefill))
    for cs, r in wl.prefill:
        kca.attn_prefill(qd[cs:cs + r], kd, vd, cs, out=out[cs:cs + r], workspace=ws)
    torch.cuda.synchronize()
    _check_status(ws)
    # Every row of chunks 0, 10, 20 and 21 (the first chunk, a middle one, the
    # last full one and the 256-row tail), plus 2,048 seeded random rows of
    # the whole prompt: the f64 oracle takes ~20 s for these on 16 cores,
    # where all 16,384 rows would take minutes.
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([
        np.arange(0, 768), np.arange(768 * 10, 768 * 11), np.arange(768 * 20, 16384),
        rng.integers(0, 16384, 2048)]))
    want = oracle_prefill(q, k, v, 0, sample, 0, "bf16", "bf16")
    assert max_err(out.cpu().numpy()[sample], want) <= 4e-3


def test_window_bf16_prefill_and_decode():
    wl = synth.window_bf16()
    k, v = _cache(0, wl.capacity, wl.capacity, "bf16")
    q = synth.draw(0, "q", (4096, 8, 256), "bf16")
    kd, vd = dev(k, "bf16"), dev(v, "bf16")
    qd = dev(q, "bf16")
    out = torch.empty((4096, 8, 256), dtype=torch.float32, device="cuda")
    for cs, r in wl.prefill:
        kca.attn_prefill(qd[cs:cs + r], kd, vd, cs, wl.window, out=out[cs:cs + r])
    rows = np.concatenate([np.arange(0, 600), np.arange(3000, 3300), np.arange(3840, 4096)])
    want = oracle_prefill(q, k, v, 0, rows, wl.window, "bf16", "bf16")
    assert max_err(out.cpu().numpy()[rows], want) <= 4e-3
    qdec = synth.draw(0, "q_decode", (len(wl.decode_ctx), 8, 256), "bf16")
    for t in (0, 1, 40, 63):
        ctx = wl.decode_ctx[t]
        o = kca.attn_decode(dev(qdec[t:t + 1], "bf16"), kd[None], vd[None], ctx, wl.window)
        w = oracle_decode(qdec[t:t + 1], k[None], v[None], ctx, wl.window, "bf16", "bf16", wl.capacity)
        assert max_err(o.cpu().numpy(), w) <= 4e-3, t


def test_ragged_long_context_decode():
    wl = synth.ragged_f16(0)
    ctx0 = np.array(wl.decode_ctx[0])
    need = ctx0 + len(wl.decode_ctx)
    k, v = _cache(0, wl.capacity, need, "f16", batch=wl.batch)
    kd, vd = dev(k, "f16"), dev(v, "f16")
    q = synth.draw(0, "q", (len(wl.decode_ctx), wl.batch, 8, 256), "f32")
    ws = kca.new_workspace(max(kca.attn_decode_workspace_bytes(c) for c in wl.decode_ctx))
    for t in (0, 31):
        o = kca.attn_decode(dev(q[t], "f32"), kd, vd, wl.decode_ctx[t], workspace=ws)
        w = oracle_decode(q[t], k, v, wl.decode_ctx[t], 0, "f32", "f16", wl.capacity)
        assert max_err(o.cpu().numpy(), w) <= 4e-3, t
    _check_status(ws)


def test_long_chunk_at_capacity_end_every_row():
    wl = synth.long_chunk_bf16()
    (cs, rows), = wl.prefill
    k, v = _cache(0, wl.capacity, wl.capacity, "bf16")
    q = synth.draw(0, "q", (rows, 8, 256), "bf16")
    out = kca.attn_prefill(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), cs)
    # every row of the chunk (each sees ~131K keys; the oracle takes ~45 s on 16 cores)
    want = oracle_prefill(q, k, v, cs, np.arange(rows), 0, "bf16", "bf16")
    assert max_err(out.cpu().numpy(), want) <= 4e-3


@pytest.mark.parametrize("q_dtype,kv_dtype", [("f32", "f16"), ("bf16", "bf16"), ("f32", "bf16")])
def test_decode_tensor_core_and_cuda_core_paths_agree(q_dtype, kv_dtype):
    cap = 20000
    ctx = [19999, 1, 63, 64, 65, 777, 12000]
    k, v = _cache(6, cap, [cap] * len(ctx), kv_dtype, batch=len(ctx))
    q = synth.draw(6, "q", (len(ctx), 8, 256), q_dtype)
    args = (dev(q, q_dtype), dev(k, kv_dtype), dev(v, kv_dtype), ctx)
    mma = kca.attn_decode(*args).cpu().numpy()
    with kca.forced_path(kca.OP_ROWS, kca.PATH_CUDA_CORE):
        simt = kca.attn_decode(*args).cpu().numpy()
    want = oracle_decode(q, k, v, ctx, 0, q_dtype, kv_dtype, cap)
    assert max_err(mma, want) <= 4e-3 and max_err(simt, want) <= 4e-3


@pytest.mark.parametrize("q_dtype,kv_dtype", [("f32", "f16"), ("f32", "f32")])
def test_decode_at_the_maximum_batch(q_dtype, kv_dtype):
    # KCA_MAX_BATCH sequences, ragged lengths including an empty context and
    # one at the capacity: tensor-core (f16) and CUDA-core (f32) kernels
    batch, cap = kca.MAX_BATCH, 2048
    ctx = synth.integers(21, "ctx", 0, cap, batch)
    ctx[0], ctx[1], ctx[2] = 0, cap, 1
    k, v = _cache(21, cap, ctx, kv_dtype, batch=batch)
    q = synth.draw(21, "q", (batch, 8, 256), q_dtype)
    ws = kca.new_workspace(kca.attn_decode_workspace_bytes(ctx))
    out = kca.attn_decode(dev(q, q_dtype), dev(k, kv_dtype), dev(v, kv_dtype), ctx, workspace=ws)
    want = oracle_decode(q, k, v, ctx, 0, q_dtype, kv_dtype, cap)
    assert max_err(out.cpu().numpy(), want) <= tol(q_dtype, kv_dtype)
    assert torch.all(out[0] == 0)
    _check_status(ws)
    one_more = batch + 1                            # past the limit: rejected before any launch
    qx = torch.zeros((one_more, 8, 256), dtype=torch.float32, device="cuda")
    kx = torch.zeros((one_more, 16, 256), dtype=torch.float16, device="cuda")
    with pytest.raises(kca.KcaError):
        kca.attn_decode(qx, kx, kx.clone(), [1] * one_more)



# ------------------------------------------- f32 (CUDA-core kernel) at size

@pytest.mark.parametrize("window", [0, 512])
def test_f32_prefill_chunk_of_768_rows_at_8192(window):
    """The CUDA-core rows kernel (f32 Q/K/V) on a full 768-row chunk at
    positions 8192..8959, every row against the oracle at the f32 bar."""
    cs, rows = 8192, 768
    k, v = _cache(31, cs + rows, cs + rows, "f32")
    q = synth.draw(31, "q", (rows, 8, 256), "f32")
    assert kca.attn_prefill_path(kca.F32, kca.F32, cs, rows, window) == 0
    ws = kca.new_workspace(kca.attn_prefill_workspace_bytes(kca.F32, kca.F32, cs, rows, window))
    out = kca.attn_prefill(dev(q, "f32"), dev(k, "f32"), dev(v, "f32"), cs, window, workspace=ws)
    want = oracle_prefill(q, k, v, cs, np.arange(rows), window, "f32", "f32")
    assert max_err(out.cpu().numpy(), want) <= 2e-6
    _check_status(ws)


def test_f32_decode_at_16k_and_64k_keys():
    """The CUDA-core rows kernel and its split merge on f32 caches: a batch
    with contexts of 16,384 and 65,536 keys (and a short one), every row
    against the oracle at the f32 bar."""
    cap = 65536
    ctx = [16384, 65536, 1000]
    k, v = _cache(32, cap, ctx, "f32", batch=len(ctx))
    q = synth.draw(32, "q", (len(ctx), 8, 256), "f32")
    ws = kca.new_workspace(kca.attn_decode_workspace_bytes(ctx))
    out = kca.attn_decode(dev(q, "f32"), dev(k, "f32"), dev(v, "f32"), ctx, workspace=ws)
    want = oracle_decode(q, k, v, ctx, 0, "f32", "f32", cap)
    assert max_err(out.cpu().numpy(), want) <= 2e-6
    _check_status(ws)
