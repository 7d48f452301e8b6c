"""GPU parity of attn_decode_dev (context lengths in device memory) against the
f64 oracle: ragged batches under a launch planned for a bound, a captured CUDA
graph replayed over changing context lengths, and out-of-range device values,
which the kernels must turn into an empty row plus a status record."""
import numpy as np
import pytest
import torch

import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth
from tests.helpers import dev, max_err, oracle_decode, oracle_threads, tol

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(cuda_ok):
    oracle_threads()
    kca.lib()


def _inputs(seed, batch, capacity, kd, qd="f32"):
    k = synth.normal(seed, "k", (batch, capacity, 256), 1.0)
    v = synth.normal(seed, "v", (batch, capacity, 256), 1.0)
    q = synth.draw(seed, "q", (batch, 8, 256), qd)
    return q, synth.to_storage(k, kd), synth.to_storage(v, kd)


def _ctx_dev(ctx):
    return torch.tensor(np.asarray(ctx, dtype=np.int64), device="cuda")


@pytest.mark.parametrize("kd", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("bound_kind", ["capacity", "max"])
def test_decode_dev_ragged_batch_matches_oracle(kd, bound_kind):
    capacity = 20480
    ctx = [0, 1, 300, 5000, 20000]
    q, k, v = _inputs(3, len(ctx), capacity, kd)
    bound = capacity if bound_kind == "capacity" else max(ctx)
    got = kca.attn_decode_dev(dev(q, "f32"), dev(k, kd), dev(v, kd), _ctx_dev(ctx), bound)
    want = oracle_decode(q, k, v, ctx, 0, "f32", kd, capacity)
    assert max_err(got.cpu().numpy(), want) <= tol("f32", kd)
    assert np.all(got[0].cpu().numpy() == 0.0)       # ctx 0: an all-zero row


def test_decode_dev_window_matches_oracle():
    capacity, window = 8192, 512
    ctx = [100, 513, 4096, 8192]
    q, k, v = _inputs(4, len(ctx), capacity, "bf16", "bf16")
    got = kca.attn_decode_dev(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), _ctx_dev(ctx), capacity,
                              window=window)
    want = oracle_decode(q, k, v, ctx, window, "bf16", "bf16", capacity)
    assert max_err(got.cpu().numpy(), want) <= tol("bf16", "bf16")


@pytest.mark.parametrize("kd", ["f16", "f32"])
def test_decode_dev_graph_replay_follows_device_context(kd):
    capacity = 16384
    batch = 3
    q, k, v = _inputs(5, batch, capacity, kd)
    qd, kd_, vd = dev(q, "f32"), dev(k, kd), dev(v, kd)
    ctx_dev = _ctx_dev([1] * batch)
    out = torch.empty((batch, 8, 256), dtype=torch.float32, device="cuda")
    ws = kca.new_workspace(kca.attn_decode_workspace_bytes([capacity] * batch))
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        kca.attn_decode_dev(qd, kd_, vd, ctx_dev, capacity, out=out, workspace=ws, stream=stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        kca.attn_decode_dev(qd, kd_, vd, ctx_dev, capacity, out=out, workspace=ws, stream=stream)
    for ctx in ([100, 5000, 16384], [16384, 1, 7777], [0, 64, 65], [16384, 16384, 16384]):
        ctx_dev.copy_(_ctx_dev(ctx))
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        want = oracle_decode(q, k, v, ctx, 0, "f32", kd, capacity)
        assert max_err(out.cpu().numpy(), want) <= tol("f32", kd), ctx
    st, detail = kca.attn_device_status(ws)
    assert st == 0, hex(detail)
    del g


@pytest.mark.parametrize("kd", ["f16", "f32"])
def test_decode_dev_out_of_range_context_is_recorded_and_empty(kd):
    capacity, bound = 4096, 2048
    ctx = [100, bound + 5, -1, bound]
    q, k, v = _inputs(6, len(ctx), capacity, kd)
    ws = kca.new_workspace(kca.attn_decode_workspace_bytes([bound] * len(ctx)))
    got = kca.attn_decode_dev(dev(q, "f32"), dev(k, kd), dev(v, kd), _ctx_dev(ctx), bound, workspace=ws)
    torch.cuda.synchronize()
    st, detail = kca.attn_device_status(ws)
    assert st == -8
    assert detail >> 24 == 10 and (detail & 0xffffff) in (1, 2)
    g = got.cpu().numpy()
    assert np.all(g[1] == 0.0) and np.all(g[2] == 0.0)
    ok = [0, 3]
    want = oracle_decode(q[ok], k[ok], v[ok], [ctx[i] for i in ok], 0, "f32", kd, capacity)
    assert max_err(g[ok], want) <= tol("f32", kd)
    assert kca.attn_device_status(ws)[0] == 0        # the read cleared it
