"""Parity in the launch configuration bench.py times: the bench's own
workload object (2 prompt replicas, 32 decode-cache replicas, one workspace
shared by all 64 decode calls), its prefill and decode captured as CUDA
graphs exactly as the timed region replays them, checked against the f64
oracle on the same seeded inputs -- every row of chunks 0, 10 and 21 plus
1,024 seeded random rows of the prompt, and every one of the 64 decode
steps -- and the bench's other configurations the same way: the decode
steps at 256 and 4,096 keys (every step), the window-512 prompt (every
row) and its 64 decode steps, and the 768-row chunk at the end of the
131,072-row cache (80 rows)."""
import os
import sys

import numpy as np
import pytest
import torch

from tests.helpers import max_err, oracle_decode, oracle_prefill, oracle_threads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bench_run(cuda_ok):
    oracle_threads()
    sys.path.insert(0, ROOT)
    import bench
    w = bench.Workload(torch.device("cuda", 0))
    w.prefill()                       # an eager step first, as the bench's warm-up
    w.decode()
    torch.cuda.synchronize()
    gp = torch.cuda.CUDAGraph()
    w.step_index = 0
    with torch.cuda.graph(gp):
        w.prefill()
    gd = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gd):
        w.decode()
    w.pre_out.fill_(float("nan"))
    w.dec_out.fill_(float("nan"))
    gp.replay()
    gd.replay()
    torch.cuda.synchronize()
    st_p = w.kca.attn_device_status(w.pre_ws)[0]
    st_d = w.kca.attn_device_status(w.dec_ws)[0]
    return bench, w, st_p, st_d


def test_bench_prefill_graph_matches_oracle(bench_run):
    bench, w, st_p, _ = bench_run
    assert st_p == 0
    x = bench._oracle_inputs(0)     # the same seeded draws as replica 0
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([np.arange(0, 768), np.arange(7680, 8448), np.arange(16128, 16384),
                                     rng.integers(0, 16384, 1024)]))
    want = oracle_prefill(x["q"], x["k"], x["v"], 0, rows, 0, "bf16", "bf16")
    assert max_err(w.pre_out.cpu().numpy()[rows], want) <= 4e-3


def test_bench_decode_graph_matches_oracle_on_every_step(bench_run):
    bench, w, _, st_d = bench_run
    assert st_d == 0
    x = bench._oracle_inputs(0)
    got = w.dec_out.cpu().numpy()
    for t, c in enumerate(w.dec_ctx):
        want = oracle_decode(x["qd"][t:t + 1], x["kd"][None], x["vd"][None], [c], 0, "f32", "f16", w.cap)
        assert max_err(got[t], want) <= 4e-3, t


@pytest.fixture(scope="module")
def other_parts(cuda_ok):
    """The bench's other configurations (decode at 256 and 4096, the window
    configuration, the long chunk), each captured as the CUDA graph the timed
    region replays, replayed once over NaN-filled outputs."""
    oracle_threads()
    sys.path.insert(0, ROOT)
    import bench
    dev = torch.device("cuda", 0)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    win = bench.WindowParts(dev, sms)
    parts = [bench.DecodeLenPart(dev, 256), bench.DecodeLenPart(dev, 4096)] + win.parts + \
        [bench.LongChunkPart(dev, sms)]
    for p in parts:
        p.run(0)
    torch.cuda.synchronize()
    graphs = []
    for p in parts:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            p.run(0)
        graphs.append(g)
    for o in (parts[0].out, parts[1].out, win.out, win.dout, parts[-1].out):
        o.fill_(float("nan"))
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    import kv_cache_attention_states_b200 as kca
    for p in parts:
        for ws in p.workspaces():
            assert kca.attn_device_status(ws)[0] == 0, p.name
    return bench, parts, win


def test_bench_small_decodes_match_oracle_on_every_step(other_parts):
    from kv_cache_attention_states_b200 import synth
    bench, parts, _ = other_parts
    for p in parts[:2]:
        wl = synth.decode_f16(p.ctx[0], bench.DECODE_STEPS)
        k = synth.draw(0, "k", (1, wl.capacity, 256), "f16")
        v = synth.draw(0, "v", (1, wl.capacity, 256), "f16")
        q = synth.draw(0, "q", (bench.DECODE_STEPS, 1, 8, 256), "f32")
        got = p.out.cpu().numpy()
        for t, c in enumerate(p.ctx):
            want = oracle_decode(q[t], k, v, [c], 0, "f32", "f16", wl.capacity)
            assert max_err(got[t], want) <= 4e-3, (p.name, t)


def test_bench_window_configuration_matches_oracle(other_parts):
    from kv_cache_attention_states_b200 import synth
    bench, _, win = other_parts
    wl = win.wl
    k = synth.draw(0, "k", (wl.capacity, 256), "bf16")
    v = synth.draw(0, "v", (wl.capacity, 256), "bf16")
    q = synth.draw(0, "q", (4096, 8, 256), "bf16")
    qd = synth.draw(0, "qd", (bench.DECODE_STEPS, 1, 8, 256), "bf16")
    want = oracle_prefill(q, k, v, 0, np.arange(4096), wl.window, "bf16", "bf16")
    assert max_err(win.out.cpu().numpy(), want) <= 4e-3
    got = win.dout.cpu().numpy()
    for t, c in enumerate(wl.decode_ctx):
        want = oracle_decode(qd[t], k[None], v[None], c, wl.window, "bf16", "bf16", wl.capacity)
        assert max_err(got[t], want) <= 4e-3, t


def test_bench_long_chunk_matches_oracle(other_parts):
    from kv_cache_attention_states_b200 import synth
    _, parts, _ = other_parts
    p = parts[-1]
    wl = synth.long_chunk_bf16()
    k = synth.draw(0, "k", (wl.capacity, 256), "bf16")
    v = synth.draw(0, "v", (wl.capacity, 256), "bf16")
    q = synth.draw(0, "q", (p.rows, 8, 256), "bf16")
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([np.arange(0, 16), np.arange(752, 768), rng.integers(0, 768, 48)]))
    want = oracle_prefill(q, k, v, p.cs, rows, 0, "bf16", "bf16")
    assert max_err(p.out.cpu().numpy()[rows], want) <= 4e-3
