"""Parity in the launch configuration bench.py times: the bench's own
workload object (2 prompt replicas, 32 decode-cache replicas, one workspace
shared by all 64 decode calls), its prefill and decode captured as CUDA
graphs exactly as the timed region replays them, checked against the f64
oracle on the same seeded inputs -- every row of chunks 0, 10 and 21 plus
1,024 seeded random rows of the prompt, and every one of the 64 decode
steps."""
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
