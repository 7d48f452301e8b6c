"""Context-split decode on one GPU: the shards' partial records
(attn_decode_partial) and their merge (attn_merge_partials) against the
oracle -- the records one by one (oracle/partial.py) and the merged output
(whole-context attention of the C oracle).  Several shards are computed on
the same GPU one after another (no kernel waits on another); the NCCL
exchange itself runs with one rank here and with two gloo ranks on the CPU
(test_multirank_cpu.py)."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth
from oracle import partial
from tests.helpers import dev, max_err, oracle_decode, oracle_threads, tol

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _setup(cuda_ok):
    oracle_threads()
    kca.lib()


def _inputs(seed, batch, cap, q_dtype, kv_dtype):
    q = synth.draw(seed, "q", (batch, 8, 256), q_dtype)
    k = synth.draw(seed, "k", (batch, cap, 256), kv_dtype)
    v = synth.draw(seed, "v", (batch, cap, 256), kv_dtype)
    return q, k, v


def _run_shards(q, k, v, ctx, cuts, window, q_dtype, kv_dtype):
    batch = q.shape[0]
    qd = dev(q, q_dtype)
    parts = torch.empty((len(cuts) - 1, kca.partial_floats(batch)), dtype=torch.float32, device="cuda")
    for i, (kb, ke) in enumerate(zip(cuts[:-1], cuts[1:])):
        ks = dev(np.ascontiguousarray(k[:, kb:ke]), kv_dtype)
        vs = dev(np.ascontiguousarray(v[:, kb:ke]), kv_dtype)
        kca.attn_decode_partial(qd, ks, vs, ctx, kb, window, part=parts[i])
    return parts


def _check_record(rec, q, k, v, ctx, kb, ke, window, q_dtype, kv_dtype):
    batch = q.shape[0]
    ml, acc = kca.split_partial(rec, batch)
    ml, acc = ml.cpu().numpy().astype(np.float64), acc.cpu().numpy().astype(np.float64)
    m, l = ml[..., 0], ml[..., 1]
    om, ol, oacc = partial.decode_partial(q, k[:, kb:ke], v[:, kb:ke], ctx, kb, window=window,
                                          q_dtype=q_dtype, kv_dtype=kv_dtype)
    empty = om == -np.inf
    assert np.all(m[empty] == -np.inf) and np.all(l[empty] == 0) and np.all(acc[empty] == 0)
    full = ~empty
    if full.any():
        # m is a reference at most 8 ln 2 below the largest score; l and acc
        # are relative to it
        assert np.all(m[full] <= om[full] + 1e-4) and np.all(m[full] >= om[full] - 8 * np.log(2) - 1e-4)
        shift = np.exp(m[full] - om[full])
        assert np.max(np.abs(l[full] * shift / ol[full] - 1)) <= 1e-4
        got = acc[full] / l[full][:, None]
        want = oacc[full] / ol[full][:, None]
        assert np.max(np.abs(got - want)) <= tol(q_dtype, kv_dtype)


@pytest.mark.parametrize("q_dtype,kv_dtype", [("f32", "f16"), ("bf16", "bf16"), ("f32", "f32")])
@pytest.mark.parametrize("window", [0, 3000])
def test_shard_records_and_merge_match_oracle(q_dtype, kv_dtype, window):
    cap = 10240
    q, k, v = _inputs(11, 3, cap, q_dtype, kv_dtype)
    ctx = [5000, 131, 9000]
    cuts = [0, 2560, 5120, 7680, 10240]
    parts = _run_shards(q, k, v, ctx, cuts, window, q_dtype, kv_dtype)
    for i, (kb, ke) in enumerate(zip(cuts[:-1], cuts[1:])):
        _check_record(parts[i], q, k, v, ctx, kb, ke, window, q_dtype, kv_dtype)
    out = kca.attn_merge_partials(parts, 3).cpu().numpy()
    want = oracle_decode(q, k, v, ctx, window, q_dtype, kv_dtype, cap)
    assert max_err(out, want) <= tol(q_dtype, kv_dtype)


def test_uneven_shards_long_context_and_empty_rows():
    # one long sequence cut unevenly, one with no context at all
    cap = 40000
    q, k, v = _inputs(12, 2, cap, "f32", "f16")
    ctx = [37777, 0]
    cuts = [0, 123, 20000, 37000, 40000]
    parts = _run_shards(q, k, v, ctx, cuts, 0, "f32", "f16")
    _check_record(parts[3], q, k, v, ctx, 37000, 40000, 0, "f32", "f16")
    out = kca.attn_merge_partials(parts, 2)
    want = oracle_decode(q, k, v, ctx, 0, "f32", "f16", cap)
    assert max_err(out.cpu().numpy(), want) <= 4e-3
    assert torch.all(out[1] == 0)
    again = kca.attn_merge_partials(parts, 2)
    assert torch.equal(out, again)                  # merged in record order: same bits


def test_one_shard_equals_attn_decode():
    cap = 16384
    q, k, v = _inputs(13, 2, cap, "f32", "f16")
    ctx = [16384, 7000]
    qd, kd, vd = dev(q, "f32"), dev(k, "f16"), dev(v, "f16")
    part = kca.attn_decode_partial(qd, kd, vd, ctx, 0)
    merged = kca.attn_merge_partials(part.view(1, -1), 2)
    direct = kca.attn_decode(qd, kd, vd, ctx)
    assert max_err(merged.cpu().numpy(), direct.cpu().numpy()) <= 1e-6


_NCCL_CHILD = r"""
import os, sys
sys.path.insert(0, sys.argv[1])
import numpy as np, torch, torch.distributed as dist
import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth
from kv_cache_attention_states_b200.context_split import decode_context_split
dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"))
q = synth.as_torch(synth.draw(14, "q", (2, 8, 256), "f32"), "f32").cuda()
k = synth.as_torch(synth.draw(14, "k", (2, 4096, 256), "f16"), "f16").cuda()
v = synth.as_torch(synth.draw(14, "v", (2, 4096, 256), "f16"), "f16").cuda()
out = decode_context_split(q, k, v, [4096, 1000], 0)
ref = kca.attn_decode(q, k, v, [4096, 1000])
torch.cuda.synchronize()
dist.destroy_process_group()
err = (out - ref).abs().max().item()
print("err", err)
sys.exit(0 if err <= 1e-6 else 1)
"""


def test_nccl_exchange_with_one_rank():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, "-c", _NCCL_CHILD, ROOT], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
