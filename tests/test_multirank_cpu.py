"""Multi-rank host paths on CPU, two gloo ranks (one process each, as the
per-GPU launch runs them):
  * bench.py's N>1 timing: the device-timed values reduce to the maximum
    over ranks, which every rank receives (the bench's data path has no
    collective: each rank runs its own replica of the workload);
  * the context-split decode exchange (context_split.exchange_partials):
    each rank's partial record reaches every rank, in rank order, and the
    merge of the gathered records is the whole-context attention.  The
    records here come from the oracle, since the ranks have no GPU."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, values, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        out[rank] = bench.max_over_ranks(values[rank], world, "cpu")
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_maximum_over_ranks():
    world = 2
    values = [[3.0, 10.0, 0.5], [7.0, 2.0, 0.5]]
    ctx = mp.get_context("spawn")          # the manager's server process too: no fork of a threaded process
    with ctx.Manager() as manager:
        out = manager.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, world, port, values, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        for r in range(world):
            assert out[r] == [7.0, 10.0, 0.5]


def _record(m, l, acc):
    """Partial record layout of attn_decode_partial: (m, l) pairs, then acc."""
    import numpy as np
    return np.concatenate([np.stack([m, l], -1).reshape(-1), acc.reshape(-1)]).astype(np.float32)


def _exchange_rank(rank, world, port, out):
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import partial
    from kv_cache_attention_states_b200 import synth
    from kv_cache_attention_states_b200.context_split import exchange_partials
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q = synth.draw(7, "q", (2, 8, 256), "f32")
        k = synth.draw(7, "k", (2, 200, 256), "f16")
        v = synth.draw(7, "v", (2, 200, 256), "f16")
        ctx = [200, 90]
        kb, ke = 100 * rank, 100 * (rank + 1)          # rank r holds positions [100 r, 100 r + 100)
        m, l, acc = partial.decode_partial(q, k[:, kb:ke], v[:, kb:ke], ctx, kb, q_dtype="f32", kv_dtype="f16")
        mine = torch.from_numpy(_record(m, l, acc))
        got = exchange_partials(mine).numpy()
        out[rank] = (got.tobytes(), mine.numpy().tobytes(), got.shape)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_context_split_exchange_gathers_records_in_rank_order():
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from oracle import partial
    from kv_cache_attention_states_b200 import synth
    world = 2
    ctx_ = mp.get_context("spawn")
    with ctx_.Manager() as manager:
        out = manager.dict()
        port = _free_port()
        procs = [ctx_.Process(target=_exchange_rank, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = {r: out[r] for r in range(world)}
    batch = 2
    n = batch * 8 * 2
    for r in range(world):
        got = np.frombuffer(res[r][0], dtype=np.float32).reshape(res[r][2])
        for src in range(world):
            assert got[src].tobytes() == res[src][1]      # every record, bit for bit, in rank order
    g = np.frombuffer(res[0][0], dtype=np.float32).reshape(res[0][2]).astype(np.float64)
    ml = g[:, :n].reshape(world, batch, 8, 2)
    acc = g[:, n:].reshape(world, batch, 8, 256)
    merged = partial.merge_partials(ml[..., 0], ml[..., 1], acc)
    q = synth.draw(7, "q", (2, 8, 256), "f32")
    k = synth.draw(7, "k", (2, 200, 256), "f16")
    v = synth.draw(7, "v", (2, 200, 256), "f16")
    want = oracle.attention(q, k.reshape(-1, 256), v.reshape(-1, 256), np.array([199, 89]), np.array([0, 200]),
                            q_dtype="f32", kv_dtype="f16")
    assert np.max(np.abs(merged - want)) <= 2e-6         # records travel as float32


def test_single_rank_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
