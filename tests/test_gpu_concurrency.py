"""Calls with their own workspaces and outputs are independent: prefill and
decode issued on two streams at once, and from two host threads at once,
give the same bits as the same calls one after the other (the library keeps
no per-call device state; its host caches are per thread or idempotent)."""
import threading

import pytest
import torch

import kv_cache_attention_states_b200 as kca

pytestmark = pytest.mark.gpu


def _inputs():
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    cap = 6000
    kp = (torch.randn((cap, 256), generator=g, device="cuda") * 0.5).bfloat16()
    vp = (torch.randn((cap, 256), generator=g, device="cuda") * 0.5).bfloat16()
    qp = (torch.randn((300, 8, 256), generator=g, device="cuda") * 0.5).bfloat16()
    kd = torch.randn((3, cap, 256), generator=g, device="cuda").half()
    vd = torch.randn((3, cap, 256), generator=g, device="cuda").half()
    qd = torch.randn((3, 8, 256), generator=g, device="cuda")
    return (qp, kp, vp), (qd, kd, vd)


def _prefill(args, stream=None):
    qp, kp, vp = args
    cs = 5000
    ws = kca.new_workspace(kca.attn_prefill_workspace_bytes(kca.BF16, kca.BF16, cs, qp.shape[0]), stream=stream)
    out = torch.empty((qp.shape[0], 8, 256), dtype=torch.float32, device="cuda")
    kca.attn_prefill(qp, kp, vp, cs, out=out, workspace=ws, stream=stream)
    return out, ws


def _decode(args, stream=None):
    qd, kd, vd = args
    ctx = [5999, 17, 4000]
    ws = kca.new_workspace(kca.attn_decode_workspace_bytes(ctx), stream=stream)
    out = torch.empty((3, 8, 256), dtype=torch.float32, device="cuda")
    kca.attn_decode(qd, kd, vd, ctx, out=out, workspace=ws, stream=stream)
    return out, ws


def test_two_streams_match_sequential(cuda_ok):
    pa, da = _inputs()
    want_p, _ = _prefill(pa)
    want_d, _ = _decode(da)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    got = []
    for _ in range(3):
        p, wsp = _prefill(pa, s1)
        d, wsd = _decode(da, s2)
        got.append((p, d, wsp, wsd, s1, s2))
    torch.cuda.synchronize()
    for p, d, wsp, wsd, a, b in got:
        assert torch.equal(p, want_p) and torch.equal(d, want_d)
        assert kca.attn_device_status(wsp, a)[0] == 0 and kca.attn_device_status(wsd, b)[0] == 0


def test_two_host_threads_match_sequential(cuda_ok):
    pa, da = _inputs()
    want_p, _ = _prefill(pa)
    want_d, _ = _decode(da)
    torch.cuda.synchronize()
    results, errors = {}, []

    def worker(name, fn, args):
        try:
            torch.cuda.set_device(0)
            s = torch.cuda.Stream()
            outs = []
            with torch.cuda.stream(s):
                for _ in range(20):
                    outs.append(fn(args, s)[0])
            s.synchronize()
            results[name] = outs
        except Exception as e:  # reported below
            errors.append(repr(e))

    th = [threading.Thread(target=worker, args=("p", _prefill, pa)),
          threading.Thread(target=worker, args=("d", _decode, da))]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=300)
    assert not errors, errors
    assert all(torch.equal(o, want_p) for o in results["p"])
    assert all(torch.equal(o, want_d) for o in results["d"])
