"""GPU parity of attn_append_kv (K/V append with RoPE) against oracle/rope.py:
the bytes written into the cache must be identical (byte work, so bit-exact),
rows outside the destinations untouched, out-of-range device destinations
skipped and recorded; and a prefill over a cache filled by the append equals
the oracle's attention over the oracle-appended cache."""
import numpy as np
import pytest
import torch

import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth
from oracle import rope
from tests.helpers import dev, max_err, oracle_prefill, oracle_threads, tol

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(cuda_ok):
    oracle_threads()
    kca.lib()


def _bytes(t):
    return t.cpu().contiguous().view(torch.uint8).numpy()


def _stored_bytes(arr):
    return np.ascontiguousarray(arr).view(np.uint8)


def _random_tables(seed, n):
    # unrelated cos and sin per element, so that any mix-up of halves shows
    cos = synth.normal(seed, "cos", (n, 256), 1.0)
    sin = synth.normal(seed, "sin", (n, 256), 1.0)
    return cos, sin


@pytest.mark.parametrize("in_dt,kv_dt", [("f32", "f32"), ("f32", "f16"), ("f32", "bf16"), ("f16", "f16"),
                                         ("bf16", "bf16"), ("bf16", "f32"), ("f16", "bf16")])
@pytest.mark.parametrize("rotate", [True, False])
def test_append_contiguous_rows_is_bit_exact(in_dt, kv_dt, rotate):
    n, rows, dst0 = 37, 100, 41
    k_new = synth.draw(1, "kn", (n, 256), in_dt, 3.0)
    v_new = synth.draw(1, "vn", (n, 256), in_dt, 3.0)
    k_cache = synth.draw(1, "kc", (rows, 256), kv_dt)
    v_cache = synth.draw(1, "vc", (rows, 256), kv_dt)
    cos, sin = _random_tables(2, n) if rotate else (None, None)
    kd, vd = dev(k_cache, kv_dt), dev(v_cache, kv_dt)
    kca.attn_append_kv(dev(k_new, in_dt), dev(v_new, in_dt), kd, vd, dst0,
                       rope_cos=torch.from_numpy(cos).cuda() if rotate else None,
                       rope_sin=torch.from_numpy(sin).cuda() if rotate else None)
    want_k, want_v = rope.append_kv(k_new, v_new, in_dt, cos, sin, k_cache, v_cache, kv_dt,
                                    np.arange(dst0, dst0 + n))
    assert np.array_equal(_bytes(kd), _stored_bytes(want_k))
    assert np.array_equal(_bytes(vd), _stored_bytes(want_v))


@pytest.mark.parametrize("kv_dt", ["f16", "bf16"])
def test_append_device_destinations_in_a_batched_cache(kv_dt):
    batch, cap = 4, 300
    ctx = [17, 299, 1, 150]                      # one decode row per sequence at ctx - 1
    dst = np.array([b * cap + c - 1 for b, c in enumerate(ctx)], dtype=np.int64)
    k_new = synth.draw(3, "kn", (batch, 256), "f32")
    v_new = synth.draw(3, "vn", (batch, 256), "f32")
    k_cache = synth.draw(3, "kc", (batch * cap, 256), kv_dt)
    v_cache = synth.draw(3, "vc", (batch * cap, 256), kv_dt)
    cos, sin = rope.rope_tables(np.array(ctx) - 1)
    kd, vd = dev(k_cache, kv_dt), dev(v_cache, kv_dt)
    kca.attn_append_kv(dev(k_new, "f32"), dev(v_new, "f32"), kd, vd, torch.from_numpy(dst).cuda(),
                       rope_cos=torch.from_numpy(cos).cuda(), rope_sin=torch.from_numpy(sin).cuda())
    want_k, want_v = rope.append_kv(k_new, v_new, "f32", cos, sin, k_cache, v_cache, kv_dt, dst)
    assert np.array_equal(_bytes(kd), _stored_bytes(want_k))
    assert np.array_equal(_bytes(vd), _stored_bytes(want_v))


def test_append_out_of_range_destination_is_skipped_and_recorded():
    rows = 64
    dst = np.array([5, rows, -3, 63], dtype=np.int64)
    k_new = synth.draw(4, "kn", (4, 256), "bf16")
    v_new = synth.draw(4, "vn", (4, 256), "bf16")
    k_cache = synth.draw(4, "kc", (rows, 256), "bf16")
    v_cache = synth.draw(4, "vc", (rows, 256), "bf16")
    kd, vd = dev(k_cache, "bf16"), dev(v_cache, "bf16")
    ws = kca.new_workspace(kca.WORKSPACE_HEADER)
    kca.attn_append_kv(dev(k_new, "bf16"), dev(v_new, "bf16"), kd, vd, torch.from_numpy(dst).cuda(),
                       workspace=ws)
    st, detail = kca.attn_device_status(ws)
    assert st == -8 and detail >> 24 == 11 and (detail & 0xffffff) in (1, 2)
    want_k, want_v = rope.append_kv(k_new, v_new, "bf16", None, None, k_cache, v_cache, "bf16", dst)
    assert np.array_equal(_bytes(kd), _stored_bytes(want_k))
    assert np.array_equal(_bytes(vd), _stored_bytes(want_v))


def test_prefill_over_an_appended_cache_matches_the_oracle():
    # A 300-row prompt appended in two chunks (RoPE at absolute positions),
    # then the second chunk's prefill, against the oracle on the oracle's cache.
    cap, first, second = 512, 200, 100
    q = synth.draw(5, "q", (second, 8, 256), "bf16")
    k_new = synth.draw(5, "kn", (first + second, 256), "bf16")
    v_new = synth.draw(5, "vn", (first + second, 256), "bf16")
    cos, sin = rope.rope_tables(np.arange(first + second))
    zero = np.zeros((cap, 256), np.uint16)
    kd, vd = dev(zero, "bf16"), dev(zero, "bf16")
    kn, vn = dev(k_new, "bf16"), dev(v_new, "bf16")
    ct, st = torch.from_numpy(cos).cuda(), torch.from_numpy(sin).cuda()
    for a, b in ((0, first), (first, first + second)):
        kca.attn_append_kv(kn[a:b], vn[a:b], kd, vd, a, rope_cos=ct[a:b], rope_sin=st[a:b])
    k_or, v_or = rope.append_kv(k_new, v_new, "bf16", cos, sin, zero, zero, "bf16", np.arange(first + second))
    assert np.array_equal(_bytes(kd), _stored_bytes(k_or))
    out = kca.attn_prefill(dev(q, "bf16"), kd, vd, first)
    want = oracle_prefill(q, k_or, v_or, first, np.arange(second), 0, "bf16", "bf16")
    assert max_err(out.cpu().numpy(), want) <= tol("bf16", "bf16")
