"""Boundary tests that need no GPU: the library loads, exports every symbol
include/kca.h declares, rejects bad arguments on the host before any CUDA
call, and its integer plans cover exactly the visible keys of every row
(J(pos) compared bit-exact with the oracle's definition)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import kv_cache_attention_states_b200 as kca

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kca.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert "attn_prefill" in names and "attn_decode" in names
    lib = kca.lib()
    for n in names:
        assert hasattr(lib, n), n


def test_every_declared_call_cites_its_passage():
    """Each declaration in kca.h sits under a comment that names the passage
    of the pages it answers to (or says that the pages have none)."""
    text = open(HEADER).read()
    blocks = [(m.start(), m.end(), m.group(0)) for m in re.finditer(r"/\*.*?\*/", text, flags=re.S)]
    code = re.sub(r"/\*.*?\*/", lambda m: " " * len(m.group(0)), text, flags=re.S)
    seen = set()
    for m in re.finditer(r"\b(attn_\w+)\s*\(", code):
        name = m.group(1)
        if name in seen:
            continue
        seen.add(name)
        before = [b for b in blocks if b[1] <= m.start()]
        assert before, name
        comment = before[-1][2]
        assert "Passage:" in comment or "no counterpart" in comment, name
    assert len(seen) == len(_declared())


def test_force_path_validates_and_restores():
    lib = kca.lib()
    assert lib.attn_force_path(3, 0) == -4 and lib.attn_force_path(0, 3) == -4 and lib.attn_force_path(1, 2) == -4
    assert lib.attn_force_path(2, 0) == 0 and lib.attn_force_path(2, -1) == 0   # op 2: the multi-row kernels
    assert lib.attn_force_path(-1, 0) == -4 and lib.attn_force_path(1, -2) == -4
    assert kca.attn_prefill_path(kca.BF16, kca.BF16, 0, 768) == 1
    with kca.forced_path(kca.OP_PREFILL, kca.PATH_ROWS):
        assert kca.attn_prefill_path(kca.BF16, kca.BF16, 0, 768) == 0
    assert kca.attn_prefill_path(kca.BF16, kca.BF16, 0, 768) == 1
    with kca.forced_path(kca.OP_PREFILL, kca.PATH_TENSOR_CORE):   # where eligible only
        assert kca.attn_prefill_path(kca.BF16, kca.BF16, 1000, 2) == 1
        assert kca.attn_prefill_path(kca.F32, kca.F32, 0, 768) == 0


def test_static_scratch_query_rejects_a_null_pointer():
    assert kca.lib().attn_decode_static_scratch(None, None) == -1


def test_header_constants_match_binding():
    text = open(HEADER).read()
    for name, val in [("KCA_MAX_CHUNK_ROWS", 768), ("KCA_MAX_POSITION", 131072),
                      ("KCA_HEAD_DIM", 256), ("KCA_N_Q_HEADS", 8), ("KCA_N_KV_HEADS", 1),
                      ("KCA_WORKSPACE_HEADER", 24832), ("KCA_MAX_BATCH", 256),
                      ("KCA_MAX_BATCH_ROWS", 15), ("KCA_I8", 3), ("KCA_I8_ROW_BYTES", 272)]:
        assert re.search(rf"#define {name} {val}\b", text), name


def test_status_strings():
    for code in range(0, -9, -1):
        assert kca.status_string(code)
    assert kca.status_string(-99) == "unknown status"


P = 0x10000  # a 16-byte aligned fake device address; validation fails before any use
KEY_TILE = 128  # keys per tensor-core KV tile (kca_plan.h)


def _prefill(**kw):
    a = dict(q=P, qd=kca.BF16, k=P, v=P, kd=kca.BF16, hq=8, hkv=1, d=256, cap=4096, cs=0, rows=768,
             ctx=768, window=0, scale=0.0625, out=P, ws=P * 2, wsb=1 << 30, stream=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return kca.lib().attn_prefill(vp(a["q"]), a["qd"], vp(a["k"]), vp(a["v"]), a["kd"], a["hq"],
                                  a["hkv"], a["d"], a["cap"], a["cs"], a["rows"], a["ctx"],
                                  a["window"], a["scale"], vp(a["out"]), vp(a["ws"]), a["wsb"],
                                  a["stream"])


def _decode(ctx=(100, 200), **kw):
    a = dict(q=P, qd=kca.F32, k=P, v=P, kd=kca.F16, hq=8, hkv=1, d=256, cap=4096, window=0,
             scale=0.0625, out=P, ws=P * 2, wsb=1 << 30, batch=None)
    a.update(kw)
    arr = np.asarray(ctx, dtype=np.int64)
    batch = len(arr) if a["batch"] is None else a["batch"]
    vp = ctypes.c_void_p
    return kca.lib().attn_decode(vp(a["q"]), a["qd"], vp(a["k"]), vp(a["v"]), a["kd"], a["hq"],
                                 a["hkv"], a["d"], a["cap"], batch,
                                 arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), a["window"],
                                 a["scale"], vp(a["out"]), vp(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(k=0), -1), (dict(v=0), -1), (dict(out=0), -1), (dict(ws=0), -1),
    (dict(hq=16), -2), (dict(hkv=2), -2), (dict(d=128), -2),
    (dict(qd=7), -3), (dict(kd=-1), -3),
    (dict(rows=0, ctx=0), -4), (dict(rows=769, ctx=769), -4), (dict(cs=-1, ctx=767), -4),
    (dict(cap=0), -4), (dict(cap=131073), -4), (dict(cs=4000, ctx=4768), -4),
    (dict(ctx=767), -4), (dict(scale=float("nan")), -4), (dict(scale=float("inf")), -4),
    (dict(scale=0.0), -4), (dict(scale=-0.0625), -4),
    (dict(q=P + 8), -6), (dict(k=P + 4), -6), (dict(v=P + 2), -6), (dict(out=P + 8), -6),
    (dict(ws=P * 2 + 16), -5),
])
def test_prefill_rejects_bad_arguments_on_the_host(kw, code):
    assert _prefill(**kw) == code


@pytest.mark.parametrize("ctx,kw,code", [
    ((1, 2), dict(q=0), -1), ((1, 2), dict(hq=4), -2), ((1, 2), dict(kd=3), -3),
    ((1, 2), dict(batch=0), -4), ((1,) * 257, dict(), -4), ((1, 4097), dict(), -4),
    ((-1, 2), dict(), -4), ((1, 2), dict(cap=131073), -4), ((1, 2), dict(scale=float("nan")), -4),
    ((1, 2), dict(scale=0.0), -4),
    ((1, 2), dict(out=P + 4), -6), ((1, 2), dict(ws=P * 2 + 128), -5),
])
def test_decode_rejects_bad_arguments_on_the_host(ctx, kw, code):
    assert _decode(ctx, **kw) == code


def _prefill_batch(ctx=(100, 200), rows=3, **kw):
    a = dict(q=P, qd=kca.F32, k=P, v=P, kd=kca.F16, hq=8, hkv=1, d=256, cap=4096, window=0,
             scale=0.0625, out=P, ws=P * 2, wsb=1 << 30, batch=None)
    a.update(kw)
    arr = np.asarray(ctx, dtype=np.int64)
    batch = len(arr) if a["batch"] is None else a["batch"]
    vp = ctypes.c_void_p
    return kca.lib().attn_prefill_batch(vp(a["q"]), a["qd"], vp(a["k"]), vp(a["v"]), a["kd"], a["hq"],
                                        a["hkv"], a["d"], a["cap"], batch, rows,
                                        arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), a["window"],
                                        a["scale"], vp(a["out"]), vp(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("ctx,rows,kw,code", [
    ((3, 9), 3, dict(q=0), -1), ((3, 9), 3, dict(ws=0), -1), ((3, 9), 3, dict(hkv=2), -2),
    ((3, 9), 3, dict(qd=9), -3), ((3, 9), 0, dict(), -4), ((16, 20), 16, dict(), -4),
    ((2, 9), 3, dict(), -4), ((3, 4097), 3, dict(), -4), ((3, 9), 3, dict(batch=0), -4),
    ((3,) * 257, 3, dict(), -4), ((3, 9), 3, dict(scale=0.0), -4), ((3, 9), 3, dict(cap=131073), -4),
    ((3, 9), 3, dict(v=P + 8), -6), ((3, 9), 3, dict(ws=P * 2 + 64), -5),
])
def test_prefill_batch_rejects_bad_arguments_on_the_host(ctx, rows, kw, code):
    assert _prefill_batch(ctx, rows, **kw) == code


def _decode_q8(ctx=(100, 200), **kw):
    a = dict(q=P, qd=kca.F32, k=P, v=P, vd=kca.F16, hq=8, hkv=1, d=256, cap=4096, window=0,
             scale=0.0625, out=P, ws=P * 2, wsb=1 << 30, batch=None)
    a.update(kw)
    arr = np.asarray(ctx, dtype=np.int64)
    batch = len(arr) if a["batch"] is None else a["batch"]
    vp = ctypes.c_void_p
    return kca.lib().attn_decode_q8(vp(a["q"]), a["qd"], vp(a["k"]), vp(a["v"]), a["vd"], a["hq"], a["hkv"],
                                    a["d"], a["cap"], batch, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                    a["window"], a["scale"], vp(a["out"]), vp(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("ctx,kw,code", [
    ((1, 2), dict(k=0), -1), ((1, 2), dict(ws=0), -1), ((1, 2), dict(hq=4), -2),
    ((1, 2), dict(vd=3), -3), ((1, 2), dict(qd=3), -3), ((1, 4097), dict(), -4), ((1, 2), dict(batch=0), -4),
    ((1, 2), dict(scale=float("nan")), -4), ((1, 2), dict(k=P + 8), -6), ((1, 2), dict(ws=P * 2 + 32), -5),
])
def test_decode_q8_rejects_bad_arguments_on_the_host(ctx, kw, code):
    assert _decode_q8(ctx, **kw) == code


def test_quantize_k_rejects_bad_arguments_on_the_host():
    lib = kca.lib()
    vp = ctypes.c_void_p
    assert lib.attn_quantize_k(None, kca.F32, 4, vp(P), None) == -1
    assert lib.attn_quantize_k(vp(P), 3, 4, vp(P), None) == -3
    assert lib.attn_quantize_k(vp(P), kca.F16, 0, vp(P), None) == -4
    assert lib.attn_quantize_k(vp(P), kca.F16, 4, vp(P + 4), None) == -6
    assert lib.attn_dot_canary(None, None) == -1


def test_prefill_batch_workspace_query_rejects_bad_arguments():
    lib = kca.lib()
    arr = np.asarray([3, 9], dtype=np.int64)
    ptr = arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
    assert lib.attn_prefill_batch_workspace_bytes(2, 4, ptr, 0) == 0      # ctx 3 < 4 rows
    assert lib.attn_prefill_batch_workspace_bytes(2, 16, ptr, 0) == 0
    assert lib.attn_prefill_batch_workspace_bytes(2, 3, None, 0) == 0


def _decode_static(ctx=(100, 200), **kw):
    a = dict(q=P, qd=kca.F32, k=P, v=P, kd=kca.F16, hq=8, hkv=1, d=256, cap=4096, window=0,
             scale=0.0625, out=P, batch=None)
    a.update(kw)
    arr = np.asarray(ctx, dtype=np.int64)
    batch = len(arr) if a["batch"] is None else a["batch"]
    vp = ctypes.c_void_p
    return kca.lib().attn_decode_static(vp(a["q"]), a["qd"], vp(a["k"]), vp(a["v"]), a["kd"], a["hq"],
                                        a["hkv"], a["d"], a["cap"], batch,
                                        arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), a["window"],
                                        a["scale"], vp(a["out"]), None)


@pytest.mark.parametrize("ctx,kw,code", [
    ((1, 2), dict(q=0), -1), ((1, 2), dict(out=0), -1), ((1, 2), dict(hq=4), -2), ((1, 2), dict(kd=3), -3),
    ((1, 2), dict(batch=0), -4), ((1,) * 257, dict(), -4), ((1, 4097), dict(), -4),
    ((1, 2), dict(scale=0.0), -4), ((1, 2), dict(out=P + 4), -6),
])
def test_decode_static_rejects_bad_arguments_before_any_device_call(ctx, kw, code):
    # the checks run before the scratch array's address is looked up, so
    # they answer even on a machine without a GPU
    assert _decode_static(ctx, **kw) == code


def _decode_dev(**kw):
    a = dict(q=P, qd=kca.F32, k=P, v=P, kd=kca.F16, hq=8, hkv=1, d=256, cap=4096, batch=2, ctx=P * 3,
             bound=4096, window=0, scale=0.0625, out=P, ws=P * 2, wsb=1 << 30)
    a.update(kw)
    vp = ctypes.c_void_p
    return kca.lib().attn_decode_dev(vp(a["q"]), a["qd"], vp(a["k"]), vp(a["v"]), a["kd"], a["hq"],
                                     a["hkv"], a["d"], a["cap"], a["batch"], vp(a["ctx"]), a["bound"],
                                     a["window"], a["scale"], vp(a["out"]), vp(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(ctx=0), -1), (dict(q=0), -1), (dict(hkv=2), -2), (dict(kd=5), -3),
    (dict(batch=0), -4), (dict(batch=257), -4), (dict(bound=4097), -4), (dict(bound=-1), -4),
    (dict(cap=131073, bound=1), -4), (dict(scale=0.0), -4),
    (dict(ctx=P * 3 + 4), -6), (dict(out=P + 4), -6), (dict(ws=P * 2 + 128), -5),
])
def test_decode_dev_rejects_bad_arguments_on_the_host(kw, code):
    assert _decode_dev(**kw) == code


def _decode_partial(ctx=(100, 5000), **kw):
    a = dict(q=P, qd=kca.F32, k=P, v=P, kd=kca.F16, hq=8, hkv=1, d=256, cap=4096, kb=4096, window=0,
             scale=0.0625, part=P, ws=P * 2, wsb=1 << 30, batch=None)
    a.update(kw)
    arr = np.asarray(ctx, dtype=np.int64)
    batch = len(arr) if a["batch"] is None else a["batch"]
    vp = ctypes.c_void_p
    return kca.lib().attn_decode_partial(vp(a["q"]), a["qd"], vp(a["k"]), vp(a["v"]), a["kd"], a["hq"],
                                         a["hkv"], a["d"], a["cap"], batch,
                                         arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), a["kb"],
                                         a["window"], a["scale"], vp(a["part"]), vp(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("ctx,kw,code", [
    ((1, 2), dict(part=0), -1), ((1, 2), dict(q=0), -1), ((1, 2), dict(d=64), -2), ((1, 2), dict(qd=9), -3),
    ((1, 2), dict(batch=0), -4), ((1,) * 257, dict(), -4), ((1, 131073), dict(), -4), ((-1, 2), dict(), -4),
    ((1, 2), dict(kb=-1), -4), ((1, 2), dict(cap=0), -4), ((1, 2), dict(kb=131072 - 4095), -4),
    ((1, 2), dict(scale=float("nan")), -4),
    ((1, 2), dict(part=P + 4), -6), ((1, 2), dict(k=P + 8), -6), ((1, 2), dict(ws=P * 2 + 128), -5),
])
def test_decode_partial_rejects_bad_arguments_on_the_host(ctx, kw, code):
    # ctx may lie past the shard (the rest of the context is on other ranks)
    assert _decode_partial(ctx, **kw) == code


@pytest.mark.parametrize("n,batch,stride,parts,out,code", [
    (2, 1, 2064, 0, P, -1), (2, 1, 2064, P, 0, -1), (0, 1, 2064, P, P, -4), (2, 0, 2064, P, P, -4),
    (2, 257, 1 << 20, P, P, -4), (2, 1, 2060, P, P, -4), (2, 1, 2066, P, P, -4), (2, 2, 2064, P, P, -4),
    (2, 1, 2064, P + 4, P, -6), (2, 1, 2064, P, P + 8, -6),
])
def test_merge_partials_rejects_bad_arguments_on_the_host(n, batch, stride, parts, out, code):
    vp = ctypes.c_void_p
    assert kca.lib().attn_merge_partials(n, batch, vp(parts), stride, vp(out), None) == code


def test_partial_record_layout():
    assert kca.partial_floats(3) == 3 * 8 * 258
    text = open(HEADER).read()
    assert re.search(r"#define KCA_PARTIAL_FLOATS\(batch\) \(\(size_t\)\(batch\) \* 8u \* 258u\)", text)


def _append(**kw):
    a = dict(k=P, v=P, it=kca.F32, n=4, cos=P * 3, sin=P * 4, kc=P * 5, vc=P * 6, kt=kca.F16, rows=100,
             dst=None, dst0=0, ws=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return kca.lib().attn_append_kv(vp(a["k"]), vp(a["v"]), a["it"], a["n"], vp(a["cos"]), vp(a["sin"]),
                                    vp(a["kc"]), vp(a["vc"]), a["kt"], a["rows"], vp(a["dst"]),
                                    a["dst0"], vp(a["ws"]), None)


@pytest.mark.parametrize("kw,code", [
    (dict(k=0), -1), (dict(vc=0), -1), (dict(cos=0), -1), (dict(sin=0), -1),
    (dict(it=3), -3), (dict(kt=-1), -3),
    (dict(n=0), -4), (dict(rows=0), -4), (dict(dst0=-1), -4), (dict(dst0=97), -4),
    (dict(k=P + 8), -6), (dict(kc=P * 5 + 2), -6), (dict(cos=P * 3 + 4), -6), (dict(dst=P * 7 + 4), -6),
])
def test_append_rejects_bad_arguments_on_the_host(kw, code):
    assert _append(**kw) == code


def _check_rows_plan(items, units, pos_of, window):
    """Every unit's items tile its visible range exactly, in order, slots unique."""
    slots = [int(s) for s in items[:, 3] if s >= 0]
    assert len(slots) == len(set(slots))
    for u in range(units):
        its = items[items[:, 0] == u]
        assert len(its) >= 1
        lo, hi = oracle.visible_range(pos_of(u), window)
        if hi < lo:
            assert len(its) == 1 and its[0, 1] == its[0, 2]
            continue
        assert its[0, 1] == lo and its[-1, 2] == hi + 1
        assert (its[1:, 1] == its[:-1, 2]).all()
        assert (its[:, 2] > its[:, 1]).all()
        if len(its) == 1:
            assert its[0, 3] == -1
        else:
            assert (its[:, 3] >= 0).all()


@pytest.mark.parametrize("cs,rows,window", [(0, 48, 0), (256, 48, 0), (1000, 15, 0), (5, 9, 3),
                                            (4090, 7, 512), (130000, 1, 0), (0, 1, 1)])
def test_prefill_rows_plan_covers_visible_keys(cs, rows, window):
    path, items = kca.attn_prefill_plan(kca.F32, kca.F32, cs, rows, window, num_sms=148)
    assert path == 0
    _check_rows_plan(items, rows, lambda u: cs + u, window)


@pytest.mark.parametrize("ctx,window", [([305], 0), ([16384], 0), ([0, 1, 2], 0), ([4097], 512),
                                        ([131072] * 8, 0), ([1024, 99999, 5, 131072], 300)])
def test_decode_plan_covers_visible_keys(ctx, window):
    for sms in (1, 7, 148):
        items = kca.attn_decode_plan(ctx, window, num_sms=sms)
        _check_rows_plan(items, len(ctx), lambda u: ctx[u] - 1, window)


def test_decode_plan_fills_one_wave():
    items = kca.attn_decode_plan([16384], 0, num_sms=148)
    assert 130 <= len(items) <= 148
    rng = np.random.default_rng(0)
    ctx = rng.integers(1024, 131041, size=8)
    items = kca.attn_decode_plan(ctx, 0, num_sms=148)
    assert len(items) <= 148


@pytest.mark.parametrize("cs,rows,window", [(0, 768, 0), (15360, 768, 0), (16128, 256, 0),
                                            (256, 48, 0), (3840, 256, 512), (130304, 768, 0),
                                            (1000, 17, 0), (7, 16, 5), (100, 200, 64),
                                            (2000, 768, 1)])
def test_prefill_tc_plan_covers_every_visible_key(cs, rows, window):
    _check_tc_plan(cs, rows, window, 148)


def _check_tc_plan(cs, rows, window, sms):
    path, items = kca.attn_prefill_plan(kca.BF16, kca.BF16, cs, rows, window, num_sms=sms)
    assert path == 1
    assert len(items) <= 2 * 80                  # the launch's item table: 80 CTA pairs
    if (rows + 31) // 32 <= sms // 2:
        assert len(items) <= 2 * (sms // 2)      # one wave of CTA pairs whenever the row tiles fit one
    kv_lo = oracle.visible_range(cs, window)[0]
    ctx = cs + rows
    n_tiles = (rows + 15) // 16
    slots = [int(s) for s in items[:, 3] if s >= 0]
    assert len(slots) == len(set(slots))
    for t in range(n_tiles):
        its = items[items[:, 0] == t]
        assert len(its) >= 1
        # items of a tile are contiguous, tile-aligned relative to kv_lo, within [kv_lo, ctx)
        assert (its[1:, 1] == its[:-1, 2]).all()
        assert ((its[:, 1] - kv_lo) % KEY_TILE == 0).all()
        assert its[0, 1] >= kv_lo and its[-1, 2] <= ctx
        covered = (int(its[0, 1]), int(its[-1, 2]))
        for r in range(16 * t, min(16 * t + 16, rows)):
            lo, hi = oracle.visible_range(cs + r, window)
            assert covered[0] <= lo and hi < covered[1]
        # tiles go in pairs (2q, 2q+1) that share their items: the first item
        # starts in the key tile of the pair's first row's lo
        lo0 = oracle.visible_range(cs + 16 * (t - t % 2), window)[0]
        assert covered[0] == kv_lo + (lo0 - kv_lo) // KEY_TILE * KEY_TILE
        if t % 2 == 1:
            assert np.array_equal(its[:, 1:3], items[items[:, 0] == t - 1][:, 1:3])
        assert (len(its) == 1) == (its[0, 3] == -1)


def test_small_chunks_and_f32_take_the_rows_path():
    assert kca.attn_prefill_path(kca.BF16, kca.BF16, 100, 15) == 0
    assert kca.attn_prefill_path(kca.BF16, kca.BF16, 100, 16) == 1
    assert kca.attn_prefill_path(kca.F32, kca.F32, 100, 768) == 0
    assert kca.attn_prefill_path(kca.F16, kca.BF16, 100, 768) == 0


def test_few_row_chunks_on_long_contexts_take_the_tensor_core_path():
    # 3-15 rows whose first row sees >= 12,288 keys: one pass over the keys
    assert kca.attn_prefill_path(kca.BF16, kca.BF16, 16381, 3) == 1
    assert kca.attn_prefill_path(kca.F16, kca.F16, 12287, 15) == 1
    assert kca.attn_prefill_path(kca.BF16, kca.BF16, 12287, 3) == 1
    assert kca.attn_prefill_path(kca.BF16, kca.BF16, 12286, 3) == 0
    assert kca.attn_prefill_path(kca.BF16, kca.BF16, 16381, 3, 4096) == 0   # window: 4096 keys
    assert kca.attn_prefill_path(kca.F32, kca.F32, 16381, 3) == 0
    # the other 2-15-row chunks on a 16-bit cache from 12,288 keys: multi-row units
    assert kca.attn_prefill_path(kca.BF16, kca.BF16, 16382, 2) == 2
    assert kca.attn_prefill_path(kca.F32, kca.BF16, 16381, 3) == 2
    assert kca.attn_prefill_path(kca.F32, kca.F16, 12287, 15) == 2
    assert kca.attn_prefill_path(kca.F32, kca.F16, 12286, 15) == 0
    assert kca.attn_prefill_path(kca.F32, kca.BF16, 16368, 16) == 0     # 16 rows: one unit per row
    assert kca.attn_prefill_path(kca.F32, kca.BF16, 16381, 3, 4096) == 0
    with kca.forced_path(kca.OP_PREFILL, kca.PATH_MULTI_ROW):
        assert kca.attn_prefill_path(kca.F32, kca.BF16, 10, 3) == 2
        assert kca.attn_prefill_path(kca.BF16, kca.BF16, 10, 1) == 0        # one row: not a unit of rows
        assert kca.attn_prefill_path(kca.F32, kca.F32, 16381, 3) == 0       # f32 cache: no multi-row kernel
    with kca.forced_path(kca.OP_ROWS, kca.PATH_CUDA_CORE):                  # multi-row units need the TC rows kernels
        assert kca.attn_prefill_path(kca.F32, kca.BF16, 16381, 3) == 0


@pytest.mark.parametrize("chunk_start,rows,window", [(20000, 15, 0), (20000, 3, 0), (130000, 8, 0), (50000, 6, 15000)])
def test_multi_row_plan_tiles_each_units_key_union(chunk_start, rows, window):
    # path 2 items: per unit of 4 or 8 consecutive rows, splits that tile the
    # union of the unit's visible keys exactly (the rows' lo .. the last
    # row's position), in order, one plan split length apart
    path, items = kca.attn_prefill_plan(kca.F32, kca.BF16, chunk_start, rows, window, num_sms=148)
    assert path == 2
    ur = 8 if rows > 4 else 4
    units = (rows + ur - 1) // ur
    assert sorted(set(items[:, 0].tolist())) == list(range(units))
    for u in range(units):
        it = items[items[:, 0] == u]
        first, last = chunk_start + u * ur, min(chunk_start + rows, chunk_start + (u + 1) * ur) - 1
        lo = max(0, first - window + 1) if window > 0 else 0
        assert it[0, 1] == lo and it[-1, 2] == last + 1
        assert (it[1:, 1] == it[:-1, 2]).all() and (it[:, 2] > it[:, 1]).all()
        assert it[:, 3].tolist() == (list(range(len(it))) if len(it) > 1 else [-1])


# Randomised checks of the same integer bookkeeping: any chunk, window and SM
# count gives plans that cover exactly what the definition J(pos) says.
from hypothesis import HealthCheck, given, settings, strategies as st


@settings(max_examples=400, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])
@given(rows=st.integers(16, 768), data=st.data(),
       window=st.one_of(st.just(0), st.integers(1, 40000)), sms=st.sampled_from([148, 132, 96, 20]))
def test_random_tensor_core_plans_cover_every_visible_key(rows, data, window, sms):
    cs = data.draw(st.integers(0, 131072 - rows))
    _check_tc_plan(cs, rows, window, sms)


@settings(max_examples=400, deadline=None, derandomize=True)
@given(rows=st.integers(1, 15), data=st.data(), window=st.one_of(st.just(0), st.integers(1, 40000)),
       sms=st.integers(1, 148))
def test_random_rows_plans_cover_every_visible_key(rows, data, window, sms):
    cs = data.draw(st.integers(0, 131072 - rows))
    path, items = kca.attn_prefill_plan(kca.F32, kca.F32, cs, rows, window, num_sms=sms)
    assert path == 0
    _check_rows_plan(items, rows, lambda u: cs + u, window)


@settings(max_examples=400, deadline=None, derandomize=True)
@given(ctx=st.lists(st.integers(0, 131072), min_size=1, max_size=16),
       window=st.one_of(st.just(0), st.integers(1, 40000)), sms=st.integers(1, 148))
def test_random_decode_plans_cover_every_visible_key(ctx, window, sms):
    items = kca.attn_decode_plan(ctx, window, num_sms=sms)
    _check_rows_plan(items, len(ctx), lambda u: ctx[u] - 1, window)


@settings(max_examples=300, deadline=None, derandomize=True)
@given(rows=st.integers(2, 15), data=st.data(), window=st.one_of(st.just(0), st.integers(12288, 40000)),
       sms=st.sampled_from([148, 132, 64]))
def test_random_multi_row_plans_tile_each_units_key_union(rows, data, window, sms):
    chunk_start = data.draw(st.integers(12288, 131072 - rows))
    path, items = kca.attn_prefill_plan(kca.F32, kca.BF16, chunk_start, rows, window, num_sms=sms)
    assert path == 2
    ur = 8 if rows > 4 else 4
    units = (rows + ur - 1) // ur
    assert sorted(set(items[:, 0].tolist())) == list(range(units))
    for u in range(units):
        it = items[items[:, 0] == u]
        first, last = chunk_start + u * ur, min(chunk_start + rows, chunk_start + (u + 1) * ur) - 1
        lo = oracle.visible_range(first, window)[0]
        assert it[0, 1] == lo and it[-1, 2] == last + 1
        assert (it[1:, 1] == it[:-1, 2]).all() and (it[:, 2] > it[:, 1]).all()
        assert it[:, 3].tolist() == (list(range(len(it))) if len(it) > 1 else [-1])
