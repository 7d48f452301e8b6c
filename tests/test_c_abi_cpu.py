"""The C ABI used from C: tests/c_abi_client.c, compiled with gcc against
include/kca.h alone and linked to the in-tree libkca.so, makes host-only
calls (status strings, integer plans, arguments rejected before any device
call) and prints what they return; the printed values must equal what the
Python binding gets from the same calls.  No GPU is needed."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import kv_cache_attention_states_b200 as kca

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CAP = (74, 33, 15)


def _digest(items):
    flat = [int(x) for x in np.asarray(items, dtype=np.int64).reshape(-1)]
    mix = 0
    for x in flat:
        mix = (mix * 1000003 + x) % 2147483647
    return len(flat) // 4, sum(flat), mix


@pytest.fixture(scope="module")
def client_output(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    lib_dir = os.path.dirname(kca.LIB_PATH)
    exe = str(tmp_path_factory.mktemp("cabi") / "client")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-O1", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_client.c"), "-L", lib_dir, "-lkca",
                    f"-Wl,-rpath,{lib_dir}", "-o", exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=120)
    return r.stdout.splitlines()


def _line(lines, prefix):
    got = [ln for ln in lines if ln.startswith(prefix)]
    assert len(got) == 1, prefix
    return got[0]


def _fields(line):
    return dict(tok.split("=", 1) for tok in line.split() if "=" in tok)


def test_status_strings_from_c(client_output):
    for s in range(0, -9, -1):
        assert _line(client_output, f"status {s} ") == f"status {s} {kca.status_string(s)}"


@pytest.mark.parametrize("cs,rows,window,dt", [(7680, 768, 0, kca.BF16), (3840, 256, 512, kca.BF16),
                                               (1000, 9, 0, kca.F32)])
def test_prefill_plan_from_c_equals_the_binding(client_output, cs, rows, window, dt):
    f = _fields(_line(client_output, f"prefill_plan {cs} {rows} {window} "))
    path, items = kca.attn_prefill_plan(dt, dt, cs, rows, window, num_sms=148, cluster_capacity=CAP)
    n, total, mix = _digest(items)
    assert f["st"] == "0"
    assert (int(f["n"]), int(f["extra"]), int(f["sum"]), int(f["mix"])) == (n, path, total, mix)


def test_decode_plan_from_c_equals_the_binding(client_output):
    f = _fields(_line(client_output, "decode_plan "))
    items, cluster = kca.attn_decode_plan([16384, 1000, 0, 131072], 0, num_sms=148, kv_dtype=kca.F16,
                                          cluster_capacity=CAP, with_cluster=True)
    n, total, mix = _digest(items)
    assert f["st"] == "0"
    assert (int(f["n"]), int(f["extra"]), int(f["sum"]), int(f["mix"])) == (n, cluster, total, mix)


def test_calls_rejected_on_the_host_from_c(client_output):
    code = {v: k for k, v in kca.STATUS.items()}
    want = {"prefill_null_q": "KCA_ERR_NULL", "prefill_heads": "KCA_ERR_GEOMETRY", "prefill_rows": "KCA_ERR_RANGE",
            "decode_dtype": "KCA_ERR_DTYPE", "decode_batch": "KCA_ERR_RANGE", "plan_capacity": "KCA_ERR_RANGE"}
    for name, status in want.items():
        assert _line(client_output, f"reject {name} ") == f"reject {name} {code[status]}"
