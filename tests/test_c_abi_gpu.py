"""The library from a plain C program on the GPU: tests/c_abi_gpu_client.c,
compiled with gcc against include/kca.h and the CUDA runtime and linked to
the in-tree libkca.so, runs a bf16 chunked prefill and an f32-query / f16
decode batch on inputs this test draws (synth) and writes to files; its
outputs are compared with the oracle at the usual tolerance."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import kv_cache_attention_states_b200 as kca
from kv_cache_attention_states_b200 import synth

from tests.helpers import max_err, oracle_decode, oracle_prefill, oracle_threads, tol

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def test_c_client_prefill_and_decode_match_the_oracle(cuda_ok, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    lib_dir = os.path.dirname(kca.LIB_PATH)
    exe = str(tmp_path / "client")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-O1", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c_abi_gpu_client.c"),
                    "-L", lib_dir, "-lkca", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{lib_dir}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", exe],
                   check=True, capture_output=True, text=True)
    cs, rows, cap = 1000, 300, 1300
    q = synth.draw(21, "q", (rows, 8, 256), "bf16")
    k = synth.draw(21, "k", (cap, 256), "bf16")
    v = synth.draw(21, "v", (cap, 256), "bf16")
    dcap, ctx = 5000, [5000, 77]
    dq = synth.draw(22, "q", (2, 8, 256), "f32")
    dk = synth.draw(22, "k", (2, dcap, 256), "f16")
    dv = synth.draw(22, "v", (2, dcap, 256), "f16")
    for name, arr in (("q", q), ("k", k), ("v", v), ("dq", dq), ("dk", dk), ("dv", dv)):
        np.ascontiguousarray(arr).tofile(str(tmp_path / f"{name}.bin"))
    r = subprocess.run([exe, str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("done")
    oracle_threads()
    got = np.fromfile(str(tmp_path / "out_prefill.bin"), dtype=np.float32).reshape(rows, 8, 256)
    want = oracle_prefill(q, k, v, cs, np.arange(rows), 0, "bf16", "bf16")
    assert max_err(got, want) <= tol("bf16", "bf16")
    got = np.fromfile(str(tmp_path / "out_decode.bin"), dtype=np.float32).reshape(2, 8, 256)
    want = oracle_decode(dq, dk, dv, ctx, 0, "f32", "f16", dcap)
    assert max_err(got, want) <= tol("f32", "f16")
