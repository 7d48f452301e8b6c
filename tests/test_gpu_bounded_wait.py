"""Failure detection without a GPU fault: every wait in the library's kernels
is bounded (kca_common.cuh).  A harness built against that header
(tests/wait_probe.cu, wait limit shortened to 1 ms) waits on an mbarrier
nothing arrives on: the wait must give up, return false, record its site in
the status word that attn_device_status reads, and leave the context usable.
A barrier that does complete must record nothing."""
import ctypes
import os
import subprocess
import tempfile

import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "kv_cache_attention_states_b200", "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def probe(cuda_ok):
    d = tempfile.mkdtemp(prefix="kca_wait_")
    so = os.path.join(d, "libwaitprobe.so")
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-shared",
                    "-Xcompiler", "-fPIC", "-I", CSRC, "-I", INCLUDE, os.path.join(HERE, "wait_probe.cu"),
                    "-o", so], check=True, capture_output=True)
    lib = ctypes.CDLL(so)
    lib.wait_probe.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_void_p]
    lib.wait_probe.restype = ctypes.c_int
    return lib


def _run(probe, arrive, site):
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    out = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    assert probe.wait_probe(status.data_ptr(), arrive, site, out.data_ptr()) == 0
    return status.cpu().tolist(), int(out.item())


def test_a_wait_nothing_completes_gives_up_and_records_its_site(probe):
    (error, detail), ok = _run(probe, 0, 9)
    assert ok == 0
    assert error == 1                     # bit 0: a bounded wait ran out
    assert (detail >> 24) == 9 and (detail & 0xFFFFFF) == 0   # site 9, block 0
    # the context is still usable: a normal kernel and a copy run afterwards
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float((x * 2).sum().item()) == 2.0 * 1023 * 1024 / 2


def test_a_completed_wait_records_nothing(probe):
    (error, detail), ok = _run(probe, 1, 9)
    assert ok == 1 and error == 0 and detail == 0
