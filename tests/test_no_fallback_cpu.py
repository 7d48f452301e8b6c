"""The product path fails loudly instead of falling back to the CPU: a
missing library raises at load time, and host (CPU) tensors are rejected by
every call before anything runs.  (The library itself also refuses, with
KCA_ERR_CUDA, anything that needs a device it cannot find.)"""
import os
import subprocess
import sys

import pytest
import torch

import kv_cache_attention_states_b200 as kca

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_missing_library_raises_at_load():
    code = ("import kv_cache_attention_states_b200 as kca\n"
            "kca.LIB_PATH = '/nonexistent/libkca.so'\n"
            "try:\n    kca.lib()\nexcept ImportError as e:\n    print('raised', e)\n")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert r.returncode == 0 and r.stdout.startswith("raised"), r.stdout + r.stderr


def test_host_tensors_are_rejected():
    q = torch.zeros((16, 8, 256), dtype=torch.bfloat16)
    k = torch.zeros((64, 256), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        kca.attn_prefill(q, k, k, 48)
    qd = torch.zeros((1, 8, 256), dtype=torch.float32)
    kd = torch.zeros((1, 64, 256), dtype=torch.float16)
    with pytest.raises(ValueError):
        kca.attn_decode(qd, kd, kd, [10])
    with pytest.raises(ValueError):
        kca.attn_decode_dev(qd, kd, kd, torch.tensor([10]), 64)


def test_a_device_query_without_a_device_is_an_error_not_a_guess():
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    # the tensor-core decode plan depends on the device's resident-cluster
    # capacity: without a device it is refused, not approximated
    with pytest.raises(kca.KcaError):
        kca.attn_decode_plan([16384], 0, kv_dtype=kca.F16)
