"""Seeded synthetic inputs for states-form KV-cache attention.

This module holds no attention arithmetic: it only draws random numbers,
rounds them to the stored element type, and describes the workloads (shapes,
positions, chunking).  Both the oracle-side tests and the CUDA-side tests and
bench draw their inputs from here, so the two sides see identical bytes.

Random streams: numpy's PCG64 seeded by SeedSequence(seed, spawn_key=(tag,)),
where tag is the CRC-32 of a stream name ("q", "k", "v", ...), so every tensor
has its own reproducible stream and the draw order does not matter.  Normal
variates come from numpy's standard_normal in float32; f16 rounding is
numpy's float32->float16 (round to nearest even), bf16 rounding is torch's
float32->bfloat16 on the CPU (round to nearest even); bf16 arrays are carried
as their uint16 bit patterns.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np

DTYPES = ("f32", "f16", "bf16")
N_Q_HEADS = 8
N_KV_HEADS = 1
HEAD_DIM = 256
SCALE = 1.0 / 16.0          # 1/sqrt(head_dim)
MAX_CHUNK = 768
MAX_POSITION = 131072


def _rng(seed: int, tag: str) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=int(seed), spawn_key=(zlib.crc32(tag.encode()),))
    return np.random.Generator(np.random.PCG64(ss))


def normal(seed: int, tag: str, shape, std: float = 1.0) -> np.ndarray:
    """i.i.d. N(0, std^2) float32 of the given shape from stream `tag`."""
    x = _rng(seed, tag).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def integers(seed: int, tag: str, lo: int, hi: int, n: int) -> np.ndarray:
    """n integers drawn uniformly from the closed range [lo, hi]."""
    return _rng(seed, tag).integers(lo, hi + 1, size=n, dtype=np.int64)


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the stored element type (bf16 -> uint16 bits)."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f16":
        return np.ascontiguousarray(x.astype(np.float16))
    if dtype == "bf16":
        import torch
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    raise ValueError(dtype)


def draw(seed: int, tag: str, shape, dtype: str, std: float = 1.0) -> np.ndarray:
    return to_storage(normal(seed, tag, shape, std), dtype)


def torch_dtype(dtype: str):
    import torch
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]


def as_torch(arr: np.ndarray, dtype: str):
    """Host torch tensor with the same bytes (bf16 bit patterns reinterpreted)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(arr))
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t


# --------------------------------------------------------------------------
# Workload descriptions (shapes, positions, chunking, dtypes, value scales).
# --------------------------------------------------------------------------

def chunks(n_rows: int, chunk: int = MAX_CHUNK, start: int = 0):
    """(chunk_start, chunk_rows) pairs covering [start, start+n_rows)."""
    out = []
    p = start
    while p < start + n_rows:
        r = min(chunk, start + n_rows - p)
        out.append((p, r))
        p += r
    return out


@dataclass
class Workload:
    name: str
    description: str
    kv_dtype: str
    q_dtype: str
    capacity: int
    std: float = 1.0
    window: int = 0
    prefill: list = field(default_factory=list)         # [(chunk_start, rows)]
    decode_ctx: list = field(default_factory=list)      # per decode step: [ctx_len per seq]
    batch: int = 1
    prefill_q_dtype: str | None = None


def tiny_f32() -> Workload:
    return Workload(
        name="tiny_f32",
        description="1 seq, f32 Q/K/V N(0,1); prefill 48 rows at positions 256-303, "
                    "then 16 decode steps at positions 304-319",
        kv_dtype="f32", q_dtype="f32", capacity=320,
        prefill=[(256, 48)], decode_ctx=[[305 + t] for t in range(16)])


def decode_f16(length: int, steps: int = 64) -> Workload:
    return Workload(
        name=f"decode_f16_{length}",
        description=f"1 seq decode, f16 K/V N(0,1), f32 q N(0,1); {steps} steps, "
                    f"step t attends ctx {length}+t",
        kv_dtype="f16", q_dtype="f32", capacity=length + steps,
        decode_ctx=[[length + t] for t in range(steps)])


def prefill_bf16_16k() -> Workload:
    return Workload(
        name="prefill_bf16_16k",
        description="16384-token prompt in 768-row chunks (21 x 768 + 256), bf16 Q/K/V "
                    "N(0,1)*0.5, causal",
        kv_dtype="bf16", q_dtype="bf16", capacity=16384, std=0.5,
        prefill=chunks(16384))


def window_bf16(steps: int = 64) -> Workload:
    return Workload(
        name="window_bf16",
        description="window 512, bf16 Q/K/V N(0,1); 4096-token prompt in 768-row chunks, "
                    f"then {steps} decode steps at positions 4096-{4096 + steps - 1}",
        kv_dtype="bf16", q_dtype="bf16", capacity=4096 + steps, window=512,
        prefill=chunks(4096), decode_ctx=[[4097 + t] for t in range(steps)])


def ragged_ctx(seed: int, batch: int = 8, steps: int = 32) -> np.ndarray:
    """Per-sequence starting context, uniform on [1024, MAX_POSITION - steps + 1]
    so that every one of the `steps` appended rows still fits the capacity."""
    return integers(seed, "ragged_ctx", 1024, MAX_POSITION - steps + 1, batch)


def ragged_f16(seed: int, batch: int = 8, steps: int = 32) -> Workload:
    ctx = ragged_ctx(seed, batch, steps)
    return Workload(
        name="ragged_f16",
        description=f"{batch} seqs, ctx drawn uniformly by the seed, f16 K/V N(0,1), "
                    f"f32 q; {steps} decode steps",
        kv_dtype="f16", q_dtype="f32", capacity=MAX_POSITION, batch=batch,
        decode_ctx=[[int(c) + t for c in ctx] for t in range(steps)])


def long_chunk_bf16() -> Workload:
    return Workload(
        name="long_chunk_bf16",
        description="one 768-row bf16 chunk at positions 130304-131071 of a 131072 cache, "
                    "N(0,1)",
        kv_dtype="bf16", q_dtype="bf16", capacity=MAX_POSITION,
        prefill=[(MAX_POSITION - MAX_CHUNK, MAX_CHUNK)])
