"""Benchmark of the states-form attention hot path on B200.

One step = PASSES passes over the headline workload, each pass a CUDA graph
of its C-ABI calls:

  prefill        the 16,384-token prompt in 768-row chunks (21 x 768 + 256),
                 bf16 Q/K/V ~ N(0,1)*0.5 (2 input replicas)        -> value
  decode         64 decode steps at context 16384..16447, f16 K/V, f32 q
                 (32 cache replicas)

value = prefill q-rows/s (a q-row is one query position with all 8 heads),
from CUDA events around the prefill graph of every pass; ms_per_step covers
whole steps.  Every other workload configuration is then timed the same way
in a region of its own (OTHER_PASSES passes per step, in this order, so
that each small working set follows a large one and its calls read cold
rows from HBM) and reported in its own object of the JSON line:

  decode_ragged  8 sequences, context drawn by the seed from [1024, 131072],
                 32 decode steps, f16 K/V, f32 q
  decode_256     64 decode steps at context 256..319, f16 K/V, f32 q
                 (64 cache replicas, one per step)
  decode_4096    64 decode steps at context 4096..4159 (64 replicas)
  window         window 512: a 4,096-token prompt in 768-row chunks, then 64
                 decode steps at positions 4096..4159, bf16 Q/K/V ~ N(0,1)
                 (the decode re-reads rows its previous step read: the window
                 slides by one row)
  long_chunk     one 768-row bf16 chunk at positions 130304..131071 of a
                 131,072-row cache
  prefill_batch  32 sequences x 4 query rows (speculative / multi-row decode)
                 per call through attn_prefill_batch, 16 calls, f16 K/V
  decode_q8_ragged  the ragged batch with int8 K rows (quantised-dot decode,
                 attn_decode_q8), f16 V

  python bench.py [--gpus N] [--steps K] [--warmup W] [--passes P] [--impl reference]
Under torchrun each rank runs its own replica of the workload (weak scaling,
no collective on the data path); rank 0 prints one JSON line.
"""
import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL_ROWS = 16384
DECODE_LEN = 16384
DECODE_STEPS = 64
DECODE_REPLICAS = 32
PREFILL_REPLICAS = 2
SMALL_DECODE_REPLICAS = 64
PASSES = 40              # passes over the headline step per timed step
OTHER_PASSES = 2         # passes over the other configurations per step (own region)
# DRAM bytes (read + write) per launch from one ncu capture of the current
# kernels, with the launch they come from; None once a kernel has changed
# since its capture.
TRAFFIC = {
    "prefill": (18.931e6 + 25.6e3, "prefill_tc_kernel, chunk 19 (768 rows at 14592)"),
    "decode": (16.919e6, "decode_mma_kernel, one call at ctx ~16.4K"),
    "decode_256": (402432.0, "decode_mma_kernel, one call at ctx ~256 (the whole last 64-row stage is loaded)"),
    "decode_4096": (4336384.0, "decode_mma_kernel, one call at ctx ~4.1K"),
    "decode_ragged": (459086080.0 + 3675136.0, "decode_mma_kernel, one call of the 8-sequence batch"),
    "window_prefill": (4518912.0, "prefill_tc_kernel, one 768-row chunk, window 512"),
    "window_decode": (595456.0, "decode_mma_kernel<bf16, bf16>, one call, window 512 (cold caches)"),
    "long_chunk": (138080256.0 + 4125184.0, "prefill_tc_kernel, the 768-row chunk at 130304"),
    "decode_q8_ragged": (350935296.0 + 3392512.0, "decode_mma_kernel<f32, int8 K, f16 V>, one call of the 8 sequences"),
    "prefill_batch": (301807360.0 + 525824.0, "rows_tc_kernel, one call of 32 sequences x 4 rows "
                                              "(its splits merged in-kernel)"),
}
E2E_FIRST = 2            # prefill chunks of the end-to-end leg's first host copy
E2E_GROUP = 4            # prefill chunks per host copy after it
METRIC = "prefill q-rows/s & decode tok/s at 16K ctx (1 B200); % of TC/HBM roofline"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0)) or None, \
            "measured"
    return 6650.0, 1590.0, None, "fallback"


def max_over_ranks(values, world: int, device):
    """Element-wise maximum over ranks of this rank's device-timed values
    (every rank calls it; the job is as slow as its slowest rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def visible(pos: int, window: int) -> int:
    """Keys a query at pos sees."""
    lo = max(0, pos - window + 1) if window > 0 else 0
    return pos - lo + 1


def prefill_flops(chunks, window=0) -> float:
    # 2 GEMMs (QK^T and PV) x 2 flop x head_dim x 8 heads per visible (query, key) pair
    pairs = 0
    for cs, r in chunks:
        if window <= 0:
            pairs += r * cs + r * (r + 1) // 2
        else:
            pairs += sum(visible(p, window) for p in range(cs, cs + r))
    return 4.0 * 256 * 8 * pairs


def decode_bytes(ctx: int, window: int = 0, kv_size: int = 2, q_size: int = 4) -> int:
    # K + V rows of the visible keys once, the query and the f32 output
    return visible(ctx - 1, window) * 256 * kv_size * 2 + 8 * 256 * (q_size + 4)


class Clocks:
    """SM clock and clock-event reasons sampled DURING the timed region.

    NVML (read-only queries) from a background thread every 2 ms, so that even
    a timed region of a few tens of milliseconds gets dozens of samples; the
    nvidia-smi CSV stream (20 ms) is the fallback when NVML is unavailable.
    Nothing here changes a GPU setting."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device):
        import threading
        self.samples, self.reasons, self.sm_max = [], set(), None
        self.proc = None
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(device)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            bits = [(n, getattr(pynvml, c)) for n, c in self.REASONS if hasattr(pynvml, c)]

            def poll():
                while not self._stop.is_set():
                    self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for n, b in bits:
                        if r & b:
                            self.reasons.add(n)
                    self._stop.wait(0.002)

            self.source = "nvml"
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            while not self.samples and self.thread.is_alive():
                time.sleep(0.0005)
        except Exception:  # NVML missing: nvidia-smi stream
            self.source = "nvidia-smi"
            self.thread = None
            self._start_smi(device)

    def _start_smi(self, device):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="kca_clocks_", suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        idx = device.index if hasattr(device, "index") and device.index is not None else 0
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={idx}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self._stop.set()
            self.thread.join()
        elif self.proc is not None:
            self.proc.terminate()
            self.proc.wait()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            smax = []
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    self.samples.append(float(f[1]))
                    smax.append(float(f[2]))
                except ValueError:
                    continue
                for n, val in zip(names, f[5:9]):
                    if val.lower() == "active":
                        self.reasons.add(n)
            self.sm_max = max(smax) if smax else None
            os.remove(self.path)
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        sm = self.samples
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": self.sm_max,
                "reasons": sorted(self.reasons), "samples": len(sm), "source": self.source}


# ------------------------------------------------------------- the workloads

class Workload:
    """Device-resident inputs of the headline configurations (the 16K prompt
    and the 64 decode steps at 16K) and the replicas that defeat L2."""

    def __init__(self, device, seed=0):
        import torch
        from kv_cache_attention_states_b200 import synth
        import kv_cache_attention_states_b200 as kca
        self.kca = kca
        pw = synth.prefill_bf16_16k()
        self.chunks = pw.prefill
        self.pre = []
        for r in range(PREFILL_REPLICAS):
            q = synth.draw(seed + r, "q", (PREFILL_ROWS, 8, 256), "bf16", pw.std)
            k = synth.draw(seed + r, "k", (PREFILL_ROWS, 256), "bf16", pw.std)
            v = synth.draw(seed + r, "v", (PREFILL_ROWS, 256), "bf16", pw.std)
            self.pre.append(tuple(synth.as_torch(x, "bf16").to(device) for x in (q, k, v)))
        self.pre_out = torch.empty((PREFILL_ROWS, 8, 256), dtype=torch.float32, device=device)
        self.pre_ws = kca.new_workspace(max(kca.attn_prefill_workspace_bytes(kca.BF16, kca.BF16, cs, r)
                                            for cs, r in self.chunks), device)
        dw = synth.decode_f16(DECODE_LEN, DECODE_STEPS)
        self.dec_ctx = [c[0] for c in dw.decode_ctx]
        self.cap = dw.capacity
        k = synth.draw(seed, "k", (1, self.cap, 256), "f16")
        v = synth.draw(seed, "v", (1, self.cap, 256), "f16")
        k0 = synth.as_torch(k, "f16").to(device)
        v0 = synth.as_torch(v, "f16").to(device)
        self.dec_kv = []
        for r in range(DECODE_REPLICAS):
            self.dec_kv.append((k0.clone(), v0.clone()))
        del k0, v0
        self.dec_q = synth.as_torch(synth.draw(seed, "q", (DECODE_STEPS, 1, 8, 256), "f32"), "f32").to(device)
        self.dec_out = torch.empty((DECODE_STEPS, 1, 8, 256), dtype=torch.float32, device=device)
        self.dec_ws = kca.new_workspace(max(kca.attn_decode_workspace_bytes([c]) for c in self.dec_ctx),
                                        device)
        self.step_index = 0

    def prefill(self):
        q, k, v = self.pre[self.step_index % PREFILL_REPLICAS]
        for cs, r in self.chunks:
            self.kca.attn_prefill(q[cs:cs + r], k, v, cs, out=self.pre_out[cs:cs + r],
                                  workspace=self.pre_ws)

    def decode(self):
        for t, c in enumerate(self.dec_ctx):
            k, v = self.dec_kv[(self.step_index * DECODE_STEPS + t) % DECODE_REPLICAS]
            self.kca.attn_decode(self.dec_q[t], k, v, [c], out=self.dec_out[t], workspace=self.dec_ws)


def _prefill_launches(kca, chunks, window, sms):
    n = 0
    for cs, r in chunks:
        path, items = kca.attn_prefill_plan(kca.BF16, kca.BF16, cs, r, window, sms)
        n += 1 + int(path == 1 and (items[:, 3] >= 0).any())
    return n


class Part:
    """One workload configuration of a pass: `run(variant)` issues its calls
    (captured once per variant as a CUDA graph), `units` counts its output
    rows or tokens, `work` its algorithmic flops (tensor-bound) or bytes
    (HBM-bound) per run."""
    name = ""
    unit = ""
    variants = 1
    bound = "hbm"
    units = 0
    work = 0.0
    launches = 0
    kernel = ""
    algorithmic = ""
    workload = ""

    def run(self, variant):
        raise NotImplementedError

    def status(self):
        return [ws for ws in self.workspaces()]

    def workspaces(self):
        return []


class PrefillPart(Part):
    name, unit, bound = "prefill", "q-rows", "tensor"
    kernel = "prefill_tc_kernel (+ its merge)"

    def __init__(self, w, sms):
        self.w = w
        self.variants = PREFILL_REPLICAS
        self.units = PREFILL_ROWS
        self.work = prefill_flops(w.chunks)
        self.launches = _prefill_launches(w.kca, w.chunks, 0, sms)
        self.algorithmic = "4*256*8*sum|J(pos)| = 1.0996e12 flop per prompt"

    def run(self, variant):
        self.w.step_index = variant
        self.w.prefill()

    def workspaces(self):
        return [self.w.pre_ws]


class HeadlineDecodePart(Part):
    name, unit, bound = "decode", "tok", "hbm"
    kernel = "decode_mma_kernel<f32 q, f16 KV> (merge in-kernel)"

    def __init__(self, w):
        self.w = w
        self.units = len(w.dec_ctx)
        self.work = float(sum(decode_bytes(c) for c in w.dec_ctx))
        self.launches = len(w.dec_ctx)
        self.algorithmic = "ctx*1024 B K/V + 16 KiB q/out per token"

    def run(self, variant):
        self.w.step_index = 0
        self.w.decode()

    def workspaces(self):
        return [self.w.dec_ws]


class DecodeLenPart(Part):
    """64 decode steps of one sequence at context L..L+63 (f16 K/V, f32 q),
    step t on cache replica t (the replicas together exceed the working set
    that L2 could hold between two visits)."""
    unit, bound = "tok", "hbm"
    kernel = "decode_mma_kernel<f32 q, f16 KV>"

    def __init__(self, device, length, seed=0):
        import torch
        import kv_cache_attention_states_b200 as kca
        from kv_cache_attention_states_b200 import synth
        self.kca = kca
        self.name = f"decode_{length}"
        wl = synth.decode_f16(length, DECODE_STEPS)
        self.ctx = [c[0] for c in wl.decode_ctx]
        self.cap = wl.capacity
        k0 = synth.as_torch(synth.draw(seed, "k", (1, self.cap, 256), "f16"), "f16").to(device)
        v0 = synth.as_torch(synth.draw(seed, "v", (1, self.cap, 256), "f16"), "f16").to(device)
        self.kv = [(k0, v0)] + [(k0.clone(), v0.clone()) for _ in range(SMALL_DECODE_REPLICAS - 1)]
        self.q = synth.as_torch(synth.draw(seed, "q", (DECODE_STEPS, 1, 8, 256), "f32"), "f32").to(device)
        self.out = torch.empty((DECODE_STEPS, 1, 8, 256), dtype=torch.float32, device=device)
        self.ws = kca.new_workspace(max(kca.attn_decode_workspace_bytes([c]) for c in self.ctx), device)
        self.units = DECODE_STEPS
        self.work = float(sum(decode_bytes(c) for c in self.ctx))
        self.launches = DECODE_STEPS
        self.algorithmic = "ctx*1024 B K/V + 16 KiB q/out per token"
        self.workload = (f"1 sequence, 64 decode steps at ctx {length}-{length + 63}, f16 K/V N(0,1), "
                         f"f32 q; {SMALL_DECODE_REPLICAS} cache replicas")

    def run(self, variant):
        for t, c in enumerate(self.ctx):
            k, v = self.kv[t % len(self.kv)]
            self.kca.attn_decode(self.q[t], k, v, [c], out=self.out[t], workspace=self.ws)

    def workspaces(self):
        return [self.ws]


class WindowParts:
    """The sliding-window configuration: a 4,096-token prompt in 768-row
    chunks, then 64 decode steps at positions 4096..4159, window 512, bf16."""

    def __init__(self, device, sms, seed=0):
        import torch
        import kv_cache_attention_states_b200 as kca
        from kv_cache_attention_states_b200 import synth
        self.kca = kca
        wl = synth.window_bf16(DECODE_STEPS)
        self.wl = wl
        self.cap = wl.capacity
        n = 4096
        self.k = synth.as_torch(synth.draw(seed, "k", (self.cap, 256), "bf16"), "bf16").to(device)
        self.v = synth.as_torch(synth.draw(seed, "v", (self.cap, 256), "bf16"), "bf16").to(device)
        self.q = synth.as_torch(synth.draw(seed, "q", (n, 8, 256), "bf16"), "bf16").to(device)
        self.qd = synth.as_torch(synth.draw(seed, "qd", (DECODE_STEPS, 1, 8, 256), "bf16"), "bf16").to(device)
        self.out = torch.empty((n, 8, 256), dtype=torch.float32, device=device)
        self.dout = torch.empty((DECODE_STEPS, 1, 8, 256), dtype=torch.float32, device=device)
        self.ws = kca.new_workspace(max(
            [kca.attn_prefill_workspace_bytes(kca.BF16, kca.BF16, cs, r, wl.window) for cs, r in wl.prefill]
            + [kca.attn_decode_workspace_bytes(c, wl.window) for c in wl.decode_ctx]), device)
        outer = self

        class Pre(Part):
            name, unit, bound = "window_prefill", "q-rows", "tensor"
            kernel = "prefill_tc_kernel (+ its merge), window 512"
            units = n
            work = prefill_flops(wl.prefill, wl.window)
            launches = _prefill_launches(kca, wl.prefill, wl.window, sms)
            algorithmic = "4*256*8*sum|J(pos)| with |J| <= 512 = 1.611e10 flop"

            def run(self, variant):
                for cs, r in wl.prefill:
                    kca.attn_prefill(outer.q[cs:cs + r], outer.k, outer.v, cs, wl.window,
                                     out=outer.out[cs:cs + r], workspace=outer.ws)

            def workspaces(self):
                return [outer.ws]

        class Dec(Part):
            name, unit, bound = "window_decode", "tok", "hbm"
            kernel = "decode_mma_kernel<bf16 q, bf16 KV>, window 512"
            units = DECODE_STEPS
            work = float(sum(decode_bytes(c[0], wl.window, 2, 2) for c in wl.decode_ctx))
            launches = DECODE_STEPS
            algorithmic = "512 keys x 1024 B K/V + 12 KiB q/out per token"

            def run(self, variant):
                k1, v1 = outer.k.view(1, outer.cap, 256), outer.v.view(1, outer.cap, 256)
                for t, c in enumerate(wl.decode_ctx):
                    kca.attn_decode(outer.qd[t], k1, v1, c, wl.window, out=outer.dout[t], workspace=outer.ws)

            def workspaces(self):
                return [outer.ws]

        self.parts = [Pre(), Dec()]


class LongChunkPart(Part):
    """One 768-row bf16 chunk at positions 130304..131071 of a 131,072-row cache."""
    name, unit, bound = "long_chunk", "q-rows", "tensor"
    kernel = "prefill_tc_kernel (+ its merge)"

    def __init__(self, device, sms, seed=0):
        import torch
        import kv_cache_attention_states_b200 as kca
        from kv_cache_attention_states_b200 import synth
        self.kca = kca
        wl = synth.long_chunk_bf16()
        self.cs, self.rows = wl.prefill[0]
        self.k = synth.as_torch(synth.draw(seed, "k", (wl.capacity, 256), "bf16"), "bf16").to(device)
        self.v = synth.as_torch(synth.draw(seed, "v", (wl.capacity, 256), "bf16"), "bf16").to(device)
        self.q = synth.as_torch(synth.draw(seed, "q", (self.rows, 8, 256), "bf16"), "bf16").to(device)
        self.out = torch.empty((self.rows, 8, 256), dtype=torch.float32, device=device)
        self.ws = kca.new_workspace(kca.attn_prefill_workspace_bytes(kca.BF16, kca.BF16, self.cs, self.rows),
                                    device)
        self.units = self.rows
        self.work = prefill_flops(wl.prefill)
        self.launches = _prefill_launches(kca, wl.prefill, 0, sms)
        self.algorithmic = "4*256*8*sum|J(pos)| = 8.222e11 flop"

    def run(self, variant):
        self.kca.attn_prefill(self.q, self.k, self.v, self.cs, out=self.out, workspace=self.ws)

    def workspaces(self):
        return [self.ws]


class RaggedPart(Part):
    """8 sequences with contexts drawn by the seed from [1024, 131072], 32
    decode steps, f16 K/V, f32 q; the 1.07 GB cache is far larger than L2."""
    name, unit, bound = "decode_ragged", "tok", "hbm"
    kernel = "decode_mma_kernel<f32 q, f16 KV>"

    def __init__(self, device):
        import torch
        import kv_cache_attention_states_b200 as kca
        from kv_cache_attention_states_b200 import synth
        self.kca = kca
        wl = synth.ragged_f16(0)
        self.wl = wl
        g = torch.Generator(device=device)
        g.manual_seed(1)
        self.k = torch.randn((wl.batch, wl.capacity, 256), generator=g, device=device).half()
        self.v = torch.randn((wl.batch, wl.capacity, 256), generator=g, device=device).half()
        self.q = torch.randn((len(wl.decode_ctx), wl.batch, 8, 256), generator=g, device=device)
        self.out = torch.empty_like(self.q)
        self.ws = kca.new_workspace(max(kca.attn_decode_workspace_bytes(c) for c in wl.decode_ctx), device)
        self.units = wl.batch * len(wl.decode_ctx)
        self.work = float(sum(sum(decode_bytes(x) for x in c) for c in wl.decode_ctx))
        self.launches = len(wl.decode_ctx)
        self.algorithmic = "ctx*1024 B K/V + 16 KiB q/out per token"
        self.mean_ctx = float(np.mean(wl.decode_ctx[0]))

    def run(self, variant):
        for t, c in enumerate(self.wl.decode_ctx):
            self.kca.attn_decode(self.q[t], self.k, self.v, c, out=self.out[t], workspace=self.ws)

    def workspaces(self):
        return [self.ws]


class BatchRowsPart(Part):
    """Batched short chunks (speculative or multi-row decode): 32 sequences
    with contexts drawn by the seed from [1024, 16384], 4 query rows each,
    16 calls (each advancing every sequence by 4 rows), f16 K/V, f32 q,
    through attn_prefill_batch."""
    name, unit, bound = "prefill_batch", "q-rows", "hbm"
    kernel = "rows_tc_kernel<f32 q, f16 KV> (tcgen05, splits merged in-kernel): 4 rows per unit"
    BATCH, ROWS, CALLS, CAP = 32, 4, 16, 16448

    def __init__(self, device, seed=0):
        import torch
        import kv_cache_attention_states_b200 as kca
        from kv_cache_attention_states_b200 import synth
        self.kca = kca
        ctx0 = synth.integers(seed, "batch_ctx", 1024, 16384, self.BATCH)
        self.ctx = [[int(c) + self.ROWS * t for c in ctx0] for t in range(self.CALLS)]
        g = torch.Generator(device=device)
        g.manual_seed(2)
        self.k = torch.randn((self.BATCH, self.CAP, 256), generator=g, device=device).half()
        self.v = torch.randn((self.BATCH, self.CAP, 256), generator=g, device=device).half()
        self.q = torch.randn((self.CALLS, self.BATCH, self.ROWS, 8, 256), generator=g, device=device)
        self.out = torch.empty_like(self.q)
        self.ws = kca.new_workspace(max(kca.attn_prefill_batch_workspace_bytes(c, self.ROWS) for c in self.ctx),
                                    device)
        self.units = self.BATCH * self.ROWS * self.CALLS
        # algorithmic bytes: each sequence's visible K/V rows once per call
        # (its rows share them), q and the f32 output
        self.work = float(sum(sum(c) * 1024 + self.BATCH * self.ROWS * 8 * 256 * 8 for c in self.ctx))
        self.launches = self.CALLS
        self.algorithmic = "ctx*1024 B K/V per sequence (shared by its 4 rows) + 16 KiB q/out per row"
        self.workload = ("32 sequences x 4 query rows at ctx drawn by the seed from [1024, 16384], 16 calls, "
                         "f16 K/V, f32 q (attn_prefill_batch)")

    def run(self, variant):
        for t, c in enumerate(self.ctx):
            self.kca.attn_prefill_batch(self.q[t], self.k, self.v, c, out=self.out[t], workspace=self.ws)

    def workspaces(self):
        return [self.ws]


class RaggedQ8Part(Part):
    """The ragged batch with int8 K (quantised-dot decode): K quantised per
    row by attn_quantize_k (272-byte packed rows), f16 V, f32 q, 32 steps."""
    name, unit, bound = "decode_q8_ragged", "tok", "hbm"
    kernel = "decode_mma_kernel<f32 q, int8 K, f16 V> (QK on int8 MMAs)"

    def __init__(self, device):
        import torch
        import kv_cache_attention_states_b200 as kca
        from kv_cache_attention_states_b200 import synth
        self.kca = kca
        wl = synth.ragged_f16(0)
        self.wl = wl
        g = torch.Generator(device=device)
        g.manual_seed(3)
        k = torch.randn((wl.batch, wl.capacity, 256), generator=g, device=device).half()
        self.k8 = kca.attn_quantize_k(k)
        del k
        self.v = torch.randn((wl.batch, wl.capacity, 256), generator=g, device=device).half()
        self.q = torch.randn((len(wl.decode_ctx), wl.batch, 8, 256), generator=g, device=device)
        self.out = torch.empty_like(self.q)
        self.ws = kca.new_workspace(max(kca.attn_decode_q8_workspace_bytes(c) for c in wl.decode_ctx), device)
        kca.attn_dot_canary()
        self.units = wl.batch * len(wl.decode_ctx)
        self.work = float(sum(sum(x * (272 + 512) + 8 * 256 * 8 for x in c) for c in wl.decode_ctx))
        self.launches = len(wl.decode_ctx)
        self.algorithmic = "ctx*(272 B int8 K row + 512 B f16 V row) + 16 KiB q/out per token"
        self.workload = ("the ragged batch (8 sequences, ctx drawn by the seed from [1024, 131072], 32 steps) "
                         "with int8 K (per-row scale) and f16 V, f32 q (attn_decode_q8)")

    def run(self, variant):
        for t, c in enumerate(self.wl.decode_ctx):
            self.kca.attn_decode_q8(self.q[t], self.k8, self.v, c, out=self.out[t], workspace=self.ws)

    def workspaces(self):
        return [self.ws]


PART_NAMES = ["decode_ragged", "decode_256", "decode_4096", "prefill", "decode", "window_prefill",
              "window_decode", "long_chunk", "prefill_batch", "decode_q8_ragged"]


def build_parts(w, device, sms, only=None):
    """The parts of one pass, in pass order (see the module docstring); with
    `only`, just that one (for profiling a single configuration)."""
    def want(*names):
        return only is None or only in names
    parts = []
    if want("decode_ragged"):
        parts.append(RaggedPart(device))
    if want("decode_256"):
        parts.append(DecodeLenPart(device, 256))
    if want("decode_4096"):
        parts.append(DecodeLenPart(device, 4096))
    if want("prefill"):
        parts.append(PrefillPart(w, sms))
    if want("decode"):
        parts.append(HeadlineDecodePart(w))
    if want("window_prefill", "window_decode"):
        parts += [p for p in WindowParts(device, sms).parts if want(p.name)]
    if want("long_chunk"):
        parts.append(LongChunkPart(device, sms))
    if want("prefill_batch"):
        parts.append(BatchRowsPart(device))
    if want("decode_q8_ragged"):
        parts.append(RaggedQ8Part(device))
    return parts


def run_cuda(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    w = Workload(dev) if args.only in (None, "prefill", "decode") else None
    parts = build_parts(w, dev, sms, args.only)
    stream = torch.cuda.current_stream()
    passes = max(1, args.passes)
    # warm-up: eager calls first (tensor-map caches, function attributes)
    for s in range(args.warmup):
        for p in parts:
            p.run(s % p.variants)
    torch.cuda.synchronize()
    graphs = None
    if not args.eager:
        graphs = {}
        for p in parts:
            graphs[p.name] = []
            for var in range(p.variants):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    p.run(var)
                graphs[p.name].append(g)
        for _ in range(2):
            for p in parts:
                for g in graphs[p.name]:
                    g.replay()
        torch.cuda.synchronize()

    def replay(p, i):
        if graphs is None:
            p.run(i % p.variants)
        else:
            graphs[p.name][i % p.variants].replay()

    def timed(region, reps):
        """K steps of `reps` passes over the parts in `region`, each part
        bracketed by CUDA events on the launching stream; returns (region ms,
        {part: ms summed over its runs}, clocks during the region)."""
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clocks = Clocks(dev)
        n = args.steps * reps
        ev = {p.name: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(n)] for p in region}
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        i = 0
        for s in range(args.steps):
            for _ in range(reps):
                for p in region:
                    e0, e1 = ev[p.name][i]
                    e0.record(stream)
                    replay(p, i)
                    e1.record(stream)
                i += 1
        end.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clk = clocks.stop()
        names = [p.name for p in region]
        vals = max_over_ranks([start.elapsed_time(end)] + [sum(a.elapsed_time(b) for a, b in ev[nm]) for nm in names],
                              world, dev)
        return vals[0], dict(zip(names, vals[1:])), clk

    # The timed region proper: the headline step (the 16K prompt and its 64
    # decode steps), replayed `passes` times per step.  The other
    # configurations follow in a region of their own.
    main = [p for p in parts if p.name in ("prefill", "decode")]
    others = [p for p in parts if p.name not in ("prefill", "decode")]
    nvtx = torch.cuda.nvtx
    res = dict(parts={p.name: p for p in parts}, part_ms={}, runs={}, passes=passes)
    if main:
        nvtx.range_push("timed steps")
        total_ms, pm, clk = timed(main, passes)
        nvtx.range_pop()
        res.update(total_ms=total_ms, clocks=clk, launches=sum(p.launches for p in main) * args.steps * passes)
        res["part_ms"].update(pm)
        res["runs"].update({nm: args.steps * passes for nm in pm})
    if others:
        reps = max(1, args.other_passes)
        nvtx.range_push("other configurations")
        other_ms, pm, clk = timed(others, reps)
        nvtx.range_pop()
        res.update(other_ms=other_ms, other_clocks=clk, other_passes=reps,
                   other_launches=sum(p.launches for p in others) * args.steps * reps)
        res["part_ms"].update(pm)
        res["runs"].update({nm: args.steps * reps for nm in pm})
    import kv_cache_attention_states_b200 as kca
    for p in parts:
        for ws in p.workspaces():
            st, detail = kca.attn_device_status(ws)
            if st != 0:
                raise RuntimeError(f"{p.name}: device status {st} detail {detail:#x}")
    if graphs is not None:
        del graphs
    if args.only is not None:
        return res
    e2e = run_e2e(w, args, stream)
    e2e["pre_ms"], e2e["dec_ms"] = max_over_ranks([e2e["pre_ms"], e2e["dec_ms"]], world, dev)
    res["e2e"] = e2e
    return res


def e2e_groups(chunks, first=None, size=None):
    """The end-to-end leg's copy groups: the first `first` chunks, then
    groups of `size`.  The outputs (f32, 1.6x the inputs' bytes) decide the
    time on the link, and the device-to-host copies start only when the
    first group has crossed and computed, so the first group is kept small."""
    first = E2E_FIRST if first is None else first
    size = E2E_GROUP if size is None else size
    groups = [list(chunks[:first])] if first > 0 else []
    rest = list(chunks[first:])
    groups += [rest[i:i + size] for i in range(0, len(rest), size)]
    return [g for g in groups if g]


def run_e2e(w, args, stream, groups=None):
    """Same metric through the public API with host buffers: each step copies
    its inputs (Q rows and the new K/V rows of every chunk, the decode query
    and its appended K/V row) from pinned host memory, runs the calls, and
    copies every output back; all inside the timed region."""
    import torch
    steps = max(1, min(args.steps, 5))
    q, k, v = w.pre[0]
    hq = q.cpu().pin_memory()
    hk = k.cpu().pin_memory()
    hv = v.cpu().pin_memory()
    hout = torch.empty(w.pre_out.shape, dtype=torch.float32).pin_memory()
    dk, dv = w.dec_kv[0]
    # Each decode step's inputs -- its query (f32) and the K and V rows it
    # appends (f16) -- sit side by side in one pinned record, so a step is
    # one host copy, the append kernel, the decode kernel and one copy back.
    qb, rb = 8 * 256 * 4, 256 * 2
    hstage = torch.empty((len(w.dec_ctx), qb + 2 * rb), dtype=torch.uint8).pin_memory()
    for t, c in enumerate(w.dec_ctx):
        hstage[t, :qb] = w.dec_q[t].cpu().reshape(-1).view(torch.uint8)
        hstage[t, qb:qb + rb] = dk[0, c - 1].cpu().view(torch.uint8)
        hstage[t, qb + rb:] = dv[0, c - 1].cpu().view(torch.uint8)
    dstage = torch.empty(qb + 2 * rb, dtype=torch.uint8, device=w.dec_q.device)
    sq = dstage[:qb].view(torch.float32).view(1, 8, 256)
    sk = dstage[qb:qb + rb].view(torch.float16).view(1, 256)
    sv = dstage[qb + rb:].view(torch.float16).view(1, 256)
    hdout = torch.empty(w.dec_out.shape, dtype=torch.float32).pin_memory()
    h2d = d2h = 0
    for cs, r in w.chunks:
        h2d += hq[cs:cs + r].numel() * 2 + 2 * hk[cs:cs + r].numel() * 2
        d2h += hout[cs:cs + r].numel() * 4
    pre_h2d, pre_d2h = h2d, d2h
    for t, c in enumerate(w.dec_ctx):
        h2d += hstage[t].numel()
        d2h += hdout[t].numel() * 4

    # Prefill streams its chunks in copy groups (e2e_groups: E2E_FIRST chunks,
    # then E2E_GROUP at a time): the inputs of group g+1 cross PCIe (copy
    # stream) while group g computes, and each group's outputs go back (a
    # second copy stream) as soon as its chunks are done.  Copies of a few
    # chunks at once keep both directions near the link rate: on one B200,
    # ms per prompt for (first, size) = (2, 4) 3.02, (1, 4) 3.06, (4, 4) 3.08,
    # (1, 3) 3.09, (1, 6) 3.09, and one copy per chunk and direction 3.70.
    # The timed region spans the first copy to the last one on the compute
    # stream.
    h2d_s = torch.cuda.Stream()
    d2h_s = torch.cuda.Stream()
    groups = e2e_groups(w.chunks) if groups is None else groups

    def step(timed):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        h2d_s.wait_stream(stream)
        d2h_s.wait_stream(stream)
        for g in groups:
            a, b = g[0][0], g[-1][0] + g[-1][1]
            with torch.cuda.stream(h2d_s):
                q[a:b].copy_(hq[a:b], non_blocking=True)
                k[a:b].copy_(hk[a:b], non_blocking=True)
                v[a:b].copy_(hv[a:b], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(h2d_s)
            stream.wait_event(ready)
            for cs, r in g:
                w.kca.attn_prefill(q[cs:cs + r], k, v, cs, out=w.pre_out[cs:cs + r], workspace=w.pre_ws,
                                   stream=stream)
            done = torch.cuda.Event()
            done.record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(done)
                hout[a:b].copy_(w.pre_out[a:b], non_blocking=True)
        stream.wait_stream(d2h_s)
        ev[1].record(stream)
        for t, c in enumerate(w.dec_ctx):
            dstage.copy_(hstage[t], non_blocking=True)
            w.kca.attn_append_kv(sk, sv, dk, dv, c - 1)
            w.kca.attn_decode(sq, dk, dv, [c], out=w.dec_out[t], workspace=w.dec_ws)
            hdout[t].copy_(w.dec_out[t], non_blocking=True)
        ev[2].record(stream)
        return ev

    step(False)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("e2e steps")
    evs = [step(True) for _ in range(steps)]
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    return dict(steps=steps, pre_ms=pre_ms, dec_ms=dec_ms, h2d=h2d, d2h=d2h, pre_h2d=pre_h2d,
                pre_d2h=pre_d2h)



# ---------------------------------------------------------- CPU oracle legs

_ORACLE_INPUTS = {}


def _oracle_inputs(seed):
    from kv_cache_attention_states_b200 import synth
    if seed not in _ORACLE_INPUTS:
        pw = synth.prefill_bf16_16k()
        dw = synth.decode_f16(DECODE_LEN, DECODE_STEPS)
        _ORACLE_INPUTS[seed] = dict(
            q=synth.draw(seed, "q", (PREFILL_ROWS, 8, 256), "bf16", pw.std),
            k=synth.draw(seed, "k", (PREFILL_ROWS, 256), "bf16", pw.std),
            v=synth.draw(seed, "v", (PREFILL_ROWS, 256), "bf16", pw.std),
            kd=synth.draw(seed, "k", (dw.capacity, 256), "f16"),
            vd=synth.draw(seed, "v", (dw.capacity, 256), "f16"),
            qd=synth.draw(seed, "q", (DECODE_STEPS, 8, 256), "f32"),
            ctx=[c[0] for c in dw.decode_ctx])
    return _ORACLE_INPUTS[seed]


def _timed(fn):
    t0 = time.perf_counter()
    fn()
    return time.perf_counter() - t0


def oracle_sample(n_rows: int, n_decode: int, seed=0):
    """Time the f64 oracle (as it stands, all host cores) on a bounded sample
    of the headline workload: n_rows prefill rows evenly spaced over the
    prompt (so their mean context equals the prompt's) and n_decode decode
    steps at context 16,384.  Returns (rows/s, tok/s, cores, description)."""
    import oracle
    from kv_cache_attention_states_b200 import synth
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    x = _oracle_inputs(seed)
    q, k, v = x["q"], x["k"], x["v"]
    rows = (np.arange(n_rows) * PREFILL_ROWS) // n_rows + PREFILL_ROWS // (2 * n_rows)
    t_pre = _timed(lambda: oracle.attention(q[rows], k, v, rows, q_dtype="bf16", kv_dtype="bf16",
                                            scale=synth.SCALE))
    kd, vd, qd = x["kd"], x["vd"], x["qd"]

    def dec():
        for t in range(n_decode):
            oracle.attention(qd[t:t + 1], kd, vd, [x["ctx"][t] - 1], kv_dtype="f16", scale=synth.SCALE)
    t_dec = _timed(dec)
    desc = (f"{n_rows} prefill rows evenly spaced over positions 0-16383 of the 16K bf16 prompt "
            f"({t_pre:.1f} s) + {n_decode} decode steps at ctx 16384 ({t_dec:.1f} s); f64 C oracle, "
            f"OpenMP over (row, head), {cores} threads")
    return n_rows / t_pre, n_decode / t_dec, cores, desc


def oracle_part_samples(seed=0):
    """The oracle on a bounded sample of every other configuration (a few
    seconds each): {part name: (units/s, sample description)}."""
    import oracle
    from kv_cache_attention_states_b200 import synth
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    out = {}
    for length, n in ((256, 64), (4096, 16)):
        wl = synth.decode_f16(length, DECODE_STEPS)
        k = synth.draw(seed, "k", (wl.capacity, 256), "f16")
        v = synth.draw(seed, "v", (wl.capacity, 256), "f16")
        q = synth.draw(seed, "q", (DECODE_STEPS, 8, 256), "f32")
        ctx = [c[0] for c in wl.decode_ctx]

        def dec():
            for t in range(n):
                oracle.attention(q[t:t + 1], k, v, [ctx[t] - 1], kv_dtype="f16", scale=synth.SCALE)
        sec = _timed(dec)
        out[f"decode_{length}"] = (n / sec, f"{n} decode steps at ctx {length}.. ({sec:.2f} s)")
    wl = synth.window_bf16(DECODE_STEPS)
    k = synth.draw(seed, "k", (wl.capacity, 256), "bf16")
    v = synth.draw(seed, "v", (wl.capacity, 256), "bf16")
    q = synth.draw(seed, "q", (4096, 8, 256), "bf16")
    qd = synth.draw(seed, "qd", (DECODE_STEPS, 8, 256), "bf16")
    rows = np.arange(0, 4096, 4)
    sec = _timed(lambda: oracle.attention(q[rows], k, v, rows, window=wl.window, q_dtype="bf16",
                                          kv_dtype="bf16", scale=synth.SCALE))
    out["window_prefill"] = (rows.size / sec, f"every 4th of the 4096 prompt rows, window 512 ({sec:.2f} s)")
    pos = np.array([c[0] - 1 for c in wl.decode_ctx])
    sec = _timed(lambda: oracle.attention(qd, k, v, pos, window=wl.window, q_dtype="bf16", kv_dtype="bf16",
                                          scale=synth.SCALE))
    out["window_decode"] = (pos.size / sec, f"all 64 decode steps, window 512 ({sec:.2f} s)")
    wl = synth.long_chunk_bf16()
    cs, r = wl.prefill[0]
    k = synth.draw(seed, "k", (wl.capacity, 256), "bf16")
    v = synth.draw(seed, "v", (wl.capacity, 256), "bf16")
    q = synth.draw(seed, "q", (r, 8, 256), "bf16")
    rows = np.arange(0, r, r // 16)
    sec = _timed(lambda: oracle.attention(q[rows], k, v, cs + rows, q_dtype="bf16", kv_dtype="bf16",
                                          scale=synth.SCALE))
    out["long_chunk"] = (rows.size / sec, f"{rows.size} rows evenly spaced over the 768-row chunk at "
                                          f"130304 ({sec:.2f} s)")
    wl = synth.ragged_f16(seed)
    ctx = wl.decode_ctx[0][:2]
    k = np.concatenate([synth.draw(seed, f"rk{b}", (c, 256), "f16") for b, c in enumerate(ctx)])
    v = np.concatenate([synth.draw(seed, f"rv{b}", (c, 256), "f16") for b, c in enumerate(ctx)])
    q = synth.draw(seed, "rq", (2, 8, 256), "f32")
    base = np.array([0, ctx[0]])
    sec = _timed(lambda: oracle.attention(q, k, v, np.array(ctx) - 1, base, kv_dtype="f16", scale=synth.SCALE))
    out["decode_ragged"] = (2 / sec, f"sequences 0-1 of the first step (ctx {ctx[0]}, {ctx[1]}; {sec:.2f} s)")
    ctx0 = synth.integers(seed, "batch_ctx", 1024, 16384, 32)[:4]
    rows = 4
    k = np.concatenate([synth.draw(seed, f"bk{b}", (int(c), 256), "f16") for b, c in enumerate(ctx0)])
    v = np.concatenate([synth.draw(seed, f"bv{b}", (int(c), 256), "f16") for b, c in enumerate(ctx0)])
    q = synth.draw(seed, "bq", (4 * rows, 8, 256), "f32")
    starts = np.concatenate([[0], np.cumsum(ctx0)[:-1]])
    pos = np.array([int(c) - rows + i for c in ctx0 for i in range(rows)])
    base = np.repeat(starts, rows)
    sec = _timed(lambda: oracle.attention(q, k, v, pos, base, kv_dtype="f16", scale=synth.SCALE))
    out["prefill_batch"] = (pos.size / sec, f"sequences 0-3 of the first call, 4 rows each ({sec:.2f} s)")
    from oracle import quant
    wl = synth.ragged_f16(seed)
    ctx = wl.decode_ctx[0][:2]
    kq = np.concatenate([synth.normal(seed, f"qk{b}", (c, 256)) for b, c in enumerate(ctx)])
    codes, scales = quant.quantize_rows(kq)
    v = np.concatenate([synth.draw(seed, f"qv{b}", (c, 256), "f16") for b, c in enumerate(ctx)])
    q = synth.draw(seed, "qq", (2, 8, 256), "f32")
    sec = _timed(lambda: quant.attention_q8(q, "f32", codes, scales, v, "f16", np.array(ctx) - 1,
                                            np.array([0, ctx[0]]), scale=synth.SCALE))
    out["decode_q8_ragged"] = (2 / sec, f"sequences 0-1 of the first step, quantised-dot oracle (numpy f64; "
                                        f"{sec:.2f} s)")
    return out, cores


def run_reference(args, rank, world):
    if rank != 0:
        return
    per_step = 24
    for _ in range(args.warmup):
        oracle_sample(4, 1)
    t0 = time.perf_counter()
    rows_s = tok_s = 0.0
    descs = []
    for _ in range(args.steps):
        r, t, cores, d = oracle_sample(per_step, 1)
        rows_s += r
        tok_s += t
        descs.append(d)
    elapsed = time.perf_counter() - t0
    value = rows_s / args.steps
    line = {"metric": METRIC, "value": value, "unit": "q-rows/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * elapsed / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": "prefill 16384 rows bf16 (768-row chunks) + 64 decode steps at "
                                   "16K f16; oracle on a bounded sample per step", "seq_len": 16384,
                       "l2": "n/a (CPU)"},
            "decode": {"value": tok_s / args.steps, "unit": "tok/s"},
            "cpu_baseline": {"value": value, "unit": "q-rows/s", "cores": cores, "kind": "oracle",
                             "sample": descs[0]},
            "e2e": {"value": value, "unit": "q-rows/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def part_object(p, ms, runs, world, hbm, tflops, tflops_sus, src, cpu=None):
    """JSON object of one configuration: throughput, roofline of its kernel
    (algorithmic work / measured time), the ncu traffic where captured."""
    sec = ms / 1e3
    per_run = sec / runs
    obj = {"workload": p.workload or p.name, "value": world * p.units * runs / sec,
           "unit": f"{p.unit}/s", "ms_per_run": 1e3 * per_run}
    if p.bound == "tensor":
        achieved = p.work / per_run / 1e12
        roof = {"kernel": p.kernel, "bound": "tensor", "achieved": achieved, "peak": tflops,
                "unit": "TFLOP/s", "frac": achieved / tflops, "peak_source": f"{src} bf16 dense (burst)"}
        if tflops_sus:
            roof["frac_of_sustained"] = achieved / tflops_sus
    else:
        achieved = p.work / per_run / 1e9
        roof = {"kernel": p.kernel, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "peak_source": f"{src} HBM copy"}
    tr = TRAFFIC.get(p.name)
    roof["traffic"] = tr[0] if tr else None
    if tr:
        roof["traffic_launch"] = tr[1]
    roof["algorithmic"] = p.algorithmic
    obj["roofline"] = roof
    if cpu is not None:
        obj["cpu_baseline"] = cpu
    return obj


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--passes", type=int, default=PASSES, help="passes over the headline step per timed step")
    ap.add_argument("--other-passes", type=int, default=OTHER_PASSES,
                    help="passes over the other configurations per step, in their own timed region")
    ap.add_argument("--impl", default="kca", choices=["kca", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch every call from Python instead of "
                    "replaying captured CUDA graphs")
    ap.add_argument("--only", choices=PART_NAMES, default=None,
                    help="time one configuration alone (profiling); prints that part's object only")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import datetime
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res = run_cuda(args, rank, world, local_rank)
    if args.only is not None:
        if rank == 0:
            hbm, tflops, tflops_sus, src = _peaks()
            p = res["parts"][args.only]
            print(json.dumps({"only": args.only, "steps": args.steps, "runs": res["runs"][args.only],
                              **part_object(p, res["part_ms"][args.only], res["runs"][args.only], world, hbm,
                                            tflops, tflops_sus, src)}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return
    cpu = parts_cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # about 10 s of the oracle on a 16-core host: 2304 prefill rows, 12 decode steps
        rows_s, tok_s, cores, desc = oracle_sample(2304, 12)
        cpu = {"value": rows_s, "unit": "q-rows/s", "cores": cores, "kind": "oracle", "sample": desc,
               "decode_tok_s": tok_s}
        samples, cores = oracle_part_samples()
        parts_cpu = {nm: {"value": v, "unit": ("q-rows/s" if nm in ("window_prefill", "long_chunk", "prefill_batch")
                                                   else "tok/s"),
                          "cores": cores if "numpy" not in d else 1, "kind": "oracle",
                          "sample": d if "numpy" in d else d + "; f64 C oracle, OpenMP over (row, head)"}
                     for nm, (v, d) in samples.items()}
        parts_cpu["decode"] = {"value": tok_s, "unit": "tok/s", "cores": cores, "kind": "oracle",
                               "sample": desc}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    hbm, tflops, tflops_sus, src = _peaks()
    K = args.steps
    parts, pm = res["parts"], res["part_ms"]

    def obj(name):
        return part_object(parts[name], pm[name], res["runs"][name], world, hbm, tflops, tflops_sus, src,
                           (parts_cpu or {}).get(name))

    pre = obj("prefill")
    e2e = res["e2e"]
    line = {
        "metric": METRIC, "value": pre["value"], "unit": "q-rows/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": res["total_ms"] / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "prefill of a 16384-token prompt in 768-row chunks (bf16, N(0,1)*0.5) "
                               "+ 64 decode steps at ctx 16384-16447 (f16 K/V, f32 q); 8 q heads / "
                               "1 KV head, head_dim 256, causal",
                   "seq_len": 16384, "global_batch": world, "parallelism": f"replicas x{world}",
                   "step": f"{res['passes']} passes over the prompt's prefill and its 64 decode steps",
                   "value": "prefill part of every pass (CUDA events); the 16K decode in 'decode'",
                   "other_configurations": f"timed after the main region, {res['other_passes']} passes per step "
                                           f"over ragged, decode_256, decode_4096, window, long_chunk, "
                                           f"prefill_batch, decode_q8_ragged ({res['other_ms'] / K:.1f} ms per step, "
                                           f"{res['other_launches']} launches, clocks {res['other_clocks']})",
                   "launch": "eager" if args.eager else "one CUDA graph per configuration of the C-ABI calls",
                   "l2": "inputs larger than L2: the 16K decode rotates 32 cache replicas (16.8 MB "
                         "each), the prompt alternates 2 input replicas (80 MB each); in the other region "
                         "the 256 / 4096 decodes rotate 64 replicas each after the 1 GB ragged batch"},
        "roofline": pre["roofline"],
        "decode": obj("decode"),
        "decode_256": obj("decode_256"),
        "decode_4096": obj("decode_4096"),
        "window": {"workload": "window 512, bf16 Q/K/V N(0,1): 4096-token prompt in 768-row chunks, then "
                               "64 decode steps at positions 4096-4159 (the decode re-reads the rows the "
                               "previous step read: sliding window)",
                   "prefill": obj("window_prefill"), "decode": obj("window_decode")},
        "long_chunk": obj("long_chunk"),
        "decode_ragged": obj("decode_ragged"),
        "prefill_batch": obj("prefill_batch"),
        "decode_q8_ragged": obj("decode_q8_ragged"),
        "e2e": {"value": world * PREFILL_ROWS * e2e["steps"] / (e2e["pre_ms"] / 1e3), "unit": "q-rows/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "decode_tok_s": world * DECODE_STEPS * e2e["steps"] / (e2e["dec_ms"] / 1e3),
                "steps": e2e["steps"]},
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
    }
    line["decode"]["workload"] = "64 decode steps at ctx 16384-16447, f16 K/V, f32 q (32 cache replicas)"
    line["decode_ragged"]["workload"] = ("8 sequences, ctx drawn by the seed from [1024, 131072] (mean "
                                         f"{parts['decode_ragged'].mean_ctx:.0f}), 32 steps, f16 K/V, f32 q")
    line["long_chunk"]["workload"] = "one 768-row bf16 chunk at positions 130304-131071 of a 131072 cache"
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
