"""Benchmark of the states-form attention hot path on B200.

One step = the whole path on one batch of synthetic input:
  * chunked causal prefill of a 16,384-token prompt in 768-row chunks
    (21 x 768 + 256), bf16 Q/K/V ~ N(0,1)*0.5, through attn_prefill, and
  * 64 single-row decode steps at context 16,384 .. 16,447, f16 K/V ~ N(0,1),
    f32 query, through attn_decode.
value = prefill q-rows/s (a q-row is one query position with all 8 heads),
timed with CUDA events around the prefill part of every step; the decode
part is reported as decode tok/s beside it; ms_per_step covers both.

L2: inputs are rotated across replicas whose total exceeds the 126 MB L2
(decode: one 16.8 MB cache replica per step index mod 32; prefill: two
input replicas), so every step reads cold rows from HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
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
# DRAM bytes (read + write) per launch from one ncu capture of the current
# kernels; reset to None whenever a kernel changes after its capture.
PREFILL_TRAFFIC = 18.931e6 + 25.6e3
DECODE_TRAFFIC = 16.919e6
E2E_GROUP = 4            # prefill chunks per host copy in the end-to-end leg
METRIC = "prefill q-rows/s & decode tok/s at 16K ctx (1 B200); % of TC/HBM roofline"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def max_over_ranks(values, world: int, device):
    """Element-wise maximum over ranks of this rank's device-timed values
    (every rank calls it; the job is as slow as its slowest rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def prefill_flops() -> float:
    # 2 GEMMs (QK^T and PV) x 2 flop x head_dim x 8 heads per visible (query, key) pair
    pairs = PREFILL_ROWS * (PREFILL_ROWS + 1) // 2
    return 4.0 * 256 * 8 * pairs


def decode_bytes(ctx: int) -> int:
    # K + V rows (f16) once, q and out (f32)
    return ctx * 256 * 2 * 2 + 2 * 8 * 256 * 4


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


# ------------------------------------------------------------- the workload

class Workload:
    """Device-resident inputs of one step (and the replicas that defeat L2)."""

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

    def launches_per_step(self) -> int:
        kca = self.kca
        n = 0
        for cs, r in self.chunks:
            path, items = kca.attn_prefill_plan(kca.BF16, kca.BF16, cs, r, 0, self.sms)
            n += 1 + int((items[:, 3] >= 0).any())
        # f16 caches take the tensor-core rows kernel, which merges its
        # splits in the same launch: one kernel per decode call.
        n += len(self.dec_ctx)
        return n

    def prefill(self):
        q, k, v = self.pre[self.step_index % PREFILL_REPLICAS]
        for cs, r in self.chunks:
            self.kca.attn_prefill(q[cs:cs + r], k, v, cs, out=self.pre_out[cs:cs + r],
                                  workspace=self.pre_ws)

    def decode(self):
        for t, c in enumerate(self.dec_ctx):
            k, v = self.dec_kv[(self.step_index * DECODE_STEPS + t) % DECODE_REPLICAS]
            self.kca.attn_decode(self.dec_q[t], k, v, [c], out=self.dec_out[t], workspace=self.dec_ws)


def run_cuda(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = Workload(dev)
    w.sms = torch.cuda.get_device_properties(dev).multi_processor_count
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        w.prefill()
        w.decode()
        w.step_index += 1
    torch.cuda.synchronize()
    graphs = None
    if not args.eager:
        # One graph per prefill input replica and one for the 64 decode steps
        # (each step visits the 32 cache replicas in the same order).
        graphs = {"pre": [], "dec": None}
        saved = w.step_index
        for r in range(PREFILL_REPLICAS):
            g = torch.cuda.CUDAGraph()
            w.step_index = r
            with torch.cuda.graph(g):
                w.prefill()
            graphs["pre"].append(g)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            w.decode()
        graphs["dec"] = g
        w.step_index = saved
        for _ in range(2):
            graphs["pre"][w.step_index % PREFILL_REPLICAS].replay()
            graphs["dec"].replay()
            w.step_index += 1
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = Clocks(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    # NVTX ranges name the phases on a profiler timeline (no cost otherwise).
    nvtx = torch.cuda.nvtx
    nvtx.range_push("timed steps")
    start.record(stream)
    for s in range(args.steps):
        ev[s][0].record(stream)
        nvtx.range_push("prefill")
        if graphs is None:
            w.prefill()
        else:
            graphs["pre"][w.step_index % PREFILL_REPLICAS].replay()
        nvtx.range_pop()
        ev[s][1].record(stream)
        nvtx.range_push("decode")
        if graphs is None:
            w.decode()
        else:
            graphs["dec"].replay()
        nvtx.range_pop()
        ev[s][2].record(stream)
        w.step_index += 1
    end.record(stream)
    nvtx.range_pop()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    total_ms = start.elapsed_time(end)
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in ev)
    total_ms, pre_ms, dec_ms = max_over_ranks([total_ms, pre_ms, dec_ms], world, dev)
    st, detail = w.kca.attn_device_status(w.pre_ws)
    st2, _ = w.kca.attn_device_status(w.dec_ws)
    if st != 0 or st2 != 0:
        raise RuntimeError(f"device status {st}/{st2} detail {detail:#x}")
    res = dict(total_ms=total_ms, pre_ms=pre_ms, dec_ms=dec_ms, clocks=clk,
               launches=w.launches_per_step() * args.steps)
    e2e = run_e2e(w, args, stream)
    e2e["pre_ms"], e2e["dec_ms"] = max_over_ranks([e2e["pre_ms"], e2e["dec_ms"]], world, dev)
    res["e2e"] = e2e
    del w, graphs
    torch.cuda.empty_cache()
    rg = run_ragged(dev, stream)
    rg["tok_s"], rg["gbs"] = [-x for x in max_over_ranks([-rg["tok_s"], -rg["gbs"]], world, dev)]
    res["ragged"] = rg
    return res


def run_e2e(w, args, stream):
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

    # Prefill streams its chunks in groups of E2E_GROUP: the inputs of group
    # g+1 cross PCIe (copy stream) while group g computes, and each group's
    # outputs go back (a second copy stream) as soon as its chunks are done.
    # Copies of a few chunks at once keep both directions near the link rate
    # (one copy per chunk and direction ran ~25 % slower on B200: 3.7 against
    # 3.2 ms per prompt).  The timed region spans the first copy to the last
    # one on the compute stream.
    h2d_s = torch.cuda.Stream()
    d2h_s = torch.cuda.Stream()
    groups = [w.chunks[i:i + E2E_GROUP] for i in range(0, len(w.chunks), E2E_GROUP)]

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


def run_ragged(device, stream):
    """The ragged long-context decode workload (8 sequences, lengths drawn by
    the seed from [1024, 131072], 32 steps, f16 K/V, f32 q), timed after the
    main region as one CUDA graph of its 32 calls: where the decode kernel
    is HBM-bound rather than latency-bound.  The 1.07 GB cache is far larger
    than L2, so no replica rotation is needed.  Reported beside the headline
    decode figure, not in it."""
    import torch
    import kv_cache_attention_states_b200 as kca
    from kv_cache_attention_states_b200 import synth
    wl = synth.ragged_f16(0)
    g = torch.Generator(device=device)
    g.manual_seed(1)
    k = torch.randn((wl.batch, wl.capacity, 256), generator=g, device=device).half()
    v = torch.randn((wl.batch, wl.capacity, 256), generator=g, device=device).half()
    q = torch.randn((len(wl.decode_ctx), wl.batch, 8, 256), generator=g, device=device)
    out = torch.empty_like(q)
    ws = kca.new_workspace(max(kca.attn_decode_workspace_bytes(c) for c in wl.decode_ctx), device)

    def steps():
        for t, c in enumerate(wl.decode_ctx):
            kca.attn_decode(q[t], k, v, c, out=out[t], workspace=ws)

    steps()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        steps()
    for _ in range(2):
        graph.replay()
    reps = 5
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("ragged decode")
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    st, detail = kca.attn_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} detail {detail:#x}")
    sec = e0.elapsed_time(e1) / 1e3
    nbytes = sum(sum(decode_bytes(x) for x in c) for c in wl.decode_ctx) * reps
    del graph, k, v
    torch.cuda.empty_cache()
    return {"tok_s": wl.batch * len(wl.decode_ctx) * reps / sec, "gbs": nbytes / sec / 1e9,
            "ms_per_step": 1e3 * sec / (reps * len(wl.decode_ctx)),
            "mean_ctx": float(np.mean(wl.decode_ctx[0]))}


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


def oracle_sample(n_rows: int, n_decode: int, seed=0):
    """Time the f64 oracle (as it stands, all host cores) on a bounded sample
    of the same workload: n_rows prefill rows evenly spaced over the prompt
    (so their mean context equals the prompt's) and n_decode decode steps at
    context 16,384.  Returns (rows/s, tok/s, cores, description)."""
    import oracle
    from kv_cache_attention_states_b200 import synth
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    x = _oracle_inputs(seed)
    q, k, v = x["q"], x["k"], x["v"]
    rows = (np.arange(n_rows) * PREFILL_ROWS) // n_rows + PREFILL_ROWS // (2 * n_rows)
    t0 = time.perf_counter()
    oracle.attention(q[rows], k, v, rows, q_dtype="bf16", kv_dtype="bf16", scale=synth.SCALE)
    t_pre = time.perf_counter() - t0
    kd, vd, qd = x["kd"], x["vd"], x["qd"]
    t0 = time.perf_counter()
    for t in range(n_decode):
        oracle.attention(qd[t:t + 1], kd, vd, [x["ctx"][t] - 1], kv_dtype="f16",
                         scale=synth.SCALE)
    t_dec = time.perf_counter() - t0
    desc = (f"{n_rows} prefill rows evenly spaced over positions 0-16383 of the 16K bf16 prompt "
            f"({t_pre:.1f} s) + {n_decode} decode steps at ctx 16384 ({t_dec:.1f} s); f64 C oracle, "
            f"OpenMP over (row, head), {cores} threads")
    return n_rows / t_pre, n_decode / t_dec, cores, desc


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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kca", choices=["kca", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch every call from Python instead of "
                    "replaying a captured CUDA graph of the step")
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
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows_s, tok_s, cores, desc = oracle_sample(768, 4)
        cpu = {"value": rows_s, "unit": "q-rows/s", "cores": cores, "kind": "oracle", "sample": desc,
               "decode_tok_s": tok_s}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    hbm, tflops, src = _peaks()
    K = args.steps
    pre_s = res["pre_ms"] / 1e3
    dec_s = res["dec_ms"] / 1e3
    value = world * PREFILL_ROWS * K / pre_s
    dec_tok_s = world * DECODE_STEPS * K / dec_s
    achieved_tf = prefill_flops() * K / pre_s / 1e12
    dec_bytes = sum(decode_bytes(c) for c in range(DECODE_LEN, DECODE_LEN + DECODE_STEPS))
    achieved_gbs = dec_bytes * K / dec_s / 1e9
    e2e = res["e2e"]
    line = {
        "metric": METRIC, "value": value, "unit": "q-rows/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": res["total_ms"] / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "prefill of a 16384-token prompt in 768-row chunks (bf16, N(0,1)*0.5) "
                               "+ 64 decode steps at ctx 16384-16447 (f16 K/V, f32 q); 8 q heads / "
                               "1 KV head, head_dim 256, causal",
                   "seq_len": 16384, "global_batch": world, "parallelism": f"replicas x{world}",
                   "value": "prefill part of each step (CUDA events); decode part in 'decode'",
                   "launch": "eager" if args.eager else "CUDA graph of the step's C-ABI calls",
                   "l2": "inputs larger than L2: decode rotates 32 cache replicas (16.8 MB each), "
                         "prefill alternates 2 input replicas (80 MB each)"},
        "roofline": {"kernel": "prefill_tc_kernel (+ its merge)", "bound": "tensor",
                     "achieved": achieved_tf, "peak": tflops, "unit": "TFLOP/s",
                     "frac": achieved_tf / tflops, "traffic": PREFILL_TRAFFIC,
                     "traffic_source": "ncu dram bytes of the chunk-19 launch (768 rows at 14592); "
                                       "profiles/prefill_tc_kernel_16k_late_chunks.md",
                     "peak_source": f"{src} bf16 dense (burst)",
                     "algorithmic": "4*256*8*sum|J(pos)| = 1.0996e12 flop per step"},
        "decode": {"value": dec_tok_s, "unit": "tok/s", "ms_per_step": res["dec_ms"] / K,
                   "roofline": {"kernel": "decode_mma_kernel<f32,f16> (merge in-kernel)", "bound": "hbm",
                                "achieved": achieved_gbs, "peak": hbm, "unit": "GB/s",
                                "frac": achieved_gbs / hbm, "traffic": DECODE_TRAFFIC,
                                "traffic_source": "ncu dram bytes of one launch at ctx ~16.4K; "
                                                  "profiles/decode_mma_kernel_16k.md",
                                "peak_source": f"{src} HBM copy",
                                "algorithmic": "ctx*1024 B K/V + 16 KiB q/out per token"}},
        "e2e": {"value": world * PREFILL_ROWS * e2e["steps"] / (e2e["pre_ms"] / 1e3), "unit": "q-rows/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "decode_tok_s": world * DECODE_STEPS * e2e["steps"] / (e2e["dec_ms"] / 1e3),
                "steps": e2e["steps"]},
        "decode_ragged": {"workload": "8 sequences, ctx drawn by the seed from [1024, 131072] "
                                      f"(mean {res['ragged']['mean_ctx']:.0f}), 32 steps, f16 K/V, f32 q; "
                                      "one CUDA graph, timed after the main region, not part of value",
                          "value": world * res["ragged"]["tok_s"], "unit": "tok/s",
                          "ms_per_step": res["ragged"]["ms_per_step"],
                          "roofline": {"kernel": "decode_mma_kernel<f32,f16>", "bound": "hbm",
                                       "achieved": res["ragged"]["gbs"], "peak": hbm, "unit": "GB/s",
                                       "frac": res["ragged"]["gbs"] / hbm,
                                       "algorithmic": "ctx*1024 B K/V + 16 KiB q/out per token"}},
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
