#!/usr/bin/env python3
"""Benchmark of the ResidualQuant decode step on B200.

One step = one decode step of the 16k-context Ouro-like workload: for each of
24 layers and 4 loops, compressed decode attention for every sequence of the
batch (96 launches), then the quantise-and-append of the new token's K/V for
every loop of every layer (anchor + 3 LS residuals, K and V: 192 launches).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rq|reference]

Prints one JSON line (rank 0).  --impl reference times the CPU oracle on a
bounded sample of the same workload.  Under torchrun (N > 1) every rank runs
the full per-GPU workload on its own sequences (weak scaling; (batch, head)
units are independent, so no collective touches the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import residual_bit_kv_b200.synth as synth  # noqa: E402

METRIC = "decode-attn tokens/s at 16k ctx"
WORKLOAD = "ouro_16k"
QUANT_WORKLOAD = "quantize_prefill"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------- plumbing --

PREHEAT_SECONDS = 2.0   # untimed replays of the step before the timed regions


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(ws, backend="nccl"):
    """One process per GPU (torchrun env); None for a single process."""
    if ws <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, dist, device) -> float:
    """The largest of every rank's value (each rank calls this at the same
    point); the value itself for a single process."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_share(w, rank: int, world: int):
    """This rank's rows of the job: the job decodes a global batch of
    world * w.batch sequences and rank r takes rows [r*B/N, (r+1)*B/N), so
    per-GPU work stays fixed as N grows (weak scaling) and every rank's
    inputs are rows of one workload, not a re-seeded copy."""
    return synth.partition(w.replace(batch=w.batch * world), rank, world)


def job_tokens_per_s(world_size: int, batch: int, ms_per_step: float) -> float:
    """Whole-job decode throughput: every rank decodes its own batch per step
    (weak scaling), the step time being the slowest rank's."""
    return world_size * batch * 1e3 / ms_per_step


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs:
    NVML every 10 ms from a thread (the device found by PCI bus id), else
    nvidia-smi every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None
        self.thread = None
        self.stop = None
        self.samples = []   # (sm_mhz, reasons bitmask)
        self.max_mhz = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            devid = getattr(props, "pci_device_id", 0)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{devid:02x}.0")
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.stop = threading.Event()

            def run():
                while not self.stop.is_set():
                    try:
                        self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                             int(reasons(h))))
                    except Exception:
                        pass
                    time.sleep(0.01)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
        except Exception:
            self._start_smi()
        time.sleep(0.05)
        return self

    def _start_smi(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.thread is not None:
            if not self.samples:
                return None
            reasons = sorted(n for n, bit in self.REASON_BITS.items()
                             if any(r & bit for _, r in self.samples))
            return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                    "sm_max_mhz": self.max_mhz, "reasons": reasons,
                    "samples": len(self.samples), "source": "nvml 10 ms"}
        if self.path is None or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi 200 ms"}


def file_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


DECODE_SOURCES = ("rq_decode_fast.cu", "rq_decode_common.cuh", "rq_internal.cuh")


def sources_sha(files) -> str:
    """sha256 over the kernel's source files (in the given order)."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "residual_bit_kv_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profile_traffic(files, profile_name: str):
    """Per-launch DRAM traffic from a committed ncu summary, if it was taken on
    the kernel sources as they stand (else None)."""
    path = os.path.join(ROOT, "profiles", profile_name)
    try:
        txt = open(path).read()
    except OSError:
        return None
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not m_sha or not m_tr:
        return None
    if m_sha.group(1) != sources_sha(files):
        return None
    return float(m_tr.group(1))


# ----------------------------------------------------------- byte accounting --

def policy_chain(L, loop, policy):
    """Loops read to rebuild `loop`: itself, then its references up to the
    anchor (loop L-1 for Last-/Next-loop, loop 0 for First-/Previous-loop)."""
    A = L - 1 if policy in ("last", "next") else 0
    comps = [loop]
    r = loop
    while r != A:
        r = A if policy in ("last", "first") else (r + 1 if policy == "next" else r - 1)
        comps.append(r)
    return comps, A


def component_bytes_per_row(w, loop, policy="last", meta_bytes=4):
    """Packed bytes of one (token, head) row of every component loop `loop`
    reads, for one side (codes + metadata (fp16 scale/offset: 4 bytes per
    group; 16-bit metadata: 2) + bf16 LS coefficient)."""
    D = w.head_dim
    comps, A = policy_chain(w.loops, loop, policy)
    tot = 0
    for r in comps:
        tot += D * w.bits[r] // 8 + (D // w.group[r]) * meta_bytes + (2 if r != A else 0)
    return tot


def decode_call_bytes(w, loop, seq_len, policy="last", meta_bytes=4):
    """Algorithmic bytes of one decode call: packed K and V of every past
    token, plus q, k_cur, v_cur (bf16) and the fp32 output."""
    bh = w.batch * w.heads
    return bh * (2 * seq_len * component_bytes_per_row(w, loop, policy, meta_bytes) +
                 w.head_dim * (2 * 3 + 4))


def quant_call_bytes(w, loop, n):
    """Algorithmic bytes of one quantise call over n tokens: the bf16 input,
    the packed output, and for a residual the packed anchor re-read."""
    rows = w.batch * w.heads * n
    D = w.head_dim
    A = w.loops - 1
    out = D * w.bits[loop] // 8 + (D // w.group[loop]) * 4 + (2 if loop != A else 0)
    ref = 0 if loop == A else D * w.bits[A] // 8 + (D // w.group[A]) * 4
    return rows * (2 * D + out + ref)


def quant_loops_bytes(w, n):
    """Algorithmic bytes of one fused call (every loop, one side) over n tokens:
    the bf16 input of every loop and the packed output; nothing is re-read."""
    rows = w.batch * w.heads * n
    D = w.head_dim
    A = w.loops - 1
    return rows * sum(2 * D + D * w.bits[l] // 8 + (D // w.group[l]) * 4 + (2 if l != A else 0)
                      for l in range(w.loops))


# --------------------------------------------------------------- rq engine --

class Engine:
    """Resident packed caches of every layer plus the step's inputs."""

    def __init__(self, w, device, keep_bf16_layers=0):
        import residual_bit_kv_b200.librq as L
        self.L = L
        self.w = w
        self.dev = device
        T = w.tokens
        self.lay = L.make_layout(w.layers, w.loops, w.batch, w.heads, w.head_dim, T + 16,
                                 w.bits, w.group, L.RQ_POLICY_LAST_LOOP)
        nb = L.rq_cache_bytes(self.lay)
        self.kbuf = torch.empty(nb, dtype=torch.uint8, device=device)
        self.vbuf = torch.empty(nb, dtype=torch.uint8, device=device)
        self.cache = L.rq_cache_bind(self.lay, self.kbuf, self.vbuf)
        self.bf16 = {}
        for layer in range(w.layers):
            for side in (0, 1):
                xs = {}
                for loop in [w.loops - 1] + list(range(w.loops - 2, -1, -1)):
                    x = synth.kv_full(w, layer, side, loop, 0, T, device=device, chunk_b=4)
                    if loop == w.loops - 1:
                        L.rq_quantize_anchor(self.cache, layer, side, x, 0, T)
                    else:
                        L.rq_quantize_append_residual(self.cache, layer, side, loop, x, 0, T)
                    if layer < keep_bf16_layers:
                        xs[loop] = x
                    else:
                        del x
                for loop, x in xs.items():
                    # bf16 baseline buffer [B, H, T+16, D] with room for the appended token
                    buf = torch.empty(w.batch, w.heads, T + 16, w.head_dim, dtype=torch.bfloat16,
                                      device=device)
                    buf[:, :, :T] = x
                    self.bf16[(layer, side, loop)] = buf
                del xs
            torch.cuda.synchronize(device)
        # step inputs: per (layer, loop) query, and the current token's K/V of
        # every loop of a layer stacked [L, B, H, D] (the append's input)
        self.q, self.kc, self.vc = {}, {}, {}
        self.kc_layer, self.vc_layer = [], []
        for layer in range(w.layers):
            kcl = torch.stack([synth.current_token(w, layer, 0, loop, device)
                               for loop in range(w.loops)]).contiguous()
            vcl = torch.stack([synth.current_token(w, layer, 1, loop, device)
                               for loop in range(w.loops)]).contiguous()
            self.kc_layer.append(kcl)
            self.vc_layer.append(vcl)
            for loop in range(w.loops):
                self.q[(layer, loop)] = synth.query(w, layer, loop, device).contiguous()
                self.kc[(layer, loop)] = kcl[loop]
                self.vc[(layer, loop)] = vcl[loop]
        self.seq = torch.full((w.batch,), T, dtype=torch.int32, device=device)
        self.out = torch.empty(w.layers, w.loops, w.batch, w.heads, w.head_dim,
                               dtype=torch.float32, device=device)
        self.ws_bytes = L.rq_decode_workspace_bytes(self.lay, T)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        L.rq_decode_workspace_init(self.ws, self.ws_bytes)
        self.bws_bytes = L.rq_decode_bf16_workspace_bytes(w.batch, w.heads, w.head_dim, T)
        self.bws = torch.zeros(self.bws_bytes, dtype=torch.uint8, device=device)
        torch.cuda.synchronize(device)

    def launches_per_step(self):
        w = self.w
        return w.layers * w.loops + w.layers

    def step(self, stream, ev=None, q=None, kc_layer=None, vc_layer=None, loops=None,
             appends=True, side=None):
        """One decode step of the looped model, in its own order: loop 1 runs
        every layer, then loop 2 every layer, ..., so each (layer, loop) decode
        call sees the query of its loop; after the final loop of a layer, one
        launch quantises and appends the new token of every loop of that
        layer, K and V.  ev: optional list collecting (start, end) event pairs
        around each decode-attention launch.  loops / appends=False select a
        part of the step (the roofline's kernel-only timings).  side: a second
        stream for the appends; each waits for its layer's final-loop decode
        and runs beside the next layers' (it writes position T, which no
        decode call of this step reads), and the step ends when both streams
        have."""
        L, w, T = self.L, self.w, self.w.tokens
        q = q or self.q
        kcl = kc_layer or self.kc_layer
        vcl = vc_layer or self.vc_layer
        final = w.loops - 1
        if side is not None:
            side.wait_stream(stream)
        for loop in (range(w.loops) if loops is None else loops):
            for layer in range(w.layers):
                if ev is not None:
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                L.rq_decode_attention(self.cache, layer, loop, q[(layer, loop)], self.seq, T,
                                      kcl[layer][loop], vcl[layer][loop], 0.0,
                                      self.out[layer, loop], self.ws, self.ws_bytes, stream)
                if ev is not None:
                    e1.record(stream)
                    ev.append((e0, e1, loop))
                if loop != final or not appends:
                    continue
                # after the final loop: quantise and append the new token (position T)
                if side is None:
                    L.rq_quantize_append_loops(self.cache, layer, kcl[layer], vcl[layer], T, 1,
                                               stream)
                else:
                    side.wait_stream(stream)
                    L.rq_quantize_append_loops(self.cache, layer, kcl[layer], vcl[layer], T, 1,
                                               side)
        if side is not None:
            stream.wait_stream(side)

    def bf16_step(self, stream, ev=None, nlayers_buf=4):
        """The same step on the uncompressed bf16 cache (loop-major, as step())."""
        L, w, T = self.L, self.w, self.w.tokens
        for loop in range(w.loops):
            for layer in range(w.layers):
                lb = layer % nlayers_buf
                k = self.bf16[(lb, 0, loop)]
                v = self.bf16[(lb, 1, loop)]
                if ev is not None:
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                L.rq_decode_attention_bf16(w.batch, w.heads, w.head_dim, self.q[(layer, loop)], k,
                                           v, T + 16, self.seq, T, self.kc[(layer, loop)],
                                           self.vc[(layer, loop)], 0.0, self.out[layer, loop],
                                           self.bws, self.bws_bytes, stream)
                if ev is not None:
                    e1.record(stream)
                    ev.append((e0, e1, loop))
                if loop == w.loops - 1:
                    for lp in range(w.loops):
                        self.bf16[(lb, 0, lp)][:, :, T].copy_(self.kc[(layer, lp)], non_blocking=True)
                        self.bf16[(lb, 1, lp)][:, :, T].copy_(self.vc[(layer, lp)], non_blocking=True)


def timed(fn, steps, warmup, stream, dist=None):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dist, "cuda")
    if dist is not None:
        dist.barrier()
    return ms


# --------------------------------------------------------- oracle (CPU) legs --

def oracle_prepare(w, b, h):
    """Set-up of one (batch, head) unit of layer 0 for the oracle: the unit's
    K/V rows of every loop generated and encoded (not timed)."""
    import oracle
    T, D = w.tokens, w.head_dim
    encs = {}
    for side in (0, 1):
        cs = synth.key_channel_scale(w, 0) if side == 0 else None
        xl = [synth.bits_of(synth.kv(w, 0, side, loop, [b], [h], 0, T, "cpu", cs)).reshape(-1, D)
              for loop in range(w.loops)]
        encs[side] = oracle.encode_side(np.stack(xl), w.bits, w.group)
    return encs


def oracle_run(w, b, h, encs, loops, q, kc, vc):
    """The oracle's decode of one unit for `loops`: reconstruction of every
    past row in fp64 and exact softmax attention (the timed work)."""
    import oracle
    T, D = w.tokens, w.head_dim
    for loop in loops:
        kh = oracle.reconstruct(encs[0], loop, w.bits, w.group).reshape(T, D)
        vh = oracle.reconstruct(encs[1], loop, w.bits, w.group).reshape(T, D)
        oracle.attention(oracle.bf16_bits_to_f64(q[loop, b, h]), kh, vh,
                         oracle.bf16_bits_to_f64(kc[loop][b, h]),
                         oracle.bf16_bits_to_f64(vc[loop][b, h]), 1.0 / np.sqrt(D))
    return len(loops)


def step_inputs_cpu(w, loops):
    q = synth.bits_of(torch.stack([synth.query(w, 0, l) for l in range(w.loops)]))
    kc = {l: synth.bits_of(synth.current_token(w, 0, 0, l)) for l in loops}
    vc = {l: synth.bits_of(synth.current_token(w, 0, 1, l)) for l in loops}
    return q, kc, vc


def oracle_decode_sample(w, pairs, loops, budget_s=None):
    """Times the oracle's decode of (b, h) units for `loops` of layer 0.
    Pairs are taken in order until `budget_s` seconds of timed work (all of
    them if None).  Encoding a pair's cache is set-up, not timed."""
    q, kc, vc = step_inputs_cpu(w, loops)
    secs, units = 0.0, 0
    for b, h in pairs:
        encs = oracle_prepare(w, b, h)
        t0 = time.perf_counter()
        units += oracle_run(w, b, h, encs, loops, q, kc, vc)
        secs += time.perf_counter() - t0
        if budget_s is not None and secs >= budget_s:
            break
    return secs, units


CPU_SAMPLE_SECONDS = 10.0
CPU_POOL_MAX_WORKERS = 64


def _pool_worker(args):
    """One oracle process (one torch thread): set-up (generation and encoding
    of its unit) untimed, then a barrier, then the timed decode of its unit
    for every loop.  Returns its timed window."""
    name, (b, h), loops, barrier = args
    torch.set_num_threads(1)
    w = synth.WORKLOADS[name]
    q, kc, vc = step_inputs_cpu(w, loops)
    encs = oracle_prepare(w, b, h)
    oracle_run(w, b, h, encs, loops[:1], q, kc, vc)   # warm: library load, page-in
    barrier.wait()
    t0 = time.perf_counter()
    units = oracle_run(w, b, h, encs, loops, q, kc, vc)
    t1 = time.perf_counter()
    return t0, t1, units


def cpu_baseline_all_cores(w):
    """The oracle's decode as independent processes on every host core
    (capped at CPU_POOL_MAX_WORKERS): one (batch, head) unit of layer 0 per
    process, every loop, each unit single-threaded; throughput = units / wall
    time of the timed windows.  (The whole layer would take several minutes of
    set-up on the host, outside the benchmark's time budget; this is a
    bounded sample of it.)"""
    import multiprocessing as mp
    ncpu = os.cpu_count() or 1
    workers = max(1, min(ncpu, CPU_POOL_MAX_WORKERS, w.batch * w.heads))
    pairs = [(i % w.batch, (5 * i) % w.heads) for i in range(workers)]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as man:
        barrier = man.Barrier(workers)
        with ctx.Pool(workers) as pool:
            res = pool.map(_pool_worker, [(w.name, pr, list(range(w.loops)), barrier)
                                          for pr in pairs])
    t0 = min(r[0] for r in res)
    t1 = max(r[1] for r in res)
    units = sum(r[2] for r in res)
    step_units = w.layers * w.loops * w.batch * w.heads
    step_s = (t1 - t0) / units * step_units
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    call_units = w.batch * w.heads   # one decode call = one loop of one layer
    return {"value": w.batch / step_s, "unit": "tokens/s", "cores": workers, "nproc": ncpu,
            "cpu_model": model, "kind": "oracle",
            "ms_per_call": (t1 - t0) / units * call_units * 1e3,
            "sample": f"{units} (batch,head,loop) decode units of layer 0 at T={w.tokens}, one "
                      f"(batch,head) per process ({t1 - t0:.1f} s wall on {workers} processes), "
                      f"scaled to {step_units} units per step ({call_units} per call)"}


def cpu_baseline(w):
    """Oracle decode on a bounded sample: (batch, head) units x 4 loops of
    layer 0 at the full 16k context until about 10 s of timed CPU work,
    scaled to the step's 24*4*B*H units."""
    pairs = [(i % w.batch, (5 * i) % w.heads) for i in range(w.batch * w.heads)]
    secs, units = oracle_decode_sample(w, pairs, list(range(w.loops)), CPU_SAMPLE_SECONDS)
    step_units = w.layers * w.loops * w.batch * w.heads
    step_s = secs / units * step_units
    return {"value": w.batch / step_s, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{units} (batch,head,loop) decode units of layer 0 at T={w.tokens} "
                      f"({secs:.1f} s timed), scaled to {step_units} units per step"}


def run_reference(args, rank):
    if rank != 0:
        return 0
    w = synth.WORKLOADS[WORKLOAD]
    pairs = [(0, 0)]
    for _ in range(args.warmup):
        oracle_decode_sample(w, pairs, [w.loops - 1])
    times = []
    for _ in range(args.steps):
        secs, units = oracle_decode_sample(w, pairs, [0])
        times.append(secs / units)
    per_unit = statistics.median(times)
    step_units = w.layers * w.loops * w.batch * w.heads
    step_s = per_unit * step_units
    value = w.batch / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded counter-based generator)",
        "config": config_of(w, max(1, args.gpus)),
        "extrapolated": ("ms_per_step is not a measured step: each timed sample decodes one "
                         "(batch, head) unit of loop 0 and the median time per unit is scaled "
                         f"to the {step_units} units of one step"),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": "per step: 1 (batch,head) unit of loop 0, layer 0 at T=16384, "
                                   f"scaled to {step_units} units"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_of(w, world=1):
    par = ("one GPU" if world == 1 else
           f"batch partition over {world} GPUs: rank r decodes batch rows "
           f"[{w.batch}r, {w.batch}r+{w.batch}) of one global batch; no collective on the path")
    return {"workload": f"{w.name}: {w.layers} layers x {w.loops} loops, batch {w.batch} per GPU, "
                        f"{w.heads} KV heads, head_dim {w.head_dim}, {w.tokens} past tokens, "
                        f"bits {list(w.bits)}, group {w.group[0]}, Last-loop anchor",
            "global_batch": w.batch * world, "seq_len": w.tokens,
            "l2": "inputs larger than L2: every decode call streams >= 0.67 GB of packed KV",
            "parallelism": par}


# --------------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="rq", choices=["rq", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--no-bf16", action="store_true", help="skip the BF16 baseline kernel")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers (default 24); smaller values give a profiling-sized case")
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per step (default 16); smaller values give a profiling-sized case")
    ap.add_argument("--no-quant", action="store_true", help="skip the prefill quantise leg")
    ap.add_argument("--no-ablation", action="store_true",
                    help="skip the shared-vs-chained deep-recurrence decode ablation")
    ap.add_argument("--only-dense", action="store_true",
                    help="run only the dense-rotation leg on one 16k layer and print its numbers "
                         "(profiling; --batch then sets its batch)")
    ap.add_argument("--only-quant", action="store_true",
                    help="run only the prefill quantise leg and print its numbers (profiling; "
                         "--batch then sets its batch)")
    args = ap.parse_args()
    ws, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank)
    dist = init_dist(ws)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from residual_bit_kv_b200 import build
    build.build()
    if args.only_dense:
        wd = synth.WORKLOADS[WORKLOAD].replace(layers=1)
        if args.batch:
            wd = wd.replace(batch=args.batch)
        print(json.dumps({"dense_rotation": bench_dense(wd, dev, torch.cuda.current_stream(dev),
                                                        args, peaks()[0])}))
        return 0
    if args.only_quant:
        print(json.dumps({"quantize": bench_quantize(dev, torch.cuda.current_stream(dev), args,
                                                     peaks()[0])}))
        return 0
    w = synth.WORKLOADS[WORKLOAD]
    if args.layers:
        w = w.replace(layers=args.layers)
    if args.batch:
        w = w.replace(batch=args.batch)
    nbuf = 0 if args.no_bf16 else 4
    eng = Engine(rank_share(w, rank, ws), dev, keep_bf16_layers=nbuf)
    w = eng.w
    stream = torch.cuda.current_stream(dev)

    hbm, hbm_kind = peaks()
    traffic = profile_traffic(DECODE_SOURCES, "decode_kernel_ouro_16k.md")
    cap = torch.cuda.Stream(dev)

    def capture(fn):
        """fn(stream) captured once as a CUDA graph (after one eager run)."""
        g = torch.cuda.CUDAGraph()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            fn(cap)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=cap):
            fn(cap)
        torch.cuda.synchronize()
        return g

    # ---- main timed region: the whole step (96 decode + 24 append launches)
    # captured once as a CUDA graph (no host work or launch gaps) and replayed
    side = torch.cuda.Stream(dev)
    graph = capture(lambda st: eng.step(st, side=side))
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    # bring the GPU to its steady power-capped clock before any timed region,
    # so the step and the kernel-only timings below see the same clocks
    t_end = time.perf_counter() + PREHEAT_SECONDS
    while time.perf_counter() < t_end:
        graph.replay()
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    with ClockSampler(local) as clk:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist, dev)
    clocks = clk.summary()
    del graph

    # ---- the roofline's kernel time: the step's 96 decode launches alone,
    # as one graph (back to back, the appends left out), and each loop's 24
    # launches as its own graph
    dec_bytes = w.layers * sum(decode_call_bytes(w, l, w.tokens) for l in range(w.loops))
    g_dec = capture(lambda st: eng.step(st, appends=False))
    dec_ms = timed(g_dec.replay, args.steps, args.warmup, stream, dist)
    del g_dec
    achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
    per_loop = {}
    for l in range(w.loops):
        g_l = capture(lambda st, l=l: eng.step(st, loops=[l], appends=False))
        t_l = timed(g_l.replay, args.steps, args.warmup, stream, dist) / w.layers
        del g_l
        per_loop[str(l)] = {"us": t_l * 1e3,
                            "gbs": decode_call_bytes(w, l, w.tokens) / (t_l * 1e-3) / 1e9}

    # ---- the same step launched call by call (host launch gaps included)
    eager_ms = timed(lambda: eng.step(stream), args.steps, args.warmup, stream, dist)

    # ---- end to end: host buffers, H2D of the step's inputs, D2H of the outputs
    pin = {k: v.cpu().pin_memory() for k, v in eng.q.items()}
    pkc = [t.cpu().pin_memory() for t in eng.kc_layer]
    pvc = [t.cpu().pin_memory() for t in eng.vc_layer]
    hout = torch.empty(eng.out.shape, dtype=torch.float32).pin_memory()
    dq = {k: torch.empty_like(v) for k, v in eng.q.items()}
    dkc = [torch.empty_like(t) for t in eng.kc_layer]
    dvc = [torch.empty_like(t) for t in eng.vc_layer]

    def copy_in():
        for k in pin:
            dq[k].copy_(pin[k], non_blocking=True)
        for i in range(len(pkc)):
            dkc[i].copy_(pkc[i], non_blocking=True)
            dvc[i].copy_(pvc[i], non_blocking=True)

    def e2e_eager_step():
        copy_in()
        eng.step(stream, None, dq, dkc, dvc)
        hout.copy_(eng.out, non_blocking=True)

    e2e_eager_ms = timed(e2e_eager_step, args.steps, args.warmup, stream, dist)

    # the public-API step on the device input buffers captured once as a CUDA
    # graph, as a serving loop would: per step the inputs are copied in from
    # pinned host memory, the graph replays and the outputs are read back
    graph_io = capture(lambda st: eng.step(st, None, dq, dkc, dvc, side=side))

    def e2e_step():
        copy_in()
        graph_io.replay()
        hout.copy_(eng.out, non_blocking=True)

    e2e_ms = timed(e2e_step, args.steps, args.warmup, stream, dist)
    del graph_io
    h2d = (sum(v.numel() for v in pin.values()) + sum(t.numel() for t in pkc) +
           sum(t.numel() for t in pvc)) * 2
    d2h = hout.numel() * 4

    # ---- BF16 baseline kernel on identical K/V (4 distinct layer buffers cycled)
    bf16 = None
    if not args.no_bf16:
        bev = []
        bms = timed(lambda: eng.bf16_step(stream), args.steps, args.warmup, stream, dist)
        eng.bf16_step(stream, bev)
        torch.cuda.synchronize()
        bdec_ms = sum(a.elapsed_time(b) for a, b, _ in bev)
        bbytes = w.layers * w.loops * w.batch * w.heads * (
            2 * w.tokens * w.head_dim * 2 + w.head_dim * (2 * 3 + 4))
        bf16 = {"tokens_per_s": w.batch * 1e3 / bms, "ms_per_step": bms,
                "decode_gbs": bbytes / (bdec_ms * 1e-3) / 1e9,
                "frac_of_hbm": bbytes / (bdec_ms * 1e-3) / 1e9 / hbm,
                "bytes_per_step": bbytes,
                "note": "same split-K engine on uncompressed bf16 K/V; 4 distinct layer buffers"}

    # ---- prefill-sized quantise (anchor + 3 residuals, K and V), separate workload
    splits0 = eng.L.rq_decode_splits(eng.lay, w.tokens)
    launches = args.steps * eng.launches_per_step()
    quant = None
    if not args.no_quant:
        quant = bench_quantize(dev, stream, args, hbm)
    ablation = None
    if not args.no_ablation:
        del eng
        torch.cuda.empty_cache()
        ablation = bench_ablation(dev, stream, args, hbm)

    cpu = cpu_all = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        cpu = cpu_baseline(w)
        cpu_all = cpu_baseline_all_cores(w)

    if rank == 0:
        value = job_tokens_per_s(ws, w.batch, ms)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded counter-based generator; Ouro-like looped KV)",
            "config": config_of(w, ws),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "traffic": traffic,
                         "kernel": "decode_fast_kernel (all loops of the step)", "peak_kind": hbm_kind,
                         "bytes_per_step": dec_bytes,
                         "kernel_time": ("CUDA events around a graph of the step's "
                                         f"{w.layers * w.loops} decode launches replayed "
                                         f"back to back: {dec_ms:.3f} ms per step")},
            "decode_per_loop": per_loop,
            "step_launch": {"timed": f"one CUDA graph per step ({w.layers * w.loops} decode + "
                                     f"{w.layers} append launches in the looped model's order: "
                                     "loop 1 over every layer, then loop 2, ...; each append on a "
                                     "second stream after its layer's final-loop decode, joined "
                                     "at the end of the step)",
                            "timed_launch_count": w.layers * w.loops + w.layers,
                            "eager_ms_per_step": eager_ms,
                            "eager_tokens_per_s": job_tokens_per_s(ws, w.batch, eager_ms)},
            "decode_splits_loop0": splits0,
            "decode_hbm_frac_of_8tbs": achieved / 8000.0,
            "e2e": {"value": job_tokens_per_s(ws, w.batch, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "path": "public API step captured as a CUDA graph on device input buffers; "
                            "per step: H2D of the inputs from pinned host memory, replay, D2H "
                            "of the output",
                    "eager_value": job_tokens_per_s(ws, w.batch, e2e_eager_ms)},
            "gpu_launches": launches,
            "clocks": clocks,
            "bf16_baseline": bf16,
            "quantize": quant,
            "ablation_shared_vs_chained": ablation,
            "cpu_baseline": cpu,
            "cpu_baseline_all_cores": cpu_all,
        }
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


POLICY_NAMES = ("last", "next", "first", "previous")


def random_rotations(w, seed):
    """Binary16 orthogonal matrices [1, H, D, D] per side (QR of Gaussians):
    stand-ins for calibrated rotations, which need model activations."""
    import numpy as np
    rng = np.random.default_rng(seed)
    rot = {}
    for side in (0, 1):
        m = np.zeros((1, w.heads, w.head_dim, w.head_dim), np.float16)
        for h in range(w.heads):
            q, r = np.linalg.qr(rng.standard_normal((w.head_dim, w.head_dim)))
            m[0, h] = (q * np.sign(np.diag(r))).astype(np.float16)
        rot[side] = torch.from_numpy(m)
    return rot


def policy_decode_step(w, policy, dev, stream, args, meta16=False, dense=False):
    """One layer of workload w stored under `policy` (16-bit metadata per
    group if meta16; dense binary16 rotations instead of the Hadamard
    transform if dense): the time of a decode step over every loop (one call
    per loop), its algorithmic bytes, the component reads, and the time of the
    fused prefill append of both sides."""
    import residual_bit_kv_b200.librq as L
    T = w.tokens
    code = {"last": L.RQ_POLICY_LAST_LOOP, "next": L.RQ_POLICY_NEXT_LOOP,
            "first": L.RQ_POLICY_FIRST_LOOP, "previous": L.RQ_POLICY_PREVIOUS_LOOP}[policy]
    lay = L.make_layout(1, w.loops, w.batch, w.heads, w.head_dim, T + 16, w.bits, w.group, code,
                        L.RQ_FLAG_META16 if meta16 else 0)
    nb = L.rq_cache_bytes(lay)
    kb = torch.empty(nb, dtype=torch.uint8, device=dev)
    vb = torch.empty(nb, dtype=torch.uint8, device=dev)
    cache = L.rq_cache_bind(lay, kb, vb)
    rot = None
    if dense:
        rot = {k: v.to(dev) for k, v in random_rotations(w, 7).items()}
        L.rq_cache_set_rotations(cache, rot[0], rot[1])
    xk = torch.stack([synth.kv_full(w, 0, 0, loop, 0, T, device=dev, chunk_b=2)
                      for loop in range(w.loops)])
    xv = torch.stack([synth.kv_full(w, 0, 1, loop, 0, T, device=dev, chunk_b=2)
                      for loop in range(w.loops)])
    prefill_ms = timed(lambda: L.rq_quantize_append_loops(cache, 0, xk, xv, 0, T, stream),
                       max(1, args.steps // 2), args.warmup, stream)
    torch.cuda.synchronize()
    del xk, xv
    q = [synth.query(w, 0, l, dev).contiguous() for l in range(w.loops)]
    kc = [synth.current_token(w, 0, 0, l, dev).contiguous() for l in range(w.loops)]
    vc = [synth.current_token(w, 0, 1, l, dev).contiguous() for l in range(w.loops)]
    seq = torch.full((w.batch,), T, dtype=torch.int32, device=dev)
    o = torch.empty(w.batch, w.heads, w.head_dim, dtype=torch.float32, device=dev)
    wsb = L.rq_decode_workspace_bytes(lay, T)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    L.rq_decode_workspace_init(ws, wsb, stream)

    def step():
        for loop in range(w.loops):
            L.rq_decode_attention(cache, 0, loop, q[loop], seq, T, kc[loop], vc[loop], 0.0, o,
                                  ws, wsb, stream)

    ms = timed(step, args.steps, args.warmup, stream)
    byt = sum(decode_call_bytes(w, l, T, policy, meta_bytes=2 if meta16 else 4)
              for l in range(w.loops))
    reads = sum(len(policy_chain(w.loops, l, policy)[0]) for l in range(w.loops))
    del kb, vb, ws, rot
    torch.cuda.empty_cache()
    return ms, byt, reads, prefill_ms


def bench_ablation(dev, stream, args, hbm):
    """Reference-policy ablation [RQ §3.2, §5.2, App. D]: decode steps of one
    layer under the shared anchors (Last-/First-loop) and the chains
    (Next-/Previous-loop).  (1) the deep-recurrence workload (8 loops, batch
    32, 40 heads, 8192 tokens, g 64): shared final-loop anchor vs the Next-loop
    chain; (2) one layer of the 16k-context Ouro-like workload (4 loops, batch
    16, 16 heads, 16384 tokens, g 32) under all four policies, the higher
    precision on the anchor loop ([2,2,2,4] for Last/Next, [4,2,2,2] for
    First/Previous, as in the pages' policy comparison)."""
    w = synth.WORKLOADS["huginn_deep"]
    T = w.tokens
    out = {"workload": f"{w.name}: 1 layer x {w.loops} loops, batch {w.batch}, {w.heads} heads, "
                       f"{T} past tokens, bits {list(w.bits)}, group {w.group[0]}"}
    for policy, name in (("last", "shared"), ("next", "chained")):
        ms, byt, reads, _ = policy_decode_step(w, policy, dev, stream, args)
        out[name] = {"ms_per_step": ms, "bytes_per_step": byt,
                     "gbs": byt / (ms * 1e-3) / 1e9, "frac_of_hbm": byt / (ms * 1e-3) / 1e9 / hbm,
                     "component_reads": reads}
    out["speedup_shared_over_chained"] = out["chained"]["ms_per_step"] / out["shared"]["ms_per_step"]
    out["bytes_ratio_chained_over_shared"] = (out["chained"]["bytes_per_step"] /
                                              out["shared"]["bytes_per_step"])
    wo = synth.WORKLOADS["ouro_16k"].replace(layers=1, bits=(2, 2, 2, 4))
    pol = {"workload": f"{wo.name}: 1 layer x {wo.loops} loops, batch {wo.batch}, {wo.heads} "
                       f"heads, {wo.tokens} past tokens, group {wo.group[0]}"}
    for policy in POLICY_NAMES:
        bits = tuple(wo.bits) if policy in ("last", "next") else tuple(wo.bits)[::-1]
        wp = wo.replace(bits=bits)
        ms, byt, reads, _ = policy_decode_step(wp, policy, dev, stream, args)
        pol[policy] = {"bits": list(bits), "ms_per_step": ms, "bytes_per_step": byt,
                       "gbs": byt / (ms * 1e-3) / 1e9, "component_reads": reads}
    pol["throughput_last_over_previous"] = pol["previous"]["ms_per_step"] / pol["last"]["ms_per_step"]
    pol["throughput_first_over_previous"] = (pol["previous"]["ms_per_step"] /
                                             pol["first"]["ms_per_step"])
    out["policies_ouro_16k_layer"] = pol
    # 16-bit metadata per group (the pages' accounting) on the same layer
    wm = synth.WORKLOADS["ouro_16k"].replace(layers=1)
    m16 = {"workload": f"{wm.name}: 1 layer x {wm.loops} loops, batch {wm.batch}, {wm.heads} "
                       f"heads, {wm.tokens} past tokens, bits {list(wm.bits)}, group {wm.group[0]}"}
    for name, flag in (("meta32", False), ("meta16", True)):
        ms, byt, _, _ = policy_decode_step(wm, "last", dev, stream, args, meta16=flag)
        mb = 2 if flag else 4
        m16[name] = {"ms_per_step": ms, "bytes_per_step": byt, "gbs": byt / (ms * 1e-3) / 1e9,
                     "frac_of_hbm": byt / (ms * 1e-3) / 1e9 / hbm,
                     "tokens_per_s_layer": wm.batch / (ms * 1e-3),
                     "bytes_per_token_head_per_loop": [
                         2 * component_bytes_per_row(wm, l, "last", mb) for l in range(wm.loops)],
                     "bits_per_element": [
                         8 * (component_bytes_per_row(wm, l, "last", mb) -
                              (component_bytes_per_row(wm, wm.loops - 1, "last", mb)
                               if l != wm.loops - 1 else 0)) / wm.head_dim
                         for l in range(wm.loops)]}
    m16["speedup_meta16_over_meta32"] = m16["meta32"]["ms_per_step"] / m16["meta16"]["ms_per_step"]
    out["metadata16_ouro_16k_layer"] = m16
    out["dense_rotation_ouro_16k_layer"] = bench_dense(wm, dev, stream, args, hbm)
    return out


def bench_dense(wm, dev, stream, args, hbm):
    """Dense binary16 rotations (tensor-core product) against the Hadamard
    transform on one layer of workload wm: the decode step over every loop and
    the fused prefill append of every loop, K and V."""
    dn = {"workload": f"{wm.name}: 1 layer x {wm.loops} loops, batch {wm.batch}, {wm.heads} "
                      f"heads, {wm.tokens} past tokens, bits {list(wm.bits)}, group {wm.group[0]}",
          "note": "random orthogonal binary16 matrices per head and side stand in for calibrated "
                  "rotations; prefill = fused append of every loop, K and V"}
    for name, flag in (("hadamard", False), ("dense", True)):
        ms, byt, _, pms = policy_decode_step(wm, "last", dev, stream, args, dense=flag)
        qb = 2 * quant_loops_bytes(wm, wm.tokens)
        dn[name] = {"decode_ms_per_step": ms, "decode_gbs": byt / (ms * 1e-3) / 1e9,
                    "decode_frac_of_hbm": byt / (ms * 1e-3) / 1e9 / hbm,
                    "prefill_ms": pms, "prefill_gbs": qb / (pms * 1e-3) / 1e9,
                    "prefill_frac_of_hbm": qb / (pms * 1e-3) / 1e9 / hbm}
    return dn


def bench_quantize(dev, stream, args, hbm):
    """Quantise-and-append of a 16k-token prefill: anchor then 3 residual loops,
    for K and V (8 launches per pass).  Reports input GB/s and the fraction of
    HBM for the bytes the pass must move."""
    import residual_bit_kv_b200.librq as L
    w = synth.WORKLOADS[QUANT_WORKLOAD]
    if args.only_quant and args.batch:
        w = w.replace(batch=args.batch)
    T = w.tokens
    lay = L.make_layout(1, w.loops, w.batch, w.heads, w.head_dim, T, w.bits, w.group,
                        L.RQ_POLICY_LAST_LOOP)
    nb = L.rq_cache_bytes(lay)
    kb = torch.empty(nb, dtype=torch.uint8, device=dev)
    vb = torch.empty(nb, dtype=torch.uint8, device=dev)
    cache = L.rq_cache_bind(lay, kb, vb)
    xs = {(s, l): synth.kv_full(w, 0, s, l, 0, T, device=dev, chunk_b=1)
          for s in (0, 1) for l in range(w.loops)}
    ev = []

    def one(record=False):
        for s in (0, 1):
            for l in [w.loops - 1] + list(range(w.loops - 2, -1, -1)):
                if record:
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                if l == w.loops - 1:
                    L.rq_quantize_anchor(cache, 0, s, xs[(s, l)], 0, T, stream)
                else:
                    L.rq_quantize_append_residual(cache, 0, s, l, xs[(s, l)], 0, T, stream)
                if record:
                    b.record(stream)
                    ev.append((a, b, l))

    ms = timed(one, args.steps, args.warmup, stream)
    one(True)
    torch.cuda.synchronize()
    # every loop of both sides in one launch (rq_quantize_append_loops)
    xk = torch.stack([xs[(0, l)] for l in range(w.loops)]).contiguous()
    xv = torch.stack([xs[(1, l)] for l in range(w.loops)]).contiguous()
    del xs
    fused_ms = timed(lambda: L.rq_quantize_append_loops(cache, 0, xk, xv, 0, T, stream),
                     args.steps, args.warmup, stream)
    fused_bytes = 2 * quant_loops_bytes(w, T)
    inp = 2 * w.loops * w.batch * w.heads * T * w.head_dim * 2
    req = 2 * sum(quant_call_bytes(w, l, T) for l in range(w.loops))
    kern_ms = sum(a.elapsed_time(b) for a, b, _ in ev)
    res_ms = sum(a.elapsed_time(b) for a, b, l in ev if l != w.loops - 1)
    res_bytes = 2 * sum(quant_call_bytes(w, l, T) for l in range(w.loops - 1))
    return {"workload": f"{w.name}: batch {w.batch}, {w.heads} heads, {T} tokens, {w.loops} loops, "
                        f"bits {list(w.bits)}, g {w.group[0]}, K and V",
            "ms_per_pass": ms, "input_gbs": inp / (ms * 1e-3) / 1e9,
            "required_gbs": req / (kern_ms * 1e-3) / 1e9,
            "frac_of_hbm": req / (kern_ms * 1e-3) / 1e9 / hbm,
            "residual_kernel_gbs": res_bytes / (res_ms * 1e-3) / 1e9,
            "residual_codes_per_pass": 2 * (w.loops - 1) * w.batch * w.heads * T * w.head_dim,
            "fused": {"ms_per_pass": fused_ms, "bytes_per_pass": fused_bytes,
                      "gbs": fused_bytes / (fused_ms * 1e-3) / 1e9,
                      "frac_of_hbm": fused_bytes / (fused_ms * 1e-3) / 1e9 / hbm,
                      "note": "every loop, K and V, one launch; the anchor is not re-read"}}


if __name__ == "__main__":
    sys.exit(main())
