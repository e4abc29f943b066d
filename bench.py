#!/usr/bin/env python
"""Benchmark of the paged decode step (KV append + paged decode attention).

The default line is the 16-layer continuous-batching trace (C5): 256 live
sequences of the Llama-3.2-1B attention shape (Hq=32, Hkv=8, head_dim 64, block
size 16) with lognormal lengths, each step appending one token per sequence and
running paged decode attention in every layer (pa_append_decode per layer;
the 100-step trace, with sequences finishing and being replaced, replayed as
often as --steps asks).  A step is one decode step of all 16 layers; the 16
layer pools (about 7.5 GB) keep the 126 MB L2 from serving the K/V reads.

Prints one JSON line (rank 0).  `value` is seq-steps/s over all ranks with
inputs resident in HBM; `e2e` repeats the measurement through the host block
manager, with each step's inputs copied up from pinned host memory in one copy
and the outputs copied back in one, inside the timed region.  `roofline`
reports the decode kernel's KV-read bandwidth against the measured HBM copy
bandwidth.  `cpu_baseline` times the fp64 CPU oracle on a bounded sample.
`also` carries the other decode workloads of the same run (C2, C3, C4; bf16
and E4M3 pools), device-timed the same way.  --config c1..c4 / pc / pf measure
one other workload as the line itself.  With --impl reference the oracle alone
is timed.

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
path has no exchange step); the timed region is bracketed by barriers and the
max over ranks is reported (weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "paged-decode seq-steps/s and KV-read HBM GB/s (fraction of B200 peak)"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0

WORKLOAD_TEXT = {
    "c1": "tiny: B=2, L=5/37 (+1 appended), Hq=2, Hkv=1, D=64, Bs=16, 8 blocks",
    "c2": "Llama-3.2-1B-shaped decode layer: B=64, Hq=32, Hkv=8, D=64, Bs=16, cached L~U[128,2048] (+1 appended), pool=needed+10%",
    "c3": "shared 1024-token prefix (4 blocks in every table) + suffix~U[256,7168] (+1), B=32, Hq=32, Hkv=8, D=64, Bs=256",
    "c4": "long context split-KV: B=4, L=32768/65536/98304/131072 (+1), Hq=64, Hkv=8, D=128, Bs=16",
    "c5": "continuous-batching trace: 16 layers (own pools), 256 live sequences, lognormal L (median 512, "
          "sigma 1, <=16384), 100 decode steps, finish p=0.01 per step with replacement, Hq=32, Hkv=8, "
          "D=64, Bs=16",
    "pf": "paged chunked prefill, Llama-3.2-1B-shaped layer: 4 sequences, 2048 new tokens each after "
          "0/512/1024/1536 cached, Hq=32, Hkv=8, D=64, Bs=16 (append of the chunk + causal attention)",
    "pc": "prefix caching + copy-on-write: host admission by token ids of 32 C3-shaped requests "
          "(1024-token shared prefix + suffix~U[256,7168], Bs=256); device copy of 8192 random "
          "blocks of the C2 geometry (Hkv=8, Bs=16, D=64) per step",
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: per config, a few hundred ms of device time)")
    ap.add_argument("--warmup", type=int, default=None, help="untimed steps after the settle period")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=["c1", "c2", "c3", "c4", "c5", "pc", "pf"], default="c5",
                    help="c5 (default): the 16-layer continuous-batching trace, one step = all 16 "
                         "layers; pc: prefix caching + copy-on-write (host admission by token ids "
                         "on the C3 request mix, device block copies)")
    ap.add_argument("--no-also", action="store_true",
                    help="c5: skip the C2/C3/C4 (bf16 and E4M3) lines measured after the headline")
    ap.add_argument("--kernel", choices=["auto", "simt", "tensor", "split"], default="auto")
    ap.add_argument("--max-ctas", type=int, default=0)
    ap.add_argument("--prefill-kernel", choices=["auto", "tcgen05", "tcgen05_ws", "mma"], default="auto",
                    help="pf: tcgen05_ws (one job per warp, O in tensor memory; auto), tcgen05 "
                         "(tensor-memory accumulators, one thread issues) or warp-level mma.sync")
    ap.add_argument("--path", choices=["fused", "separate"], default="fused",
                    help="fused: pa_append_decode; separate: pa_append_kv then pa_decode")
    ap.add_argument("--split-tokens", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU work budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--kv", choices=["bf16", "e4m3"], default="bf16",
                    help="KV cache element type (e4m3: FP8 pools with per-tensor scales, tensor kernel)")
    ap.add_argument("--rope", type=float, default=0.0,
                    help="RoPE frequency base for the fused call (q and the new K turned at position "
                         "L-1); 0 = no rotation")
    ap.add_argument("--graphs", choices=["on", "off"], default="on",
                    help="time the device-resident steps as replays of CUDA graphs captured from "
                         "the same library calls (host launch cost out of the timed region); "
                         "needs --pdl on")
    ap.add_argument("--pdl", choices=["on", "off"], default="on",
                    help="PA_FLAG_PDL: the tensor kernel plans its work while the previous kernel "
                         "runs; tables and lengths are written once before the timed region, as "
                         "the flag requires (per-call events are then left out: they would "
                         "serialise the calls)")
    args = ap.parse_args(argv)
    steps, warmup = DEFAULT_STEPS[args.config]
    if args.steps is None:
        args.steps = steps
    if args.warmup is None:
        args.warmup = warmup
    return args


# (steps, warm-up steps) when the command line gives none
DEFAULT_STEPS = {"c1": (20000, 50), "c2": (20000, 50), "c3": (10000, 50), "c4": (2000, 20),
                 "c5": (300, 10), "pc": (200, 10), "pf": (200, 10)}


# ---------------------------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------------------------
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def max_over_ranks(values, dist, device):
    """Each value's max over all ranks: the slowest rank sets a multi-GPU job's time."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def kv_read_bytes(lens, num_kv_heads, head_dim, elem_bytes=2):
    """Algorithmic K+V bytes one decode launch must read: 2 (K,V) x L x Hkv x D x elem_bytes per
    sequence (2 for bf16 pools, 1 for E4M3)."""
    return int(2 * int(np.sum(lens, dtype=np.int64)) * num_kv_heads * head_dim * elem_bytes)


def kernel_source_hash(kernel_name):
    files = {"tensor": ["decode_stream.cu", "pa_ptx.cuh", "merge.cu"],
             "split": ["decode_tensor.cu", "pa_ptx.cuh", "merge.cu"],
             "simt": ["decode_simt.cu", "merge.cu"],
             "prefill": ["prefill_tc.cu", "pa_umma.cuh", "pa_ptx.cuh"],
             "prefill_ws": ["prefill_ws.cu", "pa_umma.cuh", "pa_ptx.cuh"]}[kernel_name]
    files = files + ["pa_device.cuh", "pa_internal.h", "api.cu"]
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "pagedattention_kv_cache_pa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(config, kernel_name):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current source."""
    prof = os.path.join(ROOT, "profiles")
    if not os.path.isdir(prof):
        return None
    pat = re.compile(r"^traffic\[%s,%s\]:\s*([0-9]+)\s+bytes/launch\s+source=([0-9a-f]+)"
                     % (re.escape(config), re.escape(kernel_name)), re.M)
    want = kernel_source_hash(kernel_name)
    for name in sorted(os.listdir(prof)):
        if not name.endswith((".txt", ".md")):
            continue
        m = pat.search(open(os.path.join(prof, name)).read())
        if m and m.group(2) == want:
            return int(m.group(1))
    return None


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled during the timed region.

    NVML is polled from a thread every few milliseconds (read-only queries), so that even a
    timed region of a few tens of milliseconds gets samples; the constructor returns once
    the first sample is in.  Without NVML, `nvidia-smi -lms 100` is the fallback."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index, enabled=True, interval_s=0.004):
        self.proc = None
        self.thread = None
        self.device_index = device_index
        self.samples = []                       # (sm_mhz, sm_max_mhz, reasons)
        if not enabled:
            return
        if self._start_nvml(interval_s):
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def _start_nvml(self, interval_s):
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            handle = None
            try:                                # the CUDA device's own GPU, by UUID
                uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
                handle = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                handle = nv.nvmlDeviceGetHandleByIndex(self.device_index)
            smax = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
            bits = [nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                    nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap]
        except Exception:
            return False
        self._stop_flag = threading.Event()
        first = threading.Event()

        def poll():
            while True:
                try:
                    sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
                    self.samples.append((float(sm), float(smax),
                                         {n for n, b in zip(self.NAMES, bits) if r & b}))
                except Exception:
                    pass
                first.set()
                if self._stop_flag.wait(interval_s):
                    return

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        first.wait(2.0)
        self._nv = nv
        return True

    def _summary(self):
        if not self.samples:
            return None
        reasons = set()
        for _, _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(s for s, _, _ in self.samples),
                "sm_max_mhz": max(m for _, m, _ in self.samples),
                "reasons": sorted(reasons), "samples": len(self.samples)}

    def stop(self):
        if self.thread is not None:
            self._stop_flag.set()
            self.thread.join(5.0)
            try:
                self._nv.nvmlShutdown()
            except Exception:
                pass
            return self._summary()
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for r in out.strip().splitlines():
            r = [x.strip() for x in r.split(",")]
            if len(r) < 9:
                continue
            try:
                sm, smax = float(r[1]), float(r[2])
            except ValueError:
                continue
            self.samples.append((sm, smax, {n for n, v in zip(self.NAMES, r[5:9])
                                            if v.lower().startswith("active")}))
        return self._summary()


# ---------------------------------------------------------------------------------------------
# the reference arm: the fp64 CPU oracle
# ---------------------------------------------------------------------------------------------
def run_reference(args, rank):
    import oracle
    if rank != 0:
        return None
    if args.config == "c5":
        # each step a bounded sample of a C5 step: the model block manager's step, then the
        # oracle's decode of layer 0 for the whole batch; the rate is scaled to all 16 layers
        t = wl.Trace5()
        events = list(t.events())
        kc, vc = t.pool(0)
        q, _, _ = t.token_inputs(0, 0)
        st = {}

        def sample(i):
            if i % t.steps == 0:                     # the trace (re)starts: a fresh manager
                st["bm"] = oracle.BlockManagerModel(t.num_blocks, t.block_size, t.batch,
                                                    t.max_blocks_per_seq, t.free_order)
                for s in range(t.batch):
                    st["bm"].add_seq(s, int(t.initial_lens[s]))
            bm = st["bm"]
            _, retired, admitted = events[i % t.steps]
            for s in retired:
                bm.free_seq(s)
            for s, n in admitted:
                bm.add_seq(s, n)
            bm.append_tokens(list(range(t.batch)))
            tables = np.array([bm.table_array(s) for s in range(t.batch)], dtype=np.int32)
            oracle.paged_decode(q, kc, vc, tables, np.array(bm.lens, dtype=np.int32), t.scale)

        W, K = args.warmup, args.steps
        for i in range(W):
            sample(i)
        t0 = time.perf_counter()
        for i in range(W, W + K):
            sample(i)
        dt = time.perf_counter() - t0
        value = t.batch * K / dt / t.layers
        cb = {"value": value, "unit": "seq-steps/s", "cores": oracle.num_threads(), "kind": "oracle",
              "sample": "%d trace steps (after %d warm-up steps): the model block manager's step and the "
                        "oracle decode of layer 0 for all 256 sequences, %.1f s; the rate is scaled to all "
                        "%d layers" % (K, W, dt, t.layers)}
        return {"metric": METRIC, "value": value, "unit": "seq-steps/s", "n_gpus": args.gpus,
                "steps": K, "warmup": W, "ms_per_step": 1e3 * dt / K * t.layers,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": WORKLOAD_TEXT["c5"], "config": "c5", "batch": t.batch},
                "cpu_baseline": cb,
                "e2e": {"value": value, "unit": "seq-steps/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    if args.config == "pc":
        # the model of the prefix-caching manager admitting the C3 request mix by token ids
        rng = np.random.default_rng(wl.CONFIG_SEED_BASE + 31)
        prefix = [int(t) for t in rng.integers(0, 128256, 1024)]
        reqs = [prefix + [int(t) for t in rng.integers(0, 128256, int(rng.integers(256, 7169)))]
                for _ in range(32)]
        nb = sum(-(-len(r) // 256) for r in reqs) + 64
        m = oracle.BlockManagerModel(nb, 256, 32, 40, list(range(nb)))
        n, t0 = 0, time.perf_counter()
        while n < max(1, args.steps) * 32 and time.perf_counter() - t0 < 30.0:
            for s, r in enumerate(reqs):
                m.add_seq_tokens(s, r)
            for s in range(32):
                m.free_seq(s)
            n += 32
        dt = time.perf_counter() - t0
        v = n / dt
        return {"metric": "prefix-cached admissions/s (host model)", "value": v, "unit": "admissions/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(n, 1),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": WORKLOAD_TEXT["pc"], "config": "pc"},
                "cpu_baseline": {"value": v, "unit": "admissions/s", "cores": 1, "kind": "oracle",
                                 "sample": "%d admissions of the C3 mix by the Python model, %.1f s" % (n, dt)},
                "e2e": {"value": v, "unit": "admissions/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    b = wl.CONFIGS[args.config]()
    B, Bs = b.batch, b.block_size
    model = oracle.BlockManagerModel(b.num_blocks, Bs, B, b.max_blocks_per_seq, b.free_order)
    for s in range(B):
        L = int(b.context_lens[s])
        model.import_seq(s, L, b.block_tables[s, : -(-L // Bs)])
    slots = np.array(model.append_tokens(list(range(B))), dtype=np.int64)
    tables = np.array([model.table_array(s) for s in range(B)], dtype=np.int32)
    lens = np.array(model.lens, dtype=np.int32)
    kc, vc = b.k_cache.copy(), b.v_cache.copy()

    def one(i):
        s = i % B   # one step = one sequence's append + decode (all its heads)
        oracle.append_kv(b.k_new[s:s + 1], b.v_new[s:s + 1], slots[s:s + 1], kc, vc, in_place=True)
        oracle.paged_decode(b.q[s:s + 1], kc, vc, tables[s:s + 1], lens[s:s + 1], b.scale)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(i)
    dt = time.perf_counter() - t0
    value = args.steps / dt
    cores = oracle.num_threads()
    sample = "%d steps, each one sequence (cycling over the %d of %s) appended and decoded over all %d query heads" % (
        args.steps, B, args.config.upper(), b.num_q_heads)
    return {"metric": METRIC, "value": value, "unit": "seq-steps/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD_TEXT[args.config], "config": args.config,
                       "batch": B},
            "cpu_baseline": {"value": value, "unit": "seq-steps/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "seq-steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def single_thread_rate(step, seconds, max_steps=1000):
    """The same oracle steps on one host thread, for a bounded time (at least one step):
    (steps, seconds).  The OpenMP thread count is put back afterwards."""
    import oracle
    prev = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        n = 0
        t0 = time.perf_counter()
        while True:
            step(n)
            n += 1
            dt = time.perf_counter() - t0
            if dt >= seconds or n >= max_steps:
                return n, dt
    finally:
        oracle.set_num_threads(prev)


def cpu_baseline(b, slots, tables, lens, budget_s):
    """The oracle as it stands on the host's cores, on whole-batch steps until the budget is
    spent; then the same steps on one thread for a third of the budget."""
    import oracle
    kc, vc = b.k_cache.copy(), b.v_cache.copy()
    n = 0
    t0 = time.perf_counter()
    while True:
        oracle.append_kv(b.k_new, b.v_new, slots, kc, vc, in_place=True)
        oracle.paged_decode(b.q, kc, vc, tables, lens, b.scale)
        n += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s or n >= 1000:
            break
    n1, dt1 = single_thread_rate(lambda i: oracle.paged_decode(b.q, kc, vc, tables, lens, b.scale),
                                 budget_s / 3)
    return {"value": n * b.batch / dt, "unit": "seq-steps/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d whole-batch steps of %s (append + decode of all %d sequences x %d heads), %.1f s"
                      % (n, b.name, b.batch, b.num_q_heads, dt),
            "single_thread": {"value": n1 * b.batch / dt1, "unit": "seq-steps/s", "cores": 1,
                              "sample": "%d whole-batch decodes, %.1f s" % (n1, dt1)}}


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------
def unique_kv_bytes(tables, lens, block_size, num_kv_heads, head_dim, elem_bytes=2):
    """K+V bytes of the distinct pool rows a decode launch reads: a block shared by several
    tables (a common prefix) counts once, with the most tokens any sequence uses in it."""
    used = {}
    for row, L in zip(tables, lens):
        L = int(L)
        for i in range(-(-L // block_size)):
            blk = int(row[i])
            used[blk] = max(used.get(blk, 0), min(block_size, L - i * block_size))
    return int(2 * sum(used.values()) * num_kv_heads * head_dim * elem_bytes)


def settle(fn, seconds=0.2):
    """Untimed calls for about `seconds` of wall time before the warm-up: clocks, caches and
    the launch path reach their steady state."""
    import torch
    t0 = time.perf_counter()
    n = 0
    while True:
        fn(n)
        n += 1
        if n % 32 == 0:
            torch.cuda.synchronize()
            if time.perf_counter() - t0 >= seconds:
                return n


def _pack(specs, device):
    """One pinned host buffer and one device buffer holding several arrays at 256-byte aligned
    offsets: a step's inputs go up in one copy.  specs: [(name, numpy array)]; returns (host
    buffer, device buffer, {name: (host numpy view, device tensor view)})."""
    import torch
    offs, off = {}, 0
    for name, a in specs:
        offs[name] = off
        off += -(-a.nbytes // 256) * 256
    h_buf = torch.empty(off, dtype=torch.uint8).pin_memory()
    d_buf = torch.empty(off, dtype=torch.uint8, device=device)
    views = {}
    tdt = {np.dtype(np.uint16): torch.bfloat16, np.dtype(np.int32): torch.int32,
           np.dtype(np.int64): torch.int64}
    for name, a in specs:
        o, n = offs[name], a.nbytes
        hv = h_buf.numpy()[o:o + n].view(a.dtype).reshape(a.shape)
        hv[...] = a
        dv = d_buf[o:o + n].view(tdt[a.dtype]).view(a.shape)
        views[name] = (hv, dv)
    return h_buf, d_buf, views


def capture_graph(fn, dev):
    """A CUDA graph of the library calls fn() makes (captured on a side stream; the calls take
    the current stream, which is the capture stream inside the capture)."""
    import torch
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


class _Rt:
    """The CUDA runtime calls the e2e loop issues per step (copies, event records, stream
    waits), made straight through ctypes on the libcudart torch has loaded, on raw stream and
    event handles: a torch copy_ of pinned memory costs several microseconds of host time
    per call, which at C2's 28 us per step would be the bound."""

    def __init__(self):
        import ctypes
        import torch
        torch.cuda.init()
        self.lib = ctypes.CDLL("libcudart.so.12")
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        L = self.lib
        L.cudaMemcpyAsync.argtypes = [vp, vp, sz, ctypes.c_int, vp]
        L.cudaEventRecord.argtypes = [vp, vp]
        L.cudaStreamWaitEvent.argtypes = [vp, vp, ctypes.c_uint]
        L.cudaEventSynchronize.argtypes = [vp]
        L.cudaEventCreateWithFlags.argtypes = [ctypes.POINTER(vp), ctypes.c_uint]
        L.cudaEventDestroy.argtypes = [vp]
        self.events = []

    def _ok(self, rc, what):
        if rc != 0:
            raise RuntimeError("%s returned cudaError %d" % (what, rc))

    def event(self):
        import ctypes
        ev = ctypes.c_void_p()
        self._ok(self.lib.cudaEventCreateWithFlags(ctypes.byref(ev), 2), "cudaEventCreateWithFlags")  # no timing
        self.events.append(ev.value)
        return ev.value

    def copy(self, dst, src, nbytes, kind, stream):        # kind 1: host to device, 2: device to host
        self._ok(self.lib.cudaMemcpyAsync(dst, src, nbytes, kind, stream), "cudaMemcpyAsync")

    def record(self, ev, stream):
        self._ok(self.lib.cudaEventRecord(ev, stream), "cudaEventRecord")

    def wait(self, stream, ev):
        self._ok(self.lib.cudaStreamWaitEvent(stream, ev, 0), "cudaStreamWaitEvent")

    def sync(self, ev):
        self._ok(self.lib.cudaEventSynchronize(ev), "cudaEventSynchronize")

    def close(self):
        for ev in self.events:
            self.lib.cudaEventDestroy(ev)
        self.events = []


def run_e2e(E, warm, stream, stage, h_in, h_outs, compute, dist, dev, host_fill=None):
    """Times E end-to-end steps.  Step i copies its inputs from pinned host memory (h_in, or
    what host_fill(i) returns) into device staging buffer i % 2 on an upload stream, runs
    compute(i, bufs) on `stream` once that copy has landed, and copies the step's output (the
    last entry of bufs) back into pinned h_outs[i % 2] on a download stream, so that the two
    directions overlap each other and the compute.  An input buffer is refilled once the
    compute two steps back has read it; an output buffer is rewritten once its download two
    steps back has left.  CUDA events on `stream` bracket the whole, max over ranks."""
    import torch
    rt = _Rt()
    cs_in = torch.cuda.Stream(device=dev)
    cs_out = torch.cuda.Stream(device=dev)
    s_main, s_in, s_out = stream.cuda_stream, cs_in.cuda_stream, cs_out.cuda_stream
    ev_in = [rt.event() for _ in range(2)]
    ev_done = [rt.event() for _ in range(2)]
    ev_out = [rt.event() for _ in range(2)]
    d_ptr = [s[0].data_ptr() for s in stage]
    o_ptr = [s[1][-1].data_ptr() for s in stage]
    h_out_ptr = [h.data_ptr() for h in h_outs]
    n_out = h_outs[0].numel() * h_outs[0].element_size()
    n_in = stage[0][0].numel() * stage[0][0].element_size()
    h_in_ptr = h_in.data_ptr() if h_in is not None else None
    # a wait on an event that was never recorded returns at once: the first two steps need none

    def step(i):
        j = i & 1
        if host_fill is not None:
            rt.sync(ev_in[j])                               # the upload of step i - 2 has left its host buffer
            src = host_fill(i).data_ptr()
        else:
            src = h_in_ptr
        rt.wait(s_in, ev_done[j])                           # the compute of step i - 2 has read these inputs
        rt.copy(d_ptr[j], src, n_in, 1, s_in)
        rt.record(ev_in[j], s_in)
        rt.wait(s_main, ev_in[j])
        rt.wait(s_main, ev_out[j])                          # the download of step i - 2 has left this output
        compute(i, stage[j][1])
        rt.record(ev_done[j], s_main)
        rt.wait(s_out, ev_done[j])
        rt.copy(h_out_ptr[j], o_ptr[j], n_out, 2, s_out)
        rt.record(ev_out[j], s_out)

    for i in range(warm):
        step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cs_in.wait_event(e0)                                # no copy of the timed steps starts earlier
    cs_out.wait_event(e0)
    for i in range(E):
        step(warm + i)
    rt.wait(s_main, ev_out[(warm + E - 1) & 1])         # the last step's output is on the host
    e1.record(stream)
    torch.cuda.synchronize()
    rt.close()
    ms, = max_over_ranks([e0.elapsed_time(e1)], dist, dev)
    return ms


def run_decode(args, rank, world, dist, cfg=None, steps=None, warmup=None, e2e_steps=None, kv=None,
               with_cpu=True):
    """A decode configuration (c1..c4): one step = pa_append_decode (or the separate calls) of
    one layer for the whole batch, rotating over layer pools larger than L2 together."""
    import torch
    import pagedattention_kv_cache_pa_b200 as pa

    cfg = cfg or args.config
    K = args.steps if steps is None else steps
    W = args.warmup if warmup is None else warmup
    E = args.e2e_steps if e2e_steps is None else e2e_steps
    kv = kv or args.kv
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    b = wl.CONFIGS[cfg]()
    B, Bs, MB = b.batch, b.block_size, b.max_blocks_per_seq
    Hq, Hkv, D = b.num_q_heads, b.num_kv_heads, b.head_dim

    # (a1, a2) on the host: give each sequence its new token's slot
    bm = pa.BlockManager(b.num_blocks, Bs, B, MB, b.free_order)
    for s in range(B):
        L = int(b.context_lens[s])
        bm.import_seq(s, L, b.block_tables[s, : -(-L // Bs)])
    slots = bm.append_tokens(np.arange(B, dtype=np.int32))
    tables = bm.block_tables().copy()
    lens = bm.context_lens().copy()
    bm.close()
    max_len = int(lens.max())

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    e4m3 = kv == "e4m3"
    KS = VS = 5.0 / 448                                  # N(0,1) data: |x| <= 5 fills the E4M3 range
    pool_bytes = 2 * b.k_cache.nbytes // (2 if e4m3 else 1)
    layers = max(1, min(8, math.ceil(1.0e9 / pool_bytes)))
    desc = pa.CacheDesc.make(num_blocks=b.num_blocks, block_size=Bs, num_kv_heads=Hkv, num_q_heads=Hq,
                             head_dim=D, max_blocks_per_seq=MB)

    def pool(a):
        t = to_dev(a)
        if not e4m3:
            return t
        # E4M3 pool: every slot's rows quantized by the library's own append
        rows = t.permute(0, 2, 1, 3).reshape(-1, Hkv, D).contiguous()
        qp = torch.empty(t.shape, dtype=torch.uint8, device=dev)
        pa.pa_append_kv_e4m3(rows, rows, torch.arange(rows.shape[0], dtype=torch.int64, device=dev), KS, KS,
                             qp, qp, desc)
        return qp
    kcs = [pool(b.k_cache) for _ in range(layers)]
    vcs = [pool(b.v_cache) for _ in range(layers)]
    torch.cuda.synchronize()
    # every input of a step in one buffer (the e2e leg uploads it whole, in one copy)
    h_buf, d_buf, io = _pack([("q", b.q), ("k", b.k_new), ("v", b.v_new), ("slots", slots),
                              ("tables", tables), ("lens", lens)], dev)
    d_buf.copy_(h_buf)
    q, k_new, v_new = io["q"][1], io["k"][1], io["v"][1]
    slots_d, tables_d, lens_d = io["slots"][1], io["tables"][1], io["lens"][1]
    out = torch.empty_like(q)
    kernel = {"auto": pa.PA_KERNEL_AUTO, "simt": pa.PA_KERNEL_SIMT,
              "tensor": pa.PA_KERNEL_TENSOR, "split": pa.PA_KERNEL_TENSOR_SPLIT}[args.kernel]
    pdl = args.pdl == "on"
    kvo = dict(kv_dtype=pa.PA_KV_E4M3, k_scale=KS, v_scale=VS) if e4m3 else {}
    opts = pa.DecodeOptions(split_tokens=args.split_tokens, kernel=kernel, max_ctas=args.max_ctas,
                            flags=pa.PA_FLAG_PDL if pdl else 0, rope_theta=args.rope, **kvo)
    wsb = pa.pa_decode_workspace_size(B, max_len, desc, opts)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    plan = pa.pa_decode_describe(B, max_len, desc, opts)

    fused = args.path == "fused"
    # separate path: pa_append_kv (or pa_rope_append_kv) through the slot mapping, then pa_decode
    opts_dec = pa.DecodeOptions(split_tokens=args.split_tokens, kernel=kernel, max_ctas=args.max_ctas,
                                flags=pa.PA_FLAG_PDL if pdl else 0, **kvo)
    pos_d = torch.from_numpy(np.maximum(lens - 1, 0).astype(np.int32)).to(dev)
    q_rot = torch.empty_like(q)

    resident = (q, k_new, v_new, slots_d, tables_d, lens_d, out)

    def call(L, ev=None, bufs=resident):
        q, k_new, v_new, slots_d, tables_d, lens_d, out = bufs
        stream = torch.cuda.current_stream(dev)        # the capture stream while capturing
        if fused:
            if ev is not None:
                ev[0].record(stream)
            pa.pa_append_decode(q, k_new, v_new, kcs[L], vcs[L], tables_d, lens_d, max_len, b.scale,
                                out, ws, desc, opts, stream=stream)
            if ev is not None:
                ev[1].record(stream)
            return
        qq = q
        if args.rope > 0:
            pa.pa_rope_append_kv(q, q_rot, k_new, v_new, pos_d, slots_d, args.rope, kcs[L], vcs[L], desc,
                                 stream=stream)
            qq = q_rot
        elif e4m3:
            pa.pa_append_kv_e4m3(k_new, v_new, slots_d, KS, VS, kcs[L], vcs[L], desc, stream=stream)
        else:
            pa.pa_append_kv(k_new, v_new, slots_d, kcs[L], vcs[L], desc, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        pa.pa_decode(qq, kcs[L], vcs[L], tables_d, lens_d, max_len, b.scale, out, ws, desc, opts_dec,
                     stream=stream)
        if ev is not None:
            ev[1].record(stream)

    # correctness guard before timing: the kernel must not report device errors
    call(0)
    torch.cuda.synchronize()
    rc = pa.pa_decode_status(ws)
    if rc != 0:
        raise RuntimeError("decode reported %s" % pa.pa_status_string(rc))

    settle(lambda i: call(i % layers))
    graphs = args.graphs == "on" and pdl
    if graphs:
        # one graph of `layers` calls (one per pool, back to back as the loop below issues them)
        # and one of the remainder: K calls = K // layers full replays + the remainder
        full = capture_graph(lambda: [call(L) for L in range(layers)], dev)
        rem = capture_graph(lambda: [call(L) for L in range(K % layers)], dev) if K % layers else None
        launch_desc = "CUDA graphs of the library calls: %d calls per replay" % layers

        def timed_steps(n):
            for _ in range(n // layers):
                full.replay()
            if n % layers:
                (rem if n % layers == K % layers else
                 capture_graph(lambda: [call(L) for L in range(n % layers)], dev)).replay()
    else:
        launch_desc = "direct calls"
    for i in range(W):
        call(i % layers)
    if graphs:
        timed_steps(W)
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index, enabled=not args.no_clocks)
    t_start.record(stream)
    if graphs:
        timed_steps(K)
    else:
        for i in range(K):
            call(i % layers, None if pdl else ev_dec[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if dist is not None:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    if pdl:
        # back-to-back calls overlap: the call's share of the timed region (the whole
        # step, append included, on the separate path)
        dec_avg_ms = elapsed_ms / K
    else:
        dec_avg_ms = float(np.mean([s.elapsed_time(e) for s, e in ev_dec]))
    elapsed_ms, dec_avg_ms = max_over_ranks([elapsed_ms, dec_avg_ms], dist, dev)
    rc = pa.pa_decode_status(ws)
    if rc != 0:
        raise RuntimeError("decode reported %s during timing" % pa.pa_status_string(rc))
    value = world * B * K / (elapsed_ms / 1e3)

    # ---- e2e: every step's inputs up from pinned host memory in one copy, its output back in
    # one, on a copy stream that runs a step ahead of the compute (two device staging buffers)
    e2e = None
    if E > 0:
        _, d_buf2, io2 = _pack([("q", b.q), ("k", b.k_new), ("v", b.v_new), ("slots", slots),
                                ("tables", tables), ("lens", lens)], dev)
        out2 = torch.empty_like(out)
        stage = [(d_buf, resident), (d_buf2, tuple(io2[n][1] for n in ("q", "k", "v", "slots", "tables",
                                                                       "lens")) + (out2,))]
        h_outs = [torch.empty(out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        compute = lambda i, bufs: call(i % layers, bufs=bufs)    # noqa: E731
        if fused:
            # the same library call on raw device pointers (the binding takes ints as well):
            # its per-tensor dtype, device and contiguity checks passed above for these buffers
            raw = [tuple(t.data_ptr() for t in s[1]) for s in stage]
            kc_p, vc_p = [t.data_ptr() for t in kcs], [t.data_ptr() for t in vcs]
            ws_p, s_h = ws.data_ptr(), stream.cuda_stream

            def compute(i, bufs):
                qp, kp, vp, _, tp, lp, op = raw[i & 1]
                L = i % layers
                pa.pa_append_decode(qp, kp, vp, kc_p[L], vc_p[L], tp, lp, max_len, b.scale, op, ws_p, desc,
                                    opts, stream=s_h, num_seqs=B, workspace_bytes=wsb)
        e2e_ms = run_e2e(E, min(W, 20), stream, stage, h_buf, h_outs, compute, dist, dev)
        e2e = {"value": world * B * E / (e2e_ms / 1e3), "unit": "seq-steps/s",
               "h2d_bytes_per_step": int(h_buf.numel()), "d2h_bytes_per_step": int(h_outs[0].numel() * 2),
               "copies_per_step": {"h2d": 1, "d2h": 1}, "steps": E,
               "overlap": "uploads and downloads on two streams of their own, one step ahead of the compute",
               "host_calls": "cudaMemcpyAsync and event calls on raw handles; the library call on raw pointers"
                             if fused else "cudaMemcpyAsync and event calls on raw handles"}

    if rank != 0:
        return None

    kernel_name = {pa.PA_KERNEL_SIMT: "simt", pa.PA_KERNEL_TENSOR_SPLIT: "split"}.get(plan.kernel, "tensor")
    peak, peak_kind = measured_peaks()
    elem = 1 if e4m3 else 2
    logical = kv_read_bytes(lens, Hkv, D, elem)
    unique = unique_kv_bytes(tables, lens, Bs, Hkv, D, elem)
    kv_bytes = unique                                    # equal to logical unless blocks are shared
    achieved = kv_bytes / (dec_avg_ms / 1e3) / 1e9
    res = {
        "metric": METRIC, "value": value, "unit": "seq-steps/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 kv, bf16 q/out" if e4m3 else "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[cfg], "config": cfg,
                   "batch": B, "num_q_heads": Hq, "num_kv_heads": Hkv, "head_dim": D,
                   "block_size": Bs, "num_blocks": b.num_blocks, "mean_context": float(lens.mean()),
                   "max_context": max_len, "decode_kernel": kernel_name, "ctas": plan.ctas,
                   "split_tokens": args.split_tokens or "auto", "max_splits": plan.max_splits,
                   "call": "pa_append_decode" if fused else
                           ("pa_rope_append_kv + pa_decode" if args.rope > 0 else "pa_append_kv + pa_decode"),
                   "pdl": pdl, "launch": launch_desc, "rope_theta": args.rope, "kv_dtype": kv,
                   "l2": "inputs larger than L2: %d rotating layer pools of %.0f MB" % (layers, pool_bytes / 1e6),
                   "parallelism": "replicas x%d" % world},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "frac_of_nominal_8000": achieved / NOMINAL_HBM_GBS,
                     "traffic": profiled_traffic(cfg + ("-e4m3" if e4m3 else ""), kernel_name),
                     "kernel": ("pa_append_decode (%s)" if fused else "pa_decode (%s)") % kernel_name,
                     "algorithmic_bytes_per_launch": kv_bytes,
                     "bytes_basis": "unique pool rows (a shared prefix counted once)" if unique != logical
                                    else "K+V rows of every context",
                     "logical_bytes_per_launch": logical,
                     "avg_launch_ms": dec_avg_ms,
                     "launch_timing": "timed region / calls" if pdl else "CUDA events around each call"},
        "kv_read_gbs_step": kv_bytes * K / (elapsed_ms / 1e3) / 1e9,
        "e2e": e2e,
        # per step: the append (its own kernel unless the stream kernel fuses it), the decode
        # kernel and (split kernels, when a sequence can be cut) the merge kernel; the stream
        # kernel merges cut sequences itself
        "gpu_launches": K * ((0 if (fused and kernel_name == "tensor") else 1) + 1 +
                             (1 if (kernel_name != "tensor" and plan.max_splits > 1) else 0)),
        "clocks": clk,
    }
    if with_cpu and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(b, slots, tables, lens, args.cpu_seconds)
    del kcs, vcs
    return res


def run_ours(args, rank, world, dist):
    return run_decode(args, rank, world, dist)


# The other decode workloads, measured in the same run as the headline line (device time,
# inputs resident in HBM), so that one bench run records all of them.
ALSO = [("c2", "bf16", 6000), ("c3", "bf16", 4000), ("c4", "bf16", 1000), ("c2", "e4m3", 6000),
        ("c4", "e4m3", 1000)]


def run_also(args, rank, world, dist):
    import torch
    out = {}
    for cfg, kv, steps in ALSO:
        r = run_decode(args, rank, world, dist, cfg=cfg, steps=steps, warmup=20, e2e_steps=0, kv=kv,
                       with_cpu=False)
        torch.cuda.empty_cache()
        if r is None:
            continue
        rf = r["roofline"]
        out[cfg + ("-e4m3" if kv == "e4m3" else "")] = {
            "workload": r["config"]["workload"], "value": r["value"], "unit": r["unit"],
            "steps": r["steps"], "warmup": r["warmup"], "ms_per_step": r["ms_per_step"],
            "kv_dtype": kv, "roofline": {k: rf[k] for k in ("achieved", "peak", "frac", "unit",
                                                           "algorithmic_bytes_per_launch", "bytes_basis",
                                                           "avg_launch_ms", "traffic")},
            "clocks": r["clocks"]}
    return out


def run_c5(args, rank, world, dist):
    """C5: the continuous-batching trace.  One step = one decode step of all 16 layers for the
    256 live sequences (host block manager, then pa_append_decode per layer).  The 100-step
    trace is replayed as often as --steps asks."""
    import torch
    import pagedattention_kv_cache_pa_b200 as pa

    if args.kv != "bf16":
        raise SystemExit("--config c5 runs bf16 pools only")
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    t = wl.Trace5()
    B, Bs, MB, N = t.batch, t.block_size, t.max_blocks_per_seq, t.num_blocks
    Hq, Hkv, D, NL, S = t.num_q_heads, t.num_kv_heads, t.head_dim, t.layers, t.steps
    seqs = np.arange(B, dtype=np.int32)

    def replay():
        bm = pa.BlockManager(N, Bs, B, MB, t.free_order)
        for s in range(B):
            bm.add_seq(s, int(t.initial_lens[s]))
        for step, retired, admitted in t.events():
            for s in retired:
                bm.free_seq(s)
            for s, n in admitted:
                bm.add_seq(s, n)
            bm.append_tokens(seqs)
            yield step, bm
        bm.close()

    tables = np.empty((S, B, MB), dtype=np.int32)
    lens = np.empty((S, B), dtype=np.int32)
    for step, bm in replay():
        tables[step] = bm.block_tables()
        lens[step] = bm.context_lens()
    tables_d = torch.from_numpy(tables).to(dev)
    lens_d = torch.from_numpy(lens).to(dev)
    step_max = [int(x) for x in lens.max(axis=1)]

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    kcs, vcs, tok = [], [], []
    for layer in range(NL):
        kc, vc = t.pool(layer)
        kcs.append(to_dev(kc))
        vcs.append(to_dev(vc))
        del kc, vc
        tok.append(t.token_inputs(layer, 0))
    # q, k, v of every layer in one buffer, the outputs of every layer in another: the e2e leg
    # moves a step's inputs up in one copy and its outputs down in one
    h_tok, d_tok, io = _pack([(n % l, a) for l in range(NL) for n, a in zip(("q%d", "k%d", "v%d"), tok[l])],
                             dev)
    d_tok.copy_(h_tok)
    qs = [io["q%d" % l][1] for l in range(NL)]
    ks = [io["k%d" % l][1] for l in range(NL)]
    vs = [io["v%d" % l][1] for l in range(NL)]
    outs_all = torch.empty((NL,) + tuple(qs[0].shape), dtype=torch.bfloat16, device=dev)
    outs = [outs_all[l] for l in range(NL)]
    desc = pa.CacheDesc.make(num_blocks=N, block_size=Bs, num_kv_heads=Hkv, num_q_heads=Hq,
                             head_dim=D, max_blocks_per_seq=MB)
    kernel = {"auto": pa.PA_KERNEL_AUTO, "simt": pa.PA_KERNEL_SIMT,
              "tensor": pa.PA_KERNEL_TENSOR, "split": pa.PA_KERNEL_TENSOR_SPLIT}[args.kernel]
    pdl = args.pdl == "on"
    opts = pa.DecodeOptions(split_tokens=args.split_tokens, kernel=kernel, max_ctas=args.max_ctas,
                            flags=pa.PA_FLAG_PDL if pdl else 0, rope_theta=args.rope)
    ws = torch.zeros(pa.pa_decode_workspace_size(B, int(lens.max()), desc, opts), dtype=torch.uint8,
                     device=dev)
    plan = pa.pa_decode_describe(B, int(lens.max()), desc, opts)

    def call(s, layer, tb=None, ln=None, mx=None):
        pa.pa_append_decode(qs[layer], ks[layer], vs[layer], kcs[layer], vcs[layer],
                            tables_d[s] if tb is None else tb, lens_d[s] if ln is None else ln,
                            step_max[s] if mx is None else mx, t.scale, outs[layer], ws, desc, opts,
                            stream=torch.cuda.current_stream(dev))

    def trace_step(i):
        for layer in range(NL):
            call(i % S, layer)

    trace_step(0)
    torch.cuda.synchronize()
    rc = pa.pa_decode_status(ws)
    if rc != 0:
        raise RuntimeError("decode reported %s" % pa.pa_status_string(rc))
    first_out = outs[0].float().cpu().numpy()            # layer 0 of trace step 0, for the parity leg
    K, W = args.steps, args.warmup
    settle(trace_step)
    graphs = args.graphs == "on" and pdl
    if graphs:
        # one graph per trace step: its 16 layer calls, with that step's tables and lengths
        step_graphs = [capture_graph(lambda s=s: [call(s, layer) for layer in range(NL)], dev) for s in range(S)]
        trace_step = lambda i: step_graphs[i % S].replay()       # noqa: E731
        launch_desc = "CUDA graphs of the library calls: one per trace step (16 calls)"
    else:
        launch_desc = "direct calls"
    for i in range(W):
        trace_step(i)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K * NL)]
    t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index, enabled=not args.no_clocks)
    t0e.record(stream)
    for i in range(K):
        if graphs:
            trace_step(i)
            continue
        s = i % S
        for layer in range(NL):
            if not pdl:
                ev[i * NL + layer][0].record(stream)
            call(s, layer)
            if not pdl:
                ev[i * NL + layer][1].record(stream)
    t1e.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if dist is not None:
        dist.barrier()
    elapsed_ms = t0e.elapsed_time(t1e)
    if pdl:   # calls overlap: each gets its share of the timed region
        call_ms = np.full(K * NL, elapsed_ms / (K * NL))
    else:
        call_ms = np.array([a.elapsed_time(b) for a, b in ev])
    kv_per_call = np.array([kv_read_bytes(lens[i % S], Hkv, D) for i in range(K) for _ in range(NL)],
                           dtype=np.float64)
    gbs = float(kv_per_call.sum() / (call_ms.sum() / 1e3) / 1e9)
    elapsed_ms, = max_over_ranks([elapsed_ms], dist, dev)
    value = world * B * K / (elapsed_ms / 1e3)
    rc = pa.pa_decode_status(ws)
    if rc != 0:
        raise RuntimeError("decode reported %s during timing" % pa.pa_status_string(rc))

    # e2e: the host block manager replays the trace inside the timed region.  Per step one copy
    # up (table rows, lengths, every layer's q/k/v) and one copy down (every layer's output), on
    # a copy stream a step ahead of the compute; the host fills one of two pinned staging
    # buffers while the other's step runs.
    warm = min(args.warmup, 20)
    E = max(1, min(args.e2e_steps, S - warm))
    hosts, stage, mx_of = [], [], [0, 0]
    for _ in range(2):
        hb, db, v2 = _pack([("tables", tables[0]), ("lens", lens[0])] +
                           [(n % l, a) for l in range(NL) for n, a in zip(("q%d", "k%d", "v%d"), tok[l])], dev)
        o = torch.empty_like(outs_all)
        hosts.append((hb, v2))
        stage.append((db, (v2, o)))
    h_outs = [torch.empty(outs_all.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    trace = replay()

    def host_fill(i):
        step, bm = next(trace)                   # retire, admit, append: the host manager's step
        hb, v2 = hosts[i & 1]
        v2["tables"][0][...] = bm.block_tables()
        v2["lens"][0][...] = bm.context_lens()
        mx_of[i & 1] = int(v2["lens"][0].max())
        return hb

    def compute(i, bufs):
        v2, o = bufs
        for layer in range(NL):
            pa.pa_append_decode(v2["q%d" % layer][1], v2["k%d" % layer][1], v2["v%d" % layer][1],
                                kcs[layer], vcs[layer], v2["tables"][1], v2["lens"][1], mx_of[i & 1], t.scale,
                                o[layer], ws, desc, opts, stream=stream)

    e2e_ms = run_e2e(E, warm, stream, stage, None, h_outs, compute, dist, dev, host_fill=host_fill)
    if rank != 0:
        return None
    peak, peak_kind = measured_peaks()
    kernel_name = {pa.PA_KERNEL_SIMT: "simt", pa.PA_KERNEL_TENSOR_SPLIT: "split"}.get(plan.kernel, "tensor")
    res = {
        "metric": METRIC, "value": value, "unit": "seq-steps/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT["c5"], "config": "c5", "batch": B, "layers": NL,
                   "trace_steps": S, "step": "one decode step of all 16 layers (trace replayed as needed)",
                   "num_blocks": N, "mean_context": float(lens.mean()),
                   "decode_kernel": kernel_name, "ctas": plan.ctas, "call": "pa_append_decode per layer",
                   "pdl": pdl, "launch": launch_desc, "rope_theta": args.rope,
                   "l2": "inputs larger than L2: 16 layer pools of %.0f MB" % (2 * kcs[0].numel() * 2 / 1e6),
                   "parallelism": "replicas x%d" % world},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                     "frac": gbs / peak, "peak_kind": peak_kind,
                     "frac_of_nominal_8000": gbs / NOMINAL_HBM_GBS,
                     "traffic": profiled_traffic("c5", kernel_name),
                     "kernel": "pa_append_decode (%s)" % kernel_name,
                     "algorithmic_bytes_per_launch": float(kv_per_call.mean()),
                     "bytes_basis": "K+V rows of every context",
                     "avg_launch_ms": float(call_ms.mean()),
                     "launch_timing": "timed region / calls" if pdl else "CUDA events around each call"},
        "e2e": {"value": world * B * E / (e2e_ms / 1e3), "unit": "seq-steps/s",
                "h2d_bytes_per_step": int(hosts[0][0].numel()),
                "d2h_bytes_per_step": int(h_outs[0].numel() * 2),
                "copies_per_step": {"h2d": 1, "d2h": 1}, "steps": E,
                "includes": "host block manager (retire, admit, append) per step",
                "overlap": "uploads and downloads on two streams of their own, one step ahead of the compute"},
        "gpu_launches": K * NL * (1 if kernel_name == "tensor" else 2),   # one fused call per layer
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline_c5(t, tables, lens, args.cpu_seconds)
        if args.rope == 0:
            res["parity"] = parity_c5(t, tables, lens, first_out)
    del kcs, vcs
    return res


def parity_c5(t, tables, lens, gpu_out):
    """The first trace step's layer-0 output against the oracle on the same inputs: the step's
    K/V rows appended into the initial pool at each sequence's newest position, then the decode."""
    import oracle
    kc, vc = t.pool(0)
    q, k, v = t.token_inputs(0, 0)
    L = lens[0].astype(np.int64)
    B = len(L)
    slots = tables[0][np.arange(B), (L - 1) // t.block_size].astype(np.int64) * t.block_size + (L - 1) % t.block_size
    oracle.append_kv(k, v, slots, kc, vc, in_place=True)
    ref = oracle.paged_decode(q, kc, vc, tables[0], lens[0], t.scale)
    ok, excess = oracle.within_tolerance(gpu_out, ref)
    err = np.abs(gpu_out.astype(np.float64) - ref)
    return {"max_abs_err": float(err.max()), "max_abs_oracle": float(np.abs(ref).max()),
            "within_tolerance": ok, "worst_excess": excess, "tolerance": "1e-2 + 1e-2 |oracle|",
            "sample": "layer 0 of trace step 0 (%d sequences x %d heads), fused append + decode" % (B, t.num_q_heads)}


def cpu_baseline_c5(t, tables, lens, budget_s):
    """The oracle on layer 0 of successive trace steps (whole batch), until the budget is spent."""
    import oracle
    kc, vc = t.pool(0)
    q, _, _ = t.token_inputs(0, 0)
    n = 0
    t0 = time.perf_counter()
    while True:
        s = n % t.steps
        oracle.paged_decode(q, kc, vc, tables[s], lens[s], t.scale)
        n += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    n1, dt1 = single_thread_rate(lambda i: oracle.paged_decode(q, kc, vc, tables[i % t.steps],
                                                                lens[i % t.steps], t.scale), budget_s / 3)
    # one seq-step = one sequence through all layers: the sample covers 1 of the 16 layers
    return {"value": n * t.batch / dt / t.layers, "unit": "seq-steps/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d trace steps of layer 0 only (256 sequences x 32 heads each), %.1f s; "
                      "value scaled to all %d layers" % (n, dt, t.layers),
            "single_thread": {"value": n1 * t.batch / dt1 / t.layers, "unit": "seq-steps/s", "cores": 1,
                              "sample": "%d trace steps of layer 0 on one thread, %.1f s; value scaled "
                                        "to all %d layers" % (n1, dt1, t.layers)}}


def run_pc(args, rank, world, dist):
    """Prefix caching + copy-on-write: a step is one pa_copy_blocks of 8192 block pairs (K and
    V) on the device; the host side times admission by token ids of the C3 request mix."""
    import torch
    import pagedattention_kv_cache_pa_b200 as pa

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    # host: C3 mix, admitted by token ids, released, admitted again (steady state)
    rng = np.random.default_rng(wl.CONFIG_SEED_BASE + 31)
    Bs3, reqs = 256, []
    prefix = [int(t) for t in rng.integers(0, 128256, 1024)]
    for _ in range(32):
        reqs.append(np.asarray(prefix + [int(t) for t in rng.integers(0, 128256, int(rng.integers(256, 7169)))],
                               dtype=np.int32))
    blocks_needed = sum(-(-len(r) // Bs3) for r in reqs)
    bm = pa.BlockManager(blocks_needed + 64, Bs3, 32, 40, np.arange(blocks_needed + 64, dtype=np.int32))
    rounds, cached, total = 0, 0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < 1.0 or rounds < 3:
        for s, r in enumerate(reqs):
            c = bm.add_seq_tokens(s, r)
            if rounds >= 1:
                cached += c
                total += len(r)
        for s in range(32):
            bm.free_seq(s)
        rounds += 1
    host_s = time.perf_counter() - t0
    bm.close()
    # device: block copies of the C2 geometry
    Hkv, Bs, D, P = 8, 16, 64, 8192
    N = 2 * P + 1024
    desc = pa.CacheDesc.make(num_blocks=N, block_size=Bs, num_kv_heads=Hkv, num_q_heads=32,
                             head_dim=D, max_blocks_per_seq=1)
    kc = torch.empty((N, Hkv, Bs, D), dtype=torch.bfloat16, device=dev).normal_()
    vc = torch.empty_like(kc).normal_()
    perm = np.random.default_rng(3).permutation(N)
    pairs = torch.from_numpy(np.stack([perm[:P], perm[P:2 * P]], 1).astype(np.int32)).to(dev)
    for _ in range(args.warmup):
        pa.pa_copy_blocks(kc, vc, pairs, desc, stream=stream)
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index, enabled=not args.no_clocks)
    e0.record(stream)
    for _ in range(K):
        pa.pa_copy_blocks(kc, vc, pairs, desc, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    ms, = max_over_ranks([ms], dist, dev)
    if rank != 0:
        return None
    bytes_step = 2 * 2 * P * Hkv * Bs * D * 2            # K and V, read + write
    peak, peak_kind = measured_peaks()
    achieved = bytes_step / (ms / K / 1e3) / 1e9
    return {
        "metric": "copy-on-write block copies/s (device) and prefix-cached admissions/s (host)",
        "value": world * P * K / (ms / 1e3), "unit": "blocks/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT["pc"], "config": "pc", "pairs": P,
                   "l2": "inputs larger than L2: %d MB read per step" % (bytes_step // 2 // 1000000)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind, "traffic": None,
                     "kernel": "pa_copy_blocks", "algorithmic_bytes_per_launch": bytes_step,
                     "avg_launch_ms": ms / K},
        "host": {"admissions_per_s": rounds * 32 / host_s, "rounds": rounds,
                 "cached_token_fraction": cached / max(total, 1),
                 "prefix_token_fraction": 1024 * 32 / max(sum(len(r) for r in reqs), 1)},
        "e2e": None, "gpu_launches": K, "clocks": clk,
    }


PF_CACHED, PF_NEW = [0, 512, 1024, 1536], 2048


def prefill_flops(lens, q_lens, num_q_heads, head_dim):
    """4 * (p + 1) * D per query head and query at position p (q.K and p.V, 2 flops a MAC)."""
    f = 0
    for L, T in zip(lens, q_lens):
        pos = np.arange(L - T, L, dtype=np.int64)
        f += int(4 * (pos + 1).sum()) * head_dim * num_q_heads
    return f


def pf_cpu_baseline(b, q_h, cu, lens, B, seconds):
    """The oracle's prefill on windows of 64 consecutive queries of the chunks, for about
    `seconds`.  Visit n takes sequence n % B and window 13 (n // B) mod (chunk / 64) of it, so
    every sequence steps through its whole chunk and a cut-short run still samples early,
    middle and late positions evenly."""
    import oracle
    windows = PF_NEW // 64
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < max(1.0, seconds):
        s_ = n % B
        w = (13 * (n // B)) % windows
        end = lens[s_] - PF_NEW + 64 * (w + 1)       # the window's queries are the last 64 of `end` tokens
        qs = q_h[int(cu[s_]) + 64 * w: int(cu[s_]) + 64 * (w + 1)]
        oracle.paged_prefill(qs, b.k_cache, b.v_cache, b.block_tables[s_:s_ + 1], np.array([0, 64], np.int32),
                             np.array([end], np.int32), b.scale)
        n += 1
    dt = time.perf_counter() - t0
    return {"value": 64 * n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d windows of 64 query tokens spread evenly over the %d chunks, %.1f s" % (n, B, dt)}


def run_pf(args, rank, world, dist):
    """Chunked prefill: a step appends each sequence's new chunk and runs the causal attention."""
    import torch
    import pagedattention_kv_cache_pa_b200 as pa

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    lens = [c + PF_NEW for c in PF_CACHED]
    q_lens = [PF_NEW] * len(lens)
    b = wl.make_batch("PF", wl.CONFIG_SEED_BASE + 41, [L - 1 for L in lens], num_q_heads=32, num_kv_heads=8,
                      head_dim=64, block_size=16)
    Hq, Hkv, D, Bs = b.num_q_heads, b.num_kv_heads, b.head_dim, b.block_size
    B = len(lens)
    rng = np.random.default_rng(wl.CONFIG_SEED_BASE + 42)
    T = sum(q_lens)
    bits = lambda shape: (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    q_h, k_h, v_h = bits((T, Hq, D)), bits((T, Hkv, D)), bits((T, Hkv, D))
    slots = np.concatenate([[int(b.block_tables[s_][p // Bs]) * Bs + p % Bs for p in range(L - Tq, L)]
                            for s_, (L, Tq) in enumerate(zip(lens, q_lens))]).astype(np.int64)
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    kc, vc = to(b.k_cache), to(b.v_cache)
    q, k, v = to(q_h), to(k_h), to(v_h)
    slots_d, cu_d = torch.from_numpy(slots).to(dev), torch.from_numpy(cu).to(dev)
    lens_d = torch.tensor(lens, dtype=torch.int32, device=dev)
    tables_d = torch.from_numpy(b.block_tables).to(dev)
    desc = pa.CacheDesc.make(num_blocks=b.num_blocks, block_size=Bs, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D,
                             max_blocks_per_seq=b.max_blocks_per_seq)
    out = torch.empty_like(q)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)

    def step(qq, kk, vv):
        pa.pa_append_kv(kk, vv, slots_d, kc, vc, desc, stream=stream)
        pa.pa_prefill(qq, kc, vc, tables_d, cu_d, lens_d, PF_NEW, b.scale, out, ws, desc, stream=stream,
                      kernel=args.prefill_kernel)

    step(q, k, v)
    torch.cuda.synchronize()
    if pa.pa_decode_status(ws) != 0:
        raise RuntimeError("prefill reported an error")
    for _ in range(args.warmup):
        step(q, k, v)
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index, enabled=not args.no_clocks)
    e0.record(stream)
    for i in range(K):
        pa.pa_append_kv(k, v, slots_d, kc, vc, desc, stream=stream)
        ev[i][0].record(stream)
        pa.pa_prefill(q, kc, vc, tables_d, cu_d, lens_d, PF_NEW, b.scale, out, ws, desc, stream=stream,
                      kernel=args.prefill_kernel)
        ev[i][1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    att_ms = float(np.mean([a.elapsed_time(c) for a, c in ev]))
    ms, att_ms = max_over_ranks([ms, att_ms], dist, dev)
    # e2e: q, k, v from pinned host memory every step, the output back
    hq, hk, hv = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in (q_h, k_h, v_h))
    hout = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    E = max(1, min(args.e2e_steps, 200))
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(E):
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        step(dq, dk, dv)
        hout.copy_(out, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, = max_over_ranks([f0.elapsed_time(f1)], dist, dev)
    if rank != 0:
        return None
    flops = prefill_flops(lens, q_lens, Hq, D)
    pk = "tcgen05_ws" if args.prefill_kernel == "auto" else args.prefill_kernel   # auto at Bs = 16
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        pass
    peak, kind = (float(peaks["bf16_tflops"]), "measured") if "bf16_tflops" in peaks else (1590.0, "fallback")
    achieved = flops / (att_ms / 1e3) / 1e12
    res = {
        "metric": "paged prefill tokens/s and TFLOP/s (fraction of B200 bf16 peak)",
        "value": world * T * K / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT["pf"], "config": "pf", "sequences": B, "new_tokens": q_lens,
                   "context": lens, "call": "pa_append_kv + pa_prefill",
                   "l2": "working set (%.0f MB of KV) fits L2: prefill is compute-bound" % (2 * b.k_cache.nbytes / 1e6)},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_kind": kind,
                     "traffic": profiled_traffic("pf", "prefill_ws" if pk == "tcgen05_ws" else "prefill")
                                if pk in ("tcgen05", "tcgen05_ws") else None,
                     "kernel": "pa_prefill (%s bf16)" % {"mma": "mma.sync", "tcgen05": "tcgen05",
                                                         "tcgen05_ws": "tcgen05, warp-specialized"}[pk],
                     "algorithmic_flops_per_launch": flops, "avg_launch_ms": att_ms},
        "e2e": {"value": world * T * E / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int((q_h.nbytes + k_h.nbytes + v_h.nbytes)), "d2h_bytes_per_step": int(q_h.nbytes),
                "steps": E},
        "gpu_launches": 2 * K, "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = pf_cpu_baseline(b, q_h, cu, lens, B, args.cpu_seconds)
    return res


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.impl == "reference":
        res = run_reference(args, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist_mod
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    try:
        runner = {"c5": run_c5, "pc": run_pc, "pf": run_pf}.get(args.config, run_ours)
        res = runner(args, rank, world, dist)
        if args.config == "c5" and not args.no_also:
            also = run_also(args, rank, world, dist)
            if res is not None:
                res["also"] = also
        if res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
