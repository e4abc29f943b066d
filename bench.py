#!/usr/bin/env python
"""Benchmark of the paged decode step (KV append + paged decode attention).

One step = one decode step of one attention layer for the whole batch:
append each sequence's new token into its slot (pa_append_kv), then paged
decode attention over every cached token (pa_decode; long contexts split
across CTAs and merged in the same launch).  The default workload is the
Llama-3.2-1B-shaped layer: 64 sequences, Hq=32, Hkv=8, head_dim 64, block
size 16, cached lengths uniform in [128, 2048], blocks scattered over a pool
10 % larger than needed.  Successive steps rotate over independent copies of
the layer's pool (different addresses, > 1 GB together) so that the 126 MB L2
cannot serve the K/V reads.

Prints one JSON line (rank 0).  `value` is seq-steps/s over all ranks with
inputs resident in HBM; `e2e` repeats the measurement with each step's inputs
copied from pinned host memory and the output copied back inside the timed
region.  `roofline` reports the decode kernel's KV-read bandwidth against the
measured HBM copy bandwidth.  `cpu_baseline` times the fp64 CPU oracle on a
bounded sample.  With --impl reference the oracle alone is timed.

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
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=["c1", "c2", "c3", "c4", "c5", "pc", "pf"], default="c2",
                    help="pc: prefix caching + copy-on-write (host admission by token ids on the "
                         "C3 request mix, device block copies)")
    ap.add_argument("--trace-steps", type=int, default=200,
                    help="c5: decode steps timed (the 100-step trace replayed as needed)")
    ap.add_argument("--kernel", choices=["auto", "simt", "tensor", "split"], default="auto")
    ap.add_argument("--max-ctas", type=int, default=0)
    ap.add_argument("--prefill-kernel", choices=["auto", "tcgen05", "mma"], default="auto",
                    help="pf: tcgen05 (tensor-memory accumulators; auto) or warp-level mma.sync")
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
    ap.add_argument("--pdl", choices=["on", "off"], default="on",
                    help="PA_FLAG_PDL: the tensor kernel plans its work while the previous kernel "
                         "runs; tables and lengths are written once before the timed region, as "
                         "the flag requires (per-call events are then left out: they would "
                         "serialise the calls)")
    return ap.parse_args(argv)


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
             "prefill": ["prefill_tc.cu", "pa_umma.cuh", "pa_ptx.cuh"]}[kernel_name]
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
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index, enabled=True):
        self.proc = None
        self.device_index = device_index
        if not enabled:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# the reference arm: the fp64 CPU oracle
# ---------------------------------------------------------------------------------------------
def run_reference(args, rank):
    import oracle
    if rank != 0:
        return None
    if args.config == "c5":
        t = wl.Trace5()
        bm = oracle.BlockManagerModel(t.num_blocks, t.block_size, t.batch, t.max_blocks_per_seq,
                                      t.free_order)
        for s in range(t.batch):
            bm.add_seq(s, int(t.initial_lens[s]))
        bm.append_tokens(list(range(t.batch)))
        tables = np.array([[bm.table_array(s) for s in range(t.batch)]], dtype=np.int32)
        lens = np.array([bm.lens], dtype=np.int32)
        t.steps = 1
        cb = cpu_baseline_c5(t, tables, lens, max(1.0, args.cpu_seconds))
        return {"metric": METRIC, "value": cb["value"], "unit": "seq-steps/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / cb["value"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": WORKLOAD_TEXT["c5"], "config": "c5", "batch": t.batch},
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "seq-steps/s", "h2d_bytes_per_step": 0,
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


def cpu_baseline(b, slots, tables, lens, budget_s):
    """The oracle as it stands on the host's cores, on whole-batch steps until the budget is spent."""
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
    return {"value": n * b.batch / dt, "unit": "seq-steps/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d whole-batch steps of %s (append + decode of all %d sequences x %d heads), %.1f s"
                      % (n, b.name, b.batch, b.num_q_heads, dt)}


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------
def run_ours(args, rank, world, dist):
    import torch
    import pagedattention_kv_cache_pa_b200 as pa

    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    b = wl.CONFIGS[args.config]()
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

    e4m3 = args.kv == "e4m3"
    KS = VS = 5.0 / 448                                  # N(0,1) data: |x| <= 5 fills the E4M3 range
    pool_bytes = 2 * b.k_cache.nbytes // (2 if e4m3 else 1)
    layers = max(1, min(8, math.ceil(1.0e9 / pool_bytes)))
    desc0 = pa.CacheDesc.make(num_blocks=b.num_blocks, block_size=Bs, num_kv_heads=Hkv, num_q_heads=Hq,
                              head_dim=D, max_blocks_per_seq=MB)

    def pool(a):
        t = to_dev(a)
        if not e4m3:
            return t
        # E4M3 pool: every slot's rows quantized by the library's own append
        rows = t.permute(0, 2, 1, 3).reshape(-1, Hkv, D).contiguous()
        qp = torch.empty(t.shape, dtype=torch.uint8, device=dev)
        pa.pa_append_kv_e4m3(rows, rows, torch.arange(rows.shape[0], dtype=torch.int64, device=dev), KS, KS,
                             qp, qp, desc0)
        return qp
    kcs = [pool(b.k_cache) for _ in range(layers)]
    vcs = [pool(b.v_cache) for _ in range(layers)]
    torch.cuda.synchronize()
    q, k_new, v_new = to_dev(b.q), to_dev(b.k_new), to_dev(b.v_new)
    slots_d = torch.from_numpy(slots).to(dev)
    tables_d = torch.from_numpy(tables).to(dev)
    lens_d = torch.from_numpy(lens).to(dev)
    out = torch.empty_like(q)
    desc = pa.CacheDesc.make(num_blocks=b.num_blocks, block_size=Bs, num_kv_heads=Hkv,
                             num_q_heads=Hq, head_dim=D, max_blocks_per_seq=MB)
    kernel = {"auto": pa.PA_KERNEL_AUTO, "simt": pa.PA_KERNEL_SIMT,
              "tensor": pa.PA_KERNEL_TENSOR, "split": pa.PA_KERNEL_TENSOR_SPLIT}[args.kernel]
    pdl = args.pdl == "on"
    kvo = dict(kv_dtype=pa.PA_KV_E4M3, k_scale=KS, v_scale=VS) if e4m3 else {}
    opts = pa.DecodeOptions(split_tokens=args.split_tokens, kernel=kernel, max_ctas=args.max_ctas,
                            flags=pa.PA_FLAG_PDL if pdl else 0, rope_theta=args.rope, **kvo)
    wsb = pa.pa_decode_workspace_size(B, max_len, desc, opts)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    splits = pa.pa_decode_max_splits(B, max_len, desc, opts)

    fused = args.path == "fused"
    # separate path: pa_append_kv (or pa_rope_append_kv) through the slot mapping, then pa_decode
    opts_dec = pa.DecodeOptions(split_tokens=args.split_tokens, kernel=kernel, max_ctas=args.max_ctas,
                                flags=pa.PA_FLAG_PDL if pdl else 0, **kvo)
    pos_d = torch.from_numpy(np.maximum(lens - 1, 0).astype(np.int32)).to(dev)
    q_rot = torch.empty_like(q)

    def separate(qq, kk, vv, sl, tb, ln, L, ev=None):
        if args.rope > 0:
            pa.pa_rope_append_kv(qq, q_rot, kk, vv, pos_d, sl, args.rope, kcs[L], vcs[L], desc,
                                 stream=stream)
            qq = q_rot
        elif e4m3:
            pa.pa_append_kv_e4m3(kk, vv, sl, KS, VS, kcs[L], vcs[L], desc, stream=stream)
        else:
            pa.pa_append_kv(kk, vv, sl, kcs[L], vcs[L], desc, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        pa.pa_decode(qq, kcs[L], vcs[L], tb, ln, max_len, b.scale, out, ws, desc, opts_dec,
                     stream=stream)
        if ev is not None:
            ev[1].record(stream)

    def step(i):
        L = i % layers
        if fused:
            pa.pa_append_decode(q, k_new, v_new, kcs[L], vcs[L], tables_d, lens_d, max_len, b.scale,
                                out, ws, desc, opts, stream=stream)
        else:
            separate(q, k_new, v_new, slots_d, tables_d, lens_d, L)

    # correctness guard before timing: the kernel must not report device errors
    step(0)
    torch.cuda.synchronize()
    rc = pa.pa_decode_status(ws)
    if rc != 0:
        raise RuntimeError("decode reported %s" % pa.pa_status_string(rc))

    for i in range(args.warmup):
        step(i)
    K = args.steps
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index, enabled=not args.no_clocks)
    t_start.record(stream)
    for i in range(K):
        L = i % layers
        if fused:
            if not pdl:
                ev_dec[i][0].record(stream)
            pa.pa_append_decode(q, k_new, v_new, kcs[L], vcs[L], tables_d, lens_d, max_len, b.scale,
                                out, ws, desc, opts, stream=stream)
            if not pdl:
                ev_dec[i][1].record(stream)
        else:
            separate(q, k_new, v_new, slots_d, tables_d, lens_d, L, None if pdl else ev_dec[i])
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

    # ---- e2e: host buffers in, result out, every step -----------------------------------
    E = args.e2e_steps
    h_q = torch.from_numpy(b.q.view(np.int16)).view(torch.bfloat16).pin_memory()
    h_k = torch.from_numpy(b.k_new.view(np.int16)).view(torch.bfloat16).pin_memory()
    h_v = torch.from_numpy(b.v_new.view(np.int16)).view(torch.bfloat16).pin_memory()
    h_slots = torch.from_numpy(slots).pin_memory()
    h_tables = torch.from_numpy(tables).pin_memory()
    h_lens = torch.from_numpy(lens).pin_memory()
    h_out = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    d_q, d_k, d_v = torch.empty_like(q), torch.empty_like(k_new), torch.empty_like(v_new)
    d_slots, d_tables, d_lens = (torch.empty_like(slots_d), torch.empty_like(tables_d),
                                 torch.empty_like(lens_d))
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k, h_v, h_slots, h_tables, h_lens))
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step(i):
        L = i % layers
        for dst, src in ((d_q, h_q), (d_k, h_k), (d_v, h_v), (d_slots, h_slots),
                         (d_tables, h_tables), (d_lens, h_lens)):
            dst.copy_(src, non_blocking=True)
        if fused:
            pa.pa_append_decode(d_q, d_k, d_v, kcs[L], vcs[L], d_tables, d_lens, max_len, b.scale,
                                out, ws, desc, opts, stream=stream)
        else:
            separate(d_q, d_k, d_v, d_slots, d_tables, d_lens, L)
        h_out.copy_(out, non_blocking=True)

    for i in range(min(args.warmup, 20)):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(E):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms, = max_over_ranks([e2e_ms], dist, dev)
    e2e_value = world * B * E / (e2e_ms / 1e3)

    if rank != 0:
        return None

    # PA_KERNEL_AUTO runs the tensor-core kernel; with Hkv a multiple of 8 (every
    # workload here) that is the whole-group, stream-partitioned one
    kernel_name = {pa.PA_KERNEL_SIMT: "simt", pa.PA_KERNEL_TENSOR_SPLIT: "split"}.get(kernel, "tensor")
    peak, peak_kind = measured_peaks()
    kv_bytes = kv_read_bytes(lens, Hkv, D, 1 if e4m3 else 2)
    achieved = kv_bytes / (dec_avg_ms / 1e3) / 1e9
    res = {
        "metric": METRIC, "value": value, "unit": "seq-steps/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 kv, bf16 q/out" if e4m3 else "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.config], "config": args.config,
                   "batch": B, "num_q_heads": Hq, "num_kv_heads": Hkv, "head_dim": D,
                   "block_size": Bs, "num_blocks": b.num_blocks, "mean_context": float(lens.mean()),
                   "max_context": max_len, "decode_kernel": kernel_name,
                   "split_tokens": args.split_tokens or "auto", "max_splits": splits,
                   "call": "pa_append_decode" if fused else
                           ("pa_rope_append_kv + pa_decode" if args.rope > 0 else "pa_append_kv + pa_decode"),
                   "pdl": pdl, "rope_theta": args.rope, "kv_dtype": args.kv,
                   "l2": "inputs larger than L2: %d rotating layer pools of %.0f MB" % (layers, pool_bytes / 1e6),
                   "parallelism": "replicas x%d" % world},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "frac_of_nominal_8000": achieved / NOMINAL_HBM_GBS,
                     "traffic": profiled_traffic(args.config + ("-e4m3" if e4m3 else ""), kernel_name),
                     "kernel": ("pa_append_decode (%s)" if fused else "pa_decode (%s)") % kernel_name,
                     "algorithmic_bytes_per_launch": kv_bytes,
                     "avg_launch_ms": dec_avg_ms,
                     "launch_timing": "timed region / calls" if pdl else "CUDA events around each call"},
        "kv_read_gbs_step": kv_bytes * K / (elapsed_ms / 1e3) / 1e9,
        "e2e": {"value": e2e_value, "unit": "seq-steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": E},
        # per step: the append (its own kernel unless the tensor kernel fuses it), the decode
        # kernel and (when any sequence can be cut) the merge kernel
        "gpu_launches": K * ((0 if (fused and kernel_name == "tensor") else 1) + 1 +
                             (1 if (kernel_name == "tensor" or splits > 1) else 0)),
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(b, slots, tables, lens, args.cpu_seconds)
    return res


def run_c5(args, rank, world, dist):
    """C5: the continuous-batching trace.  One step = one decode step of all 16 layers for the
    256 live sequences (host block manager, then pa_append_decode per layer)."""
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

    kcs, vcs, qs, ks, vs, outs = [], [], [], [], [], []
    for layer in range(NL):
        kc, vc = t.pool(layer)
        kcs.append(to_dev(kc))
        vcs.append(to_dev(vc))
        del kc, vc
        q, k, v = t.token_inputs(layer, 0)
        qs.append(to_dev(q))
        ks.append(to_dev(k))
        vs.append(to_dev(v))
        outs.append(torch.empty_like(qs[-1]))
    desc = pa.CacheDesc.make(num_blocks=N, block_size=Bs, num_kv_heads=Hkv, num_q_heads=Hq,
                             head_dim=D, max_blocks_per_seq=MB)
    kernel = {"auto": pa.PA_KERNEL_AUTO, "simt": pa.PA_KERNEL_SIMT,
              "tensor": pa.PA_KERNEL_TENSOR, "split": pa.PA_KERNEL_TENSOR_SPLIT}[args.kernel]
    pdl = args.pdl == "on"
    opts = pa.DecodeOptions(split_tokens=args.split_tokens, kernel=kernel, max_ctas=args.max_ctas,
                            flags=pa.PA_FLAG_PDL if pdl else 0, rope_theta=args.rope)
    ws = torch.zeros(pa.pa_decode_workspace_size(B, int(lens.max()), desc, opts), dtype=torch.uint8,
                     device=dev)

    def call(s, layer):
        pa.pa_append_decode(qs[layer], ks[layer], vs[layer], kcs[layer], vcs[layer], tables_d[s],
                            lens_d[s], step_max[s], t.scale, outs[layer], ws, desc, opts,
                            stream=stream)

    for s in range(3):
        for layer in range(NL):
            call(s, layer)
    torch.cuda.synchronize()
    rc = pa.pa_decode_status(ws)
    if rc != 0:
        raise RuntimeError("decode reported %s" % pa.pa_status_string(rc))
    K = args.trace_steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K * NL)]
    t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index, enabled=not args.no_clocks)
    t0e.record(stream)
    for i in range(K):
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

    # e2e: the host block manager replays the trace inside the timed region; per step the
    # table rows and lengths go up, per layer q/k/v go up and the output comes back
    E = min(args.e2e_steps, S)
    h_q = [torch.from_numpy(np.ascontiguousarray(t.token_inputs(l, 0)[0]).view(np.int16)).view(torch.bfloat16).pin_memory() for l in range(NL)]
    h_k = [torch.from_numpy(np.ascontiguousarray(t.token_inputs(l, 0)[1]).view(np.int16)).view(torch.bfloat16).pin_memory() for l in range(NL)]
    h_v = [torch.from_numpy(np.ascontiguousarray(t.token_inputs(l, 0)[2]).view(np.int16)).view(torch.bfloat16).pin_memory() for l in range(NL)]
    h_out = torch.empty(outs[0].shape, dtype=torch.bfloat16).pin_memory()
    h_tab = torch.empty((B, MB), dtype=torch.int32).pin_memory()
    h_len = torch.empty((B,), dtype=torch.int32).pin_memory()
    d_q, d_k, d_v = torch.empty_like(qs[0]), torch.empty_like(ks[0]), torch.empty_like(vs[0])
    d_tab, d_len = torch.empty((B, MB), dtype=torch.int32, device=dev), torch.empty((B,), dtype=torch.int32, device=dev)
    h2d = h_tab.numel() * 4 + h_len.numel() * 4 + NL * (h_q[0].numel() + h_k[0].numel() + h_v[0].numel()) * 2
    d2h = NL * h_out.numel() * 2
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for step, bm in replay():
        if step >= E:
            break
        torch.cuda.current_stream().synchronize()   # pinned staging is reused each step
        h_tab.numpy()[:] = bm.block_tables()
        h_len.numpy()[:] = bm.context_lens()
        d_tab.copy_(h_tab, non_blocking=True)
        d_len.copy_(h_len, non_blocking=True)
        mx = int(h_len.numpy().max())
        for layer in range(NL):
            d_q.copy_(h_q[layer], non_blocking=True)
            d_k.copy_(h_k[layer], non_blocking=True)
            d_v.copy_(h_v[layer], non_blocking=True)
            pa.pa_append_decode(d_q, d_k, d_v, kcs[layer], vcs[layer], d_tab, d_len, mx, t.scale,
                                outs[layer], ws, desc, opts, stream=stream)
            h_out.copy_(outs[layer], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms, = max_over_ranks([e2e_ms], dist, dev)
    if rank != 0:
        return None
    peak, peak_kind = measured_peaks()
    kernel_name = {pa.PA_KERNEL_SIMT: "simt", pa.PA_KERNEL_TENSOR_SPLIT: "split"}.get(kernel, "tensor")
    res = {
        "metric": METRIC, "value": value, "unit": "seq-steps/s", "n_gpus": world, "steps": K,
        "warmup": 3, "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT["c5"], "config": "c5", "batch": B, "layers": NL,
                   "trace_steps": S, "num_blocks": N, "mean_context": float(lens.mean()),
                   "decode_kernel": kernel_name, "call": "pa_append_decode per layer", "pdl": pdl,
                   "rope_theta": args.rope,
                   "l2": "inputs larger than L2: 16 layer pools of %.0f MB" % (2 * kcs[0].numel() * 2 / 1e6),
                   "parallelism": "replicas x%d" % world},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                     "frac": gbs / peak, "peak_kind": peak_kind,
                     "frac_of_nominal_8000": gbs / NOMINAL_HBM_GBS,
                     "traffic": profiled_traffic("c5", kernel_name),
                     "kernel": "pa_append_decode (%s)" % kernel_name,
                     "algorithmic_bytes_per_launch": float(kv_per_call.mean()),
                     "avg_launch_ms": float(call_ms.mean()),
                     "launch_timing": "timed region / calls" if pdl else "CUDA events around each call"},
        "e2e": {"value": world * B * E / (e2e_ms / 1e3), "unit": "seq-steps/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": E,
                "includes": "host block manager (retire, admit, append) per step"},
        "gpu_launches": K * NL * 2,
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline_c5(t, tables, lens, args.cpu_seconds)
    return res


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
    # one seq-step = one sequence through all layers: the sample covers 1 of the 16 layers
    return {"value": n * t.batch / dt / t.layers, "unit": "seq-steps/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d trace steps of layer 0 only (256 sequences x 32 heads each), %.1f s; "
                      "value scaled to all %d layers" % (n, dt, t.layers)}


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
                     "traffic": None if args.prefill_kernel == "mma" else profiled_traffic("pf", "prefill"),
                     "kernel": "pa_prefill (%s bf16)" % ("mma.sync" if args.prefill_kernel == "mma" else "tcgen05"),
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
        if res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
