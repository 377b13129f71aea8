"""Benchmark of the hybrid compressed attention path on B200.

Default run: the headline workload, one CSA layer prefill, bf16, T=131072, D=2048 (projection +
compressor + lightning indexer/top-k + attention), inputs resident in HBM; `value` is tokens/s over all
ranks (each rank runs its own independent sequence: weak scaling, no collective on the data path).
Then the other workloads, each measured the same way and nested in the same JSON line under
"workloads": HCA prefill T=65536, CSA decode B=32 at a 262144-token prefix, the 8-layer CSA/HCA decode
stack B=4 at 1M context, and the V4-style stack (two HCA layers, then CSA/HCA alternating, chained
through the residual stream).  Every workload carries its roofline, end-to-end and CPU-oracle figures.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference] [--no-extra]

--workload NAME runs one workload alone (hca_prefill_T65536, csa_decode_B32_P262144,
hybrid_decode_B4_P1048576, v4_decode_B4_P1048576, csa_prefill_T131072).
"""
from __future__ import annotations

import argparse
import dataclasses
import gc
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "CSA/HCA prefill tokens/s and decode µs/step at 128K-1M ctx; % of HBM/TC roofline"

WORKLOADS = {
    "csa_prefill_T131072": ("prefill", "csa_bf16_t131072", False),
    "hca_prefill_T65536": ("prefill", "hca_bf16_t65536", False),
    "csa_decode_B32_P262144": ("decode", "csa_decode_b32_p262144", False),
    "hybrid_decode_B4_P1048576": ("decode", "hybrid_decode_b4_p1048576", False),
    "v4_decode_B4_P1048576": ("decode", "v4_decode_b4_p1048576", False),
    # the same layers with FP8 entries and FP4 indexer keys (block-scaled storage; bf16 arithmetic)
    "csa_prefill_fp8fp4_T131072": ("prefill", "csa_bf16_t131072", True),
    "csa_decode_fp8fp4_B32_P262144": ("decode", "csa_decode_b32_p262144", True),
    "hybrid_decode_fp8fp4_B4_P1048576": ("decode", "hybrid_decode_b4_p1048576", True),
}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ algorithmic work per call

# DRAM bytes per query token of the tensor-core attention kernel (query rows in, output rows out; the
# gathered key/value rows are served by L2), from an ncu capture of the same kernel at T=8192 with
# dram__bytes_read.sum + dram__bytes_write.sum = 576.9 + 499.8 MB; linear in T.
ATTEND_TC_DRAM_BYTES_PER_TOKEN = 1076.7e6 / 8192

# Rate at which 148 CTAs gather random 128-byte row segments into shared memory with 16-byte cp.async,
# measured on this B200 (the same for tables of 32 to 256 MB).
GATHER_CEILING_GBS = 7340.0


def prefill_work(spec):
    """Algorithmic flops / bytes of each call of a prefill layer (visible pairs only)."""
    T, m, k, win = spec.T, spec.m, spec.topk, spec.window
    t = np.arange(T, dtype=np.float64)
    vis = np.minimum(t // m, -(-T // m))
    nwin = np.minimum(win, t + 1)
    bpe = 2 if spec.dtype == "bf16" else 4
    w = {}
    ncols = 2 * spec.C + spec.H * spec.dh + (spec.di + spec.Hi * spec.di + spec.Hi if spec.kind == "csa" else 0)
    w["hcsa_project"] = {"flops": 2.0 * T * spec.D * ncols}
    N = -(-T // m)
    pool_ch = spec.C + (spec.di if spec.kind == "csa" else 0)
    w["compress"] = {"bytes": float(T * (2 * spec.C + (spec.di if spec.kind == "csa" else 0)) * bpe
                                    + N * pool_ch * bpe)}
    if spec.kind == "csa":
        w["csa_index_topk"] = {"flops": float(vis.sum()) * spec.Hi * spec.di * 2.0}
        nkeys = np.minimum(vis, k) + nwin
    else:
        nkeys = vis + nwin
    w["attend"] = {"flops": float(nkeys.sum()) * spec.H * spec.dh * 4.0}
    return w


def decode_bytes(spec, B, N, residual=False, lowprec=False):
    """Algorithmic HBM bytes of one decode step of one layer (weights + cache reads + writes; with the
    residual chain also the output projection and the hidden state read and written).  lowprec: entries
    of C + C/32 bytes (FP8 codes + exponents), indexer keys of di/2 + di/32 bytes (FP4)."""
    bpe = 2
    ent = spec.C + spec.C // 32 if lowprec else spec.C * bpe
    ncols = 2 * spec.C + spec.H * spec.dh + (spec.di + spec.Hi * spec.di + spec.Hi if spec.kind == "csa" else 0)
    b = spec.D * ncols * bpe                                   # weights
    if spec.kind == "csa":
        key = spec.di // 2 + spec.di // 32 if lowprec else spec.di * bpe
        b += B * N * key                                       # indexer key scan
        b += B * spec.topk * ent + B * spec.window * spec.C * bpe   # selected rows + window
    else:
        b += B * N * ent + B * spec.window * spec.C * bpe      # all entries + window
    b += B * spec.H * spec.dh * bpe * 2                        # q in, out
    if residual:
        b += spec.H * spec.dh * spec.D * bpe + B * spec.D * bpe * 2   # W_o, x in and out
    return float(b)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, sampled while the timed region runs.

    NVML is polled every 2 ms from a thread (a decode step is well under a millisecond, so the timed
    region can be shorter than nvidia-smi's sampling period); nvidia-smi -lms 200 is the fallback."""

    _REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, dev_index):
        self.samples, self.p, self.thread = [], None, None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv, self.h = pynvml, self._handle(pynvml, dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            get = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.get_reasons = get
            import threading
            self.stop_ev = threading.Event()
            self._sample()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={dev_index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                       "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    @staticmethod
    def _handle(nv, dev_index):
        """NVML handle of torch's device `dev_index` (by UUID, so CUDA_VISIBLE_DEVICES remapping is honoured)."""
        try:
            u = str(torch.cuda.get_device_properties(dev_index).uuid)
            return nv.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)
        except Exception:
            pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ent = vis.split(",")[dev_index].strip() if vis else str(dev_index)
        if ent.startswith("GPU-"):
            return nv.nvmlDeviceGetHandleByUUID(ent)
        return nv.nvmlDeviceGetHandleByIndex(int(ent))

    def _sample(self):
        sm = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
        self.samples.append((float(sm), int(self.get_reasons(self.h))))

    def _run(self):
        while not self.stop_ev.wait(0.002):
            try:
                self._sample()
            except Exception:
                return

    def stop(self):
        if self.thread is not None:
            self.stop_ev.set()
            self.thread.join(timeout=5)
            if not self.samples:
                return None
            sm = [x[0] for x in self.samples]
            reasons = sorted({name for x in self.samples for bit, name in self._REASONS.items() if x[1] & bit})
            loaded = sorted(sm)[len(sm) // 4:] or sm
            return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": float(self.max_mhz), "reasons": reasons,
                    "samples": len(sm), "source": "nvml"}
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = []
        with open(self.f.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        loaded = sorted(sm)[len(sm) // 4:] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows), "source": "nvidia-smi"}


# ------------------------------------------------------------------ distributed plumbing

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ CPU oracle timing (bounded sample)

def _host_cores():
    return len(os.sched_getaffinity(0))


def oracle_prefill_rate(spec, inp, n_rows=1024, offset=0.5, entries=None, lowprec=False):
    """Oracle throughput (tokens/s) of the whole layer, from a bounded sample of the workload's own inputs.

    The sequence-wide half (projections of the pooled columns and the compressor over all T tokens) is
    timed in full, unless `entries` = (result, seconds) of an earlier timing is passed.  The per-query half
    (query projections, indexer, top-k, attention over the real entries) is timed on n_rows query
    positions spread evenly over the sequence -- row i at (i + offset) T / n_rows, so the sample has the
    sequence's mix of visible counts -- and scaled by T / n_rows.  Returns (tokens/s, sample description,
    (result, seconds) of the sequence-wide half)."""
    import oracle
    T = spec.T
    if entries is None:
        t0 = time.perf_counter()
        res = oracle.prefill_entries(spec, inp, lowprec=lowprec)
        entries = (res, time.perf_counter() - t0)
    res, t_fixed = entries
    n_rows = min(n_rows, T)
    rows = np.unique(((np.arange(n_rows) + offset) * T / n_rows).astype(np.int64))
    t0 = time.perf_counter()
    oracle.prefill_queries(spec, inp, res, rows)
    t_q = time.perf_counter() - t0
    total = t_fixed + t_q * T / len(rows)
    sample = (f"projections + compressor over all T={T} tokens ({t_fixed:.1f} s), then query projections + "
              f"indexer + top-k + attention for {len(rows)} evenly spread query rows ({t_q:.1f} s) scaled by "
              f"T/{len(rows)}; {oracle.num_threads()} OpenMP threads on {_host_cores()} host cores; "
              f"whole-layer time {total:.1f} s")
    return T / total, sample, entries


def oracle_decode_rate(d, seq=0, lowprec=False):
    """Oracle µs per decode step, timed on one sequence of the workload's own inputs (its cache, weights
    and new token) through every layer in order -- with the residual chain, each layer's output
    projection and residual update included -- and scaled to the batch of B independent sequences.
    Returns (µs/step, sample description)."""
    import oracle
    import synth
    x = None
    elapsed = 0.0
    for li, spec in enumerate(d.layers):
        inp = synth.decode_inputs(d, li, seqs=[seq])
        inp["x"] = inp["x"][seq:seq + 1] if x is None else x
        t0 = time.perf_counter()
        x, _ = oracle.decode_stack([spec], [inp], d.P, residual=d.residual, lowprec=lowprec)
        elapsed += time.perf_counter() - t0
        if not d.residual:
            x = None
        del inp
    us = elapsed * d.B * 1e6
    sample = (f"sequence {seq} of {d.B} through all {len(d.layers)} layers (append, indexer, top-k, attention"
              f"{', output projection + residual' if d.residual else ''}) on its own cache at P={d.P} "
              f"({elapsed:.1f} s), scaled by B={d.B}; {oracle.num_threads()} OpenMP threads on "
              f"{_host_cores()} host cores")
    return us, sample


# ------------------------------------------------------------------ our arm

def run_prefill(args, spec_name, ws, rank, lowprec=False):
    import long_context_compressed_05_b200 as h
    import synth
    from long_context_compressed_05_b200.host import to_device as dev
    spec = synth.PREFILL[spec_name]
    if args.tokens:
        spec = spec.replace(T=args.tokens)
    if ws > 1:
        spec = spec.replace(seed=spec.seed + 1000 * rank)   # independent sequence per rank
    inp = synth.prefill_inputs(spec)
    x, W, B = dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"])
    layer = h.PrefillLayer(spec, lowprec=lowprec)
    stream = torch.cuda.current_stream()
    calls = ["hcsa_project", "compress"] + (["csa_index_topk"] if spec.kind == "csa" else []) + ["attend"]

    def step(evs=None):
        fns = [lambda: layer.project(x, W), lambda: layer.compress(B)]
        if spec.kind == "csa":
            fns.append(layer.index_topk)
        fns.append(layer.attend)
        for i, f in enumerate(fns):
            if evs is not None:
                evs[i][0].record(stream)
            f()
            if evs is not None:
                evs[i][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
           for _ in range(args.steps)]
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    barrier(ws)
    torch.cuda.synchronize()
    h.hcsa_launch_count(reset=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(args.steps):
        step(evs[s])
    e1.record(stream)
    torch.cuda.synchronize()
    launches = h.hcsa_launch_count()
    barrier(ws)
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(e0.elapsed_time(e1), ws) / args.steps
    phase_ms = {c: statistics.mean(evs[s][i][0].elapsed_time(evs[s][i][1]) for s in range(args.steps))
                for i, c in enumerate(calls)}
    value = ws * spec.T / (ms / 1e3)
    work = prefill_work(spec)
    hbm, tc, tc_sus, src = peaks()
    ours = {c: t for c, t in phase_ms.items() if c != "hcsa_project"}
    dom = max(ours, key=ours.get)
    wk = work[dom]
    if "flops" in wk:
        ach = wk["flops"] / (ours[dom] / 1e3) / 1e12
        traffic = None
        if dom == "attend" and spec.kind == "csa" and spec.H == 64 and spec.dh == 512 and not lowprec:
            traffic = ATTEND_TC_DRAM_BYTES_PER_TOKEN * spec.T
        roof = {"bound": "tensor", "achieved": ach, "peak": tc_sus, "unit": "TFLOP/s", "frac": ach / tc_sus,
                "traffic": traffic, "kernel": dom, "peak_kind": f"{src} bf16 sustained"}
        if dom == "attend" and spec.kind == "csa":
            # the kernel's gathered 128-byte segments of entry rows, against the rate a microbenchmark
            # measured on this B200 for random 128-byte segments moved by 16-byte cp.async into a
            # swizzled ring (148 CTAs, row indices from shared memory): 7.33-7.35 TB/s for any table
            # size from 32 to 256 MB
            ent_mb = -(-spec.T // spec.m) * spec.C * (1 if lowprec else 2) / 2 ** 20
            ceiling = GATHER_CEILING_GBS
            t = np.arange(spec.T, dtype=np.float64)
            rows = np.minimum(np.minimum(t // spec.m, -(-spec.T // spec.m)), spec.topk).sum()
            gathered = rows * spec.C * (1 + 1 / 32 if lowprec else 2)
            gbs = gathered / (ours[dom] / 1e3) / 1e9
            roof["gather"] = {"achieved": gbs, "ceiling": ceiling, "unit": "GB/s", "frac": gbs / ceiling,
                              "bytes": gathered, "entries_MB": ent_mb}
    else:
        ach = wk["bytes"] / (ours[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "traffic": None,
                "kernel": dom, "peak_kind": f"{src} hbm"}
    # end to end through the public API: pinned host x in, the whole output back to pinned host memory every
    # step (forward_host: the output rows stream back by row range while the rest of the step runs)
    e2e = None
    if not args.no_e2e:
        xh = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        xh.copy_(x)
        oh = torch.empty(layer.out.shape, dtype=layer.out.dtype, pin_memory=True)
        ke = max(1, min(args.steps, 3))
        layer.forward_host(xh, W, B, oh)   # untimed: creates the copy stream and the input buffer
        layer.wait_host()
        torch.cuda.synchronize()
        barrier(ws)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(ke):
            layer.forward_host(xh, W, B, oh)
        layer.wait_host()
        a1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(a0.elapsed_time(a1), ws) / ke
        e2e = {"value": ws * spec.T / (ems / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": xh.numel() * xh.element_size(),
               "d2h_bytes_per_step": oh.numel() * oh.element_size()}
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) inputs, N(0,1/D) weights)",
            "config": {"workload": f"{spec.kind}_prefill_{'fp8fp4' if lowprec else 'bf16'}_T{spec.T}_D{spec.D}",
                       "T": spec.T, "D": spec.D, "C": spec.C, "topk": spec.topk, "H": spec.H, "dh": spec.dh,
                       "storage": ("entries FP8 E4M3, indexer keys FP4 E2M1, power-of-two scale per 32 channels"
                                   if lowprec else "bf16"),
                       "parallelism": f"replicas x{ws} (one sequence per GPU)",
                       "l2": "inputs larger than L2 (x 0.5 GB, projections 9.7 GB)"},
            "phase_ms": phase_ms, "roofline": roof, "e2e": e2e, "gpu_launches": launches, "clocks": clocks}
    return line, (spec, inp)


def run_decode(args, spec_name, ws, rank, lowprec=False):
    import long_context_compressed_05_b200 as h
    import synth
    from long_context_compressed_05_b200.host import to_device as dev
    d = synth.DECODE[spec_name]
    if args.batch:
        import dataclasses
        d = dataclasses.replace(d, B=args.batch)
    layers, Ws, Bs, Wos, xs = [], [], [], [], None
    for li, spec in enumerate(d.layers):
        inp = synth.decode_inputs(d, li)
        cache = {k: dev(inp[k]) for k in ("entries", "win_kv", "ring_g", "idx_keys", "ring_ki") if k in inp}
        n_cap = inp["entries"].shape[1]
        if lowprec:   # the same cache stored as FP8 entries / FP4 indexer keys (library quantizer)
            p = h.params_for(spec, T=0, B=d.B, n_cap=n_cap, lowprec=True)
            rows = d.B * n_cap
            for key, what, nbytes in (("entries", h.STORE_ENTRIES, h.hcsa_entry_bytes(p, rows)),
                                      ("idx_keys", h.STORE_KEYS, h.hcsa_key_bytes(p, rows))):
                if key in cache:
                    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
                    h.hcsa_quantize_rows(p, what, cache[key].reshape(rows, -1), buf)
                    cache[key] = buf
            torch.cuda.synchronize()
        layers.append(h.DecodeLayer(spec, d.B, n_cap, cache, lowprec=lowprec))
        Ws.append(dev(inp["W_cat"]))
        Bs.append(dev(inp["B"]))
        Wos.append(dev(inp["W_o"]) if d.residual else None)
        if xs is None:
            xs = dev(inp["x"])
        del inp
    pos = torch.full((d.B,), d.P, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    xw = torch.empty_like(xs)   # the residual stream of a chained stack (restarts from xs every step)

    def step(xw=xw):
        if d.residual:
            xw.copy_(xs)
            for L, W, B, Wo in zip(layers, Ws, Bs, Wos):
                L.step(xw, W, B, pos)
                L.out_project(xw, Wo)
        else:
            for L, W, B in zip(layers, Ws, Bs):
                L.step(xs, W, B, pos)   # each layer reads the same hidden state

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    barrier(ws)
    torch.cuda.synchronize()
    h.hcsa_launch_count(reset=True)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    clocks = sampler.stop() if sampler else None
    us = max_over_ranks(e0.elapsed_time(e1), ws) / args.steps * 1e3
    # launches per step: count one eager step
    h.hcsa_launch_count(reset=True)
    step()
    torch.cuda.synchronize()
    launches = h.hcsa_launch_count() * args.steps
    hbm, tc, tc_sus, src = peaks()
    total_bytes = sum(decode_bytes(L.spec, d.B, L.p.n_cap, d.residual, lowprec) for L in layers)
    ach = total_bytes / (us / 1e6) / 1e9
    roof = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "traffic": None,
            "kernel": "whole decode step (CUDA graph)", "peak_kind": f"{src} hbm"}
    # End to end: the step's input from pinned host memory and its result (the hidden state of a chained
    # stack, else the last layer's output) back to pinned host memory, every step.  The result buffer is
    # double-buffered (a second graph writes the other one), so step i's copy back overlaps step i + 1;
    # the replay of step i + 2 waits for it.
    xh = torch.empty(xs.shape, dtype=xs.dtype, pin_memory=True)
    xh.copy_(xs)
    if d.residual:
        res = (xw, torch.empty_like(xw))
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            step(res[1])
    else:
        res = (layers[-1].out, torch.empty_like(layers[-1].out))
        layers[-1].out = res[1]
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            step()
        layers[-1].out = res[0]
    graphs = (g, g2)
    oh = torch.empty(res[0].shape, dtype=res[0].dtype, pin_memory=True)
    cs = torch.cuda.Stream()
    copied = [None, None]
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for i in range(args.steps):
        k = i & 1
        xs.copy_(xh, non_blocking=True)
        if copied[k] is not None:
            stream.wait_event(copied[k])
        graphs[k].replay()
        done = torch.cuda.Event()
        done.record(stream)
        cs.wait_event(done)
        with torch.cuda.stream(cs):
            oh.copy_(res[k], non_blocking=True)
        copied[k] = torch.cuda.Event()
        copied[k].record(cs)
    stream.wait_stream(cs)
    a1.record(stream)
    torch.cuda.synchronize()
    eus = max_over_ranks(a0.elapsed_time(a1), ws) / args.steps * 1e3
    del g, g2, graphs
    line = {"metric": METRIC, "value": us, "unit": "us/step", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) caches and inputs)",
            "config": {"workload": spec_name.replace("_b", "_fp8fp4_b", 1) if lowprec else spec_name,
                       "B": d.B, "P": d.P, "layers": len(d.layers), "residual": d.residual,
                       "storage": ("entries FP8 E4M3, indexer keys FP4 E2M1, power-of-two scale per 32 channels"
                                   if lowprec else "bf16"),
                       "parallelism": f"replicas x{ws}", "l2": "working set larger than L2",
                       "bytes_per_step": total_bytes},
            "roofline": roof,
            "e2e": {"value": eus, "unit": "us/step", "h2d_bytes_per_step": xh.numel() * xh.element_size(),
                    "d2h_bytes_per_step": oh.numel() * oh.element_size()},
            "gpu_launches": launches, "clocks": clocks}
    return line, (d, None)


DEFAULT_WORKLOAD = "csa_prefill_T131072"
# measured after the headline in the default run and nested in its line under "workloads"
EXTRA_WORKLOADS = ["hca_prefill_T65536", "csa_decode_B32_P262144", "hybrid_decode_B4_P1048576",
                   "v4_decode_B4_P1048576"]
NESTED_KEYS = ["value", "unit", "higher_is_better", "steps", "warmup", "ms_per_step", "config", "phase_ms",
               "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"]


def run_workload(args, wl, ws, rank):
    """One workload on our arm: its JSON line, with the CPU oracle baseline (rank 0, one GPU)."""
    kind, name, lowprec = WORKLOADS[wl]
    if kind == "prefill":
        line, (spec, inp) = run_prefill(args, name, ws, rank, lowprec)
    else:
        line, (d, _) = run_decode(args, name, ws, rank, lowprec)
    line["cpu_baseline"] = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle
        if kind == "prefill":
            v, sample, _ = oracle_prefill_rate(spec, inp, lowprec=lowprec)
            unit = "tokens/s"
        else:
            v, sample = oracle_decode_rate(d, lowprec=lowprec)
            unit = "us/step"
        line["cpu_baseline"] = {"value": v, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": sample}
    gc.collect()
    torch.cuda.empty_cache()
    return line


def run_reference(args, wl, ws, rank):
    """The reference arm: the CPU oracle as it stands, timed on the host cores on bounded samples of the
    same workload (rank 0 only)."""
    import oracle
    import synth
    kind, name, lowprec = WORKLOADS[wl]
    vals = []
    n = args.warmup + args.steps
    if kind == "prefill":
        spec = synth.PREFILL[name]
        inp = synth.prefill_inputs(spec)
        entries = None
        for i in range(n):
            # the sequence-wide half is timed once (first step) and reused; every step times the per-query
            # half on 64 evenly spread rows, shifted from step to step
            v, sample, entries = oracle_prefill_rate(spec, inp, n_rows=64, offset=(i + 0.5) / n, entries=entries,
                                                     lowprec=lowprec)
            if i >= args.warmup:
                vals.append(v)
        sample += f"; per step: 64 query rows shifted by (step + 0.5)/{n} of a stratum, mean over {args.steps} steps"
        unit, hib = "tokens/s", True
        ms = spec.T / statistics.mean(vals) * 1e3
        config = {"workload": f"{spec.kind}_prefill_{'fp8fp4' if lowprec else 'bf16'}_T{spec.T}_D{spec.D}",
                  "T": spec.T, "D": spec.D, "C": spec.C, "topk": spec.topk, "H": spec.H, "dh": spec.dh,
                  "parallelism": "CPU oracle on rank 0"}
    else:
        d = synth.DECODE[name]
        for i in range(n):
            v, sample = oracle_decode_rate(d, seq=i % d.B, lowprec=lowprec)
            if i >= args.warmup:
                vals.append(v)
        unit, hib = "us/step", False
        ms = statistics.mean(vals) / 1e3
        config = {"workload": name.replace("_b", "_fp8fp4_b", 1) if lowprec else name, "B": d.B, "P": d.P,
                  "layers": len(d.layers), "residual": d.residual, "parallelism": "CPU oracle on rank 0"}
    v = statistics.mean(vals)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": hib, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, the same inputs as the CUDA path; bounded sample, scaled to the workload)",
            "config": config, "gpu_launches": 0,
            "cpu_baseline": {"value": v, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=None, choices=list(WORKLOADS),
                    help="run this workload alone (default: the CSA prefill headline, then the other workloads "
                         "nested in its line)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="default run without the nested workloads")
    ap.add_argument("--tokens", type=int, default=0, help="override T of a prefill workload (profiling small cases)")
    ap.add_argument("--batch", type=int, default=0, help="override B of a decode workload (profiling small cases)")
    args = ap.parse_args()
    ws, rank, local = dist_setup()
    wl = args.workload or DEFAULT_WORKLOAD

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, wl, ws, rank)))
        return

    line = run_workload(args, wl, ws, rank)
    if args.workload is None and not args.no_extra and not args.tokens and not args.batch:
        line["workloads"] = {}
        for x in EXTRA_WORKLOADS:
            sub = run_workload(args, x, ws, rank)
            line["workloads"][x] = {k: sub.get(k) for k in NESTED_KEYS}
    if rank == 0:
        print(json.dumps(line))
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
