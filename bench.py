#!/usr/bin/env python3
"""Benchmark of the RAT+ sequence-mixer hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  prefill of the long-context layer (B=2, T=16384, H=16, Dh=128, D=64, W=128):
    fused key/value scan + dilated/windowed attention;
  decode burst of the decode-from-32K-context workload (B=64, H=16, D=64,
    W=128): 256 fused decode steps (recurrence step, cache append, split-K
    attention over the D-compressed cache), captured in one CUDA graph.
`value` is prefill tokens/s of the T=16K, D=64 layer (whole job, all ranks);
decode tokens/s is reported beside it.  Kernels are timed with CUDA events on
the stream they are launched on; multi-GPU runs are weak-scaled replicas (no
data-path collective) timed as the max over ranks.

--impl reference times the fp64 CPU oracle (the only executable statement of
the method there is) on the same workload: each step is the whole T=16K
prefill plus a few literal decode steps of the 32K-context workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL = "bf16_long_T16384_D64_W128"
DECODE = "bf16_decode_ctx32768_D64_W128"
METRIC = "RAT+ layer prefill & decode tokens/s at T=16K, D=64; % of HBM/tensor roofline"


# ----------------------------------------------------------------------------- counts
def attention_pairs(T, D, W, dense=False):
    """Exact number of (query, key) pairs of one (b, h): sum_t |K(t)|."""
    t = np.arange(T, dtype=np.int64)
    if dense or D == 1:
        return int((t + 1).sum())
    if W <= 0:
        return int((t // D + 1).sum())
    lo = np.maximum(0, t - W + 1)
    F = lambda x: np.where(x >= 0, (x + 1) // D, 0)     # #{0 <= j <= x : j mod D = D-1}
    dup = F(t - 1) - F(lo - 1)
    return int((t // D + np.minimum(W, t + 1) - dup).sum())


def prefill_counts(w):
    E = w.B * w.T * w.H * w.Dh
    esz = 4 if w.dtype == "f32" else 2
    pairs = 0
    for h in range(w.H):
        pairs += w.B * attention_pairs(w.T, w.D, w.W, dense=h in w.dense_heads)
    return {
        "scan_bytes": 5 * E * esz,                # read xk, xv, g; write hk, hv
        "attn_bytes": 4 * E * esz,                # read q, hk, hv; write o
        "attn_flops": 4 * w.Dh * pairs,           # QK^T + PV over the key sets
        "pairs": pairs,
    }


def decode_bytes_per_step(w, t):
    """Algorithmic HBM bytes of one decode token for every (b, h) at position t."""
    total = 0
    for h in range(w.H):
        Dd = 1 if h in w.dense_heads else w.D
        n_slots = t // Dd
        n_win = 0
        if w.W > 0 and Dd > 1:
            lo = max(0, t - w.W + 1)
            n_win = sum(1 for p in range(lo, t) if p % Dd != Dd - 1)
        rows = n_slots + n_win
        per = rows * 2 * w.Dh * 2                 # K and V rows read
        per += 2 * w.Dh * 4 * 2                   # fp32 state read + write (k, v)
        per += 4 * w.Dh * 2 + w.Dh * 2            # q, xk, xv, g read; o written
        per += (2 * w.Dh * 2) if w.W > 0 else 0   # ring write
        per += (2 * w.Dh * 2) if t % Dd == Dd - 1 else 0   # dilated append
        total += w.B * per
    return total


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(values, world, device=None):
    """Element-wise max of per-rank timings (every rank calls it, same order)."""
    if world == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(units_per_rank, world, seconds_max):
    """Whole-job throughput of weak-scaled replicas: all ranks' units over the
    slowest rank's time."""
    return world * units_per_rank / seconds_max


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples during the timed region (clocks and throttle reasons)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def ready(self, timeout=5.0):
        """Wait for nvidia-smi's first sample, then drop what came before the
        timed region, so that every kept sample falls inside it."""
        t0 = time.perf_counter()
        while self.proc is not None and not self.lines and time.perf_counter() - t0 < timeout:
            time.sleep(0.01)
        self.lines.clear()

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


KERNEL_SOURCES = {
    "scan_kv": ["scan.cuh", "common.cuh", "sm100.cuh"],
    "dilated_attn": ["attn_tc.cuh", "fused.cuh", "scan.cuh", "common.cuh", "sm100.cuh"],
    "decode_step": ["decode.cuh", "common.cuh"],
}


def kernel_source_hash(kernel):
    """sha256 of the source files a kernel is built from (short form)."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "recurrence_augmented_dilated_chunked_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's source has changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "kernel_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    if d.get("source_sha") != kernel_source_hash(kernel):
        return None
    return d.get("dram_bytes_per_launch")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ----------------------------------------------------------------------------- oracle
class OracleBaseline:
    """The fp64 oracle (plain C, OpenMP over rows) on the headline workloads.

    prefill(): the whole prefill of the T=16K layer, nothing sampled: the
    scan of both streams over every token of both sequences and attention of
    every query row of every head over its key set.
    decode(n): n literal decode steps (recurrence step, append, attention
    over the cache contents) for all 64 sequences of the 32K-context
    workload, continuing from the previous call's position.
    Inputs are the GPU arm's seeded inputs (rank 0), converted to fp64 once,
    outside the timed calls, as the GPU arm's inputs are resident in HBM.
    """
    DECODE_PER_STEP = 4

    def __init__(self):
        import oracle
        from recurrence_augmented_dilated_chunked_b200 import (WORKLOADS, decode_context,
                                                               decode_inputs, prefill_inputs)
        self.oracle = oracle
        oracle.build()
        self.wp, self.wd = WORKLOADS[PREFILL], WORKLOADS[DECODE]
        w = self.wp
        self.pre = [x.to(torch.float64).numpy() for x in
                    prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype, w.gate_mean, w.gate_std, seed=0)]
        wd = self.wd
        steps = wd.decode_steps
        kd, vd, kw, vw, st0 = decode_context(wd.B, wd.H, wd.Dh, wd.decode_ctx, wd.D, wd.W, seed=2)
        self.dec_in = [x.to(torch.float64).numpy() for x in
                       decode_inputs(steps, wd.B, wd.H, wd.Dh, "bf16", wd.gate_mean, wd.gate_std, seed=1)]
        oc = oracle.Cache(wd.B, wd.H, wd.Dh, wd.decode_ctx + steps, wd.D, wd.W)
        for b in range(wd.B):
            for h in range(wd.H):
                r0 = oracle.cache_row(b, h, 0, wd.H, oc.T_max, wd.D)
                m = kd[h].shape[1]
                oc.Kc[r0:r0 + m] = kd[h][b].to(torch.float64).numpy()
                oc.Vc[r0:r0 + m] = vd[h][b].to(torch.float64).numpy()
        self.ring0 = (kw.to(torch.float64).numpy().reshape(-1, wd.Dh),
                      vw.to(torch.float64).numpy().reshape(-1, wd.Dh))
        self.state0 = st0.to(torch.float64).numpy()
        self.cache = oc
        self.pos = steps          # forces a reset on the first decode call

    def prefill(self):
        q, xk, xv, g = self.pre
        w = self.wp
        t0 = time.perf_counter()
        hk = self.oracle.scan(xk, g)
        hv = self.oracle.scan(xv, g)
        self.oracle.attention(q, hk, hv, w.D, w.W)
        return time.perf_counter() - t0

    def decode(self, n):
        oc, wd = self.cache, self.wd
        if self.pos + n > wd.decode_steps:      # back to the start of the context
            oc.Kw[:], oc.Vw[:] = self.ring0
            oc.state[:] = self.state0
            oc.len[:] = wd.decode_ctx
            self.pos = 0
        t0 = time.perf_counter()
        for i in range(self.pos, self.pos + n):
            oc.decode_step(*[x[i] for x in self.dec_in])
        self.pos += n
        return time.perf_counter() - t0

    def describe(self):
        w, wd = self.wp, self.wd
        return ("fp64 oracle: the whole prefill of %s (scan of both streams over %d x %d tokens x "
                "%d channels, attention of all %d query rows x %d heads over their key sets) + "
                "%d literal decode steps of %s (%d sequences, 32K-token context) per step" % (
                    PREFILL, w.B, w.T, w.H * w.Dh, w.B * w.T, w.H, self.DECODE_PER_STEP, DECODE, wd.B))

    def measure(self):
        """One baseline step: (prefill s, decode s) and the derived rates."""
        t_pre = self.prefill()
        n = self.DECODE_PER_STEP
        t_dec = self.decode(n)
        return t_pre, t_dec

    def summary(self, t_pre, t_dec, cores):
        w, wd = self.wp, self.wd
        n = self.DECODE_PER_STEP
        return {"value": w.B * w.T / t_pre, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                "sample": self.describe(),
                "prefill": {"tokens_per_s": w.B * w.T / t_pre, "s": t_pre, "cores": cores},
                "decode": {"tokens_per_s": wd.B * n / t_dec, "s_per_token_step": t_dec / n,
                           "cores": 1, "steps": n}}


def oracle_sample():
    """The CPU baseline of the GPU line: one baseline step of the oracle."""
    ob = OracleBaseline()
    t_pre, t_dec = ob.measure()
    return ob.summary(t_pre, t_dec, ob.oracle.num_threads())


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    ob = OracleBaseline()
    cores = ob.oracle.num_threads()
    pre, dec = [], []
    for i in range(args.warmup + args.steps):
        t_pre, t_dec = ob.measure()
        if i >= args.warmup:
            pre.append(t_pre)
            dec.append(t_dec)
    w = ob.wp
    v = w.B * w.T * args.steps / sum(pre)
    base = ob.summary(sum(pre) / args.steps, sum(dec) / args.steps, cores)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": (sum(pre) + sum(dec)) / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, ob.wd, 1),
        "prefill": base["prefill"], "decode": base["decode"],
        "cpu_baseline": base,
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def bench_config(wp, wd, world):
    """The workload named by the JSON line (both arms)."""
    return {"workload": PREFILL, "B": wp.B, "T": wp.T, "H": wp.H, "Dh": wp.Dh, "D": wp.D,
            "W": wp.W, "decode_workload": DECODE, "decode_B": wd.B,
            "decode_ctx": wd.decode_ctx, "decode_steps": wd.decode_steps,
            "l2": "no flush: every step streams > 1 GB (inputs larger than L2)",
            "parallelism": "replicas x%d" % world}


# ----------------------------------------------------------------------------- GPU arm
# the fp32 workload is a parity configuration: its line is latency, not a roofline
OTHER_CONFIGS = ["bf16_1p5b_T4096_D16", "bf16_hybrid_7p6b_T8192_D4", "f32_small_T256_D4"]


def measure_config(name, dev, steps, warmup, peaks):
    """Prefill (and, where the workload has them, decode steps continuing from
    the prefill) of one more configuration, timed with CUDA events on the
    launching stream.  Reported beside the headline line, not part of it."""
    import recurrence_augmented_dilated_chunked_b200 as ratp
    from recurrence_augmented_dilated_chunked_b200 import WORKLOADS, decode_inputs, prefill_inputs
    w = WORKLOADS[name]
    stream = torch.cuda.current_stream(dev)
    q, xk, xv, g = (t.to(dev) for t in prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype,
                                                        w.gate_mean, w.gate_std, seed=0))
    hk, hv, o = (torch.empty_like(q) for _ in range(3))
    fs = torch.empty(2, w.B, w.H, w.Dh, dtype=torch.float32, device=dev)
    ws = ratp.scan_workspace(w.B, w.T, w.H, w.Dh, q.dtype, dev)
    mask = w.dense_mask if w.dense_heads else None
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(warmup + steps):
        ev = evs[i - warmup] if i >= warmup else None
        if ev:
            ev[0].record(stream)
        ratp.scan_prefill_kv(xk, xv, g, hk=hk, hv=hv, final_state=fs, workspace=ws)
        if ev:
            ev[1].record(stream)
        ratp.dilated_attn_prefill(q, hk, hv, w.D, w.W, head_mask=mask, out=o)
        if ev:
            ev[2].record(stream)
    torch.cuda.synchronize()
    ratp.last_error(dev)
    scan_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    pc = prefill_counts(w)
    scan_gbs = pc["scan_bytes"] / (scan_ms / 1e3) / 1e9
    attn_gbs = pc["attn_bytes"] / (attn_ms / 1e3) / 1e9
    attn_tfs = pc["attn_flops"] / (attn_ms / 1e3) / 1e12
    out = {"B": w.B, "T": w.T, "H": w.H, "Dh": w.Dh, "D": w.D, "W": w.W,
           "dense_heads": list(w.dense_heads),
           "prefill_tokens_per_s": w.B * w.T / ((scan_ms + attn_ms) / 1e3),
           "scan_ms": scan_ms, "scan_frac_hbm": scan_gbs / peaks["hbm_gbs"],
           "attn_ms": attn_ms, "attn_frac_hbm": attn_gbs / peaks["hbm_gbs"],
           "attn_tflops": attn_tfs, "attn_frac_tensor": attn_tfs / peaks["bf16_tflops"],
           "attn_pairs": pc["pairs"], "attn_flops": pc["attn_flops"]}
    del xk, xv, g, ws
    if w.decode_steps:
        n = w.decode_steps
        cache = ratp.KVCache(w.B, w.H, w.Dh, w.T + n, w.D, w.W, head_mask=mask, device=dev)
        cache.pack(hk, hv, w.T)
        lens = cache.lengths()
        dq, dxk, dxv, dg = (t.to(dev) for t in decode_inputs(n, w.B, w.H, w.Dh, w.dtype,
                                                              w.gate_mean, w.gate_std))
        state = fs.clone()
        dout = torch.empty(n, w.B, w.H, w.Dh, dtype=torch.bfloat16, device=dev)

        def burst():
            lens.fill_(w.T)
            state.copy_(fs)
            for i in range(n):
                cache.decode_step(dq[i], dxk[i], dxv[i], dg[i], state, out=dout[i])

        burst()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            burst()
        for _ in range(warmup):
            graph.replay()
        d_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for e in d_evs:
            e[0].record(stream)
            graph.replay()
            e[1].record(stream)
        torch.cuda.synchronize()
        ratp.last_error(dev)
        dec_ms = statistics.median(e[0].elapsed_time(e[1]) for e in d_evs) / n
        dec_bytes = sum(decode_bytes_per_step(w, w.T + i) for i in range(n)) / n
        dec_gbs = dec_bytes / (dec_ms / 1e3) / 1e9
        out.update({"decode_steps": n, "decode_tokens_per_s": w.B / (dec_ms / 1e3),
                    "decode_ms_per_step": dec_ms, "decode_frac_hbm": dec_gbs / peaks["hbm_gbs"],
                    "decode_alg_bytes_per_step": dec_bytes})
        del graph
    return out


def measure_fused(names, dev, steps, warmup, peaks):
    """The fused prefill (ratp_prefill_fused: recurrence and attention in one
    launch) beside the two-kernel path on the same inputs, timed with CUDA
    events on the launching stream.  Reported beside the headline line."""
    import recurrence_augmented_dilated_chunked_b200 as ratp
    from recurrence_augmented_dilated_chunked_b200 import WORKLOADS, prefill_inputs
    out = {}
    for name in names:
        w = WORKLOADS[name]
        stream = torch.cuda.current_stream(dev)
        q, xk, xv, g = (t.to(dev) for t in prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype,
                                                            w.gate_mean, w.gate_std, seed=0))
        hk, hv, o = (torch.empty_like(q) for _ in range(3))
        mask = w.dense_mask if w.dense_heads else None
        ws = ratp.scan_workspace(w.B, w.T, w.H, w.Dh, q.dtype, dev)
        fws = ratp.prefill_fused_workspace(w.B, w.T, w.H, w.Dh, dev)
        runs = {
            "fused": lambda: ratp.prefill_fused(q, xk, xv, g, w.D, w.W, head_mask=mask, hk=hk, hv=hv,
                                                out=o, workspace=fws),
            "two_kernel": lambda: (ratp.scan_prefill_kv(xk, xv, g, hk=hk, hv=hv, workspace=ws),
                                   ratp.dilated_attn_prefill(q, hk, hv, w.D, w.W, head_mask=mask, out=o)),
        }
        r = {}
        for key, run in runs.items():
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
            for i in range(warmup + steps):
                ev = evs[i - warmup] if i >= warmup else None
                if ev:
                    ev[0].record(stream)
                run()
                if ev:
                    ev[1].record(stream)
            torch.cuda.synchronize()
            ratp.last_error(dev)
            ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
            r[key] = {"ms": ms, "tokens_per_s": w.B * w.T / (ms / 1e3)}
        # bytes the fused call must move: read q, x_k, x_v, g; write h_k, h_v, o
        E = w.B * w.T * w.H * w.Dh
        r["fused"]["alg_bytes"] = 7 * E * 2
        r["fused"]["frac_hbm"] = 7 * E * 2 / (r["fused"]["ms"] / 1e3) / 1e9 / peaks["hbm_gbs"]
        out[name] = r
        del q, xk, xv, g, hk, hv, o
    return out


def measure_scan_variants(name, L_list, window_L, dev, steps, warmup, peaks):
    """The key/value scan of one workload with the chunk-local recurrence (the
    original RAT's blocks of L tokens) and with the fixed look-back window,
    beside the full-sequence scan, timed with CUDA events on the launching
    stream.  Reported beside the headline line, not part of it."""
    import recurrence_augmented_dilated_chunked_b200 as ratp
    from recurrence_augmented_dilated_chunked_b200 import WORKLOADS, prefill_inputs
    w = WORKLOADS[name]
    stream = torch.cuda.current_stream(dev)
    _, xk, xv, g = (t.to(dev) for t in prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype,
                                                        w.gate_mean, w.gate_std, seed=0))
    hk, hv = torch.empty_like(xk), torch.empty_like(xv)
    fs = torch.empty(2, w.B, w.H, w.Dh, dtype=torch.float32, device=dev)
    ws = ratp.scan_workspace(w.B, w.T, w.H, w.Dh, xk.dtype, dev)
    pc = prefill_counts(w)
    out = {"workload": name}
    runs = [("full_sequence", lambda: ratp.scan_prefill_kv(xk, xv, g, hk=hk, hv=hv, final_state=fs,
                                                          workspace=ws))]
    for L in L_list:
        runs.append(("chunk_local_L%d" % L,
                     lambda L=L: ratp.scan_prefill_kv(xk, xv, g, hk=hk, hv=hv, final_state=fs,
                                                      workspace=ws, L=L)))
    runs.append(("window_L%d" % window_L,
                 lambda: ratp.scan_prefill_kv_window(xk, xv, g, window_L, hk=hk, hv=hv)))
    for key, run in runs:
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for i in range(warmup + steps):
            ev = evs[i - warmup] if i >= warmup else None
            if ev:
                ev[0].record(stream)
            run()
            if ev:
                ev[1].record(stream)
        torch.cuda.synchronize()
        ratp.last_error(dev)
        ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
        gbs = pc["scan_bytes"] / (ms / 1e3) / 1e9
        out[key] = {"scan_ms": ms, "achieved_gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"]}
    del xk, xv, g, hk, hv, ws
    return out


def measure_per_sample(name, dev, steps, warmup, peaks):
    """Prefill of one workload with one dilation per sample in one attention
    launch: the first half of the batch dense (D = 1), the second half at
    D = 64 (the batch composition of active recurrence learning).  Timed
    with CUDA events on the launching stream; reported beside the headline
    line."""
    import recurrence_augmented_dilated_chunked_b200 as ratp
    from recurrence_augmented_dilated_chunked_b200 import WORKLOADS, prefill_inputs
    w = WORKLOADS[name]
    Ds = [1] * (w.B // 2) + [64] * (w.B - w.B // 2)
    stream = torch.cuda.current_stream(dev)
    q, xk, xv, g = (t.to(dev) for t in prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype,
                                                        w.gate_mean, w.gate_std, seed=0))
    hk, hv, o = (torch.empty_like(q) for _ in range(3))
    ws = ratp.scan_workspace(w.B, w.T, w.H, w.Dh, q.dtype, dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(warmup + steps):
        ev = evs[i - warmup] if i >= warmup else None
        if ev:
            ev[0].record(stream)
        ratp.scan_prefill_kv(xk, xv, g, hk=hk, hv=hv, workspace=ws)
        if ev:
            ev[1].record(stream)
        ratp.dilated_attn_prefill_per_sample(q, hk, hv, Ds, 0, out=o)
        if ev:
            ev[2].record(stream)
    torch.cuda.synchronize()
    ratp.last_error(dev)
    scan_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    pairs = sum(w.H * attention_pairs(w.T, d, 0) for d in Ds)
    flops = 4 * w.Dh * pairs
    E = w.B * w.T * w.H * w.Dh
    attn_gbs = 4 * E * 2 / (attn_ms / 1e3) / 1e9
    tfs = flops / (attn_ms / 1e3) / 1e12
    del q, xk, xv, g, hk, hv, o, ws
    return {"workload": name, "D_per_sample": Ds, "B": w.B, "T": w.T, "H": w.H, "Dh": w.Dh,
            "prefill_tokens_per_s": w.B * w.T / ((scan_ms + attn_ms) / 1e3),
            "scan_ms": scan_ms, "attn_ms": attn_ms, "attn_pairs": pairs, "attn_flops": flops,
            "attn_tflops": tfs, "attn_frac_tensor": tfs / peaks["bf16_tflops"],
            "attn_frac_hbm": attn_gbs / peaks["hbm_gbs"]}


# A 1.5B-like stack of 24 sequence mixers for the layer-wise hybrid: dense
# layers at 0 (input) and 12 (middle), every other layer at D = 64 with a
# 128-token window; decode from 32K-token contexts, 16 sequences.
STACK = {"name": "bf16_1p5b_stack24_decode_ctx32768", "layers": 24, "dense_layers": (0, 12),
         "B": 16, "H": 16, "Dh": 128, "D": 64, "W": 128, "ctx": 32768, "steps": 16}


def measure_layer_stack(dev, replays, warmup, peaks):
    """Decode token steps through the whole layer stack, each token step one
    ``ratp_decode_step_layers`` call, 16 token steps captured in one CUDA
    graph.  Caches are filled on the device with N(0, 1) rows (the values do
    not change the work).  Reported beside the headline line."""
    import recurrence_augmented_dilated_chunked_b200 as ratp
    from recurrence_augmented_dilated_chunked_b200 import Workload, decode_inputs
    S = STACK
    n, B, H, Dh, ctx = S["steps"], S["B"], S["H"], S["Dh"], S["ctx"]
    gen = torch.Generator(dev).manual_seed(5)
    dq, dxk, dxv, dg = (t.to(dev) for t in decode_inputs(n, B, H, Dh, "bf16", 2.0, 1.5, seed=6))
    layers, kinds = [], []
    for li in range(S["layers"]):
        dense = li in S["dense_layers"]
        D, W = (1, 0) if dense else (S["D"], S["W"])
        cache = ratp.KVCache(B, H, Dh, ctx + n, D, W, device=dev)
        for which in ("k", "v"):
            rows = cache.dil_rows(which)
            rows.copy_(torch.randn(rows.shape, generator=gen, device=dev, dtype=torch.float32))
            if W:
                ring = cache.ring(which)
                ring.copy_(torch.randn(ring.shape, generator=gen, device=dev, dtype=torch.float32))
                # a dilated position inside the last W holds one value in both places
                for h in range(H):
                    off, _ = cache.head_rows(h)
                    for pos in range(ctx - W, ctx):
                        if pos % D == D - 1:
                            ring[:, h, pos % W] = rows[:, off + pos // D]
        state0 = torch.randn(2, B, H, Dh, generator=gen, device=dev, dtype=torch.float32)
        out = torch.empty(n, B, H, Dh, dtype=torch.bfloat16, device=dev)
        layers.append((cache, state0, state0.clone(), out))
        kinds.append(Workload("stack", "bf16", B=B, T=0, H=H, Dh=Dh, D=D, W=W, gate_mean=2.0,
                              gate_std=1.5, decode_steps=n, decode_ctx=ctx))

    def burst():
        for cache, s0, st, _ in layers:
            cache.lengths().fill_(ctx)
            st.copy_(s0)
        for i in range(n):
            ratp.decode_step_layers([(c, dq[i], dxk[i], dxv[i], dg[i], st, o[i])
                                     for c, _, st, o in layers])

    burst()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        burst()
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        graph.replay()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(replays)]
    for e in evs:
        e[0].record(stream)
        graph.replay()
        e[1].record(stream)
    torch.cuda.synchronize()
    ratp.last_error(dev)
    # the resets at the start of a burst are part of the replay; they move
    # 2 * 24 small state copies, negligible beside the cache reads
    ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs) / n
    alg = sum(decode_bytes_per_step(w, ctx + i) for w in kinds for i in range(n)) / n
    gbs = alg / (ms / 1e3) / 1e9
    cache_bytes = sum(c.buffer.numel() for c, _, _, _ in layers)
    del graph, layers
    return {"workload": S["name"], "layers": S["layers"], "dense_layers": list(S["dense_layers"]),
            "B": B, "H": H, "Dh": Dh, "D": S["D"], "W": S["W"], "ctx": ctx,
            "token_steps_per_graph": n, "launches_per_token_step": S["layers"],
            "ms_per_token_step": ms, "tokens_per_s": B / (ms / 1e3),
            "alg_bytes_per_token_step": alg, "achieved_gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
            "cache_bytes": cache_bytes}


def run_ours(args, rank, world, local_rank):
    import recurrence_augmented_dilated_chunked_b200 as ratp
    from recurrence_augmented_dilated_chunked_b200 import (WORKLOADS, decode_context,
                                                           decode_inputs, prefill_inputs)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    ratp.load_library()
    stream = torch.cuda.current_stream(dev)
    wp, wd = WORKLOADS[PREFILL], WORKLOADS[DECODE]

    if args.only == "prefill":
        # profiling driver: prefill passes of one workload, no timing or report
        w = WORKLOADS[args.workload or PREFILL]
        q, xk, xv, g = (t.to(dev) for t in prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype,
                                                            w.gate_mean, w.gate_std, seed=rank))
        hk, hv, o = (torch.empty_like(q) for _ in range(3))
        ws = ratp.scan_workspace(w.B, w.T, w.H, w.Dh, q.dtype, dev)
        mask = w.dense_mask if w.dense_heads else None
        L = w.D if args.variant == "chunk_local" else 0
        Ds = [1] * (w.B // 2) + [64] * (w.B - w.B // 2)
        fws = ratp.prefill_fused_workspace(w.B, w.T, w.H, w.Dh, dev) if args.variant == "fused" else None
        for _ in range(args.warmup + args.steps):
            if args.variant == "fused":
                ratp.prefill_fused(q, xk, xv, g, w.D, w.W, head_mask=mask, hk=hk, hv=hv, out=o, workspace=fws)
                continue
            if args.variant == "window":
                ratp.scan_prefill_kv_window(xk, xv, g, 64, hk=hk, hv=hv)
            else:
                ratp.scan_prefill_kv(xk, xv, g, hk=hk, hv=hv, workspace=ws, L=L)
            if args.variant == "per_sample":
                ratp.dilated_attn_prefill_per_sample(q, hk, hv, Ds, w.W, head_mask=mask, out=o)
            else:
                ratp.dilated_attn_prefill(q, hk, hv, w.D, w.W, head_mask=mask, out=o)
        torch.cuda.synchronize()
        ratp.last_error(dev)
        return 0

    # ---- prefill inputs (seeded, synthetic; a different seed per rank) ----
    q, xk, xv, g = prefill_inputs(wp.B, wp.T, wp.H, wp.Dh, wp.dtype, wp.gate_mean, wp.gate_std,
                                  seed=rank)
    q_h, xk_h, xv_h, g_h = (t.pin_memory() for t in (q, xk, xv, g))
    qd, xkd, xvd, gd = (t.to(dev) for t in (q_h, xk_h, xv_h, g_h))
    hk, hv, o = (torch.empty_like(qd) for _ in range(3))
    ws = ratp.scan_workspace(wp.B, wp.T, wp.H, wp.Dh, qd.dtype, dev)
    o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()

    # ---- decode context + per-step inputs ----
    steps = wd.decode_steps
    T_max = wd.decode_ctx + steps
    kd, vd, kw, vw, st0 = decode_context(wd.B, wd.H, wd.Dh, wd.decode_ctx, wd.D, wd.W, seed=2 + rank)
    dq, dxk, dxv, dg = (t.to(dev) for t in decode_inputs(steps, wd.B, wd.H, wd.Dh, "bf16",
                                                         wd.gate_mean, wd.gate_std, seed=1 + rank))
    cache = ratp.KVCache(wd.B, wd.H, wd.Dh, T_max, wd.D, wd.W)
    kc, vc = cache.dil_rows("k"), cache.dil_rows("v")
    for h in range(wd.H):
        off, _ = cache.head_rows(h)
        n = kd[h].shape[1]
        kc[:, off:off + n] = kd[h].to(dev)
        vc[:, off:off + n] = vd[h].to(dev)
    cache.ring("k").copy_(kw.to(dev))
    cache.ring("v").copy_(vw.to(dev))
    state0 = st0.to(dev)
    state = state0.clone()
    dout = torch.empty(steps, wd.B, wd.H, wd.Dh, dtype=torch.bfloat16, device=dev)
    lens = cache.lengths()

    def decode_burst():
        lens.fill_(wd.decode_ctx)
        for i in range(steps):
            cache.decode_step(dq[i], dxk[i], dxv[i], dg[i], state, out=dout[i])

    # capture the 256-step burst once (warm the kernels first)
    decode_burst()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        decode_burst()
    torch.cuda.synchronize()
    ratp.last_error(dev)

    if args.only == "decode":
        # profiling driver: decode bursts only (graph replays), no report
        for _ in range(args.warmup + args.steps):
            graph.replay()
        torch.cuda.synchronize()
        ratp.last_error(dev)
        return 0

    def prefill(ev=None):
        if ev:
            ev[0].record(stream)
        ratp.scan_prefill_kv(xkd, xvd, gd, hk=hk, hv=hv, workspace=ws)
        if ev:
            ev[1].record(stream)
        ratp.dilated_attn_prefill(qd, hk, hv, wp.D, wp.W, out=o)
        if ev:
            ev[2].record(stream)

    for _ in range(args.warmup):
        prefill()
        graph.replay()
    torch.cuda.synchronize()
    ratp.last_error(dev)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        clk.ready()
        # keep the device busy (~1 ms, before the first event) while the host
        # queues the first step, so no host-side launch time falls between a
        # step's events
        torch.cuda._sleep(2_000_000)
        t_wall = time.perf_counter()
        for i in range(args.steps):
            prefill(evs[i])
            graph.replay()
            evs[i][3].record(stream)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if world > 1:
        torch.distributed.barrier()
    ratp.last_error(dev)
    scan_ms = [e[0].elapsed_time(e[1]) for e in evs]
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs]
    dec_ms = [e[2].elapsed_time(e[3]) for e in evs]
    total_ms = evs[0][0].elapsed_time(evs[-1][3])

    # ---- end to end through the public API with host buffers ----
    # Every step copies its q, x_k, x_v, g from pinned host memory and its o
    # back.  The copies run on their own streams (one per direction, PCIe is
    # full duplex) with two device buffer sets, so step i+1's inputs cross
    # PCIe while step i computes and step i-1's output returns.
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    host_in = (q_h, xk_h, xv_h, g_h)
    ins = [(qd, xkd, xvd, gd), tuple(torch.empty_like(t) for t in (qd, xkd, xvd, gd))]
    outs = [o, torch.empty_like(o)]
    host_out = [o_h, torch.empty(o.shape, dtype=o.dtype).pin_memory()]
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of set k landed
    ev_used = [torch.cuda.Event() for _ in range(2)]    # compute on set k done
    ev_out = [torch.cuda.Event() for _ in range(2)]     # output of set k copied out
    e_start, e_end = (torch.cuda.Event(enable_timing=True) for _ in range(2))

    def h2d(i):
        k = i & 1
        with torch.cuda.stream(s_h2d):
            if i >= 2:
                s_h2d.wait_event(ev_used[k])
            for src, dst in zip(host_in, ins[k]):
                dst.copy_(src, non_blocking=True)
            ev_in[k].record(s_h2d)

    def run_e2e(n, timed):
        torch.cuda.synchronize()
        if timed:
            e_start.record(s_h2d)
        h2d(0)
        for i in range(n):
            k = i & 1
            if i + 1 < n:
                h2d(i + 1)
            stream.wait_event(ev_in[k])
            if i >= 2:
                stream.wait_event(ev_out[k])
            q_, xk_, xv_, g_ = ins[k]
            ratp.scan_prefill_kv(xk_, xv_, g_, hk=hk, hv=hv, workspace=ws)
            ratp.dilated_attn_prefill(q_, hk, hv, wp.D, wp.W, out=outs[k])
            ev_used[k].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_used[k])
                host_out[k].copy_(outs[k], non_blocking=True)
                ev_out[k].record(s_d2h)
        if timed:
            e_end.record(s_d2h)
        torch.cuda.synchronize()

    run_e2e(args.warmup, False)
    run_e2e(args.steps, True)
    e2e_ms = e_start.elapsed_time(e_end)
    ratp.last_error(dev)

    # ---- max over ranks ----
    s_scan, s_attn, s_dec, s_total, s_e2e = max_over_ranks(
        [sum(scan_ms), sum(attn_ms), sum(dec_ms), total_ms, e2e_ms], world, dev)
    if rank != 0:
        return 0

    K = args.steps
    pc = prefill_counts(wp)
    peaks = measured_peaks()
    prefill_tokens = wp.B * wp.T
    prefill_s = (s_scan + s_attn) / 1e3
    value = job_throughput(prefill_tokens * K, world, prefill_s)
    decode_tok_s = job_throughput(wd.B * steps * K, world, s_dec / 1e3)
    scan_gbs = pc["scan_bytes"] * K / (s_scan / 1e3) / 1e9
    attn_gbs = pc["attn_bytes"] * K / (s_attn / 1e3) / 1e9
    attn_tfs = pc["attn_flops"] * K / (s_attn / 1e3) / 1e12
    dec_bytes = sum(decode_bytes_per_step(wd, wd.decode_ctx + i) for i in range(steps))
    dec_gbs = dec_bytes * K / (s_dec / 1e3) / 1e9
    kernels = {
        "scan_kv": {"ms_per_launch": s_scan / K, "achieved_gbs": scan_gbs,
                    "frac_hbm": scan_gbs / peaks["hbm_gbs"], "alg_bytes": pc["scan_bytes"]},
        "dilated_attn": {"ms_per_launch": s_attn / K, "achieved_gbs": attn_gbs,
                         "frac_hbm": attn_gbs / peaks["hbm_gbs"], "achieved_tflops": attn_tfs,
                         "frac_tensor": attn_tfs / peaks["bf16_tflops"], "alg_bytes": pc["attn_bytes"],
                         "alg_flops": pc["attn_flops"]},
        "decode_step": {"ms_per_launch": s_dec / K / steps, "achieved_gbs": dec_gbs,
                        "frac_hbm": dec_gbs / peaks["hbm_gbs"], "alg_bytes_per_launch": dec_bytes / steps},
    }
    # dominant kernel of the timed step by share of device time
    shares = {"scan_kv": s_scan, "dilated_attn": s_attn, "decode_step": s_dec}
    dom = max(shares, key=shares.get)
    kd_ = kernels[dom]
    roof = {"kernel": dom, "bound": "hbm", "achieved": kd_["achieved_gbs"], "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": kd_["frac_hbm"], "traffic": measured_traffic(dom),
            "peak_source": peaks["source"]}
    for name in kernels:
        kernels[name]["traffic"] = measured_traffic(name)
    h2d = sum(t.numel() * t.element_size() for t in (q_h, xk_h, xv_h, g_h))
    d2h = o_h.numel() * o_h.element_size()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": s_total / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(wp, wd, world),
        "prefill": {"tokens_per_s": value, "ms": (s_scan + s_attn) / K},
        "decode": {"tokens_per_s": decode_tok_s, "ms_per_token_step": s_dec / K / steps,
                   "graph": "256 decode launches per CUDA graph"},
        "kernels": kernels,
        "roofline": roof,
        "e2e": {"value": job_throughput(prefill_tokens * args.steps, world, s_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "what": "prefill through the C ABI from pinned host q/xk/xv/g to host o; "
                        "copies of step i+1 in and step i-1 out overlap step i"},
        "gpu_launches": K * (2 + steps),
        "clocks": clk.summary(),
        "wall_s": t_wall,
    }
    if not args.no_other_configs:
        # the other workloads, measured after the timed region (not part of it)
        line["other_configs"] = {n: measure_config(n, dev, min(args.steps, 5), args.warmup, peaks)
                                 for n in OTHER_CONFIGS}
        line["scan_variants"] = measure_scan_variants(PREFILL, [wp.D, 1000], 64, dev,
                                                      min(args.steps, 5), args.warmup, peaks)
        line["layer_stack_decode"] = measure_layer_stack(dev, min(args.steps, 5), args.warmup, peaks)
        line["per_sample_prefill"] = measure_per_sample("bf16_1p5b_T4096_D16", dev, min(args.steps, 5),
                                                        args.warmup, peaks)
        line["fused_prefill"] = measure_fused([PREFILL, "bf16_1p5b_T4096_D16", "bf16_hybrid_7p6b_T8192_D4"],
                                              dev, min(args.steps, 5), args.warmup, peaks)
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = oracle_sample()
    print(json.dumps(line), flush=True)
    del graph
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the per-configuration measurements of the other workloads")
    ap.add_argument("--only", choices=["prefill", "decode"], default=None,
                    help="run only this part, untimed (a driver for ncu captures)")
    ap.add_argument("--workload", default=None,
                    help="with --only prefill: the prefill workload (default: the headline one)")
    ap.add_argument("--variant", choices=["chunk_local", "per_sample", "window", "fused"], default=None,
                    help="with --only prefill: chunk-local scan (L = D), per-sample attention "
                         "(first half of the batch dense, second half at D = 64), the "
                         "fixed look-back scan (L = 64), or the fused prefill")
    args = ap.parse_args()
    if args.warmup < 3 and args.only is None:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.impl == "reference":
            return run_reference(args, rank, world)
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1 and args.impl == "ours":
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
