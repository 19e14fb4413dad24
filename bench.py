#!/usr/bin/env python
"""Benchmark of the NVFP4 hot path on B200.

One step = one W4A4 linear layer of the dense-FFN workload (the 12B hybrid
model's FFN shape): quantize the BF16 activations A [8192 x 5120] to NVFP4
(tensor amax, then block scales + codes) and run the block-scaled FP4 GEMM
against the pre-quantized weight W [20480 x 5120], writing D [8192 x 20480]
BF16.  Metric: NVFP4 GEMM TFLOP/s over the whole step (2*M*N*K per step).
The same run measures standalone quantize GB/s on the 2^28-value tensor of
the quantize sweep (the metric's second half) as ``quantize``.

Launch: ``python bench.py [--gpus N] [--steps K] [--warmup W]``; for N > 1
under torch.distributed.run, one rank per GPU.  The path has no data
exchange, so N > 1 runs N replicas (weak scaling) and only the timing is
reduced across ranks (max).  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, N, K = 8192, 20480, 5120
SWEEP_N = 1 << 28
METRIC = "NVFP4 GEMM TFLOPS (% of FP4 peak); quantize GB/s (% of HBM BW), 1 B200"
WORKLOAD = "w4a4_linear_ffn_M8192_N20480_K5120 (quantize A + block-scaled FP4 GEMM)"
L2_FLUSH_BYTES = 256 << 20
# Algorithmic bytes per value of a two-pass quantize (amax read 2 B, then
# read 2 B + write 0.5 B codes + 0.0625 B scales) and of the encode pass.
QUANT_BYTES_PER_VALUE_2PASS = 4.5625
ENCODE_BYTES_PER_VALUE = 2.5625
FP4_OVER_BF16 = 4.0        # nominal dense FP4 / BF16 tensor throughput on B200
# DRAM bytes (read + write) of one GEMM launch on this workload, per kernel,
# from an ncu capture of dram__bytes_read.sum + dram__bytes_write.sum of one
# launch at this shape: (bytes, hash of the kernel's sources when captured).
# Reported only while the sources still hash to the captured version
# (otherwise null).
GEMM_TRAFFIC = {
    "single": (87.86e6 + 291.46e6, "ea4f2dd8ebcc62e2"),
    "pair": (89.65e6 + 293.04e6, "47979815b0fae04d"),
}
GEMM_SOURCES = {"single": ("gemm.cu", "gemm.h", "ptx.cuh"),
                "pair": ("gemm_pair.cu", "gemm.h", "ptx.cuh")}


def gemm_sources_sha(kernel):
    import hashlib
    csrc = os.path.join(ROOT, "nvfp4_block_scaled_22_b200", "csrc")
    h = hashlib.sha256()
    for f in GEMM_SOURCES[kernel]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def gemm_traffic(kernel):
    nbytes, sha = GEMM_TRAFFIC[kernel]
    return nbytes if nbytes is not None and gemm_sources_sha(kernel) == sha else None


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of `values` over all ranks (identity with one
    rank): every multi-GPU time in the JSON line is the slowest rank's."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def replica_throughput(world, units_per_step, steps, total_ms):
    """Whole-job rate of `world` independent replicas (weak scaling): the
    units every rank processed over the slowest rank's time."""
    return world * units_per_step * steps / (total_ms / 1e3)


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs"), d.get("bf16_tflops"), d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons every few ms during a region."""

    REASONS = {0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x4: "sw_power_cap", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting", 0x100: "sync_boost"}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.stop_ev = threading.Event()
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop_ev.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "source": "nvml" if self.ok else "unavailable"}
        mhz = [s[0] for s in self.samples]
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = sorted({name for bit, name in self.REASONS.items() if mask & bit} - {"gpu_idle"})
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz), "source": "nvml"}


# ------------------------------------------------------------ GPU workload
class Workload:
    def __init__(self, device):
        from nvfp4_block_scaled_22_b200 import binding as nb
        from nvfp4_block_scaled_22_b200 import inputs
        self.nb = nb
        self.dev = device
        nb.lib()
        self.ws = nb.Workspace(device)
        w = inputs.ffn_weight(device=device)
        self.qw = nb.nvfp4_quantize(w, workspace=self.ws)
        del w
        self.a = inputs.ffn_activation(M, device=device)
        self.qa = nb.NVFP4Tensor.empty(M, K, device=device)
        self.d = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        self.flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        torch.cuda.synchronize()
        st = nb.nvfp4_check_status(self.ws)
        if st != 0:
            raise RuntimeError(f"setup status {st}")

    def flush(self):
        self.flush_buf.zero_()

    def quantize(self):
        self.nb.nvfp4_quantize(self.a, out=self.qa, workspace=self.ws)

    def gemm(self):
        self.nb.nvfp4_gemm(self.qa, self.qw, out=self.d, workspace=self.ws)


def time_steps(wl: Workload, steps: int, warmup: int):
    """Device time of each step (flush outside the events)."""
    for _ in range(warmup):
        wl.flush()
        wl.quantize()
        wl.gemm()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    n0 = wl.nb.nvfp4_launch_count()
    for i in range(steps):
        wl.flush()
        ev[i][0].record()
        wl.quantize()
        ev[i][1].record()
        wl.gemm()
        ev[i][2].record()
    torch.cuda.synchronize()
    launches = wl.nb.nvfp4_launch_count() - n0
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    quant_ms = [e[0].elapsed_time(e[1]) for e in ev]
    gemm_ms = [e[1].elapsed_time(e[2]) for e in ev]
    return step_ms, quant_ms, gemm_ms, launches


def time_sweep_quantize(nb, device, iters=10):
    from nvfp4_block_scaled_22_b200 import inputs
    x = inputs.sweep_tensor(SWEEP_N, device=device)
    q = nb.NVFP4Tensor.empty(x.shape[0], x.shape[1], device=device)
    ws = nb.Workspace(device)
    for _ in range(3):
        nb.nvfp4_quantize(x, out=q, workspace=ws)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    for a, b in evs:                 # 512 MiB input > L2: no flush needed
        a.record()
        nb.nvfp4_quantize(x, out=q, workspace=ws)
        b.record()
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in evs)
    # encode pass alone (caller-supplied tensor scale)
    for a, b in evs:
        a.record()
        nb.nvfp4_quantize(x, out=q, global_supplied=True, workspace=ws)
        b.record()
    torch.cuda.synchronize()
    ms1 = statistics.median(a.elapsed_time(b) for a, b in evs)
    st = nb.nvfp4_check_status(ws)
    del x, q
    return ms, ms1, st


def time_e2e(wl: Workload, steps: int, warmup: int):
    """Same step through the public API from pinned host memory: every
    step copies its A host-to-device, quantizes it, runs the GEMM and copies
    its D device-to-host, all inside the events.  Consecutive steps overlap
    on three streams, as a serving loop would run them: step i's input copy
    and step i-1's output copy use the two copy directions at once, and the
    compute of step i runs beside step i-1's output copy.  Two device
    buffers each for A and D; events order every reuse."""
    a_host = wl.a.cpu().pin_memory()
    d_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    a_dev = [torch.empty_like(wl.a) for _ in range(2)]
    d_dev = [wl.d, torch.empty_like(wl.d)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[b])        # step i-2's compute has read a_dev[b]
                a_dev[b].copy_(a_host, non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[b])
                if i >= 2:
                    s_comp.wait_event(ev_out[b])       # step i-2's D has left d_dev[b]
                wl.nb.nvfp4_quantize(a_dev[b], out=wl.qa, workspace=wl.ws)
                wl.nb.nvfp4_gemm(wl.qa, wl.qw, out=d_dev[b], workspace=wl.ws)
                ev_comp[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                d_host.copy_(d_dev[b], non_blocking=True)
                ev_out[b].record(s_out)

    def fence(ev):
        for st in (s_in, s_comp, s_out):
            st.wait_event(ev)

    cur = torch.cuda.current_stream()
    run(max(2, warmup))
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(3, min(steps, 20))
    s.record(cur)
    fence(s)
    run(n)
    for st in (s_in, s_comp, s_out):
        cur.wait_stream(st)
    e.record(cur)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / n
    return ms, a_host.numel() * 2, d_host.numel() * 2


# ------------------------------------------------------- CPU oracle timing
def oracle_sample(rows: int = 1, cols: int = 4096, seed: int = 0, threads: int = 1):
    """Oracle on a bounded sample of the step: the tensor amax over all of A
    (A's tensor scale needs it), quantize `rows` rows of A with that scale,
    and compute their first `cols` outputs of the FP64 GEMM against the
    oracle-quantized W, on `threads` host threads.  Returns (seconds, flops)."""
    import numpy as np
    import oracle
    from nvfp4_block_scaled_22_b200 import inputs
    cache = oracle_sample.__dict__.setdefault("cache", {})
    if "w" not in cache:
        w = inputs.ffn_weight()
        st, qw = oracle.quantize_parallel(w)
        a = inputs.ffn_activation(M)
        cache["w"], cache["a"] = qw, a
    qw, a = cache["w"], cache["a"]
    r0 = (seed * rows) % (M - rows + 1)
    t0 = time.perf_counter()
    st, amax = oracle.tensor_amax_parallel(a, threads)
    st, g = oracle.global_scale(amax)
    qa = oracle.quantize_with_global(a[r0:r0 + rows], g)
    ii, jj = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
    oracle.gemm_ref_parallel(qa, qw, ii.ravel(), jj.ravel(), threads)
    dt = time.perf_counter() - t0
    return dt, 2.0 * rows * cols * K


def cpu_baseline_entry():
    import oracle
    cores = oracle.host_threads()
    oracle_sample()                                   # setup (W quantized once), untimed
    dt1, f1 = oracle_sample(rows=1, threads=1)
    dtn, fn = oracle_sample(rows=cores, seed=1, threads=cores)
    return {"value": fn / dtn / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "value_1core": f1 / dt1 / 1e12,
            "sample": f"{cores} of {M} rows of A (one per thread): tensor amax over all of A, "
                      f"quantize the rows, then 4096 of {N} outputs per row of the FP64 GEMM "
                      f"(K={K}) against the oracle-quantized W, on {cores} host threads "
                      f"({dtn:.2f} s); value_1core: 1 row on one thread ({dt1:.2f} s)"}


def run_reference(args):
    import oracle
    rank, _, world = env_rank()
    if rank != 0:
        return 0
    cores = oracle.host_threads()
    oracle_sample()   # builds the oracle and quantizes W once (setup, untimed)
    for i in range(args.warmup):
        oracle_sample(rows=cores, seed=i, threads=cores)
    times, flops = [], 0.0
    for i in range(args.steps):
        dt, f = oracle_sample(rows=cores, seed=args.warmup + i, threads=cores)
        times.append(dt)
        flops = f
    total = sum(times)
    value = flops * args.steps / total / 1e12
    sample = (f"per step: {cores} rows of A quantized (after the full-tensor amax) and 4096 "
              f"outputs per row of the FP64 GEMM, K=5120, on {cores} host threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
        "config": {"workload": WORKLOAD + f" [oracle sample per step: {cores} rows x 4096 outputs]",
                   "M": M, "N": N, "K": K},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0



# ------------------------------------------------- other workloads (rows)
def _events(n):
    return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(n)]


def _timed(fn, steps, warmup, flush=None):
    """Median device time (ms) of fn() over `steps` runs, optional L2 flush
    between runs outside the events."""
    for _ in range(warmup):
        if flush is not None:
            flush()
        fn()
    torch.cuda.synchronize()
    evs = _events(steps)
    for a, b in evs:
        if flush is not None:
            flush()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs)


def workload_line(name, args, device):
    """Measure one of the other scope rows; returns a JSON-able dict."""
    from nvfp4_block_scaled_22_b200 import binding as nb
    from nvfp4_block_scaled_22_b200 import inputs
    hbm_gbs, bf16_tf, _, peak_src = measured_peaks()
    fp4_peak = bf16_tf * FP4_OVER_BF16
    ws = nb.Workspace(device)
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush = flush_buf.zero_
    line = {"impl": "ours", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "data": "synthetic", "scaling": "weak", "vs_baseline": None}

    if name == "sweep":
        rows = []
        for n in inputs.SWEEP_SIZES:
            x = inputs.sweep_tensor(n, device=device)
            q = nb.NVFP4Tensor.empty(x.shape[0], x.shape[1], device=device)
            big = 2 * n > 126e6
            ms = _timed(lambda: nb.nvfp4_quantize(x, out=q, workspace=ws), args.steps, args.warmup,
                        None if big else flush)
            ms1 = _timed(lambda: nb.nvfp4_quantize(x, out=q, global_supplied=True, workspace=ws),
                         args.steps, args.warmup, None if big else flush)
            bpv = QUANT_BYTES_PER_VALUE_2PASS if big else ENCODE_BYTES_PER_VALUE
            rows.append({"values": n, "ms": ms, "gbs": n * bpv / ms / 1e6,
                         "bytes_per_value": bpv, "ms_supplied_scale": ms1,
                         "gbs_supplied_scale": n * ENCODE_BYTES_PER_VALUE / ms1 / 1e6})
            del x, q
        top = rows[-1]
        line.update({"metric": "NVFP4 quantize GB/s (2^28 values)", "value": top["gbs"],
                     "unit": "GB/s", "higher_is_better": True, "ms_per_step": top["ms"],
                     "config": {"workload": "quantize sweep 2^20 / 2^24 / 2^28 values"},
                     "roofline": {"bound": "hbm", "achieved": top["gbs"], "peak": hbm_gbs,
                                  "unit": "GB/s", "frac": top["gbs"] / hbm_gbs,
                                  "peak_source": f"{peak_src} hbm_gbs"},
                     "rows": rows})
        return line

    if name in ("ffn16", "ffn512"):
        m = int(name[3:])
        w = inputs.ffn_weight(device=device)
        qw = nb.nvfp4_quantize(w, workspace=ws)
        del w
        a = inputs.ffn_activation(m, device=device)
        qa = nb.NVFP4Tensor.empty(m, K, device=device)
        d = torch.empty((m, N), dtype=torch.bfloat16, device=device)
        qms = _timed(lambda: nb.nvfp4_quantize(a, out=qa, workspace=ws), args.steps, args.warmup, flush)
        gms = _timed(lambda: nb.nvfp4_gemm(qa, qw, out=d, workspace=ws), args.steps, args.warmup, flush)
        flops = 2.0 * m * N * K
        wbytes = qw.nbytes() + qa.nbytes() + d.numel() * 2
        gbs = wbytes / gms / 1e6
        line.update({"metric": f"NVFP4 W4A4 linear M={m} TFLOP/s", "value": flops / (qms + gms) / 1e9,
                     "unit": "TFLOP/s", "higher_is_better": True, "ms_per_step": qms + gms,
                     "config": {"workload": f"ffn linear M={m} N={N} K={K}", "l2": "flushed"},
                     "gemm_ms": gms, "quantize_ms": qms, "gemm_tflops": flops / gms / 1e9,
                     "roofline": {"kernel": "k_gemm_nvf4", "bound": "hbm", "achieved": gbs,
                                  "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs,
                                  "algorithmic_bytes_per_launch": wbytes,
                                  "peak_source": f"{peak_src} hbm_gbs"}})
        return line

    if name == "moe":
        r = inputs.MoeRouting()
        E, H, I = inputs.MOE_EXPERTS, inputs.MOE_HIDDEN, inputs.MOE_INTER
        x = inputs.moe_activation(device=device)
        slot = r.slot_offsets.to(device)
        rows = r.rows.to(device)
        gather = r.gather.to(device)
        ident = torch.where(r.gather >= 0, torch.arange(r.padded_rows, dtype=torch.int32),
                            torch.full_like(r.gather, -1)).to(device)
        def stacked(which, n, k):
            q = nb.NVFP4Tensor.empty(E * n, k, device=device)
            g = torch.zeros(E, dtype=torch.float32, device=device)
            sfb = nb.nvfp4_scales_bytes(n, k)
            for e in range(E):
                w = inputs.moe_expert_weight(which, e, device=device)
                sub = nb.NVFP4Tensor(q.codes[e * n:(e + 1) * n], q.scales[e * sfb:(e + 1) * sfb],
                                     g[e:e + 1], n, k, nb.SF_SWIZZLED)
                nb.nvfp4_quantize(w, out=sub, workspace=ws)
            return q, g
        wu, gu = stacked("up", I, H)
        wd, gd = stacked("down", H, I)
        # X, quantized once; linear scale rows make the gather's scale reads
        # whole row pieces (the slots' copy is in the GEMM's 128x4 layout)
        qxs = nb.NVFP4Tensor.empty(inputs.MOE_TOKENS, H, nb.SF_LINEAR, device)
        qx = nb.NVFP4Tensor.empty(r.padded_rows, H, device=device)
        hbuf = torch.empty((r.padded_rows, I), dtype=torch.bfloat16, device=device)
        qh = nb.NVFP4Tensor.empty(r.padded_rows, I, device=device)
        y = torch.empty((r.padded_rows, H), dtype=torch.bfloat16, device=device)
        ev = {}

        def step(mark=False):
            # each token's row is quantized once (X's tensor scale), then its
            # NVFP4 bytes are gathered into its 8 expert slots
            nb.nvfp4_quantize(x, out=qxs, workspace=ws)
            nb.nvfp4_gather_rows(qxs, gather, out=qx, workspace=ws)
            # the up projection also yields the intermediate's tensor scale (its
            # max over the real rows, taken in the GEMM epilogue), so the
            # intermediate's quantize needs no amax pass of its own
            nb.nvfp4_grouped_gemm_out_scale(slot, rows, qx, wu, gu, I, out=hbuf,
                                            out_global=qh.global_scale, workspace=ws)
            nb.nvfp4_quantize_gather(hbuf, ident, out=qh, global_supplied=True, workspace=ws)
            if mark:
                ev["a"].record()
            nb.nvfp4_grouped_gemm(slot, rows, qh, wd, gd, H, out=y, workspace=ws)
            if mark:
                ev["b"].record()

        ms = _timed(step, args.steps, args.warmup, flush)
        ev["a"], ev["b"] = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush()
        step(mark=True)
        torch.cuda.synchronize()
        down_ms = ev["a"].elapsed_time(ev["b"])
        st = nb.nvfp4_check_status(ws)
        flops = 2.0 * r.real_rows * I * H * 2
        down_bytes = wd.nbytes() + qh.nbytes() + r.real_rows * H * 2
        gbs = down_bytes / down_ms / 1e6
        line.update({"metric": "NVFP4 MoE expert block TFLOP/s (up + down grouped GEMMs)",
                     "value": flops / ms / 1e9, "unit": "TFLOP/s", "higher_is_better": True,
                     "ms_per_step": ms,
                     "config": {"workload": f"moe {E} experts top-{inputs.MOE_TOPK} of "
                                            f"{inputs.MOE_TOKENS} tokens, hidden {H}, inter {I}",
                                "real_rows": r.real_rows, "padded_rows": r.padded_rows,
                                "l2": "flushed"},
                     "weights_bytes": wu.nbytes() + wd.nbytes(), "status": st,
                     "roofline": {"kernel": "k_gemm_nvf4 (grouped, down projection)",
                                  "bound": "hbm", "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s",
                                  "frac": gbs / hbm_gbs, "ms_per_launch": down_ms,
                                  "algorithmic_bytes_per_launch": down_bytes,
                                  "peak_source": f"{peak_src} hbm_gbs"}})
        return line

    if name == "kv":
        L, T = args.layers, inputs.KV_TOKENS
        C = inputs.KV_HEADS * inputs.KV_HEAD_DIM
        xs = [inputs.kv_tensor(l, kv, device=device).view(T, C) for l in range(L) for kv in (0, 1)]
        qs = [nb.NVFP4Tensor.empty(T, C, nb.SF_LINEAR, device) for _ in xs]
        y = torch.empty((T, C), dtype=torch.bfloat16, device=device)

        def quant_all():
            for x, q in zip(xs, qs):
                nb.nvfp4_quantize(x, out=q, workspace=ws)

        def deq_all():
            for q in qs:
                nb.nvfp4_dequantize(q, out=y)

        qms = _timed(quant_all, args.steps, args.warmup)
        dms = _timed(deq_all, args.steps, args.warmup)
        st = nb.nvfp4_check_status(ws)
        nvals = len(xs) * T * C
        qgbs = nvals * QUANT_BYTES_PER_VALUE_2PASS / qms / 1e6
        dgbs = nvals * (0.5625 + 2.0) / dms / 1e6
        per_token = sum(q.nbytes() for q in qs) // T
        line.update({"metric": "NVFP4 KV-cache quantize GB/s (32 layers x K,V, 128K tokens)",
                     "value": qgbs, "unit": "GB/s", "higher_is_better": True, "ms_per_step": qms,
                     "config": {"workload": f"kv cache {L} x {{K,V}} x [131072 x 8 x 128]"},
                     "bytes_per_token": per_token, "bytes_per_value": per_token / (2 * L * C),
                     "dequantize_ms": dms, "dequantize_gbs": dgbs, "status": st,
                     "roofline": {"kernel": "k_amax + k_encode", "bound": "hbm", "achieved": qgbs,
                                  "peak": hbm_gbs, "unit": "GB/s", "frac": qgbs / hbm_gbs,
                                  "bytes_per_value": QUANT_BYTES_PER_VALUE_2PASS,
                                  "peak_source": f"{peak_src} hbm_gbs"}})
        return line
    if name == "wgrad":
        # dW = dY^T X from the forward layouts dY [M x N], X [M x K]: both
        # operands quantized column-wise with the 16x16 Hadamard transform.
        m = inputs.WGRAD_M
        mask = inputs.rht_sign_mask(0)
        dy_t = inputs.wgrad_grad_output_t(m, device=device)
        x_t = inputs.wgrad_activation_t(m, device=device)
        dy, x = dy_t.t().contiguous(), x_t.t().contiguous()
        qa = nb.NVFP4Tensor.empty(N, m, device=device)
        qw = nb.NVFP4Tensor.empty(K, m, device=device)
        d = torch.empty((N, K), dtype=torch.bfloat16, device=device)
        ev = {k: torch.cuda.Event(enable_timing=True) for k in "abcd"}

        def step(mark=False):
            if mark:
                ev["a"].record()
            nb.nvfp4_quantize_t(dy, out=qa, sign_mask=mask, workspace=ws)
            if mark:
                ev["b"].record()
            nb.nvfp4_quantize_t(x, out=qw, sign_mask=mask, workspace=ws)
            if mark:
                ev["c"].record()
            nb.nvfp4_gemm(qa, qw, out=d, workspace=ws)
            if mark:
                ev["d"].record()

        ms = _timed(step, args.steps, args.warmup, flush)
        qa_ms, qw_ms, g_ms = [], [], []
        for _ in range(max(3, min(args.steps, 10))):
            flush()
            step(mark=True)
            torch.cuda.synchronize()
            qa_ms.append(ev["a"].elapsed_time(ev["b"]))
            qw_ms.append(ev["b"].elapsed_time(ev["c"]))
            g_ms.append(ev["c"].elapsed_time(ev["d"]))
        qa_ms, qw_ms, g_ms = (statistics.median(v) for v in (qa_ms, qw_ms, g_ms))
        # the same operand quantized row-wise from an explicit dY^T
        rw_ms = _timed(lambda: nb.nvfp4_quantize_rht(dy_t, mask, out=qa, workspace=ws),
                       args.steps, args.warmup, flush)
        # column-wise without the transform
        cw_ms = _timed(lambda: nb.nvfp4_quantize_t(dy, out=qa, workspace=ws),
                       args.steps, args.warmup, flush)
        st = nb.nvfp4_check_status(ws)
        flops = 2.0 * N * K * m
        nv = N * m
        qgbs = nv * QUANT_BYTES_PER_VALUE_2PASS / qa_ms / 1e6
        line.update({"metric": "NVFP4 Wgrad step TFLOP/s (column-wise RHT quantize of dY and X + GEMM)",
                     "value": flops / ms / 1e9, "unit": "TFLOP/s", "higher_is_better": True,
                     "ms_per_step": ms,
                     "config": {"workload": f"wgrad dW = dY^T X, {N} x {K}, {m} tokens, forward layouts, "
                                            "16x16 RHT on both operands", "sign_mask": mask,
                                "l2": "flushed"},
                     "quantize_t_rht_dy_ms": qa_ms, "quantize_t_rht_x_ms": qw_ms, "gemm_ms": g_ms,
                     "quantize_t_rht_dy_gbs": qgbs,
                     "quantize_t_dy_gbs": nv * QUANT_BYTES_PER_VALUE_2PASS / cw_ms / 1e6,
                     "quantize_rht_rowwise_dy_t_gbs": nv * QUANT_BYTES_PER_VALUE_2PASS / rw_ms / 1e6,
                     "gemm_tflops": flops / g_ms / 1e9, "status": st,
                     "roofline": {"kernel": "k_amax_t_rht + k_encode_t_rht (dY)", "bound": "hbm",
                                  "achieved": qgbs, "peak": hbm_gbs, "unit": "GB/s",
                                  "frac": qgbs / hbm_gbs,
                                  "bytes_per_value": QUANT_BYTES_PER_VALUE_2PASS,
                                  "peak_source": f"{peak_src} hbm_gbs"}})
        return line
    if name == "train":
        # One NVFP4 linear layer of the ffn, forward and backward, in the
        # recipe's roles: Fprop Y = X W^T; Dgrad dX = dY W (dY stochastically
        # rounded, W^T from the 2D blocks); Wgrad dW = dY^T X (both operands
        # column-wise with the Hadamard transform, dY stochastically rounded).
        m = inputs.WGRAD_M
        mask = inputs.rht_sign_mask(0)
        w = inputs.ffn_weight(device=device)                      # N x K
        x = inputs.ffn_activation(m, device=device)                # M x K
        dy = inputs.wgrad_grad_output_t(m, device=device).t().contiguous()   # M x N
        qw = nb.NVFP4Tensor.empty(N, K, device=device)
        qwt = nb.NVFP4Tensor.empty(K, N, device=device)
        qx = nb.NVFP4Tensor.empty(m, K, device=device)
        qdy = nb.NVFP4Tensor.empty(m, N, device=device)
        qdyt = nb.NVFP4Tensor.empty(N, m, device=device)
        qxt = nb.NVFP4Tensor.empty(K, m, device=device)
        y = torch.empty((m, N), dtype=torch.bfloat16, device=device)
        dx = torch.empty((m, K), dtype=torch.bfloat16, device=device)
        dw = torch.empty((N, K), dtype=torch.bfloat16, device=device)
        names = ["quantize_2d_w", "quantize_x", "fprop_gemm", "quantize_sr_dy", "dgrad_gemm",
                 "quantize_t_sr_rht_dy", "quantize_t_rht_x", "wgrad_gemm"]
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        seed = [0]

        def step(mark=False):
            seed[0] += 1
            ops = [lambda: nb.nvfp4_quantize_2d(w, out=qw, out_t=qwt, workspace=ws),
                   lambda: nb.nvfp4_quantize(x, out=qx, workspace=ws),
                   lambda: nb.nvfp4_gemm(qx, qw, out=y, workspace=ws),
                   lambda: nb.nvfp4_quantize_sr(dy, 2 * seed[0], out=qdy, workspace=ws),
                   lambda: nb.nvfp4_gemm(qdy, qwt, out=dx, workspace=ws),
                   lambda: nb.nvfp4_quantize_sr(dy, 2 * seed[0] + 1, out=qdyt, transposed=True,
                                                sign_mask=mask, workspace=ws),
                   lambda: nb.nvfp4_quantize_t(x, out=qxt, sign_mask=mask, workspace=ws),
                   lambda: nb.nvfp4_gemm(qdyt, qxt, out=dw, workspace=ws)]
            for i, op in enumerate(ops):
                if mark:
                    ev[i].record()
                op()
            if mark:
                ev[-1].record()

        ms = _timed(step, args.steps, args.warmup, flush)
        parts = {n: [] for n in names}
        for _ in range(max(3, min(args.steps, 10))):
            flush()
            step(mark=True)
            torch.cuda.synchronize()
            for i, n in enumerate(names):
                parts[n].append(ev[i].elapsed_time(ev[i + 1]))
        parts = {n: statistics.median(v) for n, v in parts.items()}
        st = nb.nvfp4_check_status(ws)
        flops = 3 * 2.0 * m * N * K
        gemm_ms = parts["fprop_gemm"] + parts["dgrad_gemm"] + parts["wgrad_gemm"]
        q_ms = ms - gemm_ms
        line.update({"metric": "NVFP4 linear-layer training step TFLOP/s (Fprop + Dgrad + Wgrad)",
                     "value": flops / ms / 1e9, "unit": "TFLOP/s", "higher_is_better": True,
                     "ms_per_step": ms,
                     "config": {"workload": f"ffn linear {N} x {K}, {m} tokens: 2D-block W, SR "
                                            "gradients, RHT on the Wgrad operands", "l2": "flushed"},
                     "phase_ms": parts, "gemm_tflops": flops / gemm_ms / 1e9, "status": st,
                     "roofline": {"kernel": "k_gemm_nvf4 (three GEMMs)", "bound": "tensor",
                                  "achieved": flops / gemm_ms / 1e9, "peak": fp4_peak,
                                  "unit": "TFLOP/s", "frac": flops / gemm_ms / 1e9 / fp4_peak,
                                  "quantize_share": q_ms / ms,
                                  "peak_source": f"{peak_src} bf16 x {FP4_OVER_BF16:g}"}})
        return line
    if name == "mxfp4":
        # The format the pages compare NVFP4 with: block 32, power-of-two
        # scales, no tensor scale -- quantize (one pass) and the W4A4 GEMM at
        # the headline FFN shape, plus the 2^28-value sweep tensor.
        m = 8192
        w = inputs.ffn_weight(device=device)
        qw = nb.nvfp4_quantize_mx(w, workspace=ws)
        del w
        a = inputs.ffn_activation(m, device=device)
        qa = nb.MXFP4Tensor.empty(m, K, device=device)
        d = torch.empty((m, N), dtype=torch.bfloat16, device=device)
        qms = _timed(lambda: nb.nvfp4_quantize_mx(a, out=qa, workspace=ws), args.steps, args.warmup, flush)
        gms = _timed(lambda: nb.nvfp4_gemm_mx(qa, qw, out=d, workspace=ws), args.steps, args.warmup, flush)
        xs = inputs.sweep_tensor(1 << 28, device=device)
        qs = nb.MXFP4Tensor.empty(xs.shape[0], xs.shape[1], device=device)
        sms = _timed(lambda: nb.nvfp4_quantize_mx(xs, out=qs, workspace=ws), args.steps, args.warmup)
        dms = _timed(lambda: nb.nvfp4_dequantize_mx(qs, out=xs), args.steps, args.warmup)
        st = nb.nvfp4_check_status(ws)
        flops = 2.0 * m * N * K
        mx_bpv = 2.0 + 0.5 + 1.0 / 32
        sgbs = (1 << 28) * mx_bpv / sms / 1e6
        line.update({"metric": "MXFP4 W4A4 linear M=8192 TFLOP/s (quantize A + GEMM)",
                     "value": flops / (qms + gms) / 1e9, "unit": "TFLOP/s", "higher_is_better": True,
                     "ms_per_step": qms + gms,
                     "config": {"workload": f"mxfp4 ffn linear M={m} N={N} K={K}; quantize sweep 2^28",
                                "l2": "flushed (GEMM); sweep tensors exceed L2"},
                     "gemm_ms": gms, "quantize_ms": qms, "gemm_tflops": flops / gms / 1e9,
                     "quantize_2p28_ms": sms, "quantize_2p28_gbs": sgbs,
                     "dequantize_2p28_gbs": (1 << 28) * (0.5 + 1.0 / 32 + 2.0) / dms / 1e6,
                     "bytes_per_value_quantize": mx_bpv, "status": st,
                     "roofline": {"kernel": "k_gemm_mxf4", "bound": "tensor", "achieved": flops / gms / 1e9,
                                  "peak": fp4_peak, "unit": "TFLOP/s",
                                  "frac": flops / gms / 1e9 / fp4_peak,
                                  "quantize_frac_of_hbm": sgbs / hbm_gbs,
                                  "peak_source": f"{peak_src} bf16 x {FP4_OVER_BF16:g}"}})
        return line
    if name == "consumers":
        # The steps after the path: MoE per-token combine of the expert
        # outputs (4096 tokens x top-8 x 6144) and NVFP4 -> FP8 of one KV
        # tensor (131072 x 1024).
        r = inputs.MoeRouting()
        g = torch.Generator(device=device).manual_seed(inputs.seed_for("moe", 9100))
        out = torch.randn((r.padded_rows, inputs.MOE_HIDDEN), generator=g, device=device).to(torch.bfloat16)
        slots, w = r.token_slots.to(device), r.combine_weights.to(device)
        y = torch.empty((r.tokens, inputs.MOE_HIDDEN), dtype=torch.bfloat16, device=device)
        cms = _timed(lambda: nb.nvfp4_moe_combine(out, slots, w, out=y), args.steps, args.warmup, flush)
        cbytes = r.tokens * inputs.MOE_HIDDEN * 2 * (r.topk + 1)
        x = inputs.kv_tensor(0, 0, device=device).view(inputs.KV_TOKENS, -1).contiguous()
        q = nb.nvfp4_quantize(x, layout=nb.SF_LINEAR, workspace=ws)
        f8 = torch.empty(x.shape, dtype=torch.uint8, device=device)
        sc = torch.zeros(1, dtype=torch.float32, device=device)
        fms = _timed(lambda: nb.nvfp4_dequantize_fp8(q, out=f8, scale=sc), args.steps, args.warmup, flush)
        fbytes = x.numel() * (0.5625 + 1.0)
        # gated activation + quantize of the MoE intermediate (real rows)
        gu = torch.randn((r.real_rows, 2 * inputs.MOE_INTER), generator=g, device=device).to(torch.bfloat16)
        qh = nb.NVFP4Tensor.empty(r.real_rows, inputs.MOE_INTER, device=device)
        sms_ = _timed(lambda: nb.nvfp4_quantize_swiglu(gu, out=qh, workspace=ws), args.steps, args.warmup, flush)
        sbytes = r.real_rows * inputs.MOE_INTER * (2 * 2 * 2 + 0.5625)     # two passes over gate|up
        st = nb.nvfp4_check_status(ws)
        cgbs = cbytes / cms / 1e6
        line.update({"metric": "MoE top-8 combine GB/s (4096 tokens x 6144)", "value": cgbs, "unit": "GB/s",
                     "higher_is_better": True, "ms_per_step": cms,
                     "config": {"workload": "consumers: moe combine 4096 x top-8 x 6144; kv nvfp4->fp8 "
                                            "131072 x 1024", "l2": "flushed"},
                     "combine_ms": cms, "fp8_ms": fms, "fp8_gbs": fbytes / fms / 1e6,
                     "swiglu_quantize_ms": sms_, "swiglu_quantize_gbs": sbytes / sms_ / 1e6, "status": st,
                     "roofline": {"kernel": "k_moe_combine", "bound": "hbm", "achieved": cgbs,
                                  "peak": hbm_gbs, "unit": "GB/s", "frac": cgbs / hbm_gbs,
                                  "fp8_frac": fbytes / fms / 1e6 / hbm_gbs,
                                  "peak_source": f"{peak_src} hbm_gbs"}})
        return line
    if name == "attention":
        # One decode step read straight from the NVFP4 KV cache: 32 layers,
        # each K and V [131072 tokens x 8 KV heads x 128] (the KV workload),
        # 64 query heads (8 per KV head).  The cache (4.8 GB) is far larger
        # than L2, so no flush is needed between steps.
        T, H = inputs.KV_TOKENS, inputs.KV_HEADS
        layers = []
        for layer in range(args.layers):
            kq = []
            for kv in (0, 1):
                x = inputs.kv_tensor(layer, kv, device=device).view(T, -1)
                kq.append(nb.nvfp4_quantize(x, layout=nb.SF_LINEAR, workspace=ws))
                del x
            layers.append((inputs.kv_query(layer, device=device), kq[0], kq[1]))
        heads_q = inputs.KV_QUERY_HEADS
        aws = nb.Workspace(device, nb.nvfp4_workspace_bytes(nb.OP_ATTENTION, T, heads_q, H))
        outs = [torch.empty((heads_q, 128), dtype=torch.bfloat16, device=device) for _ in layers]

        def step():
            for (qq, kk, vv), o in zip(layers, outs):
                nb.nvfp4_attention_decode(qq, kk, vv, H, out=o, workspace=aws)

        ms = _timed(step, args.steps, args.warmup)
        one = _timed(lambda: nb.nvfp4_attention_decode(layers[0][0], layers[0][1], layers[0][2], H,
                                                       out=outs[0], workspace=aws),
                     args.steps, args.warmup, flush)
        st = nb.nvfp4_check_status(ws)
        cache_bytes = len(layers) * 2 * T * H * 128 * 0.5625
        gbs = cache_bytes / ms / 1e6
        # Scores and the weighted V sum both run on the tensor cores (2 x 2
        # flops per MAC, heads_q x T x 128 MACs each); the roofline is the
        # layer's cache read (K and V codes and scales, once).
        layer_bytes = T * H * 128 * 2 * 0.5625
        achieved = layer_bytes / one / 1e6
        line.update({"metric": "NVFP4 KV-cache decode attention GB/s of cache read (32 layers x K,V, "
                               "128K tokens, 64 query / 8 KV heads)",
                     "value": gbs, "unit": "GB/s", "higher_is_better": True, "ms_per_step": ms,
                     "config": {"workload": f"attention decode {len(layers)} x {{K,V}} x [131072 x 8 x 128], "
                                            "64 query heads",
                                "l2": "inputs (4.8 GB cache) larger than L2; one-layer timing flushed"},
                     "tokens_per_s": 1e3 / ms, "ms_per_layer": one, "status": st,
                     "hbm_frac": gbs / hbm_gbs,
                     "roofline": {"kernel": "k_attn_partial + k_attn_combine (one layer)", "bound": "hbm",
                                  "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                                  "frac": achieved / hbm_gbs,
                                  "algorithmic_bytes_per_launch": layer_bytes,
                                  "tensor_flops_per_launch": 2 * 2.0 * heads_q * T * 128,
                                  "peak_source": f"{peak_src} hbm_gbs"}})
        return line
    raise ValueError(name)


# -------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the CPU oracle leg")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the standalone 2^28 quantize measurement")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--workload", default="ffn8192",
                    choices=["ffn8192", "ffn16", "ffn512", "sweep", "moe", "kv", "wgrad", "train", "mxfp4", "consumers",
                             "attention"],
                    help="ffn8192 is the headline; the others measure the remaining scope rows")
    ap.add_argument("--layers", type=int, default=32,
                    help="kv / attention workloads: layers of the KV cache (the workload has 32; "
                         "fewer give a case small enough for a multi-pass ncu capture)")
    ap.add_argument("--gemm-kernel", default="pair", choices=["single", "pair"],
                    help="GEMM kernel for M >= 256: CTA pairs on 256x256 tiles (the library "
                         "default) or one SM per 128x256 tile")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.warmup < 3:
        args.warmup = 3

    rank, local_rank, world = env_rank()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if args.workload != "ffn8192":
        if world == 1:
            line = workload_line(args.workload, args, device)
            print(json.dumps(line), flush=True)
            return 0
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = measured_peaks()
    fp4_peak = bf16_tf * FP4_OVER_BF16

    wl = Workload(device)
    wl.nb.nvfp4_set_gemm_pairs(args.gemm_kernel == "pair")
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        step_ms, quant_ms, gemm_ms, launches = time_steps(wl, args.steps, args.warmup)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    st = wl.nb.nvfp4_check_status(wl.ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after timed steps")

    total_ms = sum(step_ms)
    gemm_avg = sum(gemm_ms) / len(gemm_ms)
    quant_avg = sum(quant_ms) / len(quant_ms)
    total_ms, gemm_avg, quant_avg = max_over_ranks([total_ms, gemm_avg, quant_avg], dist, device)
    flops = 2.0 * M * N * K
    ms_per_step = total_ms / args.steps
    value = replica_throughput(world, flops, args.steps, total_ms) / 1e12
    gemm_tflops = flops / (gemm_avg / 1e3) / 1e12

    sweep_ms, sweep_ms1, sst = (float("nan"),) * 2 + (0,)
    if not args.no_sweep:
        sweep_ms, sweep_ms1, sst = time_sweep_quantize(wl.nb, device)
    e2e_ms, h2d, d2h = float("nan"), 0, 0
    if not args.no_e2e:
        e2e_ms, h2d, d2h = time_e2e(wl, args.steps, args.warmup)
    sweep_ms, sweep_ms1, e2e_ms = max_over_ranks([sweep_ms, sweep_ms1, e2e_ms], dist, device)

    if rank == 0:
        gbs_2pass = SWEEP_N * QUANT_BYTES_PER_VALUE_2PASS / (sweep_ms / 1e3) / 1e9
        gbs_1pass = SWEEP_N * ENCODE_BYTES_PER_VALUE / (sweep_ms1 / 1e3) / 1e9
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "nvfp4 (e2m1 x e4m3/16, fp32 accumulate, bf16 out)",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "flushed (256 MiB write) before every timed step",
                       "weights": "pre-quantized once, outside the timed region",
                       "gemm_kernel": "cta_pair_256x256" if args.gemm_kernel == "pair"
                       else "single_cta_128x256"},
            "roofline": {"kernel": "k_gemm_nvf4_pair" if args.gemm_kernel == "pair" else "k_gemm_nvf4",
                         "bound": "tensor",
                         "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": gemm_tflops / fp4_peak,
                         "peak_source": f"{peak_src} bf16 burst {bf16_tf} TFLOP/s x "
                                        f"{FP4_OVER_BF16:g} (nominal FP4/BF16 ratio)",
                         "traffic": gemm_traffic(args.gemm_kernel), "ms_per_launch": gemm_avg,
                         "algorithmic_flops_per_launch": flops},
            "quantize": {"workload": "quantize sweep, 2^28 BF16 values [65536 x 4096]",
                         "gbs_two_pass": gbs_2pass, "frac_two_pass": gbs_2pass / hbm_gbs,
                         "ms_two_pass": sweep_ms,
                         "gbs_supplied_scale": gbs_1pass, "frac_supplied_scale": gbs_1pass / hbm_gbs,
                         "ms_supplied_scale": sweep_ms1,
                         "bytes_per_value": {"two_pass": QUANT_BYTES_PER_VALUE_2PASS,
                                             "supplied_scale": ENCODE_BYTES_PER_VALUE},
                         "peak_gbs": hbm_gbs, "peak_source": f"{peak_src} hbm_gbs",
                         "status": sst},
            "activation_quantize_ms": quant_avg,
            "gpu_launches": launches,
            "e2e": {"value": world * flops / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms,
                    "overlap": "consecutive steps on three streams: input copy, compute, output copy"},
            "clocks": clk.summary(),
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_entry()
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
