#!/usr/bin/env python
"""Throughput of the HARP rotate + quantize path on B200.

Workload (the headline configuration): a 4096 x 4096 bf16 weight (Student-t
nu = 3 entries x 0.02, 0.5 % of input channels x 20), two-sided processor
(16,16,16) x (16,16,16) with random orthogonal blocks and random signs,
Lloyd-Max N(0,1) codebooks with group 128 at 2 and at 4 bits.

One step = the whole hot path over that weight, for each bit width, through
the public two-sided calls: harp_rotate_quantize (rotate both sides,
quantize, pack) then harp_dequantize_unrotate (decode, inverse rotation, bf16
out). Each call runs the library's pass kernels (two for this plan), which
bench.py times one by one with events the library records between them.
value = algorithmic bytes of the step (bf16 weight read and codes + fp16
scales written by each forward; codes + scales read and the bf16 weight
written by each inverse) / device time, in GB/s. The fp32 intermediate
between the passes is implementation traffic and is not credited. L2 is flushed (512 MB write) before every timed step.

--impl reference times the float64 oracle (the CPU statement of the same
computation) on the host cores instead, on a bounded sample of the same
workload. Under torchrun every rank runs an independent replica (the path has
no exchange step); the time is the maximum over ranks.
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import os
import shutil
import signal
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "rotate+quantize GB/s and % of B200 HBM peak (4096×4096 bf16, two-sided)"
ROWS = COLS = 4096
RADIX = (16, 16, 16)
BITS = (2, 4)
GROUP = 128
L2_FLUSH_BYTES = 512 << 20
WORKLOAD = ("4096x4096 bf16 weight (Student-t nu=3 x0.02, 0.5% input channels x20), two-sided "
            "HARP processor (16,16,16)x(16,16,16), random orthogonal blocks + random signs; "
            "Lloyd-Max N(0,1) group 128 at 2 and 4 bits; step = rotate+quantize then "
            "dequantize+unrotate for each bit width")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}

# DRAM bytes (read + write) per pass launch of this step, from one ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum) of the pass kernels
# built from the source whose SHA-256 prefix is "kernel_src"; writes still in
# L2 when a launch ends are counted by the next launch. When the pass-kernel
# source differs from the captured one the figures no longer describe the
# kernel and the roofline's traffic field is reported as null.
MEASURED_TRAFFIC = {"kernel_src": "7a9a4395ad575c7d", "bytes": {
    "fwd_p0_2bit": 50513920,
    "fwd_p1_2bit": 87086848,
    "fwd_p2_2bit": 67988480,
    "inv_p0_2bit": 16457216,
    "inv_p1_2bit": 87363584,
    "inv_p2_2bit": 70016512,
    "fwd_p0_4bit": 47332096,
    "fwd_p1_4bit": 87085056,
    "fwd_p2_4bit": 68019968,
    "inv_p0_4bit": 21024256,
    "inv_p1_4bit": 87330048,
    "inv_p2_4bit": 69442304,
}}
PASS_SRC = os.path.join(ROOT, "rotation_preconditioned_bit_b200", "csrc", "harp_pass.cu")


def pass_source_hash():
    import hashlib
    with open(PASS_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def measured_traffic(kernel):
    if MEASURED_TRAFFIC["kernel_src"] != pass_source_hash():
        return None
    return MEASURED_TRAFFIC["bytes"].get(kernel)


def fwd_bytes_per_elem(bits):
    return 2.0 + bits / 8.0 + 2.0 / GROUP


def inv_bytes_per_elem(bits):
    return bits / 8.0 + 2.0 / GROUP + 2.0


STEP_BYTES = ROWS * COLS * sum(fwd_bytes_per_elem(b) + inv_bytes_per_elem(b) for b in BITS)
FLOP_PER_ELEM_SIDE = 2 * sum(RADIX)      # one FMA per block coefficient per element


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def fp32_peak_tflops(sm_mhz):
    """FFMA peak: 148 SMs x 128 fp32 lanes x 2 flop x clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


# ------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            cmd = ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                   "--format=csv,noheader,nounits", "-lms", "20"]
            if shutil.which("stdbuf"):
                cmd = ["stdbuf", "-oL"] + cmd      # line-buffered: samples arrive as taken
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            time.sleep(0.3)                         # first sample before the timed region
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.05)
        self.proc.send_signal(signal.SIGINT)
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ multi-rank helpers

def max_over_ranks(ms, world, device):
    """The slowest rank's time (every rank replicates the same step; the job
    is done when the last replica is)."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.item()


def job_gbs(world, steps, total_ms):
    """Whole-job algorithmic GB/s: every rank processes STEP_BYTES per step."""
    return world * STEP_BYTES * steps / (total_ms * 1e-3) / 1e9


# ------------------------------------------------------------ GPU arm

def run_gpu(args, rank, world, local_rank):
    import numpy as np
    import torch

    import rotation_preconditioned_bit_b200 as harp
    from rotation_preconditioned_bit_b200 import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.workload("c2")
    left = harp.Plan.from_side(w.left)
    right = harp.Plan.from_side(w.right)
    cbs = [harp.Codebook("lloyd_max", b, GROUP) for b in BITS]
    x_host = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16).pin_memory()
    x = x_host.to(dev)
    ws = harp.empty_workspace(left, right, ROWS, COLS, dev)
    out = torch.empty((ROWS, COLS), dtype=torch.bfloat16, device=dev)
    outs = [harp.empty_codes(ROWS, COLS, cb, dev) for cb in cbs]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # one step = for each bit width the public two-sided forward call, then
    # the inverse call; each call launches `npass` pass kernels, timed one by
    # one with CUDA events the library records between its launches
    npass = harp.harp_pass_count(left, right, cbs[0])
    assert npass > 0, "the two-sided calls should run the pass kernels"
    pass_fma = [harp.harp_pass_fma(left, right, cbs[0], k) for k in range(npass)]
    names = [f"fwd_p{k}" for k in range(npass)] + [f"inv_p{k}" for k in range(npass)]
    kt = {f"{n}_{b}bit": [] for b in BITS for n in names}
    ev_pool = []

    def new_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record(stream)                     # creates the CUDA event before timing
        return evs

    def step(record):
        evs = []
        for cb, (codes, scales) in zip(cbs, outs):
            if record:
                ef, ei = ev_pool.pop(), ev_pool.pop()
                harp.harp_set_pass_events(ef)
            harp.harp_rotate_quantize(left, right, cb, x, codes, scales, None, ws, stream)
            if record:
                harp.harp_set_pass_events(ei)
            harp.harp_dequantize_unrotate(left, right, cb, codes, scales, out, ws, stream)
            if record:
                harp.harp_set_pass_events([])
                evs.append((cb.bits, ef, ei))
        return evs

    for _ in range(2 * len(BITS) * args.steps):
        ev_pool.append(new_events(npass + 1))
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        flush.zero_()
        step(False)
    torch.cuda.synchronize()

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    step_ms = []
    all_evs = []
    for _ in range(args.steps):
        flush.zero_()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        evs = step(True)
        s1.record(stream)
        all_evs.append((s0, s1, evs))
    torch.cuda.synchronize()
    clk = clocks.stop()
    for s0, s1, evs in all_evs:
        step_ms.append(s0.elapsed_time(s1))
        for bits, ef, ei in evs:
            for k in range(npass):
                kt[f"fwd_p{k}_{bits}bit"].append(ef[k].elapsed_time(ef[k + 1]))
                kt[f"inv_p{k}_{bits}bit"].append(ei[k].elapsed_time(ei[k + 1]))
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    if world > 1:
        torch.distributed.barrier()

    # ---- the same step with every block stage forced onto the tensor cores
    # (tcgen05, 3xTF32), timed the same way, for comparison with the
    # automatic choice above (every rank takes the same steps)
    alt = None
    if not args.no_alt:
        harp.harp_set_block_stages(harp.HARP_BLOCK_STAGES_TC)
        kt_tc = {k: [] for k in kt}
        for _ in range(args.warmup):
            flush.zero_()
            step(False)
        for _ in range(2 * len(BITS) * args.steps):
            ev_pool.append(new_events(npass + 1))
        torch.cuda.synchronize()
        alt_ms, alt_evs = [], []
        for _ in range(args.steps):
            flush.zero_()
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            evs = step(True)
            s1.record(stream)
            alt_evs.append((s0, s1, evs))
        torch.cuda.synchronize()
        harp.harp_set_block_stages(harp.HARP_BLOCK_STAGES_AUTO)
        for s0, s1, evs in alt_evs:
            alt_ms.append(s0.elapsed_time(s1))
            for bits, ef, ei in evs:
                for k in range(npass):
                    kt_tc[f"fwd_p{k}_{bits}bit"].append(ef[k].elapsed_time(ef[k + 1]))
                    kt_tc[f"inv_p{k}_{bits}bit"].append(ei[k].elapsed_time(ei[k + 1]))
        alt = (max_over_ranks(sum(alt_ms), world, dev), kt_tc)
        if world > 1:
            torch.distributed.barrier()

    # ---- end to end through the C ABI's host-buffer calls
    e2e = None
    if not args.no_e2e:
        codes_h = [torch.empty(c.shape, dtype=c.dtype).pin_memory() for c, _ in outs]
        scales_h = [torch.empty(s.shape, dtype=s.dtype).pin_memory() for _, s in outs]
        outs_h = [torch.empty((ROWS, COLS), dtype=torch.bfloat16).pin_memory() for _ in cbs]
        # the two bit widths are independent chains: each runs on its own
        # stream with its own device scratch (values, codes, scales,
        # workspace), so one chain's PCIe copies overlap the other's kernels
        streams = [stream] + [torch.cuda.Stream(dev) for _ in cbs[1:]]
        scratches = [harp.empty_host_scratch(left, right, cb, ROWS, COLS, harp.HARP_BF16, dev) for cb in cbs]
        h2d = sum(x_host.numel() * 2 + c.numel() + s.numel() * 2 for c, s in zip(codes_h, scales_h))
        d2h = sum(c.numel() + s.numel() * 2 + o.numel() * 2 for c, s, o in zip(codes_h, scales_h, outs_h))
        ws_bytes = sum(t.numel() for t in scratches)

        def e2e_step():
            # per bit width: the forward from the host weight to host codes and
            # scales, then the inverse from those host buffers to the host
            # weight, in order on that chain's stream
            start = torch.cuda.Event()
            start.record(stream)
            for i, cb in enumerate(cbs):
                st = streams[i]
                if st is not stream:
                    st.wait_event(start)
                harp.harp_rotate_quantize_host(left, right, cb, x_host, codes_h[i], scales_h[i], scratches[i], st)
                harp.harp_dequantize_unrotate_host(left, right, cb, codes_h[i], scales_h[i], outs_h[i],
                                                   scratches[i], st)
            for st in streams[1:]:
                done = torch.cuda.Event()
                done.record(st)
                stream.wait_event(done)

        for _ in range(max(2, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e_ms = []
        for _ in range(args.steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e_step()
            b.record(stream)
            b.synchronize()
            e_ms.append(a.elapsed_time(b))
        e_total = max_over_ranks(sum(e_ms), world, dev)
        e2e = {"value": round(job_gbs(world, args.steps, e_total), 2),
               "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e_total / args.steps, 4),
               "api": "harp_rotate_quantize_host + harp_dequantize_unrotate_host (two-sided): pinned host "
                      "buffers in and out; per bit width one stream, copies (cudaMemcpyAsync) and kernels in "
                      "order on it, the two widths' streams concurrent",
               "scratch_bytes": ws_bytes}
    del flush
    return total_ms, step_ms, kt, clk, e2e, npass, pass_fma, alt


WORKLOAD_NAMES = ("c1", "c3", "c4", "c5", "rht", "pq", "theta")


def workload_cpu_baseline(w, q, budget_s=1.0):
    """The float64 oracle on a bounded sample of a workload's forward call,
    on all host cores (OpenMP over rows / columns) and on one thread: the
    right pass + quantise + pack on a strip of rows and, for two-sided
    calls, the left pass on a strip of columns, each the same fraction of the
    matrix (sized to about budget_s seconds). Credited with that fraction of
    the call's algorithmic bytes."""
    import numpy as np

    import oracle
    from rotation_preconditioned_bit_b200 import synth

    rows, cols = w.rows, w.cols
    Pr = oracle.processor(w.right)
    Pl = oracle.processor(w.left) if w.left is not None else None
    in_b = 2 if w.dtype == "bf16" else 4

    def f64(a):
        return synth.bf16_bits_to_f64(a) if w.dtype == "bf16" else np.asarray(a, dtype=np.float64)

    def sample(frac):
        nr = max(1, int(round(rows * frac)))
        nc = max(1, int(round(cols * frac)))
        Xr = f64(np.ascontiguousarray(w.x[:nr]))
        Xc = f64(np.ascontiguousarray(w.x[:, :nc])) if Pl is not None else None
        t0 = time.perf_counter()
        if Pl is not None:
            Pl.rotate_cols(Xc)
        Y = Pr.rotate_rows(Xr)
        codes, scales, _, _ = oracle.quantize(q.kind, q.bits, q.group, Y, with_margins=False)
        oracle.pack(q.bits, codes)
        dt = time.perf_counter() - t0
        return dt, nr * cols, nr, nc

    out = {}
    cores = os.cpu_count() or 1
    for label, nt in (("all_cores", cores), ("single_thread", 1)):
        oracle.threads(nt)
        frac = min(1.0, (1 << 18) / (rows * cols))
        dt, _, _, _ = sample(frac)
        frac = min(1.0, frac * budget_s / max(dt, 1e-3))
        dt, elems, nr, nc = sample(frac)
        gbs = elems * (in_b + q.bits / 8.0 + 2.0 / q.group) / dt / 1e9
        strip = f"{nr}x{cols} row strip" + (f" and {rows}x{nc} column strip" if Pl is not None else "")
        out[label] = {"gbs": round(gbs, 4), "cores": oracle.threads(), "seconds": round(dt, 2),
                      "sample": f"float64 oracle, forward on a {strip} ({frac:.4f} of the matrix)"}
    oracle.threads(cores)
    return out


def run_workloads(steps, dev, names=WORKLOAD_NAMES, c3_tokens=(1, 16, 256, 8192), cpu=False):
    """The other synthetic workloads, through the public calls with inputs
    resident on the device: per call, mean device time over `steps` calls
    (CUDA events; L2 not flushed: each call streams more than L2 except c1
    and the small token counts, which also report fwd_graph_us, the time per
    call replayed from a CUDA graph),
    algorithmic GB/s (input read + codes + scales written for a forward;
    codes + scales read + output written for an inverse) and elements/s."""
    import numpy as np
    import torch

    import rotation_preconditioned_bit_b200 as harp
    from rotation_preconditioned_bit_b200 import synth

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps * 1e-3

    def graph_timed(fn, calls=20, reps=5):
        """Device time per call with the calls replayed from a CUDA graph
        (no host work between launches): the latency a serving loop that
        captures its steps sees; for small calls the plain loop above is
        bound by the host's per-call overhead instead."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(3):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(calls):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / (reps * calls) * 1e-3

    out = {}
    jobs = []
    for name in [n for n in ("c1", "c3", "c4", "c5", "rht") if n in names]:
        # the activation workload at every token count (T <= 16 is a
        # latency case: its time in microseconds is the figure to read)
        jobs += [(name, T) for T in c3_tokens] if name == "c3" else [(name, None)]
    for name, tokens in jobs:
        if name == "rht":
            # the c2 weight with Hadamard-initialised processors on both sides
            # (random signs, normalised Sylvester blocks: HARP's theta = 0 start)
            w = synth.workload("c2")
            w = dataclasses.replace(w, name="rht_4096x4096",
                           right=synth.side_draws(2, RADIX, "hadamard", synth.S_SIGNS_R, synth.S_BLOCKS_R),
                           left=synth.side_draws(2, RADIX, "hadamard", synth.S_SIGNS_L, synth.S_BLOCKS_L),
                           quants=[synth.Quant("lloyd_max", 4, GROUP)])
        elif tokens is not None:
            w = synth.workload(name, tokens=tokens)
        else:
            w = synth.workload(name)
        rows, cols = w.rows, w.cols
        if w.dtype == "bf16":
            x = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16).to(dev)
            in_b = 2
        else:
            x = torch.from_numpy(w.x).to(dev)
            in_b = 4
        right = harp.Plan.from_side(w.right)
        left = harp.Plan.from_side(w.left) if w.left is not None else None
        ws = harp.empty_workspace(left, right, rows, cols, dev) if left else None
        for q in w.quants:
            cb = harp.Codebook(q.kind, q.bits, q.group)
            codes, scales = harp.empty_codes(rows, cols, cb, dev)
            code_b = q.bits / 8.0 + 2.0 / q.group
            n = rows * cols
            key = f"{w.name}_{q.kind}{q.bits}_g{q.group}"
            t = timed(lambda: harp.harp_rotate_quantize(left, right, cb, x, codes, scales, None, ws))
            rec = {"shape": [rows, cols], "fwd_us": round(t * 1e6, 2),
                   "fwd_gbs": round(n * (in_b + code_b) / t / 1e9, 2), "fwd_elems_per_s": float(f"{n / t:.4g}")}
            if rows * cols <= 256 * 4096:
                tg = graph_timed(lambda: harp.harp_rotate_quantize(left, right, cb, x, codes, scales, None, ws))
                rec["fwd_graph_us"] = round(tg * 1e6, 2)
            if cpu:
                rec["cpu_oracle"] = workload_cpu_baseline(w, q)
            if left is not None:
                o = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
                t = timed(lambda: harp.harp_dequantize_unrotate(left, right, cb, codes, scales, o, ws))
                rec.update({"inv_us": round(t * 1e6, 2), "inv_gbs": round(n * (2 + code_b) / t / 1e9, 2),
                            "inv_elems_per_s": float(f"{n / t:.4g}")})
                rec["passes"] = harp.harp_pass_count(left, right, cb)
            out[key] = rec
        del x, ws
        torch.cuda.empty_cache()
    if "pq" in names:
        out.update(run_polarquant(timed, dev))
    if "theta" in names:
        out.update(run_theta_loads(timed, dev))
    return out


def run_polarquant(timed, dev):
    """PolarQuant's per-block workload on the 4096x4096 bf16 weight: rows of
    128 rotated by H_128 (radices (16, 8), Sylvester blocks, no signs) with
    5-bit Lloyd-Max codes (Q5), its inverse, and the fused two-stage codec
    (Q5 codes -> restored fp16 weights -> 4-bit absmax g128)."""
    import numpy as np
    import torch

    import rotation_preconditioned_bit_b200 as harp
    from rotation_preconditioned_bit_b200 import synth

    rows = cols = 4096
    n = rows * cols // 128
    w = synth.workload("c2")
    x = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16).to(dev).view(n, 128)
    plan = harp.Plan((16, 8), [harp.stage_blocks("hadamard", b, 128 // b) for b in (16, 8)])
    q5, a4 = harp.Codebook("lloyd_max", 5, 128), harp.Codebook("absmax", 4, 128)
    c5, s5 = harp.empty_codes(n, 128, q5, dev)
    c4, s4 = harp.empty_codes(n, 128, a4, dev)
    o = torch.empty((n, 128), dtype=torch.bfloat16, device=dev)
    e = rows * cols
    t_f = timed(lambda: harp.harp_rotate_quantize(None, plan, q5, x, c5, s5))
    t_i = timed(lambda: harp.harp_dequantize_unrotate(None, plan, q5, c5, s5, o))
    t_r = timed(lambda: harp.harp_requantize(plan, q5, c5, s5, n, 128, "f16", a4, c4, s4))
    b5, b4 = 5 / 8 + 2 / 128, 4 / 8 + 2 / 128
    return {"polarquant_h128_q5_4096x4096": {
        "fwd_us": round(t_f * 1e6, 2), "fwd_gbs": round(e * (2 + b5) / t_f / 1e9, 2),
        "inv_us": round(t_i * 1e6, 2), "inv_gbs": round(e * (b5 + 2) / t_i / 1e9, 2),
        "requant_q5_to_int4_us": round(t_r * 1e6, 2), "requant_gbs": round(e * (b5 + b4) / t_r / 1e9, 2)}}


def run_theta_loads(timed, dev):
    """Device time to rebuild every stage of a processor from int8-stored
    parameters (harp_plan_load_theta: Givens / Cayley times the base mixer,
    double precision), for the 4096x4096 and 8192x28672 processors."""
    import numpy as np
    import torch

    import rotation_preconditioned_bit_b200 as harp
    from rotation_preconditioned_bit_b200 import synth

    out = {}
    for name, radix in (("theta_4096_16x16x16", (16, 16, 16)), ("theta_28672_7x16x16x16", (7, 16, 16, 16)),
                        ("theta_8192_32x16x16", (32, 16, 16))):
        d = int(np.prod(radix))
        side = synth.side_draws(5, radix, "hadamard", synth.S_SIGNS_R, synth.S_BLOCKS_R)
        plan = harp.Plan.from_side(side)
        params = []
        for t, b in enumerate(radix):
            q = torch.from_numpy(synth.theta_draws(5, t, d // b, b)).to(dev)
            base = None
            if b & (b - 1):
                base = torch.from_numpy(harp.stage_blocks("hadamard", b, 1, None, side.base[t])[0]).to(dev)
            params.append((q, base))

        def load():
            for t, (q, base) in enumerate(params):
                harp.harp_plan_load_theta(plan, t, q, 0.05 / 40, base)

        t_load = timed(load)
        groups = sum(d // b for b in radix)
        out[name] = {"stages": len(radix), "groups": groups, "us": round(t_load * 1e6, 2),
                     "blocks_per_s": float(f"{groups / t_load:.4g}")}
    return out


def kernel_table(kt, npass, pass_fma):
    """Per pass kernel: mean duration, the bytes it moves itself (input read,
    output written: bf16 weight, fp32 workspace, codes + scales), the
    algorithmic bytes of the step it accounts for, and its FLOP rate: forward
    pass k applies stages whose radices sum to pass_fma[k] (one FMA per block
    coefficient per element, 2 flop each); inverse pass k applies the stages
    of forward pass npass-1-k."""
    n = ROWS * COLS
    out = {}
    for key, v in kt.items():
        if not v:
            continue
        us = 1e3 * statistics.mean(v)
        name, bits = key.rsplit("_", 1)
        b = int(bits[:-3])
        kind, pk = name.split("_p")
        k = int(pk)
        flop = n * 2 * (pass_fma[k] if kind == "fwd" else pass_fma[npass - 1 - k])
        code_b = b / 8.0 + 2.0 / GROUP
        if kind == "fwd":
            rd = 2.0 if k == 0 else 4.0
            wr = code_b if k == npass - 1 else 4.0
            alg = n * (2.0 if k == 0 else 0.0) + n * (code_b if k == npass - 1 else 0.0)
        else:
            rd = code_b if k == 0 else 4.0
            wr = 2.0 if k == npass - 1 else 4.0
            alg = n * (code_b if k == 0 else 0.0) + n * (2.0 if k == npass - 1 else 0.0)
        own = n * (rd + wr)
        out[key] = {"us": round(us, 2), "own_bytes": int(own), "own_gbs": round(own / (us * 1e-6) / 1e9, 1),
                    "alg_bytes": int(alg), "tflops": round(flop / (us * 1e-6) / 1e12, 2)}
    return out


# ------------------------------------------------------------ CPU (oracle) arm

_C2 = {}


def _c2_oracle_inputs():
    if not _C2:
        import oracle
        from rotation_preconditioned_bit_b200 import synth
        w = synth.workload("c2")
        _C2["X"] = synth.x_as_f64(w)
        _C2["P"] = (oracle.processor(w.left), oracle.processor(w.right))
    return _C2["X"], _C2["P"]


def oracle_sample(frac):
    """The float64 oracle on a sample of the step, for each bit width of the
    step: the left pass on a column strip and the right pass + quantise +
    pack + dequantise + inverse on a row strip, each a fraction `frac` of the
    weight, with the oracle's current host threads. Returns (seconds,
    algorithmic bytes credited, description)."""
    import oracle

    X, (Pl, Pr) = _c2_oracle_inputs()
    nc = max(1, int(round(COLS * frac)))
    nr = max(1, int(round(ROWS * frac)))
    t0 = time.perf_counter()
    for bits in BITS:
        T = Pl.rotate_cols(X[:, :nc])
        Y = Pr.rotate_rows(X[:nr, :])
        codes, scales, _, _ = oracle.quantize("lloyd_max", bits, GROUP, Y, with_margins=False)
        packed = oracle.pack(bits, codes)
        codes2 = oracle.unpack(bits, packed, COLS)
        Yh = oracle.dequantize("lloyd_max", bits, GROUP, codes2, scales)
        Z = Pr.rotate_rows(Yh, inverse=True)
        U = Pl.rotate_cols(T, inverse=True)
        del T, Z, U
    dt = time.perf_counter() - t0
    elems = nc * ROWS                              # both sides cover this many elements
    credited = elems * sum(fwd_bytes_per_elem(b) + inv_bytes_per_elem(b) for b in BITS)
    nt = oracle.threads()
    desc = (f"float64 oracle, the step's {' and '.join(f'{b}-bit' for b in BITS)} variants: left pass on a "
            f"{ROWS}x{nc} column strip and right pass + quantise + pack + dequantise + inverse on a "
            f"{nr}x{COLS} row strip ({frac:.4f} of the weight), {nt} host thread{'s' if nt > 1 else ''}")
    return dt, credited, desc


def pick_frac(budget_s):
    dt, _, _ = oracle_sample(1.0 / 128)
    per_full = dt * 128
    return max(1.0 / 512, min(1.0, budget_s / per_full))


def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle
    cores = oracle.threads(os.cpu_count() or 1)
    budget = max(1.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    frac = pick_frac(budget)
    for _ in range(args.warmup):
        oracle_sample(frac)
    secs, credited, desc = 0.0, 0.0, ""
    for _ in range(args.steps):
        dt, cr, desc = oracle_sample(frac)
        secs += dt
        credited += cr
    value = credited / secs / 1e9
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * secs / args.steps, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "parallelism": "replicas", "l2": "n/a (host)"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="harp", choices=["harp", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-alt", action="store_true",
                    help="skip the comparison series with every block stage on the tensor cores")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--workloads", action="store_true",
                    help="also time the c1, c3, c4 and c5 workloads (adds ~1 min of input generation)")
    ap.add_argument("--workloads-only", default=None, metavar="NAMES",
                    help="time only these workloads (comma list of " + ",".join(WORKLOAD_NAMES) +
                         ") on one GPU, print them as one JSON line and exit")
    ap.add_argument("--c3-tokens", default="1,16,256,8192", metavar="LIST",
                    help="token counts of the c3 activation workload (comma list)")
    ap.add_argument("--workload-cpu", action="store_true",
                    help="with --workloads-only: also time the float64 oracle on a bounded sample of each "
                         "forward call (all host cores and one thread, about 1 s each)")
    args = ap.parse_args()
    if args.workloads_only is not None:
        import torch
        names = tuple(n for n in args.workloads_only.split(",") if n)
        bad = [n for n in names if n not in WORKLOAD_NAMES]
        if bad:
            ap.error(f"unknown workloads {bad}")
        torch.cuda.set_device(0)
        toks = tuple(int(v) for v in args.c3_tokens.split(",") if v)
        print(json.dumps({"workloads": run_workloads(max(3, args.steps), torch.device("cuda", 0), names, toks,
                                                     cpu=args.workload_cpu)}))
        return
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    import torch
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    total_ms, step_ms, kt, clk, e2e, npass, pass_fma, alt = run_gpu(args, rank, world, local_rank)

    if rank == 0:
        peaks, peak_src = load_peaks()
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        value = job_gbs(world, args.steps, total_ms)
        ktab = kernel_table(kt, npass, pass_fma)
        # dominant kernel: largest total time in the step
        dom = max(ktab, key=lambda k: ktab[k]["us"])
        smhz = float(peaks.get("sm_max_mhz", 1965.0))
        peak_tf = fp32_peak_tflops(smhz)
        d = ktab[dom]
        roof = {"kernel": dom, "bound": "alu", "achieved": d["tflops"], "peak": round(peak_tf, 1),
                "unit": "TFLOP/s", "frac": round(d["tflops"] / peak_tf, 4),
                "traffic": measured_traffic(dom),
                "peak_source": f"FFMA: 148 SM x 128 lanes x 2 flop x {smhz:.0f} MHz (max SM clock, {peak_src})",
                "algorithmic": f"2 flop per block coefficient per element: FMA per element by forward pass {pass_fma}",
                "own_bytes_hbm_frac": round(d["own_gbs"] / hbm, 4)}
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            cores = os.cpu_count() or 1
            oracle.threads(1)
            frac = pick_frac(args.cpu_budget / 2)
            dt1, credited1, desc1 = oracle_sample(frac)
            oracle.threads(cores)
            frac_all = min(1.0, frac * cores)
            dt, credited, desc = oracle_sample(frac_all)
            cpu = {"value": round(credited / dt / 1e9, 4), "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
                   "sample": desc, "seconds": round(dt, 2),
                   "single_thread": {"value": round(credited1 / dt1 / 1e9, 4), "cores": 1, "sample": desc1,
                                     "seconds": round(dt1, 2)}}
        wl = (run_workloads(max(3, args.steps // 4), torch.device("cuda", local_rank))
              if args.workloads and world == 1 else None)
        line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOAD, "rows": ROWS, "cols": COLS, "in_dtype": "bf16",
                           "left_radix": list(RADIX), "right_radix": list(RADIX), "bits": list(BITS),
                           "group": GROUP, "parallelism": "replicas" if world > 1 else "single",
                           "l2": "flushed before every timed step (512 MB write)",
                           "step_bytes": int(STEP_BYTES)},
                "hbm_frac": round(value / world / hbm, 4), "hbm_peak_gbs": hbm, "peak_source": peak_src,
                "roofline": roof, "kernels": ktab, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": 2 * len(BITS) * npass * args.steps, "clocks": clk}
        # the metric's own call, rotate + quantize alone: per bit width the
        # forward passes' device time and the forward's algorithmic bytes
        fwd = {}
        for b in BITS:
            us = sum(ktab[f"fwd_p{k}_{b}bit"]["us"] for k in range(npass))
            gbs = ROWS * COLS * fwd_bytes_per_elem(b) / (us * 1e-6) / 1e9
            fwd[f"{b}bit"] = {"us": round(us, 2), "gbs": round(gbs, 2), "hbm_frac": round(gbs / hbm, 4)}
        line["forward_only"] = fwd
        if alt is not None:
            alt_ms, kt_tc = alt
            ktab_tc = kernel_table(kt_tc, npass, pass_fma)
            line["tensor_core_stages"] = {
                "ms_per_step": round(alt_ms / args.steps, 4),
                "value": round(job_gbs(world, args.steps, alt_ms), 2),
                "note": "same step with every block stage on tcgen05 (kind::tf32, split operands); the "
                        "headline uses the automatic choice (FFMA for 16-wide blocks)",
                "kernels_us": {k: v["us"] for k, v in ktab_tc.items()}}
        if wl is not None:
            line["workloads"] = wl
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
