#!/usr/bin/env python
"""Benchmark: KATA causal chunked forward (+ state export + one decode step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of synthetic input:
kata_chunked_forward over B=1, H=8, T=131072, d=64 bf16 (chunk C=64) with the
final state exported, then one kata_decode_step on that state.  Inputs are
resident in HBM when the timed region starts; the L2 is flushed (a 256 MiB
write) between timed steps, outside each step's events.  Timing: CUDA events
per step on the launching stream, barrier + synchronize around the K steps,
max over ranks.  Under torchrun each rank runs its own batch of independent
heads (weak scaling, no data-path collective); NCCL only carries the timing
reduction.

Printed (rank 0): one JSON line.  Besides the contract keys it carries the
roofline of the dominant kernel (timed live with CUDA events recorded by the
library around each launch), the CPU baseline (the fp64 oracle on a bounded
sample, host cores), the end-to-end number through the public API with host
buffers, the SM clocks sampled during the timed region, the decode-step
bandwidth on the 64 x 16-head decode workload, and the quadratic
(flash-attention-style) form timed on the same inputs beside a library causal
flash-attention forward of the same shape (context only).

--impl reference times the fp64 CPU oracle (the only other implementation of
this path) on a bounded sample per step, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "long_B1H8_T131072_d64_bf16"
DECODE_WORKLOAD = "recall_decode_B64H16_T32768_d64_bf16"
METRIC = "KATA chunked fwd tokens/s @T=131k,H=8,d=64 bf16; % tensor-pipe roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_TENSOR_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--chunk", type=int, default=64)
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU work budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the sub-measures beside the step (quadratic form, other workloads, sequence split)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override the workload's T (smaller cases of the same workload for profiling)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# Multi-rank plumbing (weak scaling over independent heads)
# ---------------------------------------------------------------------------


def rank_seed(base_seed, rank):
    """Each rank draws its own batch of independent heads."""
    return base_seed + 1000 * rank


def max_over_ranks(value, world, device="cuda"):
    """Max of a per-rank float over all ranks (the slowest rank sets the job
    time); identity for one rank.  Same collective on every rank."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_rank, ms_max):
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# Algorithmic work per unit (per token-head, canonical dense d^2 state form)
# ---------------------------------------------------------------------------


def alg_flops_per_token_head(kind, d, dv, C, g=1):
    """Canonical flops of the method's chunked-state form, per token and head:
    state build 2 d^2 dv + normaliser build 2 d^2; readout 2 d^2 dv + normaliser
    readout 2 d^2 + causal intra-chunk term (C + 1)(d + dv).  With g factors
    (KATA-Mg) the state has d^2 / g rows instead of d^2."""
    rows = d * d // g
    build = 2 * rows * dv + 2 * rows
    read = 2 * rows * dv + 2 * rows + (C + 1) * (d + dv)
    return {"build": build, "read": read, "forward": build + read}[kind]


def segment_length(d, C):
    """Tokens between the library's stored states (include/kata.h, argument C):
    C itself for C >= 512, else a fixed length per head size."""
    if C >= 512:
        return C
    return 1024 if d >= 64 else (512 if d >= 32 else 256)


def kernel_roofline_units(name, w, C, BH, T, n_seg, E_floats):
    """(bound, algorithmic units per launch, unit) for a kernel of the forward."""
    d = dv = w.d
    if "read" in name:
        return "tensor", BH * T * alg_flops_per_token_head("read", d, dv, C), "flop"
    if "build" in name:
        return "tensor", BH * T * alg_flops_per_token_head("build", d, dv, C), "flop"
    if "scan" in name:
        return "hbm", BH * n_seg * E_floats * 4 * 2, "byte"
    if "decode" in name:
        return "hbm", BH * (d * d * dv + d * d) * 4 * 2, "byte"
    if "expand" in name:
        return "hbm", BH * (d * d * dv + d * d) * 4 * 2, "byte"
    return "hbm", 0, "byte"


# The sources the tensor-core forward kernels (tc_read and the kernels launched
# beside it) are compiled from: a committed ncu record (profiles/traffic.json)
# holds only while these are unchanged.
TC_SOURCES = ("kata_internal.cuh", "sm100.cuh", "tc_forward.cu", "tc_layout.cuh", "tmap.cuh")


def source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kernelized_linear_attention_fwd_b200", "csrc")
    for fn in TC_SOURCES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if taken on the
    current kernel sources (profiles/traffic.json), else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        data = json.load(open(path))
        ent = data.get(kernel, {}).get(workload)
        if ent and ent.get("source_sha") == source_sha():
            return ent.get("bytes_per_launch")
    except Exception:
        return None
    return None


# ---------------------------------------------------------------------------
# Clocks during the timed region
# ---------------------------------------------------------------------------


def smi_device_id(props):
    """nvidia-smi's name for the GPU behind torch device properties `props`:
    its UUID ("GPU-..."), else its PCI bus id ("dddddddd:bb:dd.0")."""
    u = str(getattr(props, "uuid", "") or "")
    if u:
        return u if u.startswith("GPU-") else "GPU-" + u
    return "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, smi_id):
        # smi_id: the GPU as nvidia-smi names it (UUID or PCI bus id); nvidia-smi
        # ignores CUDA_VISIBLE_DEVICES, so torch's device index may name another GPU
        self.dev = smi_id
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "200"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.tmp.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample
# ---------------------------------------------------------------------------


def oracle_sample_rate(w, T, seconds, seed=0, threads=None):
    """Rows uniform in t (mean cost ~T/2 keys per row) of one head, timed with
    the oracle's own threads.  Returns (rows/s, rows, cores, seconds)."""
    import numpy as np

    from kernelized_linear_attention_fwd_b200 import inputs
    from oracle import oracle

    oracle.build()
    threads = threads or os.cpu_count() or 1
    g = np.random.default_rng(seed)
    qb, kb, vb = inputs.make_qkv(1, 1, T, w.d, w.d, w.dtype, seed=w.seed, qk=w.qk)
    q64, k64, v64 = (inputs.widen(x, w.dtype).reshape(1, T, -1) for x in (qb, kb, vb))
    # calibrate
    n0 = max(threads, 8)
    rows = g.integers(0, T, size=n0)
    t0 = time.perf_counter()
    oracle.forward_rows(q64, k64, v64, np.zeros(n0, np.int64), rows, nthreads=threads)
    dt0 = time.perf_counter() - t0
    n = int(max(threads, min(200000, n0 * seconds / max(dt0, 1e-6))))
    rows = g.integers(0, T, size=n)
    t0 = time.perf_counter()
    oracle.forward_rows(q64, k64, v64, np.zeros(n, np.int64), rows, nthreads=threads)
    dt = time.perf_counter() - t0
    return n / dt, n, threads, dt, (q64, k64, v64)


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------


def run_ours(args, rank, world):
    import torch
    import torch.distributed as dist

    import kernelized_linear_attention_fwd_b200 as K
    from kernelized_linear_attention_fwd_b200 import inputs
    from kernelized_linear_attention_fwd_b200.binding import load_library
    from kernelized_linear_attention_fwd_b200.csrc import build as kbuild

    if rank == 0 and not os.path.exists(os.path.join(ROOT, "kernelized_linear_attention_fwd_b200",
                                                     "libkata.so")):
        kbuild.build()
    if world > 1:
        dist.barrier()
    lib = load_library()
    import ctypes

    lib.kata_profile_enable.argtypes = [ctypes.c_int]
    lib.kata_profile_kernel_count.restype = ctypes.c_int
    lib.kata_profile_kernel.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_char_p),
                                        ctypes.POINTER(ctypes.c_int),
                                        ctypes.POINTER(ctypes.c_double)]

    def profile_read():
        n = lib.kata_profile_kernel_count()
        res = {}
        for i in range(max(n, 0)):
            nm, cnt, ms = ctypes.c_char_p(), ctypes.c_int(), ctypes.c_double()
            lib.kata_profile_kernel(i, ctypes.byref(nm), ctypes.byref(cnt), ctypes.byref(ms))
            res[nm.value.decode()] = (cnt.value, ms.value)
        return res

    dev = torch.cuda.current_device()
    w = inputs.WORKLOADS[args.workload]
    C = args.chunk
    B, H, T, d = w.B, w.H, (args.seq_len or w.T), w.d
    BH = B * H
    # each rank: its own batch of independent heads (seed offset by rank)
    qh, kh, vh = inputs.make_qkv(B, H, T, d, d, w.dtype, seed=rank_seed(w.seed, rank), qk=w.qk)
    q1h, k1h, v1h = inputs.make_qkv(B, H, 1, d, d, w.dtype, seed=rank_seed(w.seed, rank), qk=w.qk,
                                    tag=1)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def pinned(a):
        t = torch.from_numpy(a.view("int16") if w.dtype == "bf16" else a)
        t = t.view(torch.bfloat16) if w.dtype == "bf16" else t
        return t.pin_memory()

    hq, hk, hv = pinned(qh), pinned(kh), pinned(vh)
    hq1, hk1, hv1 = (pinned(x.reshape(B, H, d)) for x in (q1h, k1h, v1h))
    q, k, v = (x.cuda() for x in (hq, hk, hv))
    q1, k1, v1 = (x.cuda() for x in (hq1, hk1, hv1))
    out = torch.empty((B, H, T, d), dtype=tdt, device="cuda")
    out1 = torch.empty((B, H, d), dtype=tdt, device="cuda")
    state = torch.empty((B, H, d * d, d), dtype=torch.float32, device="cuda")
    zst = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
    code = 1 if w.dtype == "bf16" else 0
    ws_bytes = K.kata_chunked_forward_workspace_bytes(B, H, T, d, d, C, code)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        K.kata_chunked_forward(q, k, v, C=C, out=out, state_out=state, z_out=zst, workspace=ws,
                               stream=stream)
        K.kata_decode_step(q1, k1, v1, state, zst, out=out1, stream=stream)

    def flush():
        flush_buf.zero_()

    for _ in range(max(args.warmup, 3)):
        step()
        flush()
    torch.cuda.synchronize()
    if K.kata_get_device_status() != 0:
        raise RuntimeError("device status set during warm-up")

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(smi_device_id(torch.cuda.get_device_properties(dev)))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    lib.kata_profile_enable(1)
    for i in range(args.steps):
        flush()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    lib.kata_profile_enable(0)
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    prof = profile_read()
    ms_local = sum(step_ms) / len(step_ms)
    ms_max = max_over_ranks(ms_local, world)
    status = K.kata_get_device_status()

    # end-to-end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        hout = torch.empty((B, H, T, d), dtype=tdt).pin_memory()
        hout1 = torch.empty((B, H, d), dtype=tdt).pin_memory()
        dq1, dk1, dv1 = (torch.empty_like(x) for x in (q1, k1, v1))
        # the public host-buffer call: heads in groups, each group's copy in and
        # copy out overlapped with another group's compute
        group = max(1, BH // 8)
        hbuf = torch.empty(K.kata_chunked_forward_host_buffer_bytes(B, H, T, d, d, C, code, group),
                           dtype=torch.uint8, device="cuda")

        def e2e_step():
            K.kata_chunked_forward_host(hq, hk, hv, hout, C=C, state_out=state, z_out=zst,
                                        device_buffer=hbuf, heads_per_group=group, stream=stream)
            for dst, src in ((dq1, hq1), (dk1, hk1), (dv1, hv1)):
                dst.copy_(src, non_blocking=True)
            K.kata_decode_step(dq1, dk1, dv1, state, zst, out=out1, stream=stream)
            hout1.copy_(out1, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        eve = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        for i in range(args.steps):
            flush()
            eve[i][0].record(stream)
            e2e_step()
            eve[i][1].record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in eve) / args.steps, world)
        es = 2 if w.dtype == "bf16" else 4
        h2d = 3 * BH * T * d * es + 3 * BH * d * es
        d2h = BH * T * d * es + BH * d * es
        e2e = {"value": job_throughput(world, B * T, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "api": f"kata_chunked_forward_host ({BH // group} groups of {group} heads, "
                      "copies overlapped with compute) + kata_decode_step",
               "pcie_gbs_h2d": h2d / (e2e_ms / 1e3) / 1e9}

    # decode bandwidth on the 64 x 16-head decode workload
    decode = None
    if not args.no_decode:
        wd = inputs.WORKLOADS[DECODE_WORKLOAD]
        Bd, Hd = wd.B, wd.H
        g = torch.Generator(device="cuda")
        g.manual_seed(1234 + rank)
        Sd = torch.randn((Bd, Hd, d * d, d), generator=g, device="cuda", dtype=torch.float32)
        Sd = 0.5 * (Sd + Sd.view(Bd, Hd, d, d, d).transpose(2, 3).reshape(Bd, Hd, d * d, d))
        Zd = torch.randn((Bd, Hd, d, d), generator=g, device="cuda", dtype=torch.float32)
        Zd = Zd @ Zd.transpose(-1, -2)
        qd_, kd_, vd_ = (torch.randn((Bd, Hd, d), generator=g, device="cuda").to(tdt)
                         for _ in range(3))
        od = torch.empty((Bd, Hd, d), dtype=tdt, device="cuda")
        nd = max(10, args.steps)
        for _ in range(5):
            K.kata_decode_step(qd_, kd_, vd_, Sd, Zd, out=od, stream=stream)
        torch.cuda.synchronize()
        evd = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(nd)]
        for i in range(nd):
            evd[i][0].record(stream)
            K.kata_decode_step(qd_, kd_, vd_, Sd, Zd, out=od, stream=stream)
            evd[i][1].record(stream)
        torch.cuda.synchronize()
        dms = sorted(a.elapsed_time(b) for a, b in evd)
        dmean = max_over_ranks(sum(dms) / nd, world)
        es = 2 if w.dtype == "bf16" else 4
        dbytes = Bd * Hd * ((d * d * d + d * d) * 4 * 2 + 4 * d * es)
        peaks, src = load_peaks()
        gbs = dbytes / (dmean / 1e3) / 1e9
        decode = {"workload": DECODE_WORKLOAD, "ms_per_step": dmean,
                  "tokens_per_s": world * Bd / (dmean / 1e3), "bytes_per_step": dbytes,
                  "achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
                  "frac": gbs / peaks["hbm_gbs"], "frac_of_8tbs_spec": gbs / SPEC_HBM_GBS,
                  "peak_source": src}
        # the same steps on the packed layout (rows i <= j: half the bytes)
        Sp, Zp = K.kata_state_pack(Sd, Zd, stream=stream)
        del Sd, Zd
        pms = max_over_ranks(time_launches(
            lambda: K.kata_decode_step_packed(qd_, kd_, vd_, Sp, Zp, out=od, stream=stream),
            stream, lambda: None, nd, warm=5), world)
        R = d * (d + 1) // 2
        pbytes = Bd * Hd * ((R * d + R) * 4 * 2 + 4 * d * es)
        pgbs = pbytes / (pms / 1e3) / 1e9
        decode["packed"] = {"ms_per_step": pms, "tokens_per_s": world * Bd / (pms / 1e3),
                            "bytes_per_step": pbytes, "achieved_gbs": pgbs,
                            "frac": pgbs / peaks["hbm_gbs"], "speedup_vs_dense": dmean / pms}
        del Sp, Zp

    # the quadratic (flash-attention-style) form of the same forward
    quad = None
    if not args.no_extras:
        quad = measure_quadratic(K, q, k, v, out, stream, flush, world, rank, ms_max, n=3)
        if K.kata_get_device_status() != 0:
            raise RuntimeError("device status set by the quadratic form")

    # the chunked forward on the other forward workloads
    others = None
    if not args.no_extras and w.name == WORKLOAD:
        others = measure_other_configs(K, inputs, stream, flush)

    # one rank's compute of the sequence-sharded forward, on this GPU
    def kernel_times(fn, n):  # per-kernel device ms per call, from the library's events
        lib.kata_profile_enable(1)
        for _ in range(n):
            flush()
            fn()
        torch.cuda.synchronize()
        lib.kata_profile_enable(0)
        return {name: round(t / n, 4) for name, (c, t) in profile_read().items()}

    seq_split = None
    if not args.no_extras and w.dtype == "bf16":
        fwd_ms = sum(t for n, (c, t) in prof.items() if "decode" not in n) / args.steps
        seq_split = measure_sequence_split(K, q, k, v, C, stream, flush, fwd_ms, kernel_times)

    # KATA-Mg with two factors on the same inputs
    mg = None
    if not args.no_extras and w.dtype == "bf16" and d == 64:
        m1_ms = sum(t for n, (c, t) in prof.items() if "decode" not in n) / args.steps
        mg = measure_mg(K, q, k, v, C, stream, flush, kernel_times, m1_ms)
        if K.kata_get_device_status() != 0:
            raise RuntimeError("device status set by the two-factor forward")

    # chunk size x sequence length sweep of the long-context workload
    sweep = None
    if not args.no_extras and w.name == WORKLOAD:
        sweep = measure_chunk_sweep(K, inputs, stream, flush, kernel_times)

    if rank != 0:
        return None

    # roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    R = d * (d + 1) // 2
    E = R * (d + 1)
    L = segment_length(d, C)
    n_seg = (T + L - 1) // L
    fwd_kernels = {n: v for n, v in prof.items() if "decode" not in n}
    dom = max(fwd_kernels, key=lambda n: fwd_kernels[n][1])
    cnt, tot = fwd_kernels[dom]
    bound, units, unit = kernel_roofline_units(dom, w, C, BH, T, n_seg, E)
    per_launch_s = tot / cnt / 1e3
    if bound == "tensor":
        ach = units / per_launch_s / 1e12
        peak = peaks["bf16_tflops"]
        runit = "TFLOP/s"
    else:
        ach = units / per_launch_s / 1e9
        peak = peaks["hbm_gbs"]
        runit = "GB/s"
    roofline = {"bound": bound, "achieved": ach, "peak": peak, "unit": runit, "frac": ach / peak,
                "traffic": load_traffic(dom, args.workload), "kernel": dom,
                "kernel_ms": tot / cnt, "peak_source": f"{peak_src} (burst)",
                "algorithmic_units_per_launch": units, "algorithmic_unit": unit}
    total_launches = sum(c for c, _ in prof.values())

    cpu = None
    if not args.no_cpu_baseline:
        rate, n, cores, secs, _ = oracle_sample_rate(w, T, args.cpu_seconds)
        cpu = {"value": rate / H, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} output rows of one head, t uniform in [0, {T}) (mean {T // 2} "
                         f"keys each), {secs:.1f} s; tokens/s = rows/s / H"}

    tokens = world * B * T
    canon_tflops = BH * T * alg_flops_per_token_head("forward", d, d, C) / (ms_max / 1e3) / 1e12
    canon = {"flop_per_token_head": alg_flops_per_token_head("forward", d, d, C),
             "achieved_tflops_per_gpu": canon_tflops,
             "frac_of_measured_peak": canon_tflops / peaks["bf16_tflops"],
             "frac_of_2250_spec": canon_tflops / SPEC_TENSOR_TFLOPS,
             "note": "whole step (all kernels), canonical dense d^2 flops of the chunked form"}
    line = {
        "metric": METRIC,
        "value": job_throughput(world, B * T, ms_max),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded unit-norm q, k; N(0,1) v)",
        "config": {"workload": args.workload, "B": B, "H": H, "T": T, "d": d, "C": C,
                   "global_batch": world * B, "seq_len": T,
                   "parallelism": f"independent heads per rank x{world}",
                   "step": "chunked forward + state export + 1 decode step",
                   "l2": "flushed between steps (256 MiB write, outside step events)"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": total_launches,
        "gpu_launches_per_step": total_launches / args.steps,
        "kernels_ms_per_step": {n: t / args.steps for n, (c, t) in prof.items()},
        "clocks": clk,
        "decode": decode,
        "quadratic_form": quad,
        "sequence_split": seq_split,
        "other_workloads": others,
        "chunk_sweep": sweep,
        "mg_two_factors": mg,
        "device_status": status,
        "forward_canonical": canon,
    }
    return line


def quadratic_flops(BH, T, d, dv):
    """Algorithmic flops of the causal quadratic form: 2 d (score) + 2 dv
    (weighted values) per (query, key) pair with key <= query."""
    return BH * T * (T + 1) // 2 * 2 * (d + dv)


def time_launches(fn, stream, flush, n, warm=2):
    """Mean device ms of fn() over n launches (CUDA events on `stream`, L2
    flushed before each, outside the events)."""
    import torch

    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    for a, b in ev:
        flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / n


def library_flash_attention(q, k, v, stream, flush, n):
    """Context only: a library causal flash-attention forward (softmax
    attention) of the same shape on this GPU, the pages' point of comparison.
    FlashAttention-2 (flash_attn) if it runs here, else torch's SDPA with its
    flash backend.  Returns (backend, mean ms) or (None, reason)."""
    import torch

    errs = []
    try:
        from flash_attn import flash_attn_func

        qt, kt, vt = (x.transpose(1, 2).contiguous() for x in (q, k, v))  # [B, T, H, d]
        ms = time_launches(lambda: flash_attn_func(qt, kt, vt, causal=True), stream, flush, n)
        del qt, kt, vt
        return "flash_attn " + __import__("flash_attn").__version__, ms
    except Exception as e:  # not built for this GPU, or not installed
        errs.append(f"flash_attn: {type(e).__name__}: {str(e)[:120]}")
    try:
        from torch.nn.attention import SDPBackend, sdpa_kernel
        from torch.nn.functional import scaled_dot_product_attention as sdpa

        def run():
            with sdpa_kernel(SDPBackend.FLASH_ATTENTION):
                sdpa(q, k, v, is_causal=True)

        return "torch sdpa (flash backend)", time_launches(run, stream, flush, n)
    except Exception as e:
        errs.append(f"torch sdpa: {type(e).__name__}: {str(e)[:120]}")
    return None, "; ".join(errs)


def measure_quadratic(K, q, k, v, out, stream, flush, world, rank, chunked_ms, n):
    """The quadratic (flash-attention-style) form on the step's own inputs."""
    B, H, T, d = q.shape
    BH = B * H
    ms = max_over_ranks(time_launches(lambda: K.kata_quadratic_forward(q, k, v, out=out,
                                                                       stream=stream),
                                      stream, flush, n), world)
    peaks, src = load_peaks()
    fl = quadratic_flops(BH, T, d, d)
    tf = fl / (ms / 1e3) / 1e12
    res = {"ms": ms, "tokens_per_s": world * B * T / (ms / 1e3),
           "flop_per_launch": fl, "achieved_tflops": tf, "peak_tflops": peaks["bf16_tflops"],
           "frac": tf / peaks["bf16_tflops"], "peak_source": f"{src} (burst)",
           "flop_note": "causal pairs x 2(d + dv); masked halves of diagonal blocks not counted"}
    if rank == 0:
        backend, fa = library_flash_attention(q, k, v, stream, flush, n)
        if backend is None:
            res["library_flash_attention"] = {"unavailable": fa}
        else:
            res["library_flash_attention"] = {
                "backend": backend, "ms": fa, "achieved_tflops": fl / (fa / 1e3) / 1e12,
                "quadratic_speedup": fa / ms, "chunked_step_speedup": fa / chunked_ms,
                "note": "context only: softmax attention of the same B, H, T, d, causal"}
    return res


def measure_sequence_split(K, q, k, v, C, stream, flush, chunked_ms, kernel_times,
                           splits=(2, 8)):
    """Per-rank compute of the sequence-sharded forward, on this one GPU: the
    block of one of N ranks (T / N tokens of every head) through
    kata_chunked_state and kata_chunked_forward_from_state with N - 1 gathered
    totals as inputs (the last rank's work).  The all-gather itself is not
    run (it needs N GPUs)."""
    import torch

    from kernelized_linear_attention_fwd_b200 import sharded

    B, H, T, d = q.shape
    res = {}
    for N in splits:
        if T % N:
            continue
        Tb = T // N
        bq, bk, bv = (x[:, :, :Tb].contiguous() for x in (q, k, v))
        flat = sharded.block_state(bk, bv, C)
        gathered = flat.repeat(N, 1)  # stands in for the N gathered totals
        out = torch.empty_like(bq)
        ws = torch.empty(max(K.kata_chunked_forward_workspace_bytes(B, H, Tb, d, d, C, 1), 256),
                         dtype=torch.uint8, device=q.device)
        ns, nz = sharded.state_numel(B, H, d, d)
        S = flat[:ns].view(B, H, d * d, d)
        Z = flat[ns:].view(B, H, d, d)
        s_in, z_in = sharded.gathered_views(gathered, N - 1, B, H, d, d)

        def rank_work():  # on the current stream (the capture stream while capturing)
            K.kata_chunked_state(bk, bv, C=C, state_out=S, z_out=Z, workspace=ws)
            K.kata_chunked_forward_from_state(bq, bk, bv, s_in, z_in, C=C, out=out, workspace=ws,
                                              reuse_segment_states=True)

        eager = time_launches(rank_work, stream, flush, 5)
        # the same calls replayed from a CUDA graph: at a few hundred microseconds of
        # GPU work per rank the host cannot issue them as fast as the GPU runs them
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                rank_work()
            ms = time_launches(graph.replay, stream, flush, 10)
            del graph
        except Exception as e:  # report the eager time only
            ms, res[f"N{N}_graph_error"] = None, f"{type(e).__name__}: {str(e)[:100]}"
        best = ms if ms is not None else eager
        res[f"N{N}"] = {"tokens_per_rank": B * Tb, "per_rank_ms": ms, "per_rank_ms_eager": eager,
                        "ideal_ms": chunked_ms / N, "compute_efficiency": chunked_ms / N / best,
                        "projected_tokens_per_s": B * T / (best / 1e3),
                        "kernels_ms": kernel_times(rank_work, 3)}
        del bq, bk, bv, flat, gathered, out, ws
    res["note"] = ("one GPU: one rank's compute (state pass + forward from N-1 gathered totals "
                   "reusing the state pass's segment states, replayed from a CUDA graph) against the single-GPU forward's kernel time / N; "
                   "the all-gather of the totals (1 MiB + 16 KiB per head) is not included")
    return res


def measure_other_configs(K, inputs, stream, flush, names=("lm340m_B4H16_T16384_d64_bf16",
                                                            "small_B2H4_T4096_d32_bf16")):
    """The chunked forward (with state export) on the other forward workloads,
    inputs generated on the device, L2 flushed before each launch."""
    import torch

    peaks, _ = load_peaks()
    res = {}
    for name in names:
        w = inputs.WORKLOADS[name]
        q, k, v = inputs.make_qkv_device(w.B, w.H, w.T, w.d, w.d, seed=w.seed)
        so = torch.empty((w.B, w.H, w.d * w.d, w.d), dtype=torch.float32, device=q.device)
        zo = torch.empty((w.B, w.H, w.d, w.d), dtype=torch.float32, device=q.device)
        out = torch.empty_like(v)
        ws = torch.empty(max(K.kata_chunked_forward_workspace_bytes(w.B, w.H, w.T, w.d, w.d, w.C,
                                                                    1), 256),
                         dtype=torch.uint8, device=q.device)
        ms = time_launches(lambda: K.kata_chunked_forward(q, k, v, C=w.C, out=out, state_out=so,
                                                          z_out=zo, workspace=ws),
                           stream, flush, 10, warm=3)
        canon = w.B * w.H * w.T * alg_flops_per_token_head("forward", w.d, w.d, w.C)
        res[name] = {"ms": ms, "tokens_per_s": w.B * w.T / (ms / 1e3),
                     "canonical_tflops": canon / (ms / 1e3) / 1e12,
                     "frac_of_measured_peak": canon / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                     "path": ("fp32 CUDA cores" if w.dtype != "bf16" else "tensor cores" if w.d == 64
                              else f"tensor cores, heads of d = {w.d} read as 64 (zero-filled by TMA), two-factor layout")}
        del q, k, v, so, zo, out, ws
    return res


def measure_mg(K, q, k, v, C, stream, flush, kernel_times, m1_ms, g=2):
    """The KATA-Mg forward (g factors, state exported) on the step's own
    inputs, beside the single-factor forward: ms, tokens/s, canonical flops of
    the g-factor form against the measured peak, per-kernel times."""
    import torch

    peaks, _ = load_peaks()
    B, H, T, d = q.shape
    so = torch.empty((B, H, d * d, d), dtype=torch.float32, device=q.device)
    zo = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    out = torch.empty_like(v)
    ws = torch.empty(max(K.kata_mg_chunked_forward_workspace_bytes(B, H, T, d, d, C, g, 1), 256),
                     dtype=torch.uint8, device=q.device)

    def fwd():
        K.kata_mg_chunked_forward(q, k, v, g=g, C=C, out=out, state_out=so, z_out=zo,
                                  workspace=ws, stream=stream)

    ms = time_launches(fwd, stream, flush, 5, warm=2)
    canon = B * H * T * alg_flops_per_token_head("forward", d, d, C, g)
    res = {"g": g, "ms": ms, "tokens_per_s": B * T / (ms / 1e3),
           "canonical_flop_per_token_head": alg_flops_per_token_head("forward", d, d, C, g),
           "canonical_tflops": canon / (ms / 1e3) / 1e12,
           "frac_of_measured_peak": canon / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
           "speedup_vs_one_factor_forward": m1_ms / ms,
           "kernels_ms": kernel_times(fwd, 3)}
    del so, zo, out, ws
    return res


def measure_chunk_sweep(K, inputs, stream, flush, kernel_times, d=64,
                        Ts=(8192, 32768, 131072), Cs=(64, 128, 256, 512, 1024, 2048), H=8):
    """The chunked forward (with state export) of the long-context workload over
    sequence lengths T and chunk sizes C.  C <= 256 runs one schedule (states
    every 1024 tokens at d = 64), C >= 512 keeps a state every C tokens: the
    sweep over C >= 512 is the sweep of the segment length L, which trades
    state traffic and scan passes against intra-segment work.  Inputs drawn on
    the device, L2 flushed before each launch.  frac: canonical flops of the
    chunked form at that C against the measured peak."""
    import torch

    peaks, _ = load_peaks()
    res = {}
    for T in Ts:
        q, k, v = inputs.make_qkv_device(1, H, T, d, d, seed=0)
        so = torch.empty((1, H, d * d, d), dtype=torch.float32, device=q.device)
        zo = torch.empty((1, H, d, d), dtype=torch.float32, device=q.device)
        out = torch.empty_like(v)
        for C in Cs:
            ws = torch.empty(max(K.kata_chunked_forward_workspace_bytes(1, H, T, d, d, C, 1), 256),
                             dtype=torch.uint8, device=q.device)

            def fwd():
                K.kata_chunked_forward(q, k, v, C=C, out=out, state_out=so, z_out=zo,
                                       workspace=ws, stream=stream)

            ms = time_launches(fwd, stream, flush, 5, warm=2)
            canon = H * T * alg_flops_per_token_head("forward", d, d, C)
            L = segment_length(d, C)
            res[f"T{T}_C{C}"] = {
                "T": T, "C": C, "segment_L": L, "n_seg": (T + L - 1) // L, "ms": ms,
                "tokens_per_s": T / (ms / 1e3),
                "canonical_tflops": canon / (ms / 1e3) / 1e12,
                "frac_of_measured_peak": canon / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                "kernels_ms": kernel_times(fwd, 3)}
            del ws
        del q, k, v, so, zo, out
    return res


# ---------------------------------------------------------------------------
# Reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------


def run_reference(args):
    from kernelized_linear_attention_fwd_b200 import inputs

    w = inputs.WORKLOADS[args.workload]
    n_steps = args.steps + max(args.warmup, 3)
    per_step = max(0.5, min(3.0, 150.0 / n_steps))
    rate, n, cores, secs, arrays = oracle_sample_rate(w, w.T, per_step)
    import numpy as np

    from oracle import oracle

    q64, k64, v64 = arrays
    g = np.random.default_rng(1)
    times = []
    for i in range(n_steps):
        rows = g.integers(0, w.T, size=n)
        t0 = time.perf_counter()
        oracle.forward_rows(q64, k64, v64, np.zeros(n, np.int64), rows, nthreads=cores)
        dt = time.perf_counter() - t0
        if i >= max(args.warmup, 3):
            times.append(dt)
    mean_s = sum(times) / len(times)
    value = n / mean_s / w.H
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": mean_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded unit-norm q, k; N(0,1) v)",
        "config": {"workload": args.workload, "B": w.B, "H": w.H, "T": w.T, "d": w.d,
                   "C": args.chunk, "global_batch": w.B, "seq_len": w.T},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {n} output rows of one head, t uniform in "
                                   f"[0, {w.T}); tokens/s = rows/s / H"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    import torch

    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    line = run_ours(args, rank, world)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
