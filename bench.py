"""Benchmark of the gated delta-rule hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one chunk-parallel forward (gdr_chunk_fwd) over the training-shape
workload bf16_b8_h16_t4096_d128 (B=8, H=16, T=4096, dk=dv=128, chunk 64,
post-write read, zero initial state), inputs resident in HBM.  The same run also
times the batched decode step (gdr_decode_step, 256 sequences x 32 v-heads,
128x128 fp32 state, 64 steps with fresh inputs) and reports its HBM bandwidth.

Prints ONE JSON line on rank 0.  Under torchrun (N > 1) every rank runs the same
workload on its own GPU with its own seed (weak scaling, no collective on the data
path); the step time is the max over ranks.

Inputs (q, k, v, o: 537 MB; decode state: 537 MB) are larger than the 126 MB L2,
so no flush is done between timed iterations.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated-delta chunk-fwd tokens/s + %bf16 TC peak; decode state GB/s vs HBM peak"
CHUNK_WORKLOAD = "bf16_b8_h16_t4096_d128"
DECODE_WORKLOAD = "bf16_decode_n256_hk16_hv32_d128"
BIDIR_WORKLOAD = "bf16_bidir_16x2048_h12_d64"
VARLEN_WORKLOAD = "bf16_varlen64_h16_d128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


CHUNK_TC_SOURCES = ("chunk_tc.cu", "chunk_tc.cuh", "wy_solve.cuh", "tc_ptx.cuh", "common.cuh")
G2_TC_SOURCES = ("chunk_g2_tc.cu", "wy_solve.cuh", "tc_ptx.cuh", "common.cuh")
BWD_TC_SOURCES = ("chunk_bwd_tc.cu", "chunk_bwd.cuh", "wy_solve.cuh", "tc_ptx.cuh", "common.cuh")
BWD_SOURCES = ("chunk_bwd.cu", "chunk_bwd.cuh", "common.cuh")
# the kernels of one tensor-core backward call, with the sources of their traffic records (the
# head reduction only where several v-heads share a key head)
BWD_TC_KERNELS = (("chunk_fused_tc_save", CHUNK_TC_SOURCES), ("chunk_fused_tc_adj", CHUNK_TC_SOURCES),
                  ("bwd_chunk_dqk_tc", BWD_TC_SOURCES), ("bwd_chunk_wy_tc", BWD_TC_SOURCES),
                  ("bwd_reduce_heads4", BWD_SOURCES))
DECODE_SOURCES = ("decode.cu", "common.cuh")


def source_digest(sources) -> str:
    """First 16 hex digits of the SHA-256 of the concatenated kernel sources (the .cu file
    and the headers it includes), the revision key of a traffic record."""
    import hashlib
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "gated_delta_rule_146_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, sources, units: float):
    """Memory traffic per launch of `kernel` from the committed ncu summary
    (profiles/traffic.json): DRAM bytes read plus the bytes the SMs wrote into L2 (each write
    counted once where it enters L2; dram__bytes_write misses the lines still dirty in L2
    when the kernel ends), scaled from the captured case to `units` (rows or sequences; 1
    for a capture of the full workload); None when a kernel source has changed since the
    counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    try:
        digest = source_digest(sources)
    except OSError:
        return None
    if not rec or digest != rec["source_sha256_16"]:
        return None
    captured = rec.get("rows_captured") or rec.get("seqs_captured") or rec.get("calls_captured")
    return (rec["dram_read_bytes"] + rec["write_bytes_into_l2"]) * units / captured


def device_status(a, ws) -> str:
    """The device-side status a call left in its workspace (read after the timed region; it
    synchronises): "ok", or the status name (e.g. an fp16 operand out of range)."""
    import gated_delta_rule_146_b200 as gdr
    st = gdr.read_device_error(a, ws)
    return "ok" if st == 0 else gdr._abi.status_string(st)


def flops_per_head_token(C, dk, dv):
    """Dense chunk-form FLOPs per token per head: KK^T, QK^T, W (2C dk each), U and the
    intra output (2C dv each), W H, the state update and Q H (2 dk dv each)."""
    return 6 * C * dk + 4 * C * dv + 6 * dk * dv


# ------------------------------------------------------------------ clocks sampler

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------ replica bookkeeping

def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank float over all ranks (the step time of the slowest replica)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms_per_step: float) -> float:
    """Units per second over all replicas: every rank does the same work per step (weak
    scaling) and the step takes as long as the slowest rank."""
    return world * units_per_rank / (ms_per_step / 1e3)


# ------------------------------------------------------------------ our implementation

def bench_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import gated_delta_rule_146_b200 as gdr
    import workloads

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()

    def barrier():
        if world > 1:
            dist.barrier()

    # ---------------- chunk-parallel forward
    w = workloads.WORKLOADS[args.workload]
    if args.rows:  # a smaller case of the same kernel (profiling): fewer rows of the workload
        import dataclasses
        w = dataclasses.replace(w, B=args.rows, name=f"{w.name}[rows={args.rows}]")
    x = workloads.workload_inputs(w, seed=rank)
    d = {n: (t.to(dev) if t is not None else None) for n, t in x.items()}
    cargs = gdr.make_chunk_args(d["q"], d["v"], d["g"], d["cu_seqlens"], w.chunk, w.read_mode,
                                w.scale)
    path = gdr.chunk_fwd_path(cargs)
    ws = torch.empty(gdr.chunk_fwd_workspace_size(cargs), dtype=torch.uint8, device=dev)
    o = torch.empty_like(d["v"])
    S_final = torch.empty((cargs.n_seqs, w.Hv, w.dk, w.dv), dtype=torch.float32, device=dev)

    def step():
        gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["cu_seqlens"],
                      chunk=w.chunk, read_mode=w.read_mode, scale=w.scale, o=o, S_final=S_final,
                      workspace=ws)

    if args.only == "decode":
        args.steps = max(1, min(args.steps, 1))
    for _ in range(args.warmup if args.only != "decode" else 0):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)  # let the sampler come up before the timed region
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, world)
    statuses = {"chunk": device_status(cargs, ws)}

    tokens = int(d["q"].shape[0] * d["q"].shape[1])
    head_tokens = tokens * w.Hv
    flops = head_tokens * flops_per_head_token(w.chunk, w.dk, w.dv)
    algo_bytes = sum(t.numel() * t.element_size() for t in
                     (d["q"], d["k"], d["v"], d["g"], d["beta"], o, S_final)) + (
        d["S0"].numel() * 4 if d["S0"] is not None else 0)
    value = whole_job_rate(tokens, world, ms)
    tflops = flops / (ms / 1e3) / 1e12
    hbm_gbs = algo_bytes / (ms / 1e3) / 1e9
    launches_per_call = 2 if path == "tc" else 3

    # ---------------- same forward through the fused gating prologue (raw a, b projections)
    gating = None
    if not args.no_gating and args.only != "decode":
        a_raw, b_raw, A_h, dt_h = (t.to(dev) for t in workloads.raw_gate_inputs(
            tuple(d["g"].shape), w.Hv, w.gate_dtype, seed=rank))

        def gstep():
            gdr.chunk_fwd(d["q"], d["k"], d["v"], a_raw, b_raw, d["S0"], d["cu_seqlens"],
                          chunk=w.chunk, read_mode=w.read_mode, scale=w.scale, o=o,
                          S_final=S_final, workspace=ws, gate_A=A_h, gate_dt_bias=dt_h)

        for _ in range(args.warmup):
            gstep()
        torch.cuda.synchronize()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            gstep()
        g1.record(stream)
        torch.cuda.synchronize()
        barrier()
        gms = max_over_ranks(g0.elapsed_time(g1) / args.steps, world)
        statuses["gating_prologue"] = device_status(cargs, ws)
        gating = {"ms_per_step": gms, "value": whole_job_rate(tokens, world, gms),
                  "unit": "tokens/s", "overhead_vs_given_gates": gms / ms - 1.0,
                  "inputs": "raw a ~ N(-2,1), b ~ N(0,1) with A = -1, dt_bias = 0 "
                            "(same gate distributions as the workload)"}

    # ---------------- bidirectional workload: both directions summed in one call
    # (gdr_chunk_fwd_bidir: one grid, the two scans of a (sequence, head) as a cluster pair)
    bidir = None
    if not args.no_bidir and args.only != "decode" and not args.rows:
        bw = workloads.WORKLOADS[BIDIR_WORKLOAD]
        bx = workloads.workload_inputs(bw, seed=rank)
        bd = {n: (t.to(dev) if t is not None else None) for n, t in bx.items()}
        bo = torch.empty_like(bd["v"])
        bargs = gdr.make_chunk_args(bd["q"], bd["v"], bd["g"], bd["cu_seqlens"], bw.chunk,
                                    bw.read_mode, bw.scale)
        bws = torch.empty(gdr.chunk_fwd_bidir_workspace_size(bargs), dtype=torch.uint8,
                          device=dev)

        def bstep():
            gdr.chunk_fwd_bidir(bd["q"], bd["k"], bd["v"], bd["g"], bd["beta"], bd["g_bwd"],
                                bd["beta_bwd"], bd["cu_seqlens"], chunk=bw.chunk,
                                read_mode=bw.read_mode, scale=bw.scale, o=bo, workspace=bws)

        for _ in range(args.warmup):
            bstep()
        torch.cuda.synchronize()
        barrier()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(args.steps):
            bstep()
        b1.record(stream)
        torch.cuda.synchronize()
        barrier()
        bms = max_over_ranks(b0.elapsed_time(b1) / args.steps, world)
        statuses["bidirectional"] = device_status(bargs, bws)
        btok = int(bd["q"].shape[1])
        # the least HBM traffic of the call: q, k, v and both directions' gates read once,
        # o written once (the fp32 hand-off between the two scans of a pair is not counted)
        bbytes = sum(bd[n].numel() * bd[n].element_size() for n in ("q", "k", "v")) + sum(
            bd[n].numel() * bd[n].element_size() for n in ("g", "beta", "g_bwd", "beta_bwd")) + (
            bo.numel() * bo.element_size())
        btraffic = measured_traffic("chunk_fused_tc_pair", CHUNK_TC_SOURCES, 1)
        bidir = {"workload": bw.name, "ms_per_step": bms, "value": whole_job_rate(btok, world, bms),
                 "traffic": btraffic,
                 "unit": "tokens/s", "path": gdr.chunk_fwd_path(bargs),
                 "call": "gdr_chunk_fwd_bidir: one grid, forward and reverse scan of a "
                         "(sequence, head) as a 2-CTA cluster, fp32 sum rounded once",
                 "algorithmic_bytes": bbytes,
                 "hbm_frac": bbytes / (bms / 1e3) / 1e9 / peaks["hbm_gbs"]}

    # ---------------- varlen workload: 64 sequences of 256-8192 tokens packed in one row,
    # per-sequence initial state, S_final per sequence
    varlen = None
    if not args.no_varlen and args.only != "decode" and not args.rows:
        vw = workloads.WORKLOADS[VARLEN_WORKLOAD]
        vx = workloads.workload_inputs(vw, seed=rank)
        vd = {n: (t.to(dev) if t is not None else None) for n, t in vx.items()}
        vo = torch.empty_like(vd["v"])
        vargs = gdr.make_chunk_args(vd["q"], vd["v"], vd["g"], vd["cu_seqlens"], vw.chunk,
                                    vw.read_mode, vw.scale)
        vS = torch.empty((vargs.n_seqs, vw.Hv, vw.dk, vw.dv), dtype=torch.float32, device=dev)
        vws = torch.empty(gdr.chunk_fwd_workspace_size(vargs), dtype=torch.uint8, device=dev)

        def vstep():
            gdr.chunk_fwd(vd["q"], vd["k"], vd["v"], vd["g"], vd["beta"], vd["S0"],
                          vd["cu_seqlens"], chunk=vw.chunk, read_mode=vw.read_mode,
                          scale=vw.scale, o=vo, S_final=vS, workspace=vws)

        for _ in range(args.warmup):
            vstep()
        torch.cuda.synchronize()
        barrier()
        v0, v1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        v0.record(stream)
        vsteps = max(1, min(args.steps, 20))
        for _ in range(vsteps):
            vstep()
        v1.record(stream)
        torch.cuda.synchronize()
        barrier()
        vms = max_over_ranks(v0.elapsed_time(v1) / vsteps, world)
        statuses["varlen"] = device_status(vargs, vws)
        vtok = int(vd["q"].shape[1])
        vbytes = sum(t.numel() * t.element_size() for t in
                     (vd["q"], vd["k"], vd["v"], vd["g"], vd["beta"], vo, vd["S0"], vS))
        vgbs = vbytes / (vms / 1e3) / 1e9
        vflops = vtok * vw.Hv * flops_per_head_token(vw.chunk, vw.dk, vw.dv)
        varlen = {"workload": vw.name, "tokens": vtok, "sequences": vargs.n_seqs,
                  "ms_per_step": vms, "steps": vsteps,
                  "value": whole_job_rate(vtok, world, vms), "unit": "tokens/s",
                  "path": gdr.chunk_fwd_path(vargs),
                  "tflops": vflops / (vms / 1e3) / 1e12,
                  "roofline": {"bound": "hbm", "achieved": vgbs, "peak": peaks["hbm_gbs"],
                               "unit": "GB/s", "frac": vgbs / peaks["hbm_gbs"],
                               "algorithmic_bytes": vbytes,
                               "floor_ms": vbytes / (peaks["hbm_gbs"] * 1e9) * 1e3}}
        del vws, vo, vS, vd

    # ---------------- decode step
    dec = None
    if not args.no_decode and args.only != "chunk":
        dw = workloads.DECODE_WORKLOADS[DECODE_WORKLOAD]
        if args.decode_seqs:
            import dataclasses
            dw = dataclasses.replace(dw, N=args.decode_seqs,
                                     name=f"{dw.name}[seqs={args.decode_seqs}]")
        dx = workloads.decode_workload_inputs(dw, seed=rank)
        dd = {n: t.to(dev) for n, t in dx.items()}
        od = torch.empty((dw.N, dw.Hv, dw.dv), dtype=torch.bfloat16, device=dev)

        def dstep(t):
            gdr.decode_step(dd["q"][t], dd["k"][t], dd["v"][t], dd["g"][t], dd["beta"][t],
                            dd["S"], read_mode=dw.read_mode, scale=dw.scale, o=od)

        for t in range(min(args.warmup, dw.steps)):
            dstep(t)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for t in range(dw.steps):
            dstep(t)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        dms = max_over_ranks(e0.elapsed_time(e1) / dw.steps, world)
        dbytes = 2 * dd["S"].numel() * 4 + sum(
            dd[n][0].numel() * dd[n].element_size() for n in ("q", "k", "v", "g", "beta")) + (
            od.numel() * od.element_size())
        dgbs = dbytes / (dms / 1e3) / 1e9
        dec = {"workload": dw.name, "ms_per_step": dms, "bytes_per_step": dbytes,
               "value": world * dgbs, "unit": "GB/s",
               "roofline": {"bound": "hbm", "achieved": dgbs, "peak": peaks["hbm_gbs"],
                            "unit": "GB/s", "frac": dgbs / peaks["hbm_gbs"],
                            "traffic": measured_traffic("decode_kernel", DECODE_SOURCES, dw.N),
                            "peak_source": f"{peak_src} (hbm_gbs, copy)"}}
        # the same steps with the decode chain's output epilogue fused (gated RMSNorm of o)
        zn = torch.randn((dw.N, dw.Hv, dw.dv), device=dev).to(torch.bfloat16)
        wn = torch.ones(dw.dv, device=dev)

        def nstep(t):
            gdr.decode_step(dd["q"][t], dd["k"][t], dd["v"][t], dd["g"][t], dd["beta"][t],
                            dd["S"], read_mode=dw.read_mode, scale=dw.scale, o=od, norm_z=zn,
                            norm_weight=wn, norm_eps=1e-6)

        for t in range(min(args.warmup, dw.steps)):
            nstep(t)
        torch.cuda.synchronize()
        barrier()
        n0, n1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n0.record(stream)
        for t in range(dw.steps):
            nstep(t)
        n1.record(stream)
        torch.cuda.synchronize()
        barrier()
        nms = max_over_ranks(n0.elapsed_time(n1) / dw.steps, world)
        nbytes = dbytes + zn.numel() * zn.element_size()
        ngbs = nbytes / (nms / 1e3) / 1e9
        dec["fused_output_norm"] = {"ms_per_step": nms, "value": world * ngbs, "unit": "GB/s",
                                    "frac": ngbs / peaks["hbm_gbs"]}
    # ---------------- backward pass (gdr_chunk_bwd) on the same workload and inputs, with a
    # seeded upstream gradient dO; gradients of q, k, v, g, beta and S0
    backward = None
    if args.backward and args.only != "decode":
        gen = torch.Generator("cpu").manual_seed(1000 + rank)
        dOb = torch.randn(tuple(d["v"].shape), generator=gen).to(d["v"].dtype).to(dev)
        bargs_ = gdr.make_chunk_args(d["q"], d["v"], d["g"], d["cu_seqlens"], w.chunk,
                                     w.read_mode, w.scale)
        bws_ = torch.empty(gdr.chunk_bwd_workspace_size(bargs_), dtype=torch.uint8, device=dev)

        def bwstep():
            gdr.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dOb, d["S0"],
                          d["cu_seqlens"], None, chunk=w.chunk, read_mode=w.read_mode,
                          scale=w.scale, workspace=bws_)

        bwsteps = min(args.steps, 5)
        for _ in range(min(args.warmup, 3)):
            bwstep()
        torch.cuda.synchronize()
        barrier()
        k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k0.record(stream)
        for _ in range(bwsteps):
            bwstep()
        k1.record(stream)
        torch.cuda.synchronize()
        barrier()
        kms = max_over_ranks(k0.elapsed_time(k1) / bwsteps, world)
        statuses["backward"] = device_status(bargs_, bws_)
        # read q, k, v, g, beta, dO (and S0); write dq, dk, dv, dg, dbeta (and dS0)
        kbytes = 2 * sum(d[n].numel() * d[n].element_size() for n in ("q", "k", "v", "g", "beta"))
        kbytes += dOb.numel() * dOb.element_size()
        if d["S0"] is not None:
            kbytes += 2 * d["S0"].numel() * 4
        backward = {"workload": w.name, "ms_per_step": kms, "steps": bwsteps,
                    "value": whole_job_rate(tokens, world, kms), "unit": "tokens/s",
                    "path": gdr.chunk_bwd_path(cargs), "algorithmic_bytes": kbytes,
                    "hbm_frac": kbytes / (kms / 1e3) / 1e9 / peaks["hbm_gbs"],
                    "workspace_bytes": bws_.numel()}
        if backward["path"] == "tc":
            # measured traffic of the call's kernels, the intermediate arrays included
            # (with one v-head per key head the head reduction is not launched)
            tp = [measured_traffic(k, src, w.B) for k, src in BWD_TC_KERNELS
                  if k != "bwd_reduce_heads4" or w.Hv != w.Hk]
            backward["traffic"] = None if None in tp else sum(tp)
        del bws_

    # ---------------- GDN-2 (decoupled per-channel gates): the chunk workload on the CUDA-core
    # path and the decode steps, same inputs with g, beta per key channel and a write gate
    gdn2 = None
    if args.gdn2:
        gdn2 = {}
        if args.only != "decode":
            gg, gb, gw = (t.to(dev) for t in workloads.gdn2_gate_inputs(
                tuple(d["v"].shape[:3]), w.dk, w.dv, w.gate_dtype, seed=rank))
            g2args = gdr.make_chunk_args(d["q"], d["v"], gg, d["cu_seqlens"], w.chunk,
                                         w.read_mode, w.scale, gdn2_w=gw)
            g2ws = torch.empty(gdr.chunk_fwd_workspace_size(g2args), dtype=torch.uint8,
                               device=dev)

            def g2step():
                gdr.chunk_fwd(d["q"], d["k"], d["v"], gg, gb, d["S0"], d["cu_seqlens"],
                              chunk=w.chunk, read_mode=w.read_mode, scale=w.scale, o=o,
                              S_final=S_final, workspace=g2ws, gdn2_w=gw)

            g2steps = min(args.steps, 3)
            for _ in range(min(args.warmup, 3)):
                g2step()
            torch.cuda.synchronize()
            barrier()
            c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            c0.record(stream)
            for _ in range(g2steps):
                g2step()
            c1.record(stream)
            torch.cuda.synchronize()
            barrier()
            cms = max_over_ranks(c0.elapsed_time(c1) / g2steps, world)
            statuses["gdn2.chunk"] = device_status(g2args, g2ws)
            # the least HBM traffic of the call: q, k, v and the three gate tensors read once,
            # o and S_final written once (the tensor-core path's per-chunk records, written
            # and read back through the workspace, are not counted)
            g2bytes = sum(d[n].numel() * d[n].element_size() for n in ("q", "k", "v")) + sum(
                t.numel() * t.element_size() for t in (gg, gb, gw)) + (
                o.numel() * o.element_size() + S_final.numel() * 4)
            gdn2["chunk"] = {"workload": w.name, "ms_per_step": cms, "steps": g2steps,
                             "value": whole_job_rate(tokens, world, cms), "unit": "tokens/s",
                             "path": gdr.chunk_fwd_path(g2args),
                             "algorithmic_bytes": g2bytes,
                             "hbm_frac": g2bytes / (cms / 1e3) / 1e9 / peaks["hbm_gbs"],
                             "vs_scalar_forward": cms / ms}
            if gdn2["chunk"]["path"] == "tc":
                # measured traffic of the two kernels of a call (the records included)
                tp = [measured_traffic(k, G2_TC_SOURCES, w.B)
                      for k in ("chunk_g2_prep_tc", "chunk_g2_chain_tc")]
                gdn2["chunk"]["traffic"] = None if None in tp else sum(tp)
            del g2ws
        if dec is not None and not args.rows:
            dg, db, dwg = (t.to(dev) for t in workloads.gdn2_gate_inputs(
                (dw.steps, dw.N, dw.Hv), dw.dk, dw.dv, dw.gate_dtype, seed=rank))

            def g2dstep(t):
                gdr.decode_step(dd["q"][t], dd["k"][t], dd["v"][t], dg[t], db[t], dd["S"],
                                read_mode=dw.read_mode, scale=dw.scale, o=od, gdn2_w=dwg[t])

            for t in range(min(args.warmup, dw.steps)):
                g2dstep(t)
            torch.cuda.synchronize()
            barrier()
            e0.record(stream)
            for t in range(dw.steps):
                g2dstep(t)
            e1.record(stream)
            torch.cuda.synchronize()
            barrier()
            g2ms = max_over_ranks(e0.elapsed_time(e1) / dw.steps, world)
            g2bytes = 2 * dd["S"].numel() * 4 + sum(
                dd[n][0].numel() * dd[n].element_size() for n in ("q", "k", "v")) + sum(
                t[0].numel() * t.element_size() for t in (dg, db, dwg)) + (
                od.numel() * od.element_size())
            g2gbs = g2bytes / (g2ms / 1e3) / 1e9
            gdn2["decode"] = {"workload": dw.name, "ms_per_step": g2ms,
                              "bytes_per_step": g2bytes, "value": world * g2gbs, "unit": "GB/s",
                              "frac": g2gbs / peaks["hbm_gbs"]}
    clocks = sampler.stop()

    # ---------------- end to end through the public API with host buffers: the rows are cut
    # into blocks; each block's inputs are copied in on one stream, its forward runs on a
    # stream of its own once its copies have landed, and its o and S_final are copied out on a
    # third stream, so copies in, kernels and copies out of different blocks overlap
    e2e = None
    if not args.no_e2e:
        pin = {n: x[n].pin_memory() for n in ("q", "k", "v", "g", "beta")}
        h_o = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        h_S = torch.empty(S_final.shape, dtype=S_final.dtype).pin_memory()
        bufs = {n: torch.empty_like(d[n]) for n in pin}
        nblk = 4 if w.B % 4 == 0 else 1
        rb = w.B // nblk
        h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        cstr = [torch.cuda.Stream(device=dev) for _ in range(nblk)]
        sub = gdr.make_chunk_args(d["q"][:rb], d["v"][:rb], d["g"][:rb], None, w.chunk,
                                  w.read_mode, w.scale)
        wss = [torch.empty(gdr.chunk_fwd_workspace_size(sub), dtype=torch.uint8, device=dev)
               for _ in range(nblk)]

        def e2e_step(start_ev):
            h2d.wait_event(start_ev)
            landed = []
            with torch.cuda.stream(h2d):
                for i in range(nblk):
                    r = slice(i * rb, (i + 1) * rb)
                    for n in pin:
                        bufs[n][r].copy_(pin[n][r], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(h2d)
                    landed.append(ev)
            for i in range(nblk):
                r = slice(i * rb, (i + 1) * rb)
                cstr[i].wait_event(landed[i])
                with torch.cuda.stream(cstr[i]):
                    gdr.chunk_fwd(bufs["q"][r], bufs["k"][r], bufs["v"][r], bufs["g"][r],
                                  bufs["beta"][r], None, None, chunk=w.chunk,
                                  read_mode=w.read_mode, scale=w.scale, o=o[r],
                                  S_final=S_final[r], workspace=wss[i], stream=cstr[i])
                    done = torch.cuda.Event()
                    done.record(cstr[i])
                d2h.wait_event(done)
                with torch.cuda.stream(d2h):
                    h_o[r].copy_(o[r], non_blocking=True)
                    h_S[r].copy_(S_final[r], non_blocking=True)
            fin = torch.cuda.Event()
            fin.record(d2h)
            stream.wait_event(fin)
            return fin

        # each step starts once the previous one has copied its results out (its buffers are
        # reused), so a step's time is one batch from host memory to host memory
        n_e2e = max(1, min(args.steps, 5))
        s0 = torch.cuda.Event()
        s0.record(stream)
        e2e_step(s0)
        torch.cuda.synchronize()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        prev = a0
        for _ in range(n_e2e):
            prev = e2e_step(prev)
        a1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(a0.elapsed_time(a1) / n_e2e, world)
        e2e = {"value": whole_job_rate(tokens, world, ems), "unit": "tokens/s", "ms_per_step": ems,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in pin.values()),
               "d2h_bytes_per_step": h_o.numel() * h_o.element_size() + h_S.numel() * 4,
               "pipeline": f"{nblk} row blocks: copies in, forward and copies out overlapped "
                           "on three streams"}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "Hk": w.Hk, "Hv": w.Hv, "dk": w.dk,
                   "dv": w.dv, "chunk": w.chunk, "read_mode": w.read_mode,
                   "state": "fp32", "path": path,
                   "l2": "inputs larger than L2 (q,k,v,o 537 MB > 126 MB), no flush",
                   "parallelism": f"replicas x{world}, no collective"},
        "tflops": tflops, "pct_bf16_tc_peak": tflops / peaks["bf16_tflops"] * 100,
        "roofline": {"bound": "hbm", "achieved": hbm_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": hbm_gbs / peaks["hbm_gbs"],
                     "traffic": args.traffic if args.traffic is not None else (
                         measured_traffic("chunk_fused_tc", CHUNK_TC_SOURCES, w.B)
                         if path == "tc" and not w.n_varlen else None),
                     "algorithmic_bytes": algo_bytes, "flops": flops,
                     "tensor_frac": tflops / peaks["bf16_tflops"],
                     "timed": "whole gdr_chunk_fwd call (plan + chunk kernels), CUDA events",
                     "peak_source": f"{peak_src} (hbm_gbs copy; bf16_tflops burst)"},
        "decode": dec, "varlen": varlen, "gating_prologue": gating, "bidirectional": bidir,
        "gdn2": gdn2, "backward": backward, "e2e": e2e,
        # every timed call's device-side status word (workspace), read after the timing
        "device_status": statuses,
        "clocks": clocks,
        "gpu_launches": launches_per_call * args.steps,
    }
    return line, x, w


def cpu_oracle_sample(x, w, rows=1):
    """Time the fp64 oracle, as it stands, on `rows` rows of the workload (all heads)."""
    import oracle
    sub = {n: (t[:rows] if t is not None else None) for n, t in x.items()
           if n in ("q", "k", "v", "g", "beta")}
    oracle.build()
    t0 = time.perf_counter()
    oracle.forward(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], None, None,
                   read_mode=w.read_mode, scale=w.scale)
    dt = time.perf_counter() - t0
    tokens = rows * w.T
    cores = len(os.sched_getaffinity(0))
    threads = int(os.environ.get("OMP_NUM_THREADS", cores))
    what = "the whole workload" if rows >= w.B else f"{rows} of {w.B} rows"
    return {"value": tokens / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{what} ({rows} x {w.T} tokens x {w.Hv} heads) of {w.name}, "
                      f"fp64 per-token recurrence, {dt:.2f} s"}


def bench_reference(args, rank, world):
    """The oracle timed on the host cores: each step a bounded sample of the workload."""
    import workloads
    if rank != 0:
        return None
    w = workloads.WORKLOADS[args.workload]
    x = workloads.workload_inputs(w)
    rows = 2
    for _ in range(args.warmup):
        cpu_oracle_sample(x, w, rows)
    vals, times = [], []
    for _ in range(args.steps):
        r = cpu_oracle_sample(x, w, rows)
        vals.append(r["value"])
        times.append(rows * w.T / r["value"])
    value = statistics.median(vals)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.median(times) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "Hk": w.Hk, "Hv": w.Hv, "dk": w.dk,
                   "dv": w.dv, "chunk": w.chunk, "read_mode": w.read_mode},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle", "cores": r["cores"],
                         "sample": r["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=CHUNK_WORKLOAD)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-backward", dest="backward", action="store_false",
                    help="skip the backward-pass measurement")
    ap.add_argument("--no-gdn2", dest="gdn2", action="store_false",
                    help="skip the GDN-2 (decoupled gates) chunk and decode measurements")
    ap.add_argument("--no-bidir", action="store_true",
                    help="skip the bidirectional workload (both directions summed)")
    ap.add_argument("--no-varlen", action="store_true",
                    help="skip the varlen workload (64 packed sequences of 256-8192 tokens)")
    ap.add_argument("--no-gating", action="store_true",
                    help="skip the forward through the fused gating prologue")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["all", "chunk", "decode"], default="all",
                    help="profiling: time only one of the two hot paths")
    ap.add_argument("--decode-seqs", type=int, default=0,
                    help="profiling: run the decode step on this many sequences only")
    ap.add_argument("--rows", type=int, default=0,
                    help="run only this many rows of the forward workload (profiling a small case)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the dominant kernel from an ncu capture")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = bench_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line, x, w = bench_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_oracle_sample(x, w, rows=w.B)
        elif rank == 0:
            line["cpu_baseline"] = None
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
