#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear layer on B200.

Default workload: the 7 projections of a Llama-7B-shaped decoder block
(q, k, v, o 4096x4096; gate, up 4096->11008; down 11008->4096), frozen base
weights in NF4 with double-quantized constants, 2048 tokens, LoRA r=16,
alpha=32.  One step = forward + backward of all 7 projections through the
C ABI (qlora_linear_fwd with T kept, qlora_linear_bwd with that T): the
dequantization runs inside the fused GEMMs every step; quantization of the
weights happens once, before timing, as at model load.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 1..5] [--M m]

Prints one JSON line (rank 0).  With N > 1 (launched by torch.distributed.run)
every rank runs its own batch of the same workload (data parallel, weak
scaling) and the adapter gradients dA, dB of all projections are summed over
the ranks with one NCCL all-reduce per step.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s & NF4 weight-stream GB/s; % of roofline, 1×B200"
QUANT = {"nf4": 0, "fp4": 1}
DROPOUT_SEED = 20251
# fp32 fused multiply-adds per cycle per SM of B200 (4 sub-partitions x 32 lanes)
FMA_PER_SM_CYCLE = 128
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# dram__bytes_read.sum + dram__bytes_write.sum of the dominant kernel, averaged over its launches
# in one timed step (ncu --metrics ... --nvtx-include "timed/" python bench.py --steps 1 ..., see
# profiles/), with the hash of the code (comments aside) of the sources that define those kernels
# and their launches when the counters were taken (a later code change to any of them makes the
# figure stale: null)
_PAIR_SRC = ("common.cuh", "nf4_decode.cuh", "tc_gemm.cuh", "tc2_gemm.cuh", "qlora_nf4.cu")
_GEMV_SRC = ("common.cuh", "nf4_decode.cuh", "tc_gemm.cuh", "gemv_mma.cuh", "small_lora.cuh", "dropout.cuh",
             "qlora_nf4.cu")
TRAFFIC = {
    "workload3_M2048": {"bytes_per_launch": 54590446, "files": _PAIR_SRC, "src": "0706f491eb5d"},
    # small M: one forward chain (GEMV + T + finish) per projection
    "workload2_M1": {"bytes_per_launch": 24058496, "files": _GEMV_SRC, "src": "0853182519f5"},
}


def src_hash(files=None) -> str:
    """Hash of the code (comments and blank lines dropped) of the given CUDA sources."""
    h = hashlib.sha1()
    d = os.path.join(ROOT, "bit_nf4_quantized_quant_b200", "csrc")
    for f in sorted(files if files is not None else os.listdir(d)):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        code = [ln.split("//", 1)[0].rstrip() for ln in text.splitlines()]
        h.update(f.encode())
        h.update("\n".join(ln for ln in code if ln).encode())
    return h.hexdigest()[:12]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 200):
        self.gpu = gpu_index
        self.period_ms = period_ms
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
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
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [v for v in sm if mx and v >= 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "sm_mhz_min": min(sm) if sm else None,
                "power_w_max": max((float(r[3]) for r in rows if r[3].replace(".", "").isdigit()), default=None)}


# ---------------------------------------------------------------------------
def flops_fwd_bwd(M, N, K, r):
    # fwd: 2MNK + 2MKr (T) + 2MNr (up); bwd: 2MNK (dX) + 2MKr (U A) + 2MNr (U) + 2MKr (dA) + 2MNr (dB)
    return 4 * M * N * K + 6 * M * r * (K + N)


def main_kernel_flops(M, N, K, r):
    """Algorithmic flops of the two fused dequant-GEMM launches (fwd, bwd) of one projection."""
    return 2 * M * N * K + 2 * M * N * r, 2 * M * N * K + 2 * M * K * r


def nf4_bytes(N, K):
    nb = N * K // 64
    return N * K // 2 + nb + 8 * math.ceil(nb / 256)


def rank_batch(wl, i, M, rank, world, device):
    """Rank-local activations X [M, K] and upstream gradient dY [M, N] of projection i
    (data parallel: every rank draws its own batch; rank 0 of a 1-GPU run draws the
    workload's canonical inputs)."""
    from bit_nf4_quantized_quant_b200 import inputs
    p = wl.projections[i]
    if world == 1:
        X, _, _, dY = inputs.layer_inputs(wl, i, M, device=device)
        return X, dY
    X = inputs.normal(inputs.seed_of(wl.index, i, inputs.ROLE_X) + 7919 * rank, (M, p.K), 1.0, device)
    dY = inputs.normal(inputs.seed_of(wl.index, i, inputs.ROLE_DY) + 7919 * rank, (M, p.N), 1.0, device)
    return X, dY


def grad_layout(shapes, r):
    """Offsets of dA [r, K] and dB [N, r] of every projection in the flat gradient
    buffer that is all-reduced once per step; returns ([(offA, offB)], total)."""
    offs, off = [], 0
    for N, K in shapes:
        offs.append((off, off + r * K))
        off += r * K + N * r
    return offs, off


def build_lib():
    from bit_nf4_quantized_quant_b200 import build as lib_build
    lib_build.build()


# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from bit_nf4_quantized_quant_b200 import _ops as ops
    from bit_nf4_quantized_quant_b200 import inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = inputs.WORKLOADS[args.workload or 3]
    M = args.M or (wl.Ms[-1] if wl.Ms else 0)
    r, s = wl.r, wl.scaling
    projs = wl.projections
    peaks, peak_src = load_peaks()

    bwd = wl.backward
    small = M <= 32
    # ---- setup: weights quantized once, inputs resident in HBM.  For the
    # memory-bound sizes the weight set is replicated so that one rotation
    # through it streams more than twice the L2 capacity from HBM.
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    wset = sum(nf4_bytes(p.N, p.K) for p in projs)
    copies = max(1, math.ceil(2 * l2 / wset)) if small else 1
    layers = []
    for i, p in enumerate(projs):
        W = inputs.layer_weight(wl, i, device=dev)
        w = ops.quant4_quantize_dq(W, QUANT[args.quant])
        ws_copies = [w] + [ops.quant4_quantize_dq(W, QUANT[args.quant]) for _ in range(copies - 1)]
        del W
        _, A, B, _ = inputs.layer_inputs(wl, i, M, device=dev, with_dy=False)
        X, dY = rank_batch(wl, i, M, rank, world, dev)
        L = dict(p=p, w=w, wc=ws_copies, X=X, A=A, B=B, dY=dY,
                 Y=torch.empty((M, p.N), dtype=torch.bfloat16, device=dev),
                 T=torch.empty((M, r), dtype=torch.bfloat16, device=dev),
                 dX=torch.empty((M, p.K), dtype=torch.bfloat16, device=dev))
        layers.append(L)
    # adapter gradients of all projections in one flat buffer (one all-reduce per step)
    offs, total = grad_layout([(L["p"].N, L["p"].K) for L in layers], r)
    gbuf = torch.empty(total, dtype=torch.bfloat16, device=dev)
    for L, (oa, ob) in zip(layers, offs):
        L["dA"] = gbuf[oa:oa + r * L["p"].K].view(r, L["p"].K)
        L["dB"] = gbuf[ob:ob + L["p"].N * r].view(L["p"].N, r)
    wsb = ops.qlora_dropout_workspace_bytes if args.dropout > 0 else ops.qlora_workspace_bytes
    ws = torch.empty(max(wsb(M, L["p"].N, L["p"].K, r) for L in layers), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    it = [0]

    def fwd_call(L, w, off):
        if args.dropout > 0:
            ops.qlora_linear_fwd_dropout(L["X"], w, L["A"], L["B"], s, args.dropout, DROPOUT_SEED, off,
                                         Y=L["Y"], T_out=L["T"], ws=ws)
        else:
            ops.qlora_linear_fwd(L["X"], w, L["A"], L["B"], s, Y=L["Y"], T_out=L["T"], ws=ws)

    def bwd_call(L, w, off, g=""):
        # g selects the gradient buffer: "" the main one, "2" the second one the end-to-end
        # pipeline alternates with
        dA, dB = L["dA" + g], L["dB" + g]
        if args.dropout > 0:
            ops.qlora_linear_bwd_dropout(L["X"], L["dY"], w, L["A"], L["B"], s, args.dropout, DROPOUT_SEED, off,
                                         T=L["T"], dX=L["dX"], dA=dA, dB=dB, ws=ws)
        else:
            ops.qlora_linear_bwd(L["X"], L["dY"], w, L["A"], L["B"], s, T=L["T"], dX=L["dX"], dA=dA, dB=dB, ws=ws)

    def step(events=None, collective=True):
        c = it[0] % copies
        it[0] += 1
        for j, L in enumerate(layers):
            w = L["wc"][c]
            if events is not None:
                ops.qlora_set_kernel_events(*events[2 * j])
            off = (it[0] - 1) * len(layers) + j   # dropout: a fresh mask per step and projection
            fwd_call(L, w, off)
            if not bwd:
                continue
            if events is not None:
                ops.qlora_set_kernel_events(*events[2 * j + 1])
            bwd_call(L, w, off)
        if world > 1 and bwd and collective:
            dist.all_reduce(gbuf)

    for _ in range(args.warmup):
        step()
    c0 = ops.qlora_launch_count()
    step()
    per_step_launches = ops.qlora_launch_count() - c0
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    # ---- timed region: one CUDA graph per timed step (the library calls are
    # asynchronous and allocation-free, so a step captures as is).  The last
    # timed step also records the library's per-launch events around the fused
    # dequant-GEMM kernels: an event between two kernels ends the overlap that
    # programmatic launch gives them, so the other steps carry none.
    ev_step = args.steps - 1
    kev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(2 * len(layers))] for _ in range(args.steps)]
    for evs in kev:                 # torch creates the CUDA events lazily: record once so they exist
        for a, b in evs:
            a.record(stream)
            b.record(stream)
    torch.cuda.synchronize()
    graphs = []
    if not args.no_graph:
        for k in range(args.steps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(kev[k] if k == ev_step else None, collective=False)
            graphs.append(g)
        for g in graphs:            # upload + warm
            g.replay()
            if world > 1:
                dist.all_reduce(gbuf)
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
    clocks = ClockSampler(local_rank, args.clock_ms)
    clocks.start()
    launches0 = ops.qlora_launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    t0.record(stream)
    for k in range(args.steps):
        if graphs:
            graphs[k].replay()
            if world > 1 and bwd:
                dist.all_reduce(gbuf)
        else:
            step(kev[k] if k == ev_step else None)
    t1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = ops.qlora_launch_count() - launches0
    if graphs:   # a replayed graph launches the kernels captured from one step
        launches = per_step_launches * args.steps
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    if world > 1:
        tt = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
    assert ops.qlora_device_status() == 0, "device-side wait timed out"
    ms_per_step = ms / args.steps

    npass = 2 if bwd else 1
    flops_step, bytes_step = step_work(wl, M)
    # roofline of the dominant kernel (the fused dequant-GEMM), from its own launch events
    kflops, kms, nlaunch = 0.0, 0.0, 0
    kbytes = 0
    kev_src = "graph replay" if graphs else "timed steps"
    try:
        kev[ev_step][0][0].elapsed_time(kev[ev_step][0][1])
    except RuntimeError:
        # events inside a replayed graph could not be timed: time the kernels
        # of one step launched eagerly on the same stream
        torch.cuda.synchronize()
        step(kev[ev_step], collective=False)
        torch.cuda.synchronize()
        kev_src = "eager pass after the timed steps"
    for k in (ev_step,):
        for j, L in enumerate(layers):
            N_, K_ = L["p"].N, L["p"].K
            f_fwd, f_bwd = main_kernel_flops(M, N_, K_, r)
            # small M: the timed pair in the forward is the GEMV (which also computes T = X A^T)
            # + its finish kernel (NF4 weight, X, A, B read, Y and T written once); in the
            # backward the U / dB kernel + the dX GEMV (NF4 weight, dY, B and T read, dB
            # written once; split partials not counted)
            b_fwd = nf4_bytes(N_, K_) + 2 * (M * K_ + M * N_ + r * K_ + N_ * r + M * r)
            b_bwd = nf4_bytes(N_, K_) + 2 * (M * N_ + 2 * N_ * r + M * r)
            for h, f, bb in ((0, f_fwd, b_fwd), (1, f_bwd, b_bwd))[:npass]:
                a, b = kev[k][2 * j + h]
                kms += a.elapsed_time(b)
                kflops += f
                kbytes += bb
                nlaunch += 1
    if small:
        achieved = kbytes / (kms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "unit": "GB/s"}
    else:
        achieved = kflops / (kms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "unit": "TFLOP/s"}
        if "bf16_tflops_sustained" in peaks:
            roof["frac_of_sustained"] = round(achieved / peaks["bf16_tflops_sustained"], 4)
    tr = TRAFFIC.get(f"workload{wl.index}_M{M}")
    roof.update({"achieved": round(achieved, 2), "peak": peak, "frac": round(achieved / peak, 4),
                 "traffic": tr["bytes_per_launch"] if tr and tr.get("src") == src_hash(tr["files"]) else None,
                 "peak_source": f"{peak_src} ({'hbm copy' if small else 'cuBLAS bf16 burst'})",
                 "kernel": ("k_nf4_gemv + k_nf4_gemv_finish / k_lora_bwd_small + k_tcs_gemm (programmatic-launch pairs)"
                            if small else "k_tc_gemm / k_tc2_gemm (fwd + bwd dX)"),
                 "launches_timed": nlaunch, "avg_launch_us": round(kms / nlaunch * 1e3, 2),
                 "events_from": kev_src})

    roof["weight_copies_rotated"] = copies
    if small:
        value = bytes_step * world / (ms_per_step * 1e-3) / 1e9
        unit = "GB/s"
    else:
        value = flops_step * world / (ms_per_step * 1e-3) / 1e12
        unit = "TFLOP/s"

    # ---- end to end through the C ABI with host buffers: H2D of X, dY, D2H of Y, dX, dA, dB each step
    hX = [torch.empty_like(L["X"], device="cpu").pin_memory() for L in layers]
    hdY = [torch.empty_like(L["dY"], device="cpu").pin_memory() for L in layers]
    for h, L in zip(hX, layers):
        h.copy_(L["X"])
    for h, L in zip(hdY, layers):
        h.copy_(L["dY"])
    hout = [[torch.empty_like(L[k], device="cpu").pin_memory() for k in ("Y", "dX")] for L in layers]
    hg = torch.empty_like(gbuf, device="cpu").pin_memory()
    h2d = sum(h.numel() * 2 for h in hX) + (sum(h.numel() * 2 for h in hdY) if bwd else 0)
    d2h = sum(os_[0].numel() * 2 + (os_[1].numel() * 2 if bwd else 0) for os_ in hout) + (hg.numel() * 2 if bwd else 0)

    # When a step moves 4 MiB or more, pipelined over the projections the way a
    # caller would run it: inputs go in on one copy stream, outputs come back on
    # another, the layer calls run on the compute stream in between, so both copy
    # directions and the kernels overlap.  With a few KB per step (decode sizes)
    # the event hops between streams cost more than they hide: one stream, in
    # order.
    # Events keep each buffer's order: layer j's inputs are overwritten only after
    # the previous step's compute has read them, and its outputs (and the
    # gradient buffer) only after the previous step's copy-out has read them.
    # The adapter gradients alternate between two device buffers by step, so a step's
    # first backward does not wait for the previous step's gradients to reach the host
    # (only for those of the step before it, long since copied).
    comp = stream
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in layers]      # layer j's inputs have landed
    ev_done = [torch.cuda.Event() for _ in layers]    # layer j's calls are done
    ev_out = [torch.cuda.Event() for _ in layers]     # layer j's outputs are on the host
    ev_grad = torch.cuda.Event()
    ev_gout = [torch.cuda.Event(), torch.cuda.Event()]  # gradient buffer g is on the host
    gbufs = [gbuf, torch.empty_like(gbuf) if bwd else gbuf]
    if bwd:
        for L, (oa, ob) in zip(layers, offs):
            L["dA2"] = gbufs[1][oa:oa + r * L["p"].K].view(r, L["p"].K)
            L["dB2"] = gbufs[1][ob:ob + L["p"].N * r].view(L["p"].N, r)
    primed = [False]
    nstep = [0]

    def e2e_step_serial():
        for j, L in enumerate(layers):
            L["X"].copy_(hX[j], non_blocking=True)
            if bwd:
                L["dY"].copy_(hdY[j], non_blocking=True)
            fwd_call(L, L["w"], j)
            hout[j][0].copy_(L["Y"], non_blocking=True)
            if bwd:
                bwd_call(L, L["w"], j)
                hout[j][1].copy_(L["dX"], non_blocking=True)
        if world > 1 and bwd:
            dist.all_reduce(gbuf)
        if bwd:
            hg.copy_(gbuf, non_blocking=True)

    pipelined = h2d + d2h >= (4 << 20)

    def e2e_step():
        if not pipelined:
            return e2e_step_serial()
        g = nstep[0] & 1
        gb = gbufs[g]
        for j, L in enumerate(layers):
            with torch.cuda.stream(s_in):
                if primed[0]:
                    s_in.wait_event(ev_done[j])
                L["X"].copy_(hX[j], non_blocking=True)
                if bwd:
                    L["dY"].copy_(hdY[j], non_blocking=True)
                ev_in[j].record(s_in)
            comp.wait_event(ev_in[j])
            if primed[0]:
                comp.wait_event(ev_out[j])
            fwd_call(L, L["w"], j)
            if bwd:
                if j == 0 and nstep[0] >= 2:
                    comp.wait_event(ev_gout[g])       # this buffer's gradients of two steps ago are out
                bwd_call(L, L["w"], j, "2" if g else "")
            ev_done[j].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[j])
                hout[j][0].copy_(L["Y"], non_blocking=True)
                if bwd:
                    hout[j][1].copy_(L["dX"], non_blocking=True)
                ev_out[j].record(s_out)
        if world > 1 and bwd:
            dist.all_reduce(gb)
        if bwd:
            ev_grad.record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_grad)
                hg.copy_(gb, non_blocking=True)
                ev_gout[g].record(s_out)
        primed[0] = True
        nstep[0] += 1

    for _ in range(max(1, args.warmup // 2)):
        e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(comp)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for _ in range(args.steps):
        e2e_step()
    comp.wait_stream(s_in)
    comp.wait_stream(s_out)
    e1.record(comp)
    torch.cuda.synchronize()
    ems = e0.elapsed_time(e1)
    if world > 1:
        tt = torch.tensor([ems], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ems = float(tt.item())
    e2e_val = (flops_step if not small else bytes_step) * world / (ems / args.steps * 1e-3) / (1e12 if not small else 1e9)

    cfg = {"workload": wl.name, "quant_type": args.quant, "lora_dropout": args.dropout,
           "projections": [f"{p.name} {p.N}x{p.K}" for p in projs], "M_per_gpu": M,
           "global_batch_tokens": M * world, "r": r, "alpha": wl.alpha, "weights": "NF4 + double-quant (64/256)",
           "step": "qlora_linear_fwd + qlora_linear_bwd for every projection" +
                   (" + NCCL all-reduce of dA,dB" if world > 1 else ""),
           "l2": (f"inputs larger than L2: {bytes_step / 1e6:.0f} MB of algorithmic traffic per step" if not small else
                  f"weights rotated over {copies} copies ({copies * wset / 1e6:.0f} MB > 2x L2)"),
           "parallelism": f"dp{world}",
           "launch": "eager" if args.no_graph else "one CUDA graph per step (library calls captured as issued)"}
    out = {"metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16 (NF4 weights, fp32 accumulate)",
           "data": "synthetic (seeded)", "config": cfg, "roofline": roof,
           "e2e": {"value": round(e2e_val, 3), "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                   "copies": ("H2D and D2H on two copy streams, pipelined over the projections" if pipelined else
                              "in order on the compute stream") + "; all inside the timed region"},
           "gpu_launches": launches, "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, M, budget_s=args.cpu_seconds, quant=args.quant, dropout=args.dropout)
    return out


# ---------------------------------------------------------------------------
def run_bulk(args, rank, world, local_rank):
    """Workload 5: quantize + double-quantize all 224 tensors of a 32-layer
    7B-shaped model, then dequantize them all back (one step = both passes)."""
    import torch

    from bit_nf4_quantized_quant_b200 import _ops as ops
    from bit_nf4_quantized_quant_b200 import inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = inputs.WORKLOADS[5]
    peaks, peak_src = load_peaks()
    layers = args.layers or wl.repeat
    tensors = []
    for c in range(layers):
        for i, p in enumerate(wl.projections):
            W = inputs.layer_weight(wl, i, device=dev, copy=c + 1000 * rank)
            tensors.append((W, ops.NF4Weight.empty(p.N, p.K, dev), torch.empty_like(W)))
    params = sum(W.numel() for W, _, _ in tensors)
    nb = sum(w.codes.numel() for _, w, _ in tensors)
    ng = sum(w.scale.numel() for _, w, _ in tensors)
    qbytes = params // 2 + nb + 8 * ng
    stream = torch.cuda.current_stream()

    def step(ev=None):
        for j, (W, w, out) in enumerate(tensors):
            if ev: ev[0][j][0].record(stream)
            ops.nf4_quantize_dq(W, out=w)
            if ev: ev[0][j][1].record(stream)
        for j, (W, w, out) in enumerate(tensors):
            if ev: ev[1][j][0].record(stream)
            ops.nf4_dequant(w, out=out)
            if ev: ev[1][j][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in tensors]
          for _ in range(2)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    l0 = ops.qlora_launch_count()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    t0.record(stream)
    for k in range(args.steps):
        step(ev if k == args.steps - 1 else None)
    t1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    launches = ops.qlora_launch_count() - l0
    clk = clocks.stop()
    assert ops.qlora_device_status() == 0
    ms = t0.elapsed_time(t1) / args.steps
    step_bytes = 2 * (2 * params + qbytes)           # quantize: read bf16, write NF4; dequant: the reverse
    value = step_bytes / (ms * 1e-3) / 1e9
    tq = sum(a.elapsed_time(b) for a, b in ev[0])
    td = sum(a.elapsed_time(b) for a, b in ev[1])
    kq = (2 * params + qbytes) / (tq * 1e-3) / 1e9
    kd = (2 * params + qbytes) / (td * 1e-3) / 1e9
    dom = ("k_quantize_dq", kq, tq) if tq >= td else ("k_dequant", kd, td)
    roof = {"bound": "hbm", "unit": "GB/s", "achieved": round(dom[1], 1), "peak": peaks["hbm_gbs"],
            "frac": round(dom[1] / peaks["hbm_gbs"], 4), "traffic": None,
            "peak_source": f"{peak_src} (hbm copy)", "kernel": dom[0], "launches_timed": len(tensors),
            "avg_launch_us": round(dom[2] / len(tensors) * 1e3, 2),
            "other": {"k_quantize_dq_GBps": round(kq, 1), "k_dequant_GBps": round(kd, 1)}}
    # e2e: host bf16 weights in, NF4 + dequantized weights out, for one layer (7 tensors) per step
    hW = [W.cpu().pin_memory() for W, _, _ in tensors[:7]]
    hout = [torch.empty_like(W, device="cpu").pin_memory() for W, _, _ in tensors[:7]]
    hq = [(torch.empty_like(w.packed, device="cpu").pin_memory(), torch.empty_like(w.codes, device="cpu").pin_memory())
          for _, w, _ in tensors[:7]]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for k in range(args.steps):
        for j, (W, w, out) in enumerate(tensors[:7]):
            W.copy_(hW[j], non_blocking=True)
            ops.nf4_quantize_dq(W, out=w)
            ops.nf4_dequant(w, out=out)
            hq[j][0].copy_(w.packed, non_blocking=True)
            hq[j][1].copy_(w.codes, non_blocking=True)
            hout[j].copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    p7 = sum(W.numel() for W, _, _ in tensors[:7])
    q7 = sum(w.packed.numel() + w.codes.numel() + 8 * w.scale.numel() for _, w, _ in tensors[:7])
    e2e = 2 * (2 * p7 + q7) / (e0.elapsed_time(e1) / args.steps * 1e-3) / 1e9
    out = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 -> NF4 + int8/fp32 constants -> bf16", "data": "synthetic (seeded)",
            "config": {"workload": wl.name, "tensors": len(tensors), "params": params,
                       "step": "nf4_quantize_dq then nf4_dequant over every tensor",
                       "l2": f"inputs larger than L2: {step_bytes / 1e9:.1f} GB per step"},
            "roofline": roof,
            "e2e": {"value": round(e2e, 1), "unit": "GB/s", "h2d_bytes_per_step": 2 * p7,
                    "d2h_bytes_per_step": 2 * p7 + sum(w.packed.numel() + w.codes.numel() for _, w, _ in tensors[:7])},
            "gpu_launches": launches, "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = bulk_cpu_baseline(wl)
    return out


def run_merge(args, rank, world, local_rank):
    """Dequantize-and-merge of the 7 projections of the 7B block (r = 16, s = 2):
    W' + s B A in bf16, one nf4_dequant_merge per projection per step.  Each rank
    merges its own copy (weak scaling)."""
    import torch

    from bit_nf4_quantized_quant_b200 import _ops as ops
    from bit_nf4_quantized_quant_b200 import inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = inputs.WORKLOADS[3]
    peaks, peak_src = load_peaks()
    r, s = wl.r, wl.scaling
    layers = []
    for i, p in enumerate(wl.projections):
        W = inputs.layer_weight(wl, i, device=dev)
        w = ops.quant4_quantize_dq(W, QUANT[args.quant])
        del W
        _, A, B, _ = inputs.layer_inputs(wl, i, 1, device=dev, with_dy=False)
        layers.append((w, A, B, torch.empty((p.N, p.K), dtype=torch.bfloat16, device=dev)))
    stream = torch.cuda.current_stream()

    def step(ev=None):
        for j, (w, A, B, out) in enumerate(layers):
            if ev: ev[j][0].record(stream)
            ops.nf4_dequant_merge(w, A, B, s, out=out)
            if ev: ev[j][1].record(stream)

    for _ in range(args.warmup):
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in layers]
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    l0 = ops.qlora_launch_count()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        step(ev if k == args.steps - 1 else None)
    t1.record(stream)
    torch.cuda.synchronize()
    launches = ops.qlora_launch_count() - l0
    clk = clocks.stop()
    assert ops.qlora_device_status() == 0
    ms = t0.elapsed_time(t1) / args.steps
    params = sum(p.N * p.K for p in wl.projections)
    step_bytes = sum(nf4_bytes(p.N, p.K) + 2 * p.N * p.K + 2 * r * (p.N + p.K) for p in wl.projections)
    step_flops = sum(2 * p.N * p.K * r for p in wl.projections)
    kms = sum(a.elapsed_time(b) for a, b in ev)
    mhz = peaks.get("sm_max_mhz", 1965.0)
    fma_peak = 148 * FMA_PER_SM_CYCLE * 2 * mhz * 1e6 / 1e12
    achieved = step_flops / (kms * 1e-3) / 1e12
    roof = {"bound": "alu", "unit": "TFLOP/s", "achieved": round(achieved, 2), "peak": round(fma_peak, 1),
            "frac": round(achieved / fma_peak, 4), "traffic": None,
            "peak_source": f"fp32 fma pipe: 148 SMs x {FMA_PER_SM_CYCLE} fma/cycle x 2 flop x {mhz:.0f} MHz "
                           f"(sm_max_mhz, {peak_src})",
            "kernel": "k_dequant_merge", "launches_timed": len(layers),
            "avg_launch_us": round(kms / len(layers) * 1e3, 2),
            "hbm": {"achieved_GBps": round(step_bytes / (kms * 1e-3) / 1e9, 1), "peak": peaks["hbm_gbs"],
                    "frac": round(step_bytes / (kms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}}
    out = {"metric": METRIC, "value": round(step_bytes / (ms * 1e-3) / 1e9, 1), "unit": "GB/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "NF4/FP4 + bf16 adapters -> bf16 (fp32 fma chain)",
           "data": "synthetic (seeded)",
           "config": {"workload": "dequantize-and-merge llama7b block (7 projections)", "quant_type": args.quant,
                      "r": r, "alpha": wl.alpha, "params": params,
                      "step": "nf4_dequant_merge of every projection",
                      "l2": f"inputs larger than L2: {step_bytes / 1e6:.0f} MB per step"},
           "roofline": roof, "gpu_launches": launches, "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = merge_cpu_baseline(wl, args.quant)
    return out


def run_adamw(args, rank, world, local_rank):
    """One 8-bit AdamW step over every LoRA adapter of a 32-layer 7B model (the 7
    projections per layer at r = 16: 40.0M bf16 parameters in one flat buffer, more
    than twice L2 with its states)."""
    import torch

    from bit_nf4_quantized_quant_b200 import _ops as ops
    from bit_nf4_quantized_quant_b200 import inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = inputs.WORKLOADS[3]
    peaks, peak_src = load_peaks()
    n = 32 * sum(wl.r * (p.N + p.K) for p in wl.projections)
    p = inputs.normal(5000, (n,), 0.01, device=dev)
    g = inputs.normal(5001, (n,), 1e-3, device=dev)
    st = ops.AdamW8State.zeros(n, device=dev)
    stream = torch.cuda.current_stream()
    k = [0]

    def step():
        k[0] += 1
        ops.adamw_8bit_step(p, g, st, k[0], 2e-4, 0.9, 0.999, 1e-8, 0.01)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    l0 = ops.qlora_launch_count()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    launches = ops.qlora_launch_count() - l0
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / args.steps
    nblk = math.ceil(n / 256)
    step_bytes = n * (2 + 2 + 1 + 1) + n * (2 + 1 + 1) + nblk * 16   # read p, g, codes; write p, codes; scales
    gbs = step_bytes / (ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "unit": "GB/s", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
            "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": None, "peak_source": f"{peak_src} (hbm copy)",
            "kernel": "k_adamw8", "launches_timed": args.steps, "avg_launch_us": round(ms * 1e3, 2)}
    out = {"metric": METRIC, "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16 params/grads, E4M3 moment codes + fp32 block scales, fp32 update",
           "data": "synthetic (seeded)",
           "config": {"workload": "8-bit AdamW step, all LoRA adapters of a 32-layer 7B model (r=16, 7 projections)",
                      "params": n, "block": 256,
                      "l2": f"inputs larger than L2: {step_bytes / 1e6:.0f} MB per step"},
           "roofline": roof, "gpu_launches": launches, "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = adamw_cpu_baseline(n // 32)
    return out


def adamw_cpu_baseline(n):
    """The oracle's AdamW step (C, one thread) on one layer's adapters, as GB/s of the
    same byte accounting (the rate stands for the whole model)."""
    import numpy as np

    import oracle
    from bit_nf4_quantized_quant_b200 import inputs
    p = inputs.bf16_bits(inputs.normal(5000, (n,), 0.01)).copy()
    g = inputs.bf16_bits(inputs.normal(5001, (n,), 1e-3)).copy()
    st = oracle.adamw8_state(n)
    t0 = time.perf_counter()
    k = 0
    while k < 3 or time.perf_counter() - t0 < 2.0:
        k += 1
        oracle.adamw8_step(p, g, st, k, 2e-4, 0.9, 0.999, 1e-8, 0.01)
    dt = (time.perf_counter() - t0) / k
    step_bytes = n * 10 + math.ceil(n / 256) * 16
    return {"value": round(step_bytes / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{k} oracle steps over one layer's adapters ({n} params), C, one thread; "
                      f"{dt * 1e3:.1f} ms per step; the rate stands for all 32 layers"}


def merge_cpu_baseline(wl, quant, rows=64):
    """The oracle's dequantize-and-merge on `rows` rows of each projection (C, one
    thread per projection), scaled to the whole weight (every row costs the same)."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np

    import oracle
    from bit_nf4_quantized_quant_b200 import inputs
    jobs = []
    for i, p in enumerate(wl.projections):
        W = inputs.layer_weight(wl, i)
        q = oracle.quantize_dq_qt(inputs.bf16_bits(W), QUANT[quant])
        _, A, B, _ = inputs.layer_inputs(wl, i, 1, with_dy=False)
        jobs.append((q, inputs.bf16_bits(A), inputs.bf16_bits(B), np.arange(rows) * (p.N // rows)))

    def one(job):
        q, A, B, rr = job
        t0 = time.perf_counter()
        oracle.dequant_merge(q, A, B, wl.scaling, rows=rr)
        return time.perf_counter() - t0

    with ThreadPoolExecutor(len(jobs)) as pool:
        times = list(pool.map(one, jobs))
    full = sum(t * p.N / rows for t, p in zip(times, wl.projections))      # serial-equivalent seconds
    step_bytes = sum(nf4_bytes(p.N, p.K) + 2 * p.N * p.K + 2 * wl.r * (p.N + p.K) for p in wl.projections)
    return {"value": round(step_bytes / full / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows} rows of each of the 7 projections merged by the C oracle ({sum(times):.1f} s), "
                      f"time scaled by N/{rows} per projection (extrapolated), one core per projection counted serially"}


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n + [1])
    except Exception:
        return os.cpu_count() or 1


def step_work(wl, M):
    """Algorithmic work of one step of a workload at M tokens: (flops, bytes).

    flops: 4MNK + 6Mr(K+N) per projection for forward + backward, 2MNK + 2Mr(K+N)
    for the forward alone.  bytes: the NF4 weight once per pass (4.12890625 bit per
    parameter) plus every activation, adapter and output tensor read or written once.
    """
    r = wl.r
    flops = bytes_ = 0
    for p in wl.projections:
        N_, K_ = p.N, p.K
        if wl.backward:
            flops += flops_fwd_bwd(M, N_, K_, r)
            bytes_ += 2 * nf4_bytes(N_, K_) + 2 * (M * K_ + r * K_ + N_ * r + M * N_)
            bytes_ += 2 * (M * N_ + M * K_ + M * K_ + r * K_ + N_ * r + M * r)
        else:
            flops += 2 * M * N_ * K_ + 2 * M * r * (K_ + N_)
            bytes_ += nf4_bytes(N_, K_) + 2 * (M * K_ + r * K_ + N_ * r + M * N_)
    return flops, bytes_


class OracleStep:
    """One step of a workload on the CPU oracle, timed on the host cores.

    Per projection: the oracle's dequantization of the whole NF4 weight (C, run
    over row ranges on a thread pool of all host cores: ctypes releases the GIL)
    and its widening to fp64, charged once per step as a layer call would; then
    the fp64 forward (+ backward) on `rows` of the M tokens (numpy, BLAS on all
    host cores), whose time is scaled by M / rows -- every token costs the same
    in these products, so the extrapolation is linear and is labelled as such.
    Quantization happens once before timing, as at model load."""

    def __init__(self, wl, M, rows=64, quant="nf4", dropout=0.0):
        import numpy as np
        from concurrent.futures import ThreadPoolExecutor

        import oracle
        from bit_nf4_quantized_quant_b200 import inputs
        self.wl, self.M = wl, M
        self.rows = min(rows, M)
        self.dropout = dropout
        self.ncores = os.cpu_count() or 1
        self.pool = ThreadPoolExecutor(self.ncores)
        self.state = []
        for i, p in enumerate(wl.projections):
            W = inputs.layer_weight(wl, i)
            q = oracle.quantize_dq_qt(inputs.bf16_bits(W), QUANT[quant])
            X, A, B, dY = inputs.layer_inputs(wl, i, self.rows, with_dy=wl.backward)
            self.state.append((q, inputs.to_f64(X), inputs.to_f64(A), inputs.to_f64(B),
                               inputs.to_f64(dY) if dY is not None else None,
                               np.array_split(np.arange(p.N), self.ncores)))
        self.flops, self.bytes = step_work(wl, M)

    def run(self):
        """Returns the step's time in seconds, extrapolated to M tokens."""
        import numpy as np

        import oracle
        total = 0.0
        s = self.wl.scaling
        for q, X, A, B, dY, chunks in self.state:
            t0 = time.perf_counter()
            parts = list(self.pool.map(lambda rr: oracle.dequant_qt(q, rr), chunks))
            Wd = oracle.bf16_to_f32(np.concatenate(parts)).astype(np.float64)
            t1 = time.perf_counter()
            if self.dropout > 0:
                keep = oracle.dropout_mask(DROPOUT_SEED, 0, X.shape[0], X.shape[1], self.dropout)
                c = oracle.dropout_scale(self.dropout)
                oracle.linear_fwd_dropout(X, Wd, A, B, s, keep, c)
                if dY is not None:
                    oracle.linear_bwd_dropout(X, dY, Wd, A, B, s, keep, c)
            else:
                oracle.linear_fwd(X, Wd, A, B, s)
                if dY is not None:
                    oracle.linear_bwd(X, dY, Wd, A, B, s)
            t2 = time.perf_counter()
            total += (t1 - t0) + (t2 - t1) * self.M / self.rows
        return total

    def value(self, seconds):
        if self.M <= 32:
            return self.bytes / seconds / 1e9, "GB/s"
        return self.flops / seconds / 1e12, "TFLOP/s"

    def sample_text(self, nsteps):
        return (f"{nsteps} oracle step(s) of all {len(self.wl.projections)} projections: dequant of each full NF4 "
                f"weight (C, {self.ncores} threads over row ranges) + fp64 fwd{'+bwd' if self.wl.backward else ''} "
                f"(numpy, {_threads()} BLAS threads) on {self.rows} of {self.M} tokens, the product time scaled "
                f"by {self.M}/{self.rows} (extrapolated); quantization once, untimed")


def cpu_baseline(wl, M, budget_s=20.0, quant="nf4", dropout=0.0):
    """The oracle, as it stands, on the host cores over a bounded sample."""
    if wl.index == 5:
        return bulk_cpu_baseline(wl)
    st = OracleStep(wl, M, quant=quant, dropout=dropout)
    st.run()                                     # warm: first touch of the fp64 buffers
    t0 = time.perf_counter()
    times = []
    while not times or time.perf_counter() - t0 < budget_s / 2:
        times.append(st.run())
    v, unit = st.value(statistics.mean(times))
    return {"value": round(v, 6), "unit": unit, "cores": st.ncores, "kind": "oracle",
            "sample": st.sample_text(len(times))}


def bulk_cpu_baseline(wl):
    """Workload 5 on the oracle: quantize + double-quantize then dequantize one
    7-tensor layer (the tensors in parallel on host threads); GB/s of the same
    byte accounting as the GPU line (read 2 B + write 0.516 B per parameter, each way)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    from bit_nf4_quantized_quant_b200 import inputs
    Ws = [inputs.bf16_bits(inputs.layer_weight(wl, i)) for i in range(len(wl.projections))]

    def one(Wb):
        q = oracle.quantize_dq(Wb)
        oracle.dequant(q)
        return Wb.size

    with ThreadPoolExecutor(len(Ws)) as pool:
        t0 = time.perf_counter()
        params = sum(pool.map(one, Ws))
        dt = time.perf_counter() - t0
    qbytes = sum(nf4_bytes(p.N, p.K) for p in wl.projections)
    v = 2 * (2 * params + qbytes) / dt / 1e9
    return {"value": round(v, 3), "unit": "GB/s", "cores": len(Ws), "kind": "oracle",
            "sample": f"one layer (7 tensors, {params} params) quantized + dequantized by the C oracle, one thread "
                      f"per tensor; {dt:.1f} s; the rate stands for the whole 32-layer set"}


def run_reference(args):
    """The oracle as the reference arm: host cores, one bounded sample per step."""
    from bit_nf4_quantized_quant_b200 import inputs
    wl = inputs.WORKLOADS[args.workload or 3]
    if wl.index == 5:
        cb = bulk_cpu_baseline(wl)
        value, unit, ms, sample = cb["value"], cb["unit"], None, cb["sample"]
        cores = cb["cores"]
    else:
        M = args.M or wl.Ms[-1]
        st = OracleStep(wl, M)
        for _ in range(args.warmup):
            st.run()
        times = [st.run() for _ in range(args.steps)]
        ms = statistics.mean(times) * 1e3
        value, unit = st.value(statistics.mean(times))
        sample, cores = st.sample_text(args.steps), st.ncores
    cfg = {"workload": wl.name, "M": args.M or (wl.Ms[-1] if wl.Ms else 0), "r": wl.r, "alpha": wl.alpha}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3) if ms else None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic (seeded)", "config": cfg,
            "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def sub_results(args, rank, world, local_rank):
    """The memory-bound half of the metric, measured in the same process after the
    headline line: decode GEMV (workload 2, M = 1), the single 4096^2 linear
    (workload 1, M = 16, fwd+bwd) and the bulk quantize + dequantize round trip
    (workload 5), each with its own roofline entry, clocks and CPU baseline."""
    import copy

    import torch
    subs = []
    for wlx, M, op, quant, dropout in ((2, 1, "linear", "nf4", 0.0), (1, 16, "linear", "nf4", 0.0),
                                       (5, 0, "linear", "nf4", 0.0), (2, 1, "linear", "fp4", 0.0),
                                       (3, 0, "merge", "nf4", 0.0), (3, 0, "adamw", "nf4", 0.0),
                                       (3, 2048, "linear", "nf4", 0.05)):
        torch.cuda.empty_cache()
        a = copy.copy(args)
        a.workload, a.M, a.op, a.quant, a.dropout = wlx, M, op, quant, dropout
        a.cpu_seconds = min(args.cpu_seconds, 8.0)
        if op == "merge":
            o = run_merge(a, rank, world, local_rank)
        elif op == "adamw":
            o = run_adamw(a, rank, world, local_rank)
        else:
            o = run_bulk(a, rank, world, local_rank) if wlx == 5 else run_ours(a, rank, world, local_rank)
        o.pop("metric", None)
        o["config"]["M"] = M
        subs.append(o)
    return subs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=0, choices=[0, 1, 2, 3, 4, 5],
                    help="0 (default): the 7B block at M = 2048 as the headline line, with the decode GEMV (M = 1), "
                         "the single 4096^2 linear (M = 16) and the bulk quantize round trip as sub_results")
    ap.add_argument("--no-sub", action="store_true", help="default workload: skip the sub_results")
    ap.add_argument("--quant", choices=["nf4", "fp4"], default="nf4", help="4-bit quant type of the frozen weights")
    ap.add_argument("--dropout", type=float, default=0.0, help="LoRA dropout rate of the linear-layer step")
    ap.add_argument("--op", choices=["linear", "merge", "adamw"], default="linear",
                    help="merge: time nf4_dequant_merge over the 7B block's projections; adamw: one 8-bit AdamW "
                         "step over every adapter of a 32-layer 7B model")
    ap.add_argument("--layers", type=int, default=0, help="workload 5: number of 7-tensor layers (default 32)")
    ap.add_argument("--M", type=int, default=0, help="tokens per GPU (default: the workload's largest)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed steps eagerly instead of as CUDA graphs")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--clock-ms", type=int, default=200, help="nvidia-smi clock sampling period during the timed region")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        if rank == 0:                 # one rank (re)builds the in-tree library if a source is newer
            build_lib()
        dist.barrier()
    build_lib()
    try:
        if args.op == "merge":
            out = run_merge(args, rank, world, local_rank)
        elif args.op == "adamw":
            out = run_adamw(args, rank, world, local_rank)
        elif args.workload == 5:
            out = run_bulk(args, rank, world, local_rank)
        else:
            out = run_ours(args, rank, world, local_rank)
        if args.workload == 0 and args.op == "linear" and world == 1 and not args.no_sub:
            out["sub_results"] = sub_results(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
