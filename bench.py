#!/usr/bin/env python
"""Throughput of the DDTS recurrence (Rodimus) on B200, as one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline: tokens/s of the chunked forward on the 130M-scale layer workload
(B=8, H=6, T=2048, d_k=64, d_v=128, bf16 in / fp32 state, chunk 64); tokens =
B*T per step, all heads included.  Inputs are resident in HBM; the L2 is flushed
(256 MB write) before every timed step because the inputs (101 MB) fit in it.
With N > 1 (torchrun, one rank per GPU) every rank runs its own batch of the
same size (weak scaling: the sequences are independent, there is no data-path
exchange), time is the max over ranks and `value` counts all ranks' tokens.

At N = 1 the same line also carries, under "workloads", the long-context
forward (B=1, H=16, T=32768, d_k=d_v=128, S_T returned), the training
forward+backward (B=4, H=16, T=4096, d_k=64, d_v=128), the same backward with
every 16th head given one chunk too wide for one decay reference (those heads
are recomputed by the exact CUDA-core backward), the batched decode (B=256,
H=16, d_k=64, d_v=128, 1024 steps in one CUDA graph), the forward variants
(gates before their activations, rank-16 beta_hat, feedthrough), ShortConv
and SW-SKA, each with the roofline of its kernels, and the fp64 oracle timed on
the host cores.

`--impl reference` times the fp64 CPU oracle (the only reference: the pages
publish no implementation) on bounded samples of the headline workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_linear_attention_ddts_b200.workloads import (SKA_DEC, SKA_FWD, WORKLOADS,  # noqa: E402
                                                        draw_decode, draw_lowrank, draw_workload)

SEQ = ("q", "k", "v", "g", "tau", "beta")
METRIC = "DDTS recurrence tokens/s (fwd, fwd+bwd, decode) on 1 B200; % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def fwd_bytes(w, with_state_out):
    """Algorithmic bytes of one forward: every input read once, every output
    written once (bf16 sequences, fp32 states)."""
    e = 2 if w.dtype == "bf16" else 4
    bh = w.B * w.H
    b = bh * w.T * e * (4 * w.dk + 3 * w.dv)
    if w.s0_std:
        b += bh * w.dk * w.dv * 4
    if with_state_out:
        b += bh * w.dk * w.dv * 4
    return b


def bwd_bytes(w):
    """Backward: q,k,g,tau,v,beta,dO read, dq,dk,dg,dtau,dv,dbeta written, S_0 read,
    dS_0 written."""
    e = 2 if w.dtype == "bf16" else 4
    bh = w.B * w.H
    return bh * w.T * e * (8 * w.dk + 5 * w.dv) + 2 * bh * w.dk * w.dv * 4


def decode_bytes(w):
    """One decode step: state read and written (fp32), q,k,g,tau,v,beta read, o written."""
    bh = w.B * w.H
    return bh * (2 * w.dk * w.dv * 4 + 2 * (4 * w.dk + 2 * w.dv) + 2 * w.dv)


def chunk_flops_fwd(w, C=64):
    # per token-head: causal half of Qt Kt^T and A V (C+1)(dk+dv), inter-chunk Q S and K^T V 4 dk dv
    return w.B * w.H * w.T * ((C + 1) * (w.dk + w.dv) + 4 * w.dk * w.dv)


def chunk_flops_bwd(w, C=64):
    return w.B * w.H * w.T * ((C + 1) * (3 * w.dk + 2 * w.dv) + 10 * w.dk * w.dv)


# sources (kernel file and the device headers it includes) that a stored ncu
# traffic figure is keyed to: the figure is reported only while they are unchanged
_DEV_HDR = ["tc_ptx.cuh", "tc_common.cuh", "rdm_common.cuh", "launch.h"]
FWD_SRC = ["tc_fwd.cu"] + _DEV_HDR
BWD_SRC = ["tc_bwd.cu"] + _DEV_HDR
DECODE_SRC = ["decode.cu", "rdm_common.cuh", "launch.h"]
SKA_SRC = ["ska.cu", "ska_launch.h"] + _DEV_HDR
CONV_SRC = ["shortconv.cu", "conv_launch.h"] + _DEV_HDR
SIMT_SRC = ["simt.cu", "rdm_common.cuh", "launch.h"]


def src_sha(*names):
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "gated_linear_attention_ddts_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def ncu_counters(kernel, source_files, workload):
    """Counters of one ncu capture of `kernel` on `workload` from the committed
    summary (profiles/ncu_counters.json), or None when the kernel's source
    changed since that capture: DRAM bytes per launch, the tensor-pipe
    utilisation and the DRAM throughput ncu reported."""
    p = os.path.join(ROOT, "profiles", "ncu_counters.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{kernel}@{workload}")
    if not d or d.get("src_sha") != src_sha(*source_files):
        return None
    return d


def roofline(bytes_, flops, ms, pk, counters, timed_alone=True):
    """Roofline object of one kernel: achieved = algorithmic bytes (or flops) per
    launch / measured time.  `counters` (ncu_counters) adds the DRAM traffic of
    a launch and the captured kernel's tensor-pipe and DRAM utilisation."""
    traffic = counters.get("dram_bytes_per_launch") if counters else None
    t = ms / 1e3
    ach_gbs = bytes_ / t / 1e9
    ach_tf = flops / t / 1e12
    tf_peak = pk["bf16_tflops"] if timed_alone else pk["bf16_tflops_sustained"]
    t_hbm = bytes_ / (pk["hbm_gbs"] * 1e9)
    t_tc = flops / (tf_peak * 1e12)
    if t_hbm >= t_tc:
        out = {"bound": "hbm", "achieved": round(ach_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
               "frac": round(ach_gbs / pk["hbm_gbs"], 4), "traffic": traffic,
               "algorithmic_bytes": int(bytes_), "peak_source": pk["source"]}
    else:
        out = {"bound": "tensor", "achieved": round(ach_tf, 2), "peak": tf_peak, "unit": "TFLOP/s",
               "frac": round(ach_tf / tf_peak, 4), "traffic": traffic,
               "algorithmic_flops": int(flops), "peak_source": pk["source"]}
    if counters:
        out["ncu"] = {k: counters[k] for k in ("tensor_pipe_pct", "dram_throughput_pct",
                                               "dram_gbs", "issue_active_pct", "duration_us")
                      if k in counters}
    return out


class ClockSampler:
    """Polls NVML (SM clock, max clock, clock-event reasons) every 2 ms."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hi = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hi)
                u = u.decode() if isinstance(u, bytes) else u
                if u.endswith(uuid) or uuid.endswith(u.replace("GPU-", "")):
                    h = hi
            if h is None and pynvml.nvmlDeviceGetCount() == 1:
                h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.nv, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = h is not None
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.th.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def time_steps(fn, K, W, flush=None, barrier=None):
    """Device time of each of K steps (CUDA events on the launching stream),
    after W untimed warm-up steps; flush (if any) runs between steps, outside
    the events.  Barrier + synchronize on both sides of the timed loop."""
    for _ in range(W):
        if flush is not None:
            flush()
        fn()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    for a, b in ev:
        if flush is not None:
            flush()
        a.record(st)
        fn()
        b.record(st)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    return [a.elapsed_time(b) for a, b in ev]


# ------------------------------------------------------------ workloads
def fwd_workspace(rdm, x, dev):
    """Scratch that lets the forward cut sequences into segments (allocated
    once, outside the timed region); False when the forward needs none."""
    n = rdm.rdm_ddts_fwd_workspace_size(*(x[k] for k in SEQ))
    return torch.empty(n, dtype=torch.uint8, device=dev) if n else False


def run_headline(rdm, w, K, W, dev, flush, barrier, pk, rank):
    x = draw_workload(w, device=dev, seed=w.seed + 1000 * rank)
    o = torch.empty(w.B, w.H, w.T, w.dv, dtype=torch.bfloat16, device=dev)
    wsf = fwd_workspace(rdm, x, dev)
    fn = lambda: rdm.rdm_ddts_fwd(*(x[n] for n in SEQ), x["S0"], o, workspace=wsf)
    with ClockSampler(dev) as clk:
        times = time_steps(fn, K, W, flush, barrier)
    status = rdm.rdm_ddts_sync_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    # end to end through the public API with pinned host buffers
    hx = {n: x[n].cpu().pin_memory() for n in SEQ}
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    dx = {n: torch.empty_like(x[n]) for n in SEQ}

    def e2e_step():
        for n in SEQ:
            dx[n].copy_(hx[n], non_blocking=True)
        rdm.rdm_ddts_fwd(*(dx[n] for n in SEQ), None, o, workspace=wsf)
        ho.copy_(o, non_blocking=True)

    e2e_times = time_steps(e2e_step, max(3, min(K, 10)), 2, None, barrier)
    h2d = sum(hx[n].numel() * hx[n].element_size() for n in SEQ)
    d2h = ho.numel() * ho.element_size()
    return times, clk.summary(), e2e_times, h2d, d2h


def run_extras(rdm, dev, pk, K):
    out = {}
    # long-context forward, S_T returned (inputs 940 MB > L2: no flush needed)
    w = WORKLOADS[2]
    x = draw_workload(w, device=dev)
    o = torch.empty(w.B, w.H, w.T, w.dv, dtype=torch.bfloat16, device=dev)
    ST = torch.empty(w.B, w.H, w.dk, w.dv, device=dev)
    wsf = fwd_workspace(rdm, x, dev)
    t = time_steps(lambda: rdm.rdm_ddts_fwd(*(x[n] for n in SEQ), x["S0"], o, ST, workspace=wsf),
                   max(3, K // 2), 2)
    ms = statistics.mean(t)
    out["long_context_fwd"] = {
        "workload": w.name, "value": w.B * w.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
        "gpu_launches_per_step": 1,
        "roofline": roofline(fwd_bytes(w, True), chunk_flops_fwd(w), ms, pk,
                             ncu_counters("tc_fwd_kernel", FWD_SRC, 2))}
    del x, o, ST, wsf
    # headline forward with the gate activations fused (inputs are the
    # pre-activations; same bytes)
    w = WORKLOADS[1]
    x = draw_workload(w, device=dev, preact=True)
    o = torch.empty(w.B, w.H, w.T, w.dv, dtype=torch.bfloat16, device=dev)
    n = rdm.rdm_ddts_fwd_workspace_size(*(x[k] for k in SEQ), gates="preact")
    wsf = torch.empty(n, dtype=torch.uint8, device=dev) if n else False
    fl = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    t = time_steps(lambda: rdm.rdm_ddts_fwd(*(x[k] for k in SEQ), x["S0"], o, workspace=wsf,
                                            gates="preact"), max(3, K // 2), 3, lambda: fl.zero_())
    ms = statistics.mean(t)
    out["fused_gates_fwd"] = {
        "workload": w.name + ", gates passed before softplus/sigmoid", "value": w.B * w.T / (ms / 1e3),
        "unit": "tokens/s", "ms_per_step": ms, "gpu_launches_per_step": 1,
        "roofline": roofline(fwd_bytes(w, False), chunk_flops_fwd(w), ms, pk,
                             ncu_counters("tc_fwd_kernel", FWD_SRC, "1pre"))}
    # the same with a rank-16 beta_hat built on chip from u [B,T,16] and w_up
    # [H,16,dv]: beta's pre-activation is no longer read
    u, wu = draw_lowrank(w.B, w.H, w.T, w.dv, 16, seed=w.seed + 40, device=dev)
    t = time_steps(lambda: rdm.rdm_ddts_fwd(*(x[k] for k in SEQ[:5]), None, x["S0"], o, workspace=wsf,
                                            gates="preact", beta_lowrank=(u, wu)),
                   max(3, K // 2), 3, lambda: fl.zero_())
    ms = statistics.mean(t)
    lr_bytes = fwd_bytes(w, False) - w.B * w.H * w.T * w.dv * 2 + u.numel() * 2 + wu.numel() * 4
    out["lowrank_beta_fwd"] = {
        "workload": w.name + ", gates passed before their activations, rank-16 beta_hat",
        "value": w.B * w.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
        "gpu_launches_per_step": 1,
        "roofline": roofline(lr_bytes, chunk_flops_fwd(w) + 2 * w.B * w.H * w.T * 16 * w.dv, ms, pk,
                             ncu_counters("tc_fwd_kernel", FWD_SRC, "1lr"))}
    del x, o, wsf, fl, u, wu
    # training forward + backward (forward saves chunk states for the backward)
    w = WORKLOADS[3]
    x = draw_workload(w, device=dev)
    o = torch.empty(w.B, w.H, w.T, w.dv, dtype=torch.bfloat16, device=dev)
    saved = torch.empty(rdm.rdm_ddts_saved_states_size(w.B, w.H, w.T, w.dk, w.dv, 64) // 4,
                        device=dev)
    grads = {n: torch.empty_like(x[r]) for n, r in (("dq", "q"), ("dk", "k"), ("dg", "g"),
                                                     ("dtau", "tau"), ("dv", "v"), ("dbeta", "beta"))}
    grads["dS0"] = torch.empty_like(x["S0"])
    ws_n = rdm.rdm_ddts_bwd_workspace_size(*(x[n] for n in SEQ), x["S0"], x["dO"], None, saved)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev)
    wsf = fwd_workspace(rdm, x, dev)
    fwd = lambda: rdm.rdm_ddts_fwd(*(x[n] for n in SEQ), x["S0"], o, None, saved, workspace=wsf)
    bwd = lambda: rdm.rdm_ddts_bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], None, saved,
                                   grads=grads, workspace=ws)
    Kb = max(3, K // 4)
    tf = time_steps(fwd, Kb, 2)
    tb = time_steps(bwd, Kb, 2)
    msf, msb = statistics.mean(tf), statistics.mean(tb)
    fb = fwd_bytes(w, False)  # the saved chunk states are scratch, not algorithmic traffic
    out["training_fwd_bwd"] = {
        "workload": w.name, "value": w.B * w.T / ((msf + msb) / 1e3), "unit": "tokens/s",
        "ms_per_step": msf + msb, "ms_fwd": msf, "ms_bwd": msb,
        # forward kernel; backward kernel, the flagged-head list and the exact
        # re-run (local and full passes of both sweeps over 8 segments, the carry
        # fix-up: small grids that exit at once when no head is flagged)
        "gpu_launches_per_step": 8,
        "roofline_fwd": roofline(fb, chunk_flops_fwd(w), msf, pk,
                                 ncu_counters("tc_fwd_kernel", FWD_SRC, 3)),
        "roofline_bwd": roofline(bwd_bytes(w), chunk_flops_bwd(w), msb, pk,
                                 ncu_counters("tc_bwd_kernel", BWD_SRC, 3)),
        "roofline_step": roofline(fb + bwd_bytes(w), chunk_flops_fwd(w) + chunk_flops_bwd(w),
                                  msf + msb, pk, None)}
    # the same backward with one chunk of every 16th head too wide for one decay
    # reference (g scaled up 40x there): those heads are recomputed whole by the
    # exact CUDA-core backward, which this line prices
    gw = x["g"].float()
    gw[:, ::16, 64 * 20:64 * 21] *= 40.0
    x["g"] = gw.clamp(min=0.05).to(torch.bfloat16)
    del gw
    fwd()
    tw = time_steps(bwd, max(3, K // 8), 2)
    msw = statistics.mean(tw)
    out["training_bwd_wide_heads"] = {
        "workload": w.name + ", one chunk in every 16th head too wide for one reference",
        "value": w.B * w.T / (msw / 1e3), "unit": "tokens/s", "ms_per_step": msw,
        "ms_bwd_without": msb, "wide_heads": w.B * ((w.H + 15) // 16),
        # backward kernel, the flagged-head list and the five exact re-run launches
        "gpu_launches_per_step": 7,
        # the backward's algorithmic bytes over the whole step: the recomputed heads
        # are latency-bound token-serial sweeps, not a bandwidth problem
        "roofline": roofline(bwd_bytes(w), chunk_flops_bwd(w), msw, pk, None),
        "ncu_exact_sweeps": {"reverse": ncu_counters("simt_bwd_rsweep", SIMT_SRC, "wide3"),
                             "forward": ncu_counters("simt_bwd_fsweep", SIMT_SRC, "wide3")}}
    del x, o, saved, grads, ws, wsf
    # headline forward with the feedthrough o_t += d (.) v_t (same algorithmic
    # bytes plus d; v is re-read from L2 in the store stage)
    w = WORKLOADS[1]
    x = draw_workload(w, device=dev)
    o = torch.empty(w.B, w.H, w.T, w.dv, dtype=torch.bfloat16, device=dev)
    dfe = torch.randn(w.H, w.dv, device=dev, generator=torch.Generator(device=dev).manual_seed(3))
    wsf = fwd_workspace(rdm, x, dev)
    fl = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    t = time_steps(lambda: rdm.rdm_ddts_fwd(*(x[k] for k in SEQ), x["S0"], o, workspace=wsf,
                                            feedthrough=dfe), max(3, K // 2), 3, lambda: fl.zero_())
    ms = statistics.mean(t)
    out["feedthrough_fwd"] = {
        "workload": w.name + ", feedthrough o += d * v", "value": w.B * w.T / (ms / 1e3),
        "unit": "tokens/s", "ms_per_step": ms, "gpu_launches_per_step": 1,
        "roofline": roofline(fwd_bytes(w, False) + w.H * w.dv * 4, chunk_flops_fwd(w), ms, pk,
                             ncu_counters("tc_fwd_kernel", FWD_SRC, "1feed"))}
    del x, o, wsf, dfe
    # ShortConv (width 4, SiLU) forward + backward on the q, k and v tensors of
    # the same layer (D = 64, 64, 128)
    gen = torch.Generator(device=dev).manual_seed(4)
    convs = []
    for D in (w.dk, w.dk, w.dv):
        xc = torch.randn(w.B, w.H, w.T, D, device=dev, generator=gen).to(torch.bfloat16)
        wc = torch.randn(w.H, D, 4, device=dev, generator=gen) / 4
        bc = torch.randn(w.H, D, device=dev, generator=gen) * 0.1
        gy = torch.randn(w.B, w.H, w.T, D, device=dev, generator=gen).to(torch.bfloat16)
        outs = dict(dx=torch.empty_like(xc), dw=torch.empty_like(wc), dbias=torch.empty_like(bc))
        convs.append((xc, wc, bc, gy, torch.empty_like(xc), outs))

    # the three tensors in one batched forward and one batched backward launch
    fwd_many = [dict(x=xc, weight=wc, bias=bc, y=yc) for xc, wc, bc, gy, yc, outs in convs]
    bwd_many = [dict(x=xc, weight=wc, bias=bc, grad_y=gy, out=outs) for xc, wc, bc, gy, yc, outs in convs]

    def conv_step():
        rdm.rdm_shortconv_fwd_many(fwd_many, silu=True)
        rdm.rdm_shortconv_bwd_many(bwd_many, silu=True)

    # short kernels: replayed as one CUDA graph so that the step is timed on the
    # device, not through the Python binding's per-call overhead
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        conv_step()
        gconv = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gconv, stream=side):
            conv_step()
    torch.cuda.current_stream().wait_stream(side)
    t = time_steps(lambda: gconv.replay(), max(3, K // 2), 3, lambda: fl.zero_())
    ms = statistics.mean(t)
    cb = w.B * w.H * w.T * 2 * (w.dk + w.dk + w.dv) * (2 + 3)   # fwd: x, y; bwd: x, dy, dx
    out["shortconv_fwd_bwd"] = {
        "workload": "ShortConv width 4 + SiLU, fwd+bwd over q, k, v of " + w.name,
        "value": w.B * w.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
        # one batched forward and one batched backward kernel (the weight gradients
        # are zeroed by memsets, not counted)
        "gpu_launches_per_step": 2, "cuda_graph": True,
        "roofline": roofline(cb, 0, ms, pk, None)}
    del gconv, convs, fl
    out.update(run_ska(rdm, dev, pk, K))
    # batched decode, 1024 steps captured in one CUDA graph
    w = WORKLOADS[4]
    steps = w.T
    xd = draw_decode(w.B, w.H, w.dk, w.dv, steps, torch.bfloat16, seed=w.seed, device=dev)
    S = torch.zeros(w.B, w.H, w.dk, w.dv, device=dev)
    od = torch.empty(steps, w.B, w.H, w.dv, dtype=torch.bfloat16, device=dev)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for s in range(2):  # warm-up before capture
            rdm.rdm_ddts_decode_step(*(xd[n][s] for n in SEQ), S, od[s])
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for s in range(steps):
                rdm.rdm_ddts_decode_step(*(xd[n][s] for n in SEQ), S, od[s])
    torch.cuda.current_stream().wait_stream(side)
    t = time_steps(lambda: g.replay(), 5, 2)
    ms = statistics.mean(t)
    per = ms / steps
    out["decode"] = {
        "workload": w.name, "value": w.B * steps / (ms / 1e3), "unit": "tokens/s",
        "ms_per_step": per, "ms_per_graph": ms, "gpu_launches_per_step": 1,
        "roofline": roofline(decode_bytes(w), 2 * w.B * w.H * w.dk * w.dv * 3, per, pk,
                             ncu_counters("decode_kernel", DECODE_SRC, 4), timed_alone=False)}
    del g, xd, S, od
    return out


def ska_keys(T, window):
    """Query-key pairs inside the sliding window: sum_t min(t + 1, window)."""
    n = min(T, window)
    return n * (n + 1) // 2 + (T - n) * window


def run_ska(rdm, dev, pk, K):
    """Sliding-window shared-key attention of the Rodimus+ block: the forward
    on a 130M-scale layer and batched decode against ring KV caches."""
    out = {}
    B, H, T, d, win = SKA_FWD
    gen = torch.Generator(device=dev).manual_seed(5)
    q = torch.randn(B, H, T, d, device=dev, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, T, d, device=dev, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, H, T, d, device=dev, generator=gen).to(torch.bfloat16)
    o = torch.empty_like(v)
    fl = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    t = time_steps(lambda: rdm.rdm_ska_fwd(q, k, v, win, o=o), max(3, K // 2), 3, lambda: fl.zero_())
    ms = statistics.mean(t)
    pairs = B * H * ska_keys(T, win)
    out["ska_fwd"] = {
        "workload": f"SW-SKA forward B{B} H{H} T{T} d_k=d_v={d} window {win} (one shared key head)",
        "value": B * T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
        "gpu_launches_per_step": 1,
        "roofline": roofline(2 * (B * H * T * 3 * d + B * T * d), 2 * pairs * 2 * d, ms, pk,
                             ncu_counters("ska_fwd_kernel", SKA_SRC, "ska1")),
        "exp2_per_step": pairs}
    del q, k, v, o
    # decode: rings full (positions from 1000 on), STEPS tokens per CUDA graph
    B, H, d, win, steps = SKA_DEC
    kc = torch.randn(B, win, d, device=dev, generator=gen).to(torch.bfloat16)
    vc = torch.randn(B, H, win, d, device=dev, generator=gen).to(torch.bfloat16)
    xq = torch.randn(steps, B, H, d, device=dev, generator=gen).to(torch.bfloat16)
    xk = torch.randn(steps, B, d, device=dev, generator=gen).to(torch.bfloat16)
    xv = torch.randn(steps, B, H, d, device=dev, generator=gen).to(torch.bfloat16)
    od = torch.empty(steps, B, H, d, dtype=torch.bfloat16, device=dev)
    pos = torch.full((B,), 1000, dtype=torch.int32, device=dev)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        rdm.rdm_ska_decode(xq[0], xk[0], xv[0], kc, vc, pos, o=od[0])
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for s_ in range(steps):
                rdm.rdm_ska_decode(xq[s_], xk[s_], xv[s_], kc, vc, pos, o=od[s_])
    torch.cuda.current_stream().wait_stream(side)
    t = time_steps(lambda: g.replay(), 5, 2)
    ms = statistics.mean(t)
    per = ms / steps
    # per step: every cached key row once, every cached value row once, q, k, v
    # in, o out, the new key and value rows written
    by = 2 * (B * win * d + B * H * win * d + B * H * d * 3 + B * d * 2 + B * H * d)
    out["ska_decode"] = {
        "workload": f"SW-SKA decode B{B} H{H} d_k=d_v={d} window {win}, full rings, "
                    f"{steps} steps per CUDA graph",
        "value": B * steps / (ms / 1e3), "unit": "tokens/s", "ms_per_step": per,
        "ms_per_graph": ms, "gpu_launches_per_step": 2, "cuda_graph": True,
        "roofline": roofline(by, 2 * B * H * win * 2 * d, per, pk,
                             ncu_counters("ska_decode_kernel", SKA_SRC, "ska4"), timed_alone=False)}
    del g, kc, vc, xq, xk, xv, od
    return out


def cpu_oracle_rate(w, min_seconds=10.0, max_seconds=30.0, heads=None):
    """fp64 oracle tokens/s on the host cores over repeated full passes (or a
    head subset) of workload w."""
    import oracle
    nthreads = oracle.default_threads()
    H = heads or w.H
    x = draw_workload(w, device="cpu", H=H)
    xs = [oracle._f64(x[n]) for n in SEQ]
    done, t0 = 0, time.time()
    while True:
        oracle.fwd(*xs, nthreads=nthreads)
        done += 1
        el = time.time() - t0
        if el >= min_seconds or el >= max_seconds:
            break
    tokens = done * w.B * w.T * H / w.H
    return tokens / el, nthreads, f"{done} fp64 oracle forward passes over B={w.B}, H={H} " \
                                   f"of {w.H} heads, T={w.T} ({el:.1f} s)"


# ------------------------------------------------------------------ main
def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of `values` over all ranks of the process group
    (the values themselves without one)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_value(tokens_per_rank, world, ms_per_step):
    """Whole-job tokens/s: every rank processes its own batch in the step time
    of the slowest rank."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="headline workload only")
    a = ap.parse_args()
    K, W = a.steps, max(3, a.warmup)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    w = WORKLOADS[1]
    cfg = {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d_k": w.dk, "d_v": w.dv,
           "chunk": 64, "global_batch": w.B * world, "seq_len": w.T,
           "parallelism": f"replicas x{world} (sequences independent)",
           "l2": "flushed (256 MB write) before every timed step"}

    if a.impl == "reference":
        if rank != 0:
            return 0
        times = []
        rate_samples = []
        import oracle
        nthreads = oracle.default_threads()
        xr = draw_workload(w, device="cpu", H=2)
        xs = [oracle._f64(xr[n]) for n in SEQ]
        for i in range(W + K):
            t0 = time.time()
            oracle.fwd(*xs, nthreads=nthreads)
            dt = time.time() - t0
            if i >= W:
                times.append(dt)
        mean = statistics.mean(times)
        tokens = w.B * w.T * 2 / w.H
        val = tokens / mean
        sample = f"each step: fp64 oracle forward over B={w.B}, 2 of {w.H} heads, T={w.T}"
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": mean * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return 0

    import gated_linear_attention_ddts_b200 as rdm
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    barrier = (lambda: dist.barrier()) if dist else None
    pk = peaks()
    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush = lambda: flush_buf.zero_()

    times, clocks, e2e_times, h2d, d2h = run_headline(rdm, w, K, W, dev, flush, barrier, pk, rank)
    total, e2e_ms = max_over_ranks([sum(times), sum(e2e_times) / len(e2e_times)], dist, dev)
    ms = total / K
    tokens = w.B * w.T * world
    value = weak_scaling_value(w.B * w.T, world, ms)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; generators in "
        "gated_linear_attention_ddts_b200/workloads.py)", "config": cfg,
        "token_heads_per_s": value * w.H,
        "roofline": roofline(fwd_bytes(w, False), chunk_flops_fwd(w), ms, pk,
                             ncu_counters("tc_fwd_kernel", FWD_SRC, 1)),
        "clocks": clocks,
        "e2e": {"value": weak_scaling_value(w.B * w.T, world, e2e_ms), "unit": "tokens/s",
                "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": K,
    }
    if world == 1 and rank == 0:
        if not a.no_extras:
            line["workloads"] = run_extras(rdm, dev, pk, K)
        val, cores, sample = cpu_oracle_rate(w)
        line["cpu_baseline"] = {"value": val, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
