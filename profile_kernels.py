#!/usr/bin/env python
"""Small launches of each kernel, the command that profiler captures wrap.

    python profile_kernels.py fwd1|fwd1pre|fwd1feed|fwd1lr|fwd2|fwdbwd3|bwdwide3|decode4|conv1|ska1|ska4

One workload per call: the mode draws its inputs on the device, runs the
kernel(s) three times and synchronises.  fwd1 is the 130M-scale layer forward
(B8 H6 T2048 d_k64 d_v128), fwd1pre the same with the gates passed before
their activations, fwd2 the long-context forward (B1 H16 T32768 d_k=d_v=128),
fwdbwd3 the training forward (saving chunk states) and backward (B4 H16 T4096
d_k64 d_v128), bwdwide3 the same with one chunk of every 16th head too wide for
one decay reference (g scaled by 40 there; the exact backward recomputes those
heads), decode4 four steps of the batched decode (B256 H16 d_k64 d_v128;
only 4 steps of inputs are drawn instead of 1024, the kernel is the same),
fwd1feed the 130M-scale layer forward with the feedthrough, fwd1lr the same
layer with the gates passed before their activations and a rank-16 beta_hat, conv1 the
ShortConv forward and backward (width 4, SiLU) on a q-shaped tensor of that
layer (B8 H6 T2048 D64), ska1 the sliding-window shared-key attention forward
(B8 H12 T2048 d_k=d_v=64, window 512) and ska4 its batched decode step against
full ring caches (B256 H16 d_k=d_v=128, window 512).
Exit status 0 only when the library's device status word is clear."""
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import gated_linear_attention_ddts_b200 as rdm  # noqa: E402
from gated_linear_attention_ddts_b200.workloads import (SKA_DEC, SKA_FWD, WORKLOADS,  # noqa: E402
                                                        draw_decode, draw_lowrank, draw_workload)

SEQ = ("q", "k", "v", "g", "tau", "beta")


def main(mode: str) -> int:
    if mode in ("fwd1", "fwd1pre", "fwd1feed", "fwd2", "fwd1lr"):
        w = WORKLOADS[2 if mode == "fwd2" else 1]
        pre = mode in ("fwd1pre", "fwd1lr")
        x = draw_workload(w, device="cuda", preact=pre)
        d = torch.randn(w.H, w.dv, device="cuda") if mode == "fwd1feed" else None
        lr = draw_lowrank(w.B, w.H, w.T, w.dv, 16, seed=w.seed + 40, device="cuda") \
            if mode == "fwd1lr" else None
        for _ in range(3):
            rdm.rdm_ddts_fwd(*(x[n] for n in SEQ[:5]), None if lr else x["beta"], x["S0"],
                             return_state=w.return_state, gates="preact" if pre else "activated",
                             feedthrough=d, beta_lowrank=lr)
    elif mode == "conv1":
        w = WORKLOADS[1]
        x = torch.randn(w.B, w.H, w.T, w.dk, device="cuda").to(torch.bfloat16)
        wt = torch.randn(w.H, w.dk, 4, device="cuda") / 4
        b = torch.randn(w.H, w.dk, device="cuda") * 0.1
        gy = torch.randn_like(x)
        for _ in range(3):
            rdm.rdm_shortconv_fwd(x, wt, b, None, silu=True)
            rdm.rdm_shortconv_bwd(x, wt, b, None, gy, None, silu=True)
    elif mode in ("ska1", "ska4"):
        gen = torch.Generator(device="cuda").manual_seed(5)
        if mode == "ska1":
            B, H, T, d, win = SKA_FWD
            q = torch.randn(B, H, T, d, device="cuda", generator=gen).to(torch.bfloat16)
            k = torch.randn(B, T, d, device="cuda", generator=gen).to(torch.bfloat16)
            v = torch.randn(B, H, T, d, device="cuda", generator=gen).to(torch.bfloat16)
            for _ in range(3):
                rdm.rdm_ska_fwd(q, k, v, win)
        else:
            B, H, d, win, _ = SKA_DEC
            kc = torch.randn(B, win, d, device="cuda", generator=gen).to(torch.bfloat16)
            vc = torch.randn(B, H, win, d, device="cuda", generator=gen).to(torch.bfloat16)
            q = torch.randn(B, H, d, device="cuda", generator=gen).to(torch.bfloat16)
            k = torch.randn(B, d, device="cuda", generator=gen).to(torch.bfloat16)
            v = torch.randn(B, H, d, device="cuda", generator=gen).to(torch.bfloat16)
            pos = torch.full((B,), 1000, dtype=torch.int32, device="cuda")
            for _ in range(3):
                rdm.rdm_ska_decode(q, k, v, kc, vc, pos)
    elif mode in ("fwdbwd3", "bwdwide3"):
        w = WORKLOADS[3]
        x = draw_workload(w, device="cuda")
        if mode == "bwdwide3":
            gw = x["g"].float()
            gw[:, ::16, 64 * 20:64 * 21] *= 40.0
            x["g"] = gw.clamp(min=0.05).to(torch.bfloat16)
        saved = torch.empty(rdm.rdm_ddts_saved_states_size(w.B, w.H, w.T, w.dk, w.dv, 64) // 4,
                            device="cuda")
        for _ in range(3):
            rdm.rdm_ddts_fwd(*(x[n] for n in SEQ), x["S0"], saved_states=saved)
            rdm.rdm_ddts_bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], None, saved)
    elif mode == "decode4":
        w = WORKLOADS[4]
        xd = draw_decode(w.B, w.H, w.dk, w.dv, 4, device="cuda")
        S = torch.zeros(w.B, w.H, w.dk, w.dv, device="cuda")
        for s in range(4):
            rdm.rdm_ddts_decode_step(*(xd[n][s] for n in SEQ), S)
    else:
        raise SystemExit(f"unknown mode {mode}")
    torch.cuda.synchronize()
    st = rdm.rdm_ddts_sync_status()
    print(mode, "status", st)
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main(sys.argv[1]))
