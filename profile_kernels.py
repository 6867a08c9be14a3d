#!/usr/bin/env python
"""Small launches of each kernel, the command that profiler captures wrap.

    python profile_kernels.py fwd1|fwd1pre|fwd2|fwdbwd3|decode4

One workload per call: the mode draws its inputs on the device, runs the
kernel(s) three times and synchronises.  fwd1 is the 130M-scale layer forward
(B8 H6 T2048 d_k64 d_v128), fwd1pre the same with the gates passed before
their activations, fwd2 the long-context forward (B1 H16 T32768 d_k=d_v=128),
fwdbwd3 the training forward (saving chunk states) and backward (B4 H16 T4096
d_k64 d_v128), decode4 four steps of the batched decode (B256 H16 d_k64 d_v128;
only 4 steps of inputs are drawn instead of 1024, the kernel is the same).
Exit status 0 only when the library's device status word is clear."""
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import gated_linear_attention_ddts_b200 as rdm  # noqa: E402
from gated_linear_attention_ddts_b200.workloads import (WORKLOADS, draw_decode,  # noqa: E402
                                                        draw_workload)

SEQ = ("q", "k", "v", "g", "tau", "beta")


def main(mode: str) -> int:
    if mode in ("fwd1", "fwd1pre", "fwd2"):
        w = WORKLOADS[2 if mode == "fwd2" else 1]
        pre = mode == "fwd1pre"
        x = draw_workload(w, device="cuda", preact=pre)
        for _ in range(3):
            rdm.rdm_ddts_fwd(*(x[n] for n in SEQ), x["S0"], return_state=w.return_state,
                             gates="preact" if pre else "activated")
    elif mode == "fwdbwd3":
        w = WORKLOADS[3]
        x = draw_workload(w, device="cuda")
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
