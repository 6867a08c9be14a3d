"""Small launches of each kernel for profiler captures (one workload per call).

    python -m gated_linear_attention_ddts_b200.profile_kernels fwd1|fwd2|fwdbwd3|decode4

Each mode draws its workload on the device, runs the kernel(s) a few times and
synchronises; it is the command that profiler captures wrap (the decode mode
draws only 4 steps of inputs instead of 1024, the kernel is the same)."""
import sys

import torch

import gated_linear_attention_ddts_b200 as rdm
from gated_linear_attention_ddts_b200.workloads import WORKLOADS, draw_decode, draw_workload

SEQ = ("q", "k", "v", "g", "tau", "beta")


def main(mode: str) -> int:
    if mode in ("fwd1", "fwd2"):
        w = WORKLOADS[1 if mode == "fwd1" else 2]
        x = draw_workload(w, device="cuda")
        for _ in range(3):
            rdm.rdm_ddts_fwd(*(x[n] for n in SEQ), x["S0"], return_state=w.return_state)
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
