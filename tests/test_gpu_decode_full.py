"""The batched decode workload at its full size against the fp64 oracle.

B=256, H=16, d_k=64, d_v=128, 1024 single-token steps on an fp32 state that
stays in HBM, bf16 per-step inputs; the GPU runs the 1024 steps as one CUDA
graph of rdm_ddts_decode_step launches, exactly as the bench times them.  The
oracle then replays the same 1024 steps token by token in float64 on the host
cores.  Checked: o of every step for every (b,h), and the state after the last
step (sequential inference on a fixed-size state: paperhub.cn OpenReview
rebuttal, answer to Q2).  This is where the fp32 rounding of the state
accumulates over many steps, which a short decode cannot show."""
import numpy as np
import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
import oracle
from gated_linear_attention_ddts_b200.workloads import WORKLOADS, draw_decode
from tests.parity import TOL, assert_close, max_rel_err

pytestmark = pytest.mark.gpu
SEQ = ("q", "k", "v", "g", "tau", "beta")


def test_config4_decode_full_size(cuda_ok):
    w = WORKLOADS[4]
    steps = w.T
    xd = draw_decode(w.B, w.H, w.dk, w.dv, steps, torch.bfloat16, seed=w.seed, device="cuda")
    S = torch.zeros(w.B, w.H, w.dk, w.dv, device="cuda")
    od = torch.empty(steps, w.B, w.H, w.dv, dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        # one eager call (first-use set-up) on a scratch state, then the graph
        scratch = torch.zeros_like(S)
        rdm.rdm_ddts_decode_step(*(xd[n][0] for n in SEQ), scratch, od[0])
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for s in range(steps):
                rdm.rdm_ddts_decode_step(*(xd[n][s] for n in SEQ), S, od[s])
    torch.cuda.current_stream().wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    del g

    S_ref = np.zeros((w.B, w.H, w.dk, w.dv))
    worst = 0.0
    for s in range(steps):
        o_ref = oracle.decode_step(*(xd[n][s].cpu() for n in SEQ), S_ref)
        e = max_rel_err(od[s], o_ref)
        worst = max(worst, e)
        assert e <= TOL[torch.bfloat16], f"config 4 o at step {s}: max rel err {e:.3e}"
        if s in (0, steps // 2, steps - 1):
            assert_close(od[s], o_ref, TOL[torch.bfloat16], f"config 4 o step {s}")
    assert_close(S, S_ref, TOL[torch.bfloat16], "config 4 final state")
    print(f"config 4: worst o error over {steps} steps {worst:.3e}")
