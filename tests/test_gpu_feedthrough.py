"""The feedthrough o_t += d (.) v_t (the d_t of the paper's Eq. (11), the SSM
feedthrough per the paperhub.cn OpenReview rebuttal's answer to Q6) on every
GPU path, against the fp64 oracle: the tensor-core forward (whole chunks,
narrow windows, sequence segments), the exact float32 path, the decode step,
and both backward paths including the gradient of d."""
import numpy as np
import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
import oracle
from gated_linear_attention_ddts_b200.workloads import draw_decode, draw_sequence
from tests.parity import TOL, assert_close

pytestmark = pytest.mark.gpu
SEQ = ("q", "k", "v", "g", "tau", "beta")
GR = ("dq", "dk", "dv", "dg", "dtau", "dbeta", "dS0")


def feed_weights(H, dv, seed):
    return torch.randn(H, dv, generator=torch.Generator().manual_seed(seed)) * 0.5


def dev(x):
    return {n: (t.cuda() if t is not None else None) for n, t in x.items()}


@pytest.mark.parametrize("dk,dv,T,B,H", [(64, 128, 200, 2, 2), (64, 64, 64 * 9 + 5, 1, 2),
                                         (128, 64, 130, 2, 3), (128, 128, 64 * 8, 1, 1)])
def test_feedthrough_forward_tc(cuda_ok, dk, dv, T, B, H):
    x = draw_sequence(B, H, T, dk, dv, torch.bfloat16, seed=900 + T + dk + dv, s0_std=0.1)
    d = feed_weights(H, dv, T)
    dx = dev(x)
    o, ST = rdm.rdm_ddts_fwd(*(dx[n] for n in SEQ), dx["S0"], impl="tc", return_state=True,
                             feedthrough=d.cuda())
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"], d=d)
    assert_close(o, o_ref, TOL[torch.bfloat16], "o with feedthrough")
    assert_close(ST, S_ref, TOL[torch.bfloat16], "S_T with feedthrough")


@pytest.mark.parametrize("chunk", [16, 64])
def test_feedthrough_forward_tc_windows(cuda_ok, chunk):
    """Wide decay: 16- and single-token windows write o rows directly."""
    x = draw_sequence(1, 2, 150, 64, 128, torch.bfloat16, seed=931, s0_std=0.1)
    x["g"] = (x["g"].float() * 40.0).to(torch.bfloat16)
    d = feed_weights(2, 128, 931)
    dx = dev(x)
    o, _ = rdm.rdm_ddts_fwd(*(dx[n] for n in SEQ), dx["S0"], impl="tc", chunk=chunk,
                            feedthrough=d.cuda())
    torch.cuda.synchronize()
    o_ref, _ = oracle.fwd(*(x[n] for n in SEQ), x["S0"], d=d)
    assert_close(o, o_ref, TOL[torch.bfloat16], f"o with feedthrough, chunk {chunk}")


def test_feedthrough_forward_fp32(cuda_ok):
    x = draw_sequence(2, 3, 77, 16, 32, torch.float32, seed=941, s0_std=0.1)
    d = feed_weights(3, 32, 941)
    dx = dev(x)
    o, ST = rdm.rdm_ddts_fwd(*(dx[n] for n in SEQ), dx["S0"], return_state=True,
                             feedthrough=d.cuda())
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"], d=d)
    assert_close(o, o_ref, 1e-4, "fp32 o with feedthrough")
    assert_close(ST, S_ref, 1e-4, "fp32 S_T with feedthrough")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_feedthrough_decode(cuda_ok, dtype):
    B, H, dk, dv, steps = 3, 4, 64, 128, 5
    xd = draw_decode(B, H, dk, dv, steps, dtype, seed=951)
    d = feed_weights(H, dv, 951)
    S = torch.zeros(B, H, dk, dv, device="cuda")
    S_ref = np.zeros((B, H, dk, dv))
    for t in range(steps):
        o = rdm.rdm_ddts_decode(*(xd[n][t].cuda() for n in SEQ), S, feedthrough=d.cuda())
        o_ref = oracle.decode_step(*(xd[n][t] for n in SEQ), S_ref, d=d)
        torch.cuda.synchronize()
        assert_close(o, o_ref, TOL[dtype], f"decode o with feedthrough, step {t}")
    assert_close(S, S_ref, TOL[dtype], "decode state with feedthrough")


@pytest.mark.parametrize("impl,dtype,dv,T", [("tc", torch.bfloat16, 128, 130),
                                             ("tc", torch.bfloat16, 64, 64 * 9 + 3),
                                             ("simt", torch.float32, 32, 45),
                                             ("simt", torch.bfloat16, 128, 70)])
def test_feedthrough_backward(cuda_ok, impl, dtype, dv, T):
    dk = 64 if impl == "tc" else 16
    x = draw_sequence(2, 2, T, dk, dv, dtype, seed=961 + T, s0_std=0.1, with_dO=True)
    d = feed_weights(2, dv, 961 + T)
    dST = 0.1 * torch.randn(2, 2, dk, dv, generator=torch.Generator().manual_seed(T))
    dx = dev(x)
    gr = rdm.rdm_ddts_bwd(*(dx[n] for n in SEQ), dx["S0"], dx["dO"], dST.cuda(), impl=impl,
                          feedthrough=d.cuda())
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    ref = oracle.bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], dST, d=d)
    tol = TOL[dtype]
    for n in GR:
        assert_close(gr[n], ref[n], tol, f"{impl} {n} with feedthrough")
    assert_close(gr["dfeed"], ref["dd"], tol, f"{impl} grad of the feedthrough weights")
