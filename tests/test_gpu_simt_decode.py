"""GPU parity of the exact CUDA-core path and of the decode step against the
fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
import oracle
from gated_linear_attention_ddts_b200.workloads import WORKLOADS, draw_decode, draw_sequence
from tests.parity import TOL, assert_close, np64

pytestmark = pytest.mark.gpu


def dev_inputs(x):
    return {n: (t.cuda() if t is not None else None) for n, t in x.items()}


def test_config0_fp32_forward(cuda_ok):
    w = WORKLOADS[0]
    x = draw_sequence(w.B, w.H, w.T, w.dk, w.dv, torch.float32, seed=w.seed)
    d = dev_inputs(x)
    o, ST = rdm.rdm_ddts_fwd(d["q"], d["k"], d["v"], d["g"], d["tau"], d["beta"],
                             impl="simt", return_state=True)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["tau"], x["beta"])
    assert_close(o, o_ref, 1e-4, "o")
    assert_close(ST, S_ref, 1e-4, "S_T")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv,T", [(16, 32, 1), (32, 16, 77), (64, 128, 130), (128, 64, 65)])
def test_simt_forward_shapes(cuda_ok, dtype, dk, dv, T):
    x = draw_sequence(2, 3, T, dk, dv, dtype, seed=100 + T, s0_std=0.1)
    d = dev_inputs(x)
    saved = torch.empty(rdm.rdm_ddts_saved_states_size(2, 3, T, dk, dv, 64) // 4,
                        device="cuda")
    o, ST = rdm.rdm_ddts_fwd(d["q"], d["k"], d["v"], d["g"], d["tau"], d["beta"], d["S0"],
                             saved_states=saved, impl="simt", return_state=True)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["tau"], x["beta"], x["S0"])
    assert_close(o, o_ref, TOL[dtype], "o")
    assert_close(ST, S_ref, TOL[dtype], "S_T")
    # saved chunk-start states: chunk c holds the state before token 64c
    nc = (T + 63) // 64
    sv = saved.view(2, 3, nc, dk, dv)
    for c in range(nc):
        if c == 0:
            ref = np64(x["S0"])
        else:
            _, ref = oracle.fwd(*(x[n][:, :, :64 * c] for n in ("q", "k", "v", "g", "tau",
                                                                "beta")), x["S0"])
        assert_close(sv[:, :, c], ref, TOL[dtype], f"saved state {c}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv,T", [(16, 32, 9), (64, 128, 70), (128, 32, 33), (32, 16, 48),
                                     (128, 128, 40)])
def test_simt_backward(cuda_ok, dtype, dk, dv, T):
    x = draw_sequence(1, 2, T, dk, dv, dtype, seed=200 + T, s0_std=0.1, with_dO=True)
    dST = torch.randn(1, 2, dk, dv, generator=torch.Generator().manual_seed(5)) * 0.1
    d = dev_inputs(x)
    gr = rdm.rdm_ddts_bwd(d["q"], d["k"], d["v"], d["g"], d["tau"], d["beta"], d["S0"],
                          d["dO"], dST.cuda(), impl="simt")
    torch.cuda.synchronize()
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["g"], x["tau"], x["beta"], x["S0"], x["dO"],
                     dST)
    for n in ("dq", "dk", "dv", "dg", "dtau", "dbeta", "dS0"):
        assert_close(gr[n], ref[n], TOL[dtype], n)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 128), (128, 128), (32, 64)])
def test_decode_steps(cuda_ok, dtype, dk, dv):
    B, H, steps = 3, 5, 6
    x = draw_decode(B, H, dk, dv, steps, dtype, seed=300 + dk)
    S0 = torch.randn(B, H, dk, dv, generator=torch.Generator().manual_seed(1)) * 0.1
    S = S0.cuda()
    S_ref = np.ascontiguousarray(np64(S0))
    for t in range(steps):
        xt = {n: x[n][t].cuda() for n in x}
        o = rdm.rdm_ddts_decode_step(xt["q"], xt["k"], xt["v"], xt["g"], xt["tau"],
                                     xt["beta"], S)
        o_ref = oracle.decode_step(*(x[n][t] for n in ("q", "k", "v", "g", "tau", "beta")),
                                   S_ref)
        torch.cuda.synchronize()
        assert_close(o, o_ref, TOL[dtype], f"o step {t}")
    assert_close(S, S_ref, TOL[dtype], "final state")


def test_decode_steps_match_forward(cuda_ok):
    """T decode steps on the GPU reproduce the GPU forward over the same T tokens."""
    B, H, T, dk, dv = 2, 2, 40, 64, 128
    x = draw_sequence(B, H, T, dk, dv, torch.bfloat16, seed=401, s0_std=0.1)
    d = dev_inputs(x)
    o, ST = rdm.rdm_ddts_fwd(d["q"], d["k"], d["v"], d["g"], d["tau"], d["beta"], d["S0"],
                             return_state=True)
    S = d["S0"].clone()
    for t in range(T):
        ot = rdm.rdm_ddts_decode_step(*(d[n][:, :, t].contiguous() for n in
                                        ("q", "k", "v", "g", "tau", "beta")), S)
        assert_close(ot, o[:, :, t], 2e-2, f"step {t}")
    assert_close(S, ST, 2e-2, "state")


def test_empty_sequence(cuda_ok):
    x = draw_sequence(1, 2, 0, 64, 64, torch.bfloat16, seed=7, s0_std=0.1)
    d = dev_inputs(x)
    o, ST = rdm.rdm_ddts_fwd(d["q"], d["k"], d["v"], d["g"], d["tau"], d["beta"], d["S0"],
                             return_state=True)
    torch.cuda.synchronize()
    assert o.numel() == 0
    assert torch.equal(ST, d["S0"])


def test_sync_status_clean(cuda_ok):
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv,T", [(16, 32, 1024 + 37), (64, 128, 2100)])
def test_simt_backward_segmented(cuda_ok, dtype, dk, dv, T):
    """Sequences of 1024 tokens and more run the exact backward in segments (two
    and four here): local maps, folds, full passes and the carry fix-up."""
    x = draw_sequence(1, 2, T, dk, dv, dtype, seed=250 + T, s0_std=0.1, with_dO=True)
    dST = torch.randn(1, 2, dk, dv, generator=torch.Generator().manual_seed(6)) * 0.1
    d = dev_inputs(x)
    gr = rdm.rdm_ddts_bwd(d["q"], d["k"], d["v"], d["g"], d["tau"], d["beta"], d["S0"],
                          d["dO"], dST.cuda(), impl="simt")
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["g"], x["tau"], x["beta"], x["S0"], x["dO"],
                     dST)
    for n in ("dq", "dk", "dv", "dg", "dtau", "dbeta", "dS0"):
        assert_close(gr[n], ref[n], TOL[dtype], f"segmented {n}")
