"""GPU parity of the fused gate activations (g, tau, beta passed before their
softplus / sigmoid / sigmoid) against the fp64 oracle in the same mode, through
the C ABI: tensor-core forward (one CTA per sequence and segmented) and
backward, the exact CUDA-core path in float32, and agreement with the
activated-input path on the same draws."""
import numpy as np
import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
import oracle
from gated_linear_attention_ddts_b200.workloads import draw_sequence
from tests.parity import assert_close

pytestmark = pytest.mark.gpu
SEQ = ("q", "k", "v", "g", "tau", "beta")
GR = ("dq", "dk", "dv", "dg", "dtau", "dbeta", "dS0")


def dev(x):
    return {n: (t.cuda() if t is not None else None) for n, t in x.items()}


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 65, 200, 64 * 9 + 3])
def test_preact_forward_tc(cuda_ok, dk, dv, T):
    x = draw_sequence(1, 2, T, dk, dv, torch.bfloat16, seed=500 + T + dk + dv, s0_std=0.1,
                      preact=True)
    d = dev(x)
    o, ST = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), d["S0"], impl="tc", gates="preact",
                             return_state=True)
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"], preact=True)
    assert_close(o, o_ref, 2e-2, "o")
    assert_close(ST, S_ref, 2e-2, "S_T")


def test_preact_matches_activated_inputs(cuda_ok):
    """Same draws through both modes (the activated mode gets the activations
    rounded to bf16, so the bar is the bf16 one)."""
    xp = draw_sequence(2, 3, 300, 64, 128, torch.bfloat16, seed=77, s0_std=0.1, preact=True)
    xa = draw_sequence(2, 3, 300, 64, 128, torch.bfloat16, seed=77, s0_std=0.1)
    dp, da = dev(xp), dev(xa)
    o1, S1 = rdm.rdm_ddts_fwd(*(dp[n] for n in SEQ), dp["S0"], gates="preact", return_state=True)
    o2, S2 = rdm.rdm_ddts_fwd(*(da[n] for n in SEQ), da["S0"], return_state=True)
    torch.cuda.synchronize()
    assert_close(o1, o2.float().cpu().numpy(), 2e-2, "o preact vs activated")
    assert_close(S1, S2.cpu().numpy(), 2e-2, "S_T preact vs activated")


def test_preact_forward_simt_fp32(cuda_ok):
    x = draw_sequence(1, 2, 150, 16, 32, torch.float32, seed=91, s0_std=0.1, preact=True)
    d = dev(x)
    o, ST = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), d["S0"], gates="preact", return_state=True)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"], preact=True)
    assert_close(o, o_ref, 1e-4, "o fp32")
    assert_close(ST, S_ref, 1e-4, "S_T fp32")


@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("T", [130, 64 * 9 + 3])
def test_preact_backward_tc(cuda_ok, dv, T):
    x = draw_sequence(1, 2, T, 64, dv, torch.bfloat16, seed=700 + T + dv, s0_std=0.1,
                      with_dO=True, preact=True)
    dST = 0.1 * torch.randn(1, 2, 64, dv, generator=torch.Generator().manual_seed(T))
    d = dev(x)
    saved = torch.empty(rdm.rdm_ddts_saved_states_size(1, 2, T, 64, dv, 64) // 4, device="cuda")
    rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), d["S0"], saved_states=saved, gates="preact")
    gr = rdm.rdm_ddts_bwd(*(d[n] for n in SEQ), d["S0"], d["dO"], dST.cuda(), saved,
                          gates="preact")
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    ref = oracle.bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], dST, preact=True)
    for n in GR:
        assert_close(gr[n], ref[n], 2e-2, f"preact {n}")


@pytest.mark.parametrize("T", [100, 64 * 9 + 3])
def test_preact_backward_tc_states_recomputed(cuda_ok, T):
    """No saved states passed: the backward recomputes them with a forward
    launch of its own, which has to activate the gates too."""
    x = draw_sequence(1, 2, T, 64, 128, torch.bfloat16, seed=710 + T, s0_std=0.1,
                      with_dO=True, preact=True)
    d = dev(x)
    gr = rdm.rdm_ddts_bwd(*(d[n] for n in SEQ), d["S0"], d["dO"], None, None, impl="tc",
                          gates="preact")
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    ref = oracle.bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], preact=True)
    for n in GR:
        assert_close(gr[n], ref[n], 2e-2, f"preact, states recomputed: {n}")


def test_preact_backward_simt_fp32(cuda_ok):
    x = draw_sequence(1, 2, 90, 16, 32, torch.float32, seed=93, s0_std=0.1, with_dO=True,
                      preact=True)
    d = dev(x)
    gr = rdm.rdm_ddts_bwd(*(d[n] for n in SEQ), d["S0"], d["dO"], gates="preact")
    torch.cuda.synchronize()
    ref = oracle.bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], preact=True)
    for n in GR:
        assert_close(gr[n], ref[n], 1e-4, f"preact fp32 {n}")
