"""GPU parity of the low-rank beta_hat (Rodimus*, digest.lyk-ai.com summary,
"Method": beta_hat from low-rank matrices; read as sigmoid(u_t . w_up[h]) with
a per-token factor u shared by the heads) against the fp64 oracle, through the
C ABI: the tensor-core forward that builds beta_hat on chip (one CTA per
sequence and segmented, ranks 8 and 16, chunks 16 to 64), the backward on both
paths (factor gradients du and dw_up and every other gradient), agreement with
the full-rank pre-activation path on the expanded pre-activation, the
130M-scale layer on sampled heads, and the argument checks."""
import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
import oracle
from gated_linear_attention_ddts_b200.workloads import WORKLOADS, draw_lowrank, draw_sequence
from tests.parity import assert_close

pytestmark = pytest.mark.gpu
SEQ = ("q", "k", "v", "g", "tau")
TOL = 2e-2


def inputs(B, H, T, dk, dv, r, seed, dtype=torch.bfloat16, with_dO=False):
    x = draw_sequence(B, H, T, dk, dv, dtype, seed=seed, s0_std=0.1, preact=True,
                      with_dO=with_dO)
    u, w = draw_lowrank(B, H, T, dv, r, dtype, seed=seed + 1)
    return x, u, w


def cuda(x):
    return {n: (t.cuda() if t is not None else None) for n, t in x.items()}


@pytest.mark.parametrize("r", [8, 16])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 65, 64 * 9 + 3])
def test_lowrank_forward_tc(cuda_ok, r, dk, dv, T):
    x, u, w = inputs(1, 2, T, dk, dv, r, seed=900 + T + dk + dv + r)
    d = cuda(x)
    o, ST = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), None, d["S0"], gates="preact",
                             beta_lowrank=(u.cuda(), w.cuda()), return_state=True)
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    o_ref, S_ref = oracle.fwd_lowrank(*(x[n] for n in SEQ), u, w, x["S0"])
    assert_close(o, o_ref, TOL, f"low-rank o r={r}")
    assert_close(ST, S_ref, TOL, f"low-rank S_T r={r}")


@pytest.mark.parametrize("chunk", [16, 32])
def test_lowrank_forward_small_chunks_and_segments(cuda_ok, chunk):
    """Sequences long enough to be cut into segments (workspace given), and the
    narrower chunk sizes of the tensor-core kernel."""
    x, u, w = inputs(1, 1, 64 * 24 + 7, 64, 128, 16, seed=31 + chunk)
    d = cuda(x)
    for ws in (None, False):  # allocated workspace (segments), then none
        o, ST = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), None, d["S0"], gates="preact",
                                 beta_lowrank=(u.cuda(), w.cuda()), return_state=True,
                                 chunk=chunk, workspace=ws)
        torch.cuda.synchronize()
        o_ref, S_ref = oracle.fwd_lowrank(*(x[n] for n in SEQ), u, w, x["S0"])
        assert_close(o, o_ref, TOL, f"chunk {chunk} workspace {ws is None}")
        assert_close(ST, S_ref, TOL, f"chunk {chunk} S_T")


def test_lowrank_matches_full_rank_preact(cuda_ok):
    """The same sequence with beta's pre-activation expanded on the host and
    rounded to bf16 (the full-rank path's input), against the fused path."""
    x, u, w = inputs(2, 3, 300, 64, 128, 16, seed=5)
    pre = torch.einsum("btr,hrj->bhtj", u.float(), w).to(torch.bfloat16).contiguous()
    d = cuda(x)
    o1, S1 = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), None, d["S0"], gates="preact",
                              beta_lowrank=(u.cuda(), w.cuda()), return_state=True)
    o2, S2 = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), pre.cuda(), d["S0"], gates="preact",
                              return_state=True)
    torch.cuda.synchronize()
    assert_close(o1, o2.float().cpu().numpy(), TOL, "fused vs expanded o")
    assert_close(S1, S2.cpu().numpy(), TOL, "fused vs expanded S_T")


@pytest.mark.parametrize("impl,dtype,dk,dv,T", [("tc", torch.bfloat16, 64, 128, 64 * 5 + 9),
                                               ("tc", torch.bfloat16, 64, 64, 200),
                                               ("simt", torch.float32, 16, 32, 77)])
def test_lowrank_backward(cuda_ok, impl, dtype, dk, dv, T):
    x, u, w = inputs(2, 2, T, dk, dv, 8, seed=61 + T, dtype=dtype, with_dO=True)
    dST = 0.1 * torch.randn(2, 2, dk, dv, generator=torch.Generator().manual_seed(T))
    d = cuda(x)
    gr = rdm.rdm_ddts_bwd(*(d[n] for n in SEQ), None, d["S0"], d["dO"], dST.cuda(), None,
                          gates="preact", beta_lowrank=(u.cuda(), w.cuda()), impl=impl)
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    ref = oracle.bwd_lowrank(*(x[n] for n in SEQ), u, w, x["S0"], x["dO"], dST)
    tol = TOL if dtype == torch.bfloat16 else 1e-4
    for n in ("dq", "dk", "dv", "dg", "dtau", "dS0", "du", "dw_up"):
        assert_close(gr[n], ref[n], tol, f"low-rank {impl} {n}")


def test_lowrank_layer_forward_sampled_heads(cuda_ok):
    """130M-scale layer (B8 H6 T2048 d_k64 d_v128), rank 16, in the launch the
    benchmark times; two (batch, head) pairs against the oracle on them alone
    (the factor u is shared by the heads, so each pair needs only its rows)."""
    w1 = WORKLOADS[1]
    x = draw_sequence(w1.B, w1.H, w1.T, w1.dk, w1.dv, torch.bfloat16, seed=w1.seed, preact=True)
    u, w = draw_lowrank(w1.B, w1.H, w1.T, w1.dv, 16, seed=w1.seed + 40)
    d = cuda(x)
    o, _ = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), None, None, gates="preact",
                            beta_lowrank=(u.cuda(), w.cuda()))
    o = o.cpu()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    for b, h in ((0, 0), (7, 5)):
        sl = {n: x[n][b:b + 1, h:h + 1] for n in SEQ}
        ref, _ = oracle.fwd_lowrank(*(sl[n] for n in SEQ), u[b:b + 1], w[h:h + 1])
        assert_close(o[b:b + 1, h:h + 1], ref, TOL, f"layer b={b} h={h}")


def test_lowrank_argument_checks(cuda_ok):
    x, u, w = inputs(1, 2, 70, 64, 64, 8, seed=3)
    d = cuda(x)
    lr = (u.cuda(), w.cuda())
    with pytest.raises(rdm.RdmError) as e:  # activated gates
        rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), None, None, beta_lowrank=lr)
    assert e.value.status == rdm.RDM_ERR_INVALID_ARG
    u4 = torch.zeros(1, 70, 4, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rdm.RdmError) as e:  # rank 4
        rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), None, None, gates="preact",
                         beta_lowrank=(u4, torch.zeros(2, 4, 64, device="cuda")))
    assert e.value.status == rdm.RDM_ERR_UNSUPPORTED
    with pytest.raises(rdm.RdmError) as e:  # the exact path does not build beta on chip
        rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), None, None, gates="preact", beta_lowrank=lr,
                         impl="simt")
    assert e.value.status == rdm.RDM_ERR_UNSUPPORTED
