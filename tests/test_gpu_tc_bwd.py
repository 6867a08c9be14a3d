"""GPU parity of the tensor-core chunked backward against the fp64 oracle,
through the C ABI: every gradient (q, k, v, g, tau, beta_hat, S_0), with and
without an upstream dS_T, with saved or recomputed chunk states, ragged tails,
wide-decay heads (exact re-run path), sequences cut into segments (one CTA
each) and the full training workload (sampled heads)."""
import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
import oracle
from gated_linear_attention_ddts_b200.workloads import WORKLOADS, draw_sequence, draw_workload
from tests.parity import assert_close

pytestmark = pytest.mark.gpu
TOL = 2e-2
SEQ = ("q", "k", "v", "g", "tau", "beta")
GR = ("dq", "dk", "dv", "dg", "dtau", "dbeta", "dS0")


def gpu_bwd(x, dST=None, use_saved=True, impl="tc"):
    d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    B, H, T, dk = d["q"].shape
    dv = d["v"].shape[-1]
    saved = None
    if use_saved:
        saved = torch.empty(rdm.rdm_ddts_saved_states_size(B, H, T, dk, dv, 64) // 4,
                            device="cuda")
        rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), d["S0"], saved_states=saved)
    gr = rdm.rdm_ddts_bwd(*(d[n] for n in SEQ), d["S0"], d["dO"],
                          dST.cuda() if dST is not None else None, saved, impl=impl)
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    return gr


def check(x, dST, gr, what=""):
    ref = oracle.bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], dST)
    for n in GR:
        assert_close(gr[n], ref[n], TOL, f"{what} {n}")


@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("T", [1, 63, 64, 130, 200])
def test_tc_backward_small(cuda_ok, dv, T):
    x = draw_sequence(2, 2, T, 64, dv, torch.bfloat16, seed=2000 + T + dv, s0_std=0.1,
                      with_dO=True)
    dST = 0.1 * torch.randn(2, 2, 64, dv, generator=torch.Generator().manual_seed(T))
    check(x, dST, gpu_bwd(x, dST), "dST given")
    check(x, None, gpu_bwd(x, None, use_saved=False), "no dST, states recomputed")


def test_tc_backward_matches_simt(cuda_ok):
    x = draw_sequence(2, 3, 300, 64, 128, torch.bfloat16, seed=88, s0_std=0.1, with_dO=True)
    a = gpu_bwd(x, impl="tc")
    b = gpu_bwd(x, impl="simt", use_saved=False)
    for n in GR:
        assert_close(a[n], b[n], TOL, f"tc vs simt {n}")


@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("T", [64 * 8, 64 * 13 + 21])
def test_tc_backward_segmented(cuda_ok, dv, T):
    """Two heads leave most SMs idle: each sequence is cut into segments whose R
    maps and decay-gradient carries are folded across CTAs.  Every gradient
    against the oracle, with and without dS_T, and against the exact path."""
    x = draw_sequence(1, 2, T, 64, dv, torch.bfloat16, seed=4000 + T + dv, s0_std=0.1,
                      with_dO=True)
    dST = 0.1 * torch.randn(1, 2, 64, dv, generator=torch.Generator().manual_seed(T + 1))
    g1 = gpu_bwd(x, dST)
    check(x, dST, g1, "segmented, dST given")
    check(x, None, gpu_bwd(x, None, use_saved=False), "segmented, no dST, states recomputed")
    g2 = gpu_bwd(x, dST, impl="simt", use_saved=False)
    for n in GR:
        assert_close(g1[n], g2[n], TOL, f"segmented vs exact {n}")


def test_tc_backward_segmented_wide_decay(cuda_ok):
    """A head with a too-wide chunk in one segment only: the whole head is re-run
    exactly, the other head keeps the segmented result."""
    x = draw_sequence(1, 2, 64 * 10 + 3, 64, 128, torch.bfloat16, seed=17, s0_std=0.1,
                      with_dO=True)
    x["g"] = x["g"].float()
    x["g"][:, 1, 64 * 7:64 * 8] *= 40.0
    x["g"] = x["g"].clamp(min=0.05).to(torch.bfloat16)
    check(x, None, gpu_bwd(x), "segmented, one wide chunk")


def test_tc_backward_segmented_no_decay(cuda_ok):
    """R-only passes over a later half with tau = 0 (alpha = 1: plain sums of
    q dO^T over whole segments) and g = 0 on no channel (dg needs g > 0)."""
    x = draw_sequence(1, 2, 64 * 12 + 7, 64, 128, torch.bfloat16, seed=59, s0_std=0.1,
                      with_dO=True)
    x["tau"][:, :, 64 * 6:] = 0
    dST = 0.1 * torch.randn(1, 2, 64, 128, generator=torch.Generator().manual_seed(59))
    check(x, dST, gpu_bwd(x, dST), "segmented, no decay in the later half")


@pytest.mark.parametrize("scale", [3.0, 40.0])
def test_tc_backward_wide_decay(cuda_ok, scale):
    """Heads whose chunk decay span exceeds one reference are re-run exactly."""
    x = draw_sequence(1, 3, 150, 64, 64, torch.bfloat16, seed=6, s0_std=0.1, with_dO=True)
    x["g"] = x["g"].float()
    x["g"][:, 1] *= scale          # only head 1 is wide
    x["g"] = x["g"].clamp(min=0.05).to(torch.bfloat16)
    check(x, None, gpu_bwd(x), f"scale {scale}")


def test_workload3_backward_sampled(cuda_ok):
    w = WORKLOADS[3]
    x = draw_workload(w, device="cuda")
    saved = torch.empty(rdm.rdm_ddts_saved_states_size(w.B, w.H, w.T, w.dk, w.dv, 64) // 4,
                        device="cuda")
    rdm.rdm_ddts_fwd(*(x[n] for n in SEQ), x["S0"], saved_states=saved)
    gr = rdm.rdm_ddts_bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], None, saved)
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    for (b, h) in [(0, 0), (3, 15)]:
        xs = {n: x[n][b:b + 1, h:h + 1].cpu() for n in SEQ + ("dO", "S0")}
        ref = oracle.bwd(*(xs[n] for n in SEQ), xs["S0"], xs["dO"])
        for n in GR:
            assert_close(gr[n][b:b + 1, h:h + 1], ref[n], TOL, f"head ({b},{h}) {n}")


@pytest.mark.parametrize("dv", [64, 128])
def test_tc_backward_wide_decay_preact_feedthrough(cuda_ok, dv):
    """A wide head under gates passed before their activations and with the
    feedthrough: the exact re-run then activates g, tau and beta itself, takes
    the chain factors to the pre-activations and adds the feedthrough's term to
    dv."""
    from tests.test_gpu_feedthrough import feed_weights
    T = 64 * 3 + 17
    x = draw_sequence(1, 3, T, 64, dv, torch.bfloat16, seed=31 + dv, s0_std=0.1, with_dO=True,
                      preact=True)
    g = x["g"].float()
    g[:, 1, 70:110] = g[:, 1, 70:110] * 4.0 + 12.0  # softplus ~ 12: one chunk of head 1 is wide
    x["g"] = g.to(torch.bfloat16)
    d = feed_weights(3, dv, 31 + dv)
    dST = 0.1 * torch.randn(1, 3, 64, dv, generator=torch.Generator().manual_seed(dv))
    dx = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    gr = rdm.rdm_ddts_bwd(*(dx[n] for n in SEQ), dx["S0"], dx["dO"], dST.cuda(), impl="tc",
                          gates="preact", feedthrough=d.cuda())
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    ref = oracle.bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], dST, preact=True, d=d)
    for n in GR:
        assert_close(gr[n], ref[n], TOL, f"wide head, preact, feedthrough: {n}")
    assert_close(gr["dfeed"], ref["dd"], TOL, "wide head: grad of the feedthrough weights")


def test_tc_backward_wide_decay_long(cuda_ok):
    """A wide head in a sequence long enough for the exact re-run to go in
    segments, with gates passed before their activations and the feedthrough."""
    from tests.test_gpu_feedthrough import feed_weights
    T = 1024 + 300
    x = draw_sequence(1, 2, T, 64, 128, torch.bfloat16, seed=41, s0_std=0.1, with_dO=True,
                      preact=True)
    g = x["g"].float()
    g[:, 0, 700:760] = g[:, 0, 700:760] * 4.0 + 12.0
    x["g"] = g.to(torch.bfloat16)
    d = feed_weights(2, 128, 41)
    dST = 0.1 * torch.randn(1, 2, 64, 128, generator=torch.Generator().manual_seed(41))
    dx = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    gr = rdm.rdm_ddts_bwd(*(dx[n] for n in SEQ), dx["S0"], dx["dO"], dST.cuda(), impl="tc",
                          gates="preact", feedthrough=d.cuda())
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    ref = oracle.bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], dST, preact=True, d=d)
    for n in GR:
        assert_close(gr[n], ref[n], TOL, f"long wide head: {n}")


def test_workload3_backward_wide_heads_sampled(cuda_ok):
    """The bench's wide-heads backward (every 16th head with one chunk's g x40,
    re-run exactly in 8 segments of 512 tokens): a wide and a plain head against
    the oracle."""
    w = WORKLOADS[3]
    x = draw_workload(w, device="cuda")
    gw = x["g"].float()
    gw[:, ::16, 64 * 20:64 * 21] *= 40.0
    x["g"] = gw.clamp(min=0.05).to(torch.bfloat16)
    del gw
    saved = torch.empty(rdm.rdm_ddts_saved_states_size(w.B, w.H, w.T, w.dk, w.dv, 64) // 4,
                        device="cuda")
    rdm.rdm_ddts_fwd(*(x[n] for n in SEQ), x["S0"], saved_states=saved)
    gr = rdm.rdm_ddts_bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], None, saved)
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    for (b, h) in [(1, 0), (2, 5)]:
        xs = {n: x[n][b:b + 1, h:h + 1].cpu() for n in SEQ + ("dO", "S0")}
        ref = oracle.bwd(*(xs[n] for n in SEQ), xs["S0"], xs["dO"])
        for n in GR:
            assert_close(gr[n][b:b + 1, h:h + 1], ref[n], TOL, f"wide-heads workload ({b},{h}) {n}")
