"""GPU parity of the tensor-core (tcgen05) chunked forward against the fp64
oracle, through the C ABI: ragged tails, initial/final states, saved chunk
states, wide-decay windows, the special cases g = 0 and tau = 0, sequences cut
into segments (one CTA each), and the full-size workloads (sampled heads)."""
import numpy as np
import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
import oracle
from gated_linear_attention_ddts_b200.workloads import WORKLOADS, draw_sequence, draw_workload
from tests.parity import assert_close, np64

pytestmark = pytest.mark.gpu
TOL = 2e-2
SEQ = ("q", "k", "v", "g", "tau", "beta")


def run_tc(x, want_saved=False, impl="tc", workspace=None):
    d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    B, H, T, dk = d["q"].shape
    dv = d["v"].shape[-1]
    saved = None
    if want_saved:
        saved = torch.full((rdm.rdm_ddts_saved_states_size(B, H, T, dk, dv, 64) // 4,),
                           float("nan"), device="cuda")
    o, ST = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), d.get("S0"), saved_states=saved, impl=impl,
                             return_state=True, workspace=workspace)
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    return o, ST, saved


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_tc_forward_small(cuda_ok, dk, dv, T):
    x = draw_sequence(2, 2, T, dk, dv, torch.bfloat16, seed=1000 + T + dk + dv, s0_std=0.1)
    o, ST, saved = run_tc(x, want_saved=True)
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    assert_close(o, o_ref, TOL, "o")
    assert_close(ST, S_ref, TOL, "S_T")
    nc = (T + 63) // 64
    sv = saved.view(2, 2, nc, dk, dv)
    for c in range(nc):
        ref = np64(x["S0"]) if c == 0 else oracle.fwd(*(x[n][:, :, :64 * c] for n in SEQ),
                                                      x["S0"])[1]
        assert_close(sv[:, :, c], ref, TOL, f"saved state {c}")


def test_tc_matches_simt_path(cuda_ok):
    x = draw_sequence(3, 2, 300, 64, 128, torch.bfloat16, seed=77, s0_std=0.1)
    o1, S1, _ = run_tc(x, impl="tc")
    o2, S2, _ = run_tc(x, impl="simt")
    assert_close(o1, o2, TOL, "o tc vs simt")
    assert_close(S1, S2, TOL, "S_T tc vs simt")


@pytest.mark.parametrize("scale,why", [(3.0, "windows of 16"), (40.0, "windows of 1"),
                                       (400.0, "single-token windows, alpha underflows")])
def test_tc_wide_decay_windows(cuda_ok, scale, why):
    """g*tau large enough that one 64-token reference cannot hold the decay
    span: the kernel falls back to shorter windows and stays exact."""
    x = draw_sequence(1, 2, 150, 64, 64, torch.bfloat16, seed=5, s0_std=0.1)
    x["g"] = (x["g"].float() * scale).to(torch.bfloat16)
    # mix: some channels with tiny decay so long memory and short memory coexist
    x["g"][:, :, :, :8] = (x["g"][:, :, :, :8].float() / scale / 10).to(torch.bfloat16)
    o, ST, _ = run_tc(x)
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    assert_close(o, o_ref, TOL, f"o ({why})")
    assert_close(ST, S_ref, TOL, f"S_T ({why})")


def test_tc_g_zero_and_tau_zero(cuda_ok):
    x = draw_sequence(1, 2, 130, 64, 128, torch.bfloat16, seed=9, s0_std=0.2)
    xg = dict(x, g=torch.zeros_like(x["g"]))          # alpha = 1, alpha_hat = 0: S stays S_0
    o, ST, _ = run_tc(xg)
    assert_close(o, np.einsum("bhij,bhti->bhtj", np64(x["S0"]), np64(x["q"])), TOL, "g=0 o")
    assert_close(ST, np64(x["S0"]), 1e-6, "g=0 S_T")
    xt = dict(x, tau=torch.zeros_like(x["tau"]))      # alpha = alpha_hat = 1: prefix sums
    o, ST, _ = run_tc(xt)
    vh = np64(x["beta"]) * np64(x["v"])
    S = np64(x["S0"])[:, :, None] + np.cumsum(np64(x["k"])[..., :, None] * vh[..., None, :], 2)
    assert_close(o, np.einsum("bhtij,bhti->bhtj", S, np64(x["q"])), TOL, "tau=0 o")
    assert_close(ST, S[:, :, -1], TOL, "tau=0 S_T")


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("scale", [1.0, 6.0])
def test_chunk_size_invariance(cuda_ok, dk, dv, scale):
    """The chunked tensor-core kernel evaluated with chunks of 16, 32 and 64
    tokens (impl="tc": every one of them runs on the tensor cores) gives the same
    output, final state and saved chunk-start states up to rounding, against
    the oracle and against chunk 64.  Chunk 128 runs the exact path and joins
    the comparison.  scale 6 widens the decay so that some chunks are narrowed
    to 16-token or single-token windows inside the kernel as well.  (Chunkwise
    form: paperhub.cn OpenReview rebuttal, "Efficient Parallelization".)"""
    B, H, T = 1, 2, 300
    x = draw_sequence(B, H, T, dk, dv, torch.bfloat16, seed=61 + dk + dv, s0_std=0.1)
    x["g"] = (x["g"].float() * scale).to(torch.bfloat16)
    d = {n: x[n].cuda() for n in SEQ}
    S0 = x["S0"].cuda()
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    ref = None
    for chunk in (64, 32, 16, 128):
        impl = "tc" if chunk <= 64 else "auto"
        saved = torch.full((rdm.rdm_ddts_saved_states_size(B, H, T, dk, dv, chunk) // 4,),
                           float("nan"), device="cuda")
        o, ST = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), S0, saved_states=saved, chunk=chunk,
                                 impl=impl, return_state=True)
        torch.cuda.synchronize()
        assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
        assert_close(o, o_ref, TOL, f"o chunk {chunk}")
        assert_close(ST, S_ref, TOL, f"S_T chunk {chunk}")
        nc = (T + chunk - 1) // chunk
        sv = saved.view(B, H, nc, dk, dv)
        for c in sorted({1, nc // 2, nc - 1}):
            sref = oracle.fwd(*(x[n][:, :, :chunk * c] for n in SEQ), x["S0"])[1]
            assert_close(sv[:, :, c], sref, TOL, f"saved state {c} of chunk {chunk}")
        if ref is None:
            ref = (o.float().cpu().numpy(), ST.cpu().numpy())
        else:
            assert_close(o, ref[0], TOL, f"o chunk {chunk} vs 64")
            assert_close(ST, ref[1], TOL, f"S_T chunk {chunk} vs 64")


@pytest.mark.parametrize("chunk", [16, 32])
def test_chunk_size_segmented(cuda_ok, chunk):
    """Small chunks inside sequence segments (state-only passes, folded maps)."""
    x = draw_sequence(1, 2, 64 * 11 + 21, 64, 128, torch.bfloat16, seed=71 + chunk, s0_std=0.1)
    assert segments_used(x)
    d = {n: x[n].cuda() for n in SEQ}
    o, ST = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), x["S0"].cuda(), chunk=chunk, impl="tc",
                             return_state=True)
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    assert_close(o, o_ref, TOL, f"o chunk {chunk}")
    assert_close(ST, S_ref, TOL, f"S_T chunk {chunk}")


def test_tc_split_invariance(cuda_ok):
    """fwd(T1) then fwd(T2, S_0 = S_T1) equals fwd(T1 + T2) on the GPU."""
    x = draw_sequence(2, 3, 320, 64, 128, torch.bfloat16, seed=21, s0_std=0.1)
    o, ST, _ = run_tc(x)
    a = {n: x[n][:, :, :128].contiguous() for n in SEQ}
    b = {n: x[n][:, :, 128:].contiguous() for n in SEQ}
    oa, Sa, _ = run_tc(dict(a, S0=x["S0"]))
    ob, Sb, _ = run_tc(dict(b, S0=Sa.cpu()))
    assert_close(torch.cat([oa, ob], 2), o, TOL, "split o")
    assert_close(Sb, ST, TOL, "split S_T")


def segments_used(x):
    d = {n: x[n].cuda() for n in SEQ}
    return rdm.rdm_ddts_fwd_workspace_size(*(d[n] for n in SEQ), impl="tc") > 0


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("T", [64 * 8, 64 * 13 + 37])
def test_tc_forward_segmented(cuda_ok, dk, dv, T):
    """Two heads leave most SMs idle, so each sequence is cut into segments that
    separate CTAs run; their state maps are folded across CTAs.  Output, final
    state and saved chunk states against the oracle, and against one CTA per
    sequence (no workspace)."""
    x = draw_sequence(1, 2, T, dk, dv, torch.bfloat16, seed=3000 + T + dk + dv, s0_std=0.1)
    assert segments_used(x)
    o, ST, saved = run_tc(x, want_saved=True)
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    assert_close(o, o_ref, TOL, "o")
    assert_close(ST, S_ref, TOL, "S_T")
    nc = (T + 63) // 64
    sv = saved.view(1, 2, nc, dk, dv)
    for c in sorted({1, nc // 3, nc // 2, (2 * nc) // 3, nc - 1}):
        ref = oracle.fwd(*(x[n][:, :, :64 * c] for n in SEQ), x["S0"])[1]
        assert_close(sv[:, :, c], ref, TOL, f"saved state {c}")
    o1, S1, _ = run_tc(x, workspace=False)
    assert_close(o, o1.float().cpu().numpy(), TOL, "o segmented vs one CTA")
    assert_close(ST, S1.cpu().numpy(), TOL, "S_T segmented vs one CTA")


@pytest.mark.parametrize("scale", [3.0, 40.0])
def test_tc_segmented_wide_decay(cuda_ok, scale):
    """Narrow windows inside segments; decay products across segments that
    underflow to zero for the short-memory channels."""
    x = draw_sequence(1, 1, 64 * 9 + 5, 64, 128, torch.bfloat16, seed=41, s0_std=0.1)
    x["g"] = (x["g"].float() * scale).to(torch.bfloat16)
    x["g"][:, :, :, :8] = (x["g"][:, :, :, :8].float() / scale / 10).to(torch.bfloat16)
    assert segments_used(x)
    o, ST, _ = run_tc(x)
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    assert_close(o, o_ref, TOL, "o")
    assert_close(ST, S_ref, TOL, "S_T")


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64)])
def test_tc_segmented_special_gates(cuda_ok, dk, dv):
    """State-only passes that sum outer products with no decay at all (tau = 0:
    alpha = alpha_hat = 1) over half of the sequence, and channels with g = 0
    (alpha = 1; alpha_hat = 0 where tau > 0, 1 where tau = 0)."""
    x = draw_sequence(1, 2, 64 * 12 + 7, dk, dv, torch.bfloat16, seed=53 + dk, s0_std=0.1)
    x["tau"][:, :, :64 * 6] = 0
    x["g"][:, :, :, :8] = 0
    assert segments_used(x)
    o, ST, saved = run_tc(x, want_saved=True)
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    assert_close(o, o_ref, TOL, "o")
    assert_close(ST, S_ref, TOL, "S_T")
    nc = (64 * 12 + 7 + 63) // 64
    sv = saved.view(1, 2, nc, dk, dv)
    for c in (3, 6, 9):
        ref = oracle.fwd(*(x[n][:, :, :64 * c] for n in SEQ), x["S0"])[1]
        assert_close(sv[:, :, c], ref, TOL, f"saved state {c}")


@pytest.mark.parametrize("B,H,T", [(1, 40, 64 * 12 + 9), (4, 25, 130)])
def test_tc_forward_wide_slices(cuda_ok, B, H, T):
    """Head counts for which one CTA takes all 128 value columns of a head:
    40 heads (segmented three ways on a 148-SM part) and 100 heads (one
    segment, one wave)."""
    x = draw_sequence(B, H, T, 64, 128, torch.bfloat16, seed=50 + B * H, s0_std=0.1)
    o, ST, _ = run_tc(x)
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    assert_close(o, o_ref, TOL, "o")
    assert_close(ST, S_ref, TOL, "S_T")


def test_tc_segmented_repeat_calls(cuda_ok):
    """The same workspace serves back-to-back calls (flags tagged per launch)."""
    x = draw_sequence(1, 2, 64 * 12, 64, 128, torch.bfloat16, seed=43, s0_std=0.1)
    d = {n: x[n].cuda() for n in SEQ}
    ws = torch.empty(rdm.rdm_ddts_fwd_workspace_size(*(d[n] for n in SEQ)), dtype=torch.uint8,
                     device="cuda")
    S0 = x["S0"].cuda()
    outs = [rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), S0, workspace=ws, return_state=True)
            for _ in range(3)]
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    for o, ST in outs:
        assert_close(o, o_ref, TOL, "o")
        assert_close(ST, S_ref, TOL, "S_T")


def sampled_check(w, heads, device_inputs=True):
    x = draw_workload(w, device="cuda")
    o, ST = rdm.rdm_ddts_fwd(*(x[n] for n in SEQ), x["S0"], return_state=True)
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    for (b, h) in heads:
        xs = {n: x[n][b:b + 1, h:h + 1].cpu() for n in SEQ}
        s0 = x["S0"][b:b + 1, h:h + 1].cpu() if x["S0"] is not None else None
        o_ref, S_ref = oracle.fwd(*(xs[n] for n in SEQ), s0)
        assert_close(o[b:b + 1, h:h + 1], o_ref, TOL, f"workload {w.name[:12]} o head ({b},{h})")
        assert_close(ST[b:b + 1, h:h + 1], S_ref, TOL, f"workload {w.name[:12]} S_T head ({b},{h})")


def test_workload1_full_size_sampled(cuda_ok):
    sampled_check(WORKLOADS[1], [(0, 0), (3, 2), (7, 5)])


def test_workload2_full_size_sampled(cuda_ok):
    sampled_check(WORKLOADS[2], [(0, 0), (0, 15)])


def test_workload3_forward_sampled(cuda_ok):
    sampled_check(WORKLOADS[3], [(0, 0), (3, 15)])
