"""The failure path of the bounded on-device waits, made to run out on purpose.

Sequence-segmented tensor-core launches have CTAs that wait for a flag another
CTA publishes; the SW-SKA forward waits for its value tiles and ShortConv for
its staged tiles.  With the test hooks set, the flags are never published (the
tiles never loaded) and the waits are bounded by about 10 ms of SM clock: the waiting CTAs give up, every
role of the CTA unwinds (its own waits being bounded too), copies and MMAs in
flight are drained, and the kernel returns with the device status word set.
The host then reads RDM_ERR_TIMEOUT from rdm_ddts_sync_status, and the next
normal call on the same context runs and matches the oracle.  No wait is left
unbounded and nothing faults: the kernel returns on its own."""
import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
import oracle
from gated_linear_attention_ddts_b200.workloads import draw_sequence
from tests.parity import assert_close

pytestmark = pytest.mark.gpu
SEQ = ("q", "k", "v", "g", "tau", "beta")
TOL = 2e-2
SHORT = 20_000_000  # SM clock cycles, about 10 ms


def segmented_inputs(seed):
    x = draw_sequence(1, 2, 64 * 12 + 5, 64, 128, torch.bfloat16, seed=seed, s0_std=0.1,
                      with_dO=True)
    d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    assert rdm.rdm_ddts_fwd_workspace_size(*(d[n] for n in SEQ), impl="tc") > 0
    return x, d


def with_hooks(limit, withhold, fn):
    rdm.rdm_ddts_set_test_hooks(limit, withhold)
    try:
        fn()
        return rdm.rdm_ddts_sync_status()
    finally:
        rdm.rdm_ddts_set_test_hooks(0, 0)


def test_forward_wait_runs_out_and_reports_timeout(cuda_ok):
    x, d = segmented_inputs(81)
    st = with_hooks(SHORT, 1, lambda: rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), d["S0"], impl="tc",
                                                         return_state=True))
    assert st == rdm.RDM_ERR_TIMEOUT
    # the context is still usable and the status word was cleared by the read
    o, ST = rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), d["S0"], impl="tc", return_state=True)
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    assert_close(o, o_ref, TOL, "o after a timed-out call")
    assert_close(ST, S_ref, TOL, "S_T after a timed-out call")


def test_backward_wait_runs_out_and_reports_timeout(cuda_ok):
    x, d = segmented_inputs(82)
    args = (*(d[n] for n in SEQ), d["S0"], d["dO"])
    assert rdm.rdm_ddts_bwd_workspace_size(*(d[n] for n in SEQ), impl="tc") > 0
    st = with_hooks(SHORT, 1, lambda: rdm.rdm_ddts_bwd(*args, impl="tc"))
    assert st == rdm.RDM_ERR_TIMEOUT
    gr = rdm.rdm_ddts_bwd(*args, impl="tc")
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    ref = oracle.bwd(*(x[n] for n in SEQ), x["S0"], x["dO"])
    for n in ("dq", "dk", "dv", "dg", "dtau", "dbeta", "dS0"):
        assert_close(gr[n], ref[n], TOL, f"{n} after a timed-out call")


def test_short_limit_alone_changes_nothing(cuda_ok):
    """The shortened bound with the flags published: no wait comes near it."""
    x, d = segmented_inputs(83)
    out = {}
    st = with_hooks(SHORT, 0, lambda: out.update(
        r=rdm.rdm_ddts_fwd(*(d[n] for n in SEQ), d["S0"], impl="tc", return_state=True)))
    assert st == rdm.RDM_OK
    o_ref, S_ref = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    assert_close(out["r"][0], o_ref, TOL, "o with the short bound")
    assert_close(out["r"][1], S_ref, TOL, "S_T with the short bound")


def test_ska_forward_wait_runs_out_and_reports_timeout(cuda_ok):
    """SW-SKA forward with its value tiles withheld: the P V waits run out, the
    roles unwind (the softmax warps of a pair give up together), the kernel
    returns with the status word set, and the next call matches the oracle."""
    g = torch.Generator().manual_seed(83)
    q = torch.randn(1, 2, 300, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 300, 64, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, 300, 64, generator=g).to(torch.bfloat16)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    st = with_hooks(SHORT, 1, lambda: rdm.rdm_ska_fwd(qd, kd, vd, 100))
    assert st == rdm.RDM_ERR_TIMEOUT
    o = rdm.rdm_ska_fwd(qd, kd, vd, 100)
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    assert_close(o, oracle.ska_fwd(q, k, v, 100), TOL, "SW-SKA o after a timed-out call")


def test_shortconv_staging_wait_runs_out_and_reports_timeout(cuda_ok):
    """ShortConv forward and backward with their staging copies withheld: the
    staging waits run out, every block leaves together (nothing is left in
    flight), the status word reports the timeout, and the next calls match the
    oracle."""
    g = torch.Generator().manual_seed(84)
    x = torch.randn(1, 2, 700, 64, generator=g).to(torch.bfloat16)
    w = torch.randn(2, 64, 4, generator=g) / 4
    b = torch.randn(2, 64, generator=g) * 0.1
    gy = torch.randn(1, 2, 700, 64, generator=g).to(torch.bfloat16)
    xd, wd, bd, gyd = x.cuda(), w.cuda(), b.cuda(), gy.cuda()
    st = with_hooks(SHORT, 1, lambda: rdm.rdm_shortconv_fwd(xd, wd, bd, None, silu=True))
    assert st == rdm.RDM_ERR_TIMEOUT
    st = with_hooks(SHORT, 1, lambda: rdm.rdm_shortconv_bwd(xd, wd, bd, None, gyd, None, silu=True))
    assert st == rdm.RDM_ERR_TIMEOUT
    y, _ = rdm.rdm_shortconv_fwd(xd, wd, bd, None, silu=True)
    gr = rdm.rdm_shortconv_bwd(xd, wd, bd, None, gyd, None, silu=True)
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
    y_ref, _ = oracle.shortconv_fwd(x, w, b, None, silu=True)
    ref = oracle.shortconv_bwd(x, w, b, None, gy, None, silu=True)
    assert_close(y, y_ref, TOL, "ShortConv y after a timed-out call")
    for n in ("dx", "dw", "dbias"):
        assert_close(gr[n], ref[n], TOL, f"ShortConv {n} after a timed-out call")
