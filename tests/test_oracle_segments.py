"""The identities the exact backward's sequence segments rest on, checked on the
fp64 oracle (CPU): the state recurrence and the gradient recurrence are affine
across any cut of the sequence, with the segment's decay product e^L (L the sum
of log alpha = -g tau over its tokens) as the linear part.  A segment's map is
obtained by running it from a zero start; folding the maps reproduces the
whole-sequence results, and the decay-gradient carry into a segment is fin plus
the dG sums of the segments after it."""
import numpy as np
import torch

import oracle
from gated_linear_attention_ddts_b200.workloads import draw_sequence

SEQ = ("q", "k", "v", "g", "tau", "beta")
CUTS = (0, 11, 26, 40)  # three segments of a 40-token sequence


def _seq(seed):
    x = draw_sequence(1, 2, 40, 4, 3, torch.float32, seed=seed, s0_std=0.3, with_dO=True)
    return {n: (t.double() if t is not None else None) for n, t in x.items()}


def _sl(x, a, b):
    return {n: x[n][:, :, a:b] for n in SEQ + ("dO",)}


def _log_alpha(x, a, b):  # [B,H,dk]: sum over tokens a..b-1 of -g tau
    return (-(x["g"][:, :, a:b] * x["tau"][:, :, a:b])).sum(2).numpy()


def test_state_map_folds_across_segments():
    x = _seq(61)
    _, S_T = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    S = x["S0"].numpy().copy()
    for a, b in zip(CUTS[:-1], CUTS[1:]):
        s = _sl(x, a, b)
        _, S_loc = oracle.fwd(*(s[n] for n in SEQ), None)  # the segment from a zero start
        S = np.exp(_log_alpha(x, a, b))[..., None] * S + np.asarray(S_loc)
    assert np.allclose(S, np.asarray(S_T), rtol=1e-12, atol=1e-12)


def test_gradient_map_folds_across_segments():
    """dS_0 of the whole sequence from dS_T equals the fold, last segment first,
    of each segment's map C_out = diag(e^L) C_in + C_loc, where C_loc is the
    segment's own dS_0 from a zero dS_T (C = alpha o dS at a cut)."""
    x = _seq(62)
    dST = torch.randn(1, 2, 4, 3, generator=torch.Generator().manual_seed(3), dtype=torch.float64)
    ref = oracle.bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], dST)
    C = dST.numpy().copy()
    for a, b in reversed(list(zip(CUTS[:-1], CUTS[1:]))):
        s = _sl(x, a, b)
        loc = oracle.bwd(*(s[n] for n in SEQ), None, s["dO"], None)
        C = np.exp(_log_alpha(x, a, b))[..., None] * C + np.asarray(loc["dS0"])
    assert np.allclose(C, np.asarray(ref["dS0"]), rtol=1e-11, atol=1e-12)


def test_decay_gradient_total_balances():
    """Within segment j, d log alpha_t = (the segment's own suffix sum of dG) +
    carry_j, with carry_j = rowsum(dS_T o S_T) + the dG sums of later segments;
    dG_u = q_u dq_u - khat_u dkhat_u, and d log alpha relates to the gradients
    by dg = -tau d log alpha + (d alpha_hat / dg) k dkhat.  Checked through the
    identity sum over all tokens of dG + rowsum(dS_T o S_T) = rowsum(dS_0 o S_0)
    (the total decay gradient of a sequence equals that of its start state)."""
    x = _seq(63)
    dST = torch.randn(1, 2, 4, 3, generator=torch.Generator().manual_seed(4), dtype=torch.float64)
    _, S_T = oracle.fwd(*(x[n] for n in SEQ), x["S0"])
    r = oracle.bwd(*(x[n] for n in SEQ), x["S0"], x["dO"], dST)
    q, k, g, tau = (x[n].numpy() for n in ("q", "k", "g", "tau"))
    ah = np.where(tau == 0, 1.0, g ** tau)
    # dkhat = dk / alpha_hat where alpha_hat > 0
    dkh = np.asarray(r["dk"]) / ah
    dG = q * np.asarray(r["dq"]) - ah * k * dkh
    lhs = dG.sum(2) + (dST.numpy() * np.asarray(S_T)).sum(-1)
    rhs = (np.asarray(r["dS0"]) * x["S0"].numpy()).sum(-1)
    assert np.allclose(lhs, rhs, rtol=1e-9, atol=1e-10)
