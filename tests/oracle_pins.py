"""Pins of the fp64 oracle against facts the definition fixes.

Each check raises AssertionError on a mismatch.  They take an optional `lib`
(an oracle library opened with ``oracle.load_library``) so that the same checks
can be run against deliberately broken builds of the oracle (mutants): every
plausible slip in the oracle must make at least one of them fail.

Definition (Rodimus*, digest.lyk-ai.com summary, "Method": alpha = exp(-g*tau),
alpha_hat = g^tau; state S_t = diag(alpha_t) S_{t-1} + (alpha_hat_t k_t)(beta_t v_t)^T,
o_t = S_t^T q_t, diagonal along n = d_k per the paperhub.cn rebuttal).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rand_inputs(rng, B, H, T, dk, dv, g_lo=0.05, g_hi=2.0, tau_lo=0.05, tau_hi=1.0, s0=0.5):
    return dict(
        q=rng.standard_normal((B, H, T, dk)),
        k=rng.standard_normal((B, H, T, dk)),
        v=rng.standard_normal((B, H, T, dv)),
        g=rng.uniform(g_lo, g_hi, (B, H, T, dk)),
        tau=rng.uniform(tau_lo, tau_hi, (B, H, T, dk)),
        beta=rng.uniform(0.1, 1.0, (B, H, T, dv)),
        S0=s0 * rng.standard_normal((B, H, dk, dv)),
    )


def close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    scale = max(1.0, float(np.max(np.abs(b)))) if b.size else 1.0
    err = float(np.max(np.abs(a - b))) / scale if a.size else 0.0
    assert err <= tol, f"{what}: max abs err / max(1,|ref|) = {err:.3e} > {tol:.1e}"


# ------------------------------------------------------------------ forward pins
def check_worked_example(lib=None):
    """Hand-derived T=3 example (tests/golden/ddts_worked_example_T3.json)."""
    fx = json.load(open(os.path.join(GOLDEN, "ddts_worked_example_T3.json")))
    shp = lambda a: np.asarray(a, dtype=np.float64)[None, None]
    o, ST = oracle.fwd(shp(fx["q"]), shp(fx["k"]), shp(fx["v"]), shp(fx["g"]), shp(fx["tau"]),
                       shp(fx["beta"]), shp(fx["S0"]), lib=lib)
    close(o[0, 0], fx["expected_o"], fx["tolerance"], "worked example o")
    close(ST[0, 0], fx["expected_ST"], fx["tolerance"], "worked example S_T")


def check_T1_closed_form(lib=None, seed=1):
    """T = 1: o_1 = S_0^T (alpha_1*q_1) + (khat_1 . q_1) vhat_1 and
    S_1 = diag(alpha_1) S_0 + khat_1 vhat_1^T."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, 2, 3, 1, 5, 4)
    o, ST = oracle.fwd(**x, lib=lib)
    al = np.exp(-x["g"][:, :, 0] * x["tau"][:, :, 0])
    kh = x["g"][:, :, 0] ** x["tau"][:, :, 0] * x["k"][:, :, 0]
    vh = x["beta"][:, :, 0] * x["v"][:, :, 0]
    q = x["q"][:, :, 0]
    o_ref = np.einsum("bhij,bhi->bhj", x["S0"], al * q) + np.sum(kh * q, -1)[..., None] * vh
    S_ref = al[..., None] * x["S0"] + kh[..., :, None] * vh[..., None, :]
    close(o[:, :, 0], o_ref, 1e-13, "T=1 o")
    close(ST, S_ref, 1e-13, "T=1 S_1")


def check_g_zero(lib=None, seed=2):
    """g = 0 (tau > 0): alpha = 1, alpha_hat = 0, so S_t = S_0 and o_t = S_0^T q_t;
    with S_0 = 0 everything is zero."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, 1, 2, 9, 4, 3)
    x["g"][:] = 0.0
    o, ST = oracle.fwd(**x, lib=lib)
    close(o, np.einsum("bhij,bhti->bhtj", x["S0"], x["q"]), 1e-13, "g=0 o")
    close(ST, x["S0"], 1e-15, "g=0 S_T")
    x["S0"] = None
    o, ST = oracle.fwd(**x, lib=lib)
    assert np.all(o == 0.0) and np.all(ST == 0.0)


def check_tau_zero(lib=None, seed=3):
    """tau -> 0: alpha = 1 and alpha_hat = 1 (0^0 = 1 too), i.e. plain
    cumulative linear attention S_t = S_0 + sum_{s<=t} k_s vhat_s^T, checked
    against numpy prefix sums of outer products."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, 2, 2, 11, 3, 5)
    for tau_val, tol in ((0.0, 1e-13), (1e-8, 1e-6)):
        x["tau"][:] = tau_val
        # 0^0 = 1 at tau = 0 exactly; for tau > 0 the limit needs g > 0
        x["g"][0, 0, :, 0] = 0.0 if tau_val == 0.0 else 0.3
        o, ST = oracle.fwd(**x, lib=lib)
        vh = x["beta"] * x["v"]
        S = x["S0"][:, :, None] + np.cumsum(x["k"][..., :, None] * vh[..., None, :], axis=2)
        close(o, np.einsum("bhtij,bhti->bhtj", S, x["q"]), tol, f"tau={tau_val} o")
        close(ST, S[:, :, -1], tol, f"tau={tau_val} S_T")


def quadratic_form(x):
    """Brute force O(T^2):  o_t = sum_{s<=t} (prod_{r=s+1..t} alpha_r * khat_s)^T q_t vhat_s
    + S_0^T (prod_{r<=t} alpha_r * q_t), products taken explicitly."""
    q, k, v, g, tau, beta, S0 = (x[n] for n in ("q", "k", "v", "g", "tau", "beta", "S0"))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    al = np.exp(-g * tau)
    kh = g ** tau * k
    vh = beta * v
    o = np.zeros((B, H, T, dv))
    for b in range(B):
        for h in range(H):
            for t in range(T):
                for s in range(t + 1):
                    w = np.ones(dk)
                    for r in range(s + 1, t + 1):
                        w = w * al[b, h, r]
                    o[b, h, t] += np.dot(w * kh[b, h, s], q[b, h, t]) * vh[b, h, s]
                w = np.ones(dk)
                for r in range(t + 1):
                    w = w * al[b, h, r]
                o[b, h, t] += S0[b, h].T @ (w * q[b, h, t])
    return o


def check_quadratic(lib=None, seed=4):
    rng = np.random.default_rng(seed)
    for (T, dk, dv) in ((16, 4, 3), (7, 2, 6)):
        x = rand_inputs(rng, 1, 2, T, dk, dv, g_lo=0.0, g_hi=3.0)
        o, _ = oracle.fwd(**x, lib=lib)
        close(o, quadratic_form(x), 1e-12, f"quadratic form T={T}")


def check_linearity(lib=None, seed=5):
    """o is linear in (vhat, S_0) jointly: scaling beta and S_0 by c scales o
    and S_T by c; superposing two v's (with their S_0's) superposes outputs."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, 1, 2, 10, 4, 3)
    o, ST = oracle.fwd(**x, lib=lib)
    y = dict(x, beta=2.5 * x["beta"], S0=2.5 * x["S0"])
    o2, ST2 = oracle.fwd(**y, lib=lib)
    close(o2, 2.5 * o, 1e-13, "scale o")
    close(ST2, 2.5 * ST, 1e-13, "scale S_T")
    x2 = rand_inputs(rng, 1, 2, 10, 4, 3)
    ya = dict(x, v=x2["v"], S0=x2["S0"])
    oa, _ = oracle.fwd(**ya, lib=lib)
    yb = dict(x, v=x["v"] + x2["v"], S0=x["S0"] + x2["S0"])
    ob, _ = oracle.fwd(**yb, lib=lib)
    close(ob, o + oa, 1e-12, "superposition")


def check_split_and_decode(lib=None, seed=6):
    """fwd(T1) then fwd(T2, S_0 = S_T1) == fwd(T1+T2); T decode steps == fwd(T)."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, 2, 1, 13, 3, 4)
    o, ST = oracle.fwd(**x, lib=lib)
    cut = lambda a, sl: a[:, :, sl]
    seq = ("q", "k", "v", "g", "tau", "beta")
    a = {n: cut(x[n], slice(0, 5)) for n in seq}
    b = {n: cut(x[n], slice(5, None)) for n in seq}
    oa, Sa = oracle.fwd(**a, S0=x["S0"], lib=lib)
    ob, Sb = oracle.fwd(**b, S0=Sa, lib=lib)
    close(np.concatenate([oa, ob], 2), o, 1e-13, "split o")
    close(Sb, ST, 1e-13, "split S_T")
    S = np.ascontiguousarray(x["S0"].copy())
    for t in range(13):
        ot = oracle.decode_step(*(x[n][:, :, t] for n in seq), S, lib=lib)
        close(ot, o[:, :, t], 1e-13, f"decode step {t}")
    close(S, ST, 1e-13, "decode final state")


# ----------------------------------------------------------------- backward pins
def loss_value(x, dO, dST, lib=None):
    o, ST = oracle.fwd(**x, lib=lib)
    return float(np.sum(o * dO) + np.sum(ST * dST))


def check_bwd_finite_differences(lib=None, seed=7):
    """Central differences (h = 1e-6) of L = <o, dO> + <S_T, dS_T> against the
    oracle's reverse mode, for every input including S_0 and the upstream dS_T."""
    rng = np.random.default_rng(seed)
    B, H, T, dk, dv = 1, 1, 6, 3, 2
    x = rand_inputs(rng, B, H, T, dk, dv, g_lo=0.1, g_hi=3.0, tau_lo=0.05, tau_hi=1.0)
    dO = rng.standard_normal((B, H, T, dv))
    dST = rng.standard_normal((B, H, dk, dv))
    gr = oracle.bwd(**x, dO=dO, dST=dST, lib=lib)
    names = dict(q="dq", k="dk", v="dv", g="dg", tau="dtau", beta="dbeta", S0="dS0")
    h = 1e-6
    for n, gn in names.items():
        num = np.zeros_like(x[n])
        for idx in np.ndindex(x[n].shape):
            xp = {m: a.copy() for m, a in x.items()}
            xp[n][idx] += h
            lp = loss_value(xp, dO, dST, lib)
            xp[n][idx] -= 2 * h
            lm = loss_value(xp, dO, dST, lib)
            num[idx] = (lp - lm) / (2 * h)
        close(gr[gn], num, 2e-7, f"finite differences {gn}")
    # no upstream dS_T (NULL) is the same as a zero dS_T
    gr0 = oracle.bwd(**x, dO=dO, dST=None, lib=lib)
    grz = oracle.bwd(**x, dO=dO, dST=np.zeros_like(dST), lib=lib)
    for gn in names.values():
        close(gr0[gn], grz[gn], 0.0, f"dS_T=None vs zeros {gn}")


def torch_loop_grads(x, dO, dST):
    """Gradients of a naive fp64 torch loop by torch.autograd (a library
    routine independent of the oracle's hand-written reverse mode)."""
    import torch
    t = {n: torch.tensor(a, dtype=torch.float64, requires_grad=True) for n, a in x.items()}
    S = t["S0"]
    outs = []
    T = x["q"].shape[2]
    for s in range(T):
        al = torch.exp(-t["g"][:, :, s] * t["tau"][:, :, s])
        kh = torch.pow(t["g"][:, :, s], t["tau"][:, :, s]) * t["k"][:, :, s]
        vh = t["beta"][:, :, s] * t["v"][:, :, s]
        S = al[..., :, None] * S + kh[..., :, None] * vh[..., None, :]
        outs.append((S * t["q"][:, :, s][..., :, None]).sum(-2))
    o = torch.stack(outs, 2)
    L = (o * torch.tensor(dO)).sum() + (S * torch.tensor(dST)).sum()
    L.backward()
    return {n: t[n].grad.numpy() for n in t}


def check_bwd_autograd(lib=None, seed=8):
    rng = np.random.default_rng(seed)
    # T = 70 crosses the oracle's 64-token checkpoint boundary
    B, H, T, dk, dv = 1, 2, 70, 4, 3
    x = rand_inputs(rng, B, H, T, dk, dv, g_lo=0.05, g_hi=1.0)
    dO = rng.standard_normal((B, H, T, dv))
    dST = rng.standard_normal((B, H, dk, dv))
    gr = oracle.bwd(**x, dO=dO, dST=dST, lib=lib)
    ref = torch_loop_grads(x, dO, dST)
    names = dict(q="dq", k="dk", v="dv", g="dg", tau="dtau", beta="dbeta", S0="dS0")
    for n, gn in names.items():
        close(gr[gn], ref[n], 1e-11, f"autograd {gn}")


# ------------------------------------------------- gate pre-activations (fused mode)
def check_preact_matches_torch_activations(lib=None, seed=9):
    """preact=True equals the plain recurrence on inputs activated by torch's own
    softplus / sigmoid (a library routine, independent of the oracle)."""
    import torch
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, 2, 2, 13, 3, 4)
    pre = dict(g=rng.normal(-1.0, 1.5, x["g"].shape), tau=rng.normal(0.0, 2.0, x["tau"].shape),
               beta=rng.normal(0.0, 2.0, x["beta"].shape))
    pre["g"][0, 0, 0, 0], pre["tau"][0, 0, 0, 0] = 40.0, -40.0   # far tails of both activations
    t = {n: torch.from_numpy(pre[n]) for n in pre}
    act = dict(g=torch.nn.functional.softplus(t["g"]).numpy(), tau=torch.sigmoid(t["tau"]).numpy(),
               beta=torch.sigmoid(t["beta"]).numpy())
    o1, S1 = oracle.fwd(x["q"], x["k"], x["v"], pre["g"], pre["tau"], pre["beta"], x["S0"],
                        lib=lib, preact=True)
    o2, S2 = oracle.fwd(x["q"], x["k"], x["v"], act["g"], act["tau"], act["beta"], x["S0"], lib=lib)
    close(o1, o2, 1e-12, "preact o")
    close(S1, S2, 1e-12, "preact S_T")


def check_preact_special_values(lib=None):
    """softplus(0) = ln 2 and sigmoid(0) = 1/2 exactly: zero pre-activations give
    g = ln 2, tau = beta_hat = 1/2 everywhere."""
    rng = np.random.default_rng(10)
    x = rand_inputs(rng, 1, 1, 5, 2, 3)
    z = lambda a: np.zeros_like(a)
    o1, S1 = oracle.fwd(x["q"], x["k"], x["v"], z(x["g"]), z(x["tau"]), z(x["beta"]), x["S0"],
                        lib=lib, preact=True)
    f = lambda a, c: np.full_like(a, c)
    o2, S2 = oracle.fwd(x["q"], x["k"], x["v"], f(x["g"], math.log(2.0)), f(x["tau"], 0.5),
                        f(x["beta"], 0.5), x["S0"], lib=lib)
    close(o1, o2, 1e-14, "zero pre-activations o")
    close(S1, S2, 1e-14, "zero pre-activations S_T")


def check_preact_bwd_finite_differences(lib=None, seed=11):
    """Gradients with respect to the pre-activations: central differences."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, 1, 1, 6, 3, 2)
    pre = dict(g=rng.normal(-0.5, 1.0, x["g"].shape), tau=rng.normal(0.0, 1.0, x["tau"].shape),
               beta=rng.normal(0.0, 1.0, x["beta"].shape))
    dO = rng.standard_normal(x["v"].shape)
    dST = rng.standard_normal(x["S0"].shape)

    def loss(p):
        o, ST = oracle.fwd(x["q"], x["k"], x["v"], p["g"], p["tau"], p["beta"], x["S0"], lib=lib,
                           preact=True)
        return float(np.sum(o * dO) + np.sum(ST * dST))

    gr = oracle.bwd(x["q"], x["k"], x["v"], pre["g"], pre["tau"], pre["beta"], x["S0"], dO, dST,
                    lib=lib, preact=True)
    h = 1e-6
    for n, gn in (("g", "dg"), ("tau", "dtau"), ("beta", "dbeta")):
        num = np.zeros_like(pre[n])
        for idx in np.ndindex(pre[n].shape):
            pp = {m: pre[m].copy() for m in pre}
            pm = {m: pre[m].copy() for m in pre}
            pp[n][idx] += h
            pm[n][idx] -= h
            num[idx] = (loss(pp) - loss(pm)) / (2 * h)
        close(gr[gn], num, 2e-7, f"preact {gn} finite differences")


PREACT_PINS = [check_preact_matches_torch_activations, check_preact_special_values,
               check_preact_bwd_finite_differences]


# ------------------------------------------ feedthrough o_t += d (.) v_t (Eq. (11)'s d_t)
def check_feedthrough_dead_state(lib=None, seed=12):
    """k = 0 and S_0 = 0 keep the state at zero, so o_t = d (.) v_t exactly (per
    head: d is [H, d_v], broadcast over batch and time)."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, 2, 3, 7, 4, 5)
    x["k"][:] = 0.0
    x["S0"][:] = 0.0
    d = rng.standard_normal((3, 5))
    o, ST = oracle.fwd(**x, d=d, lib=lib)
    close(o, d[None, :, None, :] * x["v"], 0.0, "dead state: o = d v")
    close(ST, np.zeros_like(ST), 0.0, "dead state: S_T")


def check_feedthrough_linearity(lib=None, seed=13):
    """o(d) - o(0) = d (.) v_t and S_T does not depend on d; the decode step
    agrees with the forward token by token."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, 2, 2, 9, 3, 4)
    d = rng.standard_normal((2, 4))
    o1, S1 = oracle.fwd(**x, d=d, lib=lib)
    o0, S0 = oracle.fwd(**x, lib=lib)
    close(o1 - o0, d[None, :, None, :] * x["v"], 1e-13, "o(d) - o(0)")
    close(S1, S0, 0.0, "S_T independent of d")
    S = np.ascontiguousarray(x["S0"].copy())
    seq = ("q", "k", "v", "g", "tau", "beta")
    for t in range(x["q"].shape[2]):
        ot = oracle.decode_step(*(x[n][:, :, t] for n in seq), S, d=d, lib=lib)
        close(ot, o1[:, :, t], 1e-13, f"decode with d, step {t}")


def check_feedthrough_bwd(lib=None, seed=14):
    """Reverse mode with the feedthrough: central differences of L = <o, dO> +
    <S_T, dS_T> for v and for d itself (d summed over the batch), and
    torch.autograd through the naive loop."""
    import torch
    rng = np.random.default_rng(seed)
    B, H, T, dk, dv = 2, 2, 5, 3, 2
    x = rand_inputs(rng, B, H, T, dk, dv, g_lo=0.1, g_hi=2.0)
    d = rng.standard_normal((H, dv))
    dO = rng.standard_normal((B, H, T, dv))
    dST = rng.standard_normal((B, H, dk, dv))
    gr = oracle.bwd(**x, dO=dO, dST=dST, d=d, lib=lib)

    def loss(xx, dd):
        o, ST = oracle.fwd(**xx, d=dd, lib=lib)
        return float(np.sum(o * dO) + np.sum(ST * dST))

    h = 1e-6
    num_d = np.zeros_like(d)
    for idx in np.ndindex(d.shape):
        dp, dm = d.copy(), d.copy()
        dp[idx] += h
        dm[idx] -= h
        num_d[idx] = (loss(x, dp) - loss(x, dm)) / (2 * h)
    close(gr["dd"], num_d, 2e-7, "finite differences dd")
    num_v = np.zeros_like(x["v"])
    for idx in np.ndindex(x["v"].shape):
        xp = {m: a.copy() for m, a in x.items()}
        xp["v"][idx] += h
        lp = loss(xp, d)
        xp["v"][idx] -= 2 * h
        num_v[idx] = (lp - loss(xp, d)) / (2 * h)
    close(gr["dv"], num_v, 2e-7, "finite differences dv with feedthrough")
    t = {n: torch.tensor(a, dtype=torch.float64, requires_grad=True) for n, a in x.items()}
    td = torch.tensor(d, dtype=torch.float64, requires_grad=True)
    S = t["S0"]
    outs = []
    for s in range(T):
        al = torch.exp(-t["g"][:, :, s] * t["tau"][:, :, s])
        kh = torch.pow(t["g"][:, :, s], t["tau"][:, :, s]) * t["k"][:, :, s]
        S = al[..., :, None] * S + kh[..., :, None] * (t["beta"][:, :, s] * t["v"][:, :, s])[..., None, :]
        outs.append((S * t["q"][:, :, s][..., :, None]).sum(-2) + td[None] * t["v"][:, :, s])
    L = (torch.stack(outs, 2) * torch.tensor(dO)).sum() + (S * torch.tensor(dST)).sum()
    L.backward()
    close(gr["dd"], td.grad.numpy(), 1e-11, "autograd dd")
    for n, gn in dict(q="dq", k="dk", v="dv", g="dg", tau="dtau", beta="dbeta", S0="dS0").items():
        close(gr[gn], t[n].grad.numpy(), 1e-11, f"autograd with feedthrough {gn}")


FEED_PINS = [check_feedthrough_dead_state, check_feedthrough_linearity, check_feedthrough_bwd]


# ------------------------------------------------ ShortConv (causal depthwise convolution)
def conv_inputs(rng, B=2, H=3, T=11, D=5, W=4):
    return dict(x=rng.standard_normal((B, H, T, D)), w=rng.standard_normal((H, D, W)),
                bias=rng.standard_normal((H, D)), xs=rng.standard_normal((B, H, W - 1, D)))


def check_conv_width_one(lib=None, seed=20):
    """W = 1: y = w (.) x + bias, element-wise; the carried state is empty."""
    rng = np.random.default_rng(seed)
    c = conv_inputs(rng, W=1)
    y, xs_out = oracle.shortconv_fwd(c["x"], c["w"], c["bias"], None, lib=lib)
    close(y, c["w"][None, :, None, :, 0] * c["x"] + c["bias"][None, :, None, :], 1e-14, "W=1")
    assert xs_out.shape == (2, 3, 0, 5)


def check_conv_numpy_convolve(lib=None, seed=21):
    """Every channel of every head equals numpy.convolve (full mode, first T
    outputs) of that channel's sequence with its filter (zero carried state)."""
    rng = np.random.default_rng(seed)
    for W in (2, 3, 4):
        c = conv_inputs(rng, W=W)
        y, _ = oracle.shortconv_fwd(c["x"], c["w"], None, None, lib=lib)
        ref = np.zeros_like(y)
        B, H, T, D = y.shape
        for b, h, ch in np.ndindex(B, H, D):
            ref[b, h, :, ch] = np.convolve(c["x"][b, h, :, ch], c["w"][h, ch])[:T]
        close(y, ref, 1e-13, f"numpy.convolve W={W}")


def check_conv_impulse_and_state(lib=None, seed=22):
    """An impulse at token t0 returns the filter at t0..t0+W-1 (causality: nothing
    before t0); a sequence cut in two with the state carried across equals the
    whole sequence, outputs and final state."""
    rng = np.random.default_rng(seed)
    c = conv_inputs(rng, T=12, W=4)
    x = np.zeros_like(c["x"])
    x[:, :, 5, :] = 1.0
    y, _ = oracle.shortconv_fwd(x, c["w"], None, None, lib=lib)
    assert np.all(y[:, :, :5] == 0.0) and np.all(y[:, :, 9:] == 0.0)
    close(y[:, :, 5:9], np.broadcast_to(np.moveaxis(c["w"], -1, 1)[None], y[:, :, 5:9].shape),
          0.0, "impulse response")
    for silu in (False, True):
        yw, sw = oracle.shortconv_fwd(c["x"], c["w"], c["bias"], c["xs"], silu=silu, lib=lib)
        for cut in (1, 2, 7):
            y1, s1 = oracle.shortconv_fwd(c["x"][:, :, :cut], c["w"], c["bias"], c["xs"], silu=silu,
                                          lib=lib)
            y2, s2 = oracle.shortconv_fwd(c["x"][:, :, cut:], c["w"], c["bias"], s1, silu=silu, lib=lib)
            close(np.concatenate([y1, y2], 2), yw, 1e-13, f"cut at {cut}")
            close(s2, sw, 0.0, f"state after cut at {cut}")
        close(sw, c["x"][:, :, -3:], 0.0, "final state = last W-1 inputs")


def check_conv_silu_and_grads(lib=None, seed=23):
    """SiLU output equals torch's silu of the linear output; the reverse mode
    equals torch.autograd through torch's grouped conv1d (left padding W-1 with
    the carried state, flipped filters) and central differences."""
    import torch
    rng = np.random.default_rng(seed)
    c = conv_inputs(rng, B=2, H=2, T=6, D=3, W=3)
    ylin, _ = oracle.shortconv_fwd(c["x"], c["w"], c["bias"], c["xs"], lib=lib)
    ysil, _ = oracle.shortconv_fwd(c["x"], c["w"], c["bias"], c["xs"], silu=True, lib=lib)
    close(ysil, torch.nn.functional.silu(torch.from_numpy(ylin)).numpy(), 1e-14, "silu")
    dy = rng.standard_normal(ylin.shape)
    dso = rng.standard_normal(c["xs"].shape)
    for silu in (False, True):
        gr = oracle.shortconv_bwd(c["x"], c["w"], c["bias"], c["xs"], dy, dso, silu=silu, lib=lib)
        t = {n: torch.tensor(a, dtype=torch.float64, requires_grad=True) for n, a in c.items()}
        B, H, T, D = c["x"].shape
        W = c["w"].shape[-1]
        seq = torch.cat([t["xs"], t["x"]], 2)                           # [B,H,W-1+T,D]
        inp = seq.permute(0, 1, 3, 2).reshape(B, H * D, W - 1 + T)
        wt = torch.flip(t["w"], [-1]).reshape(H * D, 1, W)
        z = torch.nn.functional.conv1d(inp, wt, t["bias"].reshape(H * D), groups=H * D)
        z = z.reshape(B, H, D, T).permute(0, 1, 3, 2)
        yt = torch.nn.functional.silu(z) if silu else z
        st = seq[:, :, T:]                                               # last W-1 inputs
        L = (yt * torch.tensor(dy)).sum() + (st * torch.tensor(dso)).sum()
        L.backward()
        for n, gn in (("x", "dx"), ("w", "dw"), ("bias", "dbias"), ("xs", "dxs")):
            close(gr[gn], t[n].grad.numpy(), 1e-12, f"conv autograd {gn} silu={silu}")
    # central differences on one weight and one state entry (silu on)
    gr = oracle.shortconv_bwd(c["x"], c["w"], c["bias"], c["xs"], dy, dso, silu=True, lib=lib)

    def loss(cc):
        y, s = oracle.shortconv_fwd(cc["x"], cc["w"], cc["bias"], cc["xs"], silu=True, lib=lib)
        return float(np.sum(y * dy) + np.sum(s * dso))

    h = 1e-6
    for n, idx, gn in (("w", (1, 2, 0), "dw"), ("xs", (0, 1, 1, 2), "dxs"), ("x", (1, 0, 5, 1), "dx")):
        cp = {m: a.copy() for m, a in c.items()}
        cm = {m: a.copy() for m, a in c.items()}
        cp[n][idx] += h
        cm[n][idx] -= h
        close(gr[gn][idx], (loss(cp) - loss(cm)) / (2 * h), 1e-7, f"conv finite difference {gn}")


CONV_PINS = [check_conv_width_one, check_conv_numpy_convolve, check_conv_impulse_and_state,
             check_conv_silu_and_grads]

# ------------------------------------------------------- low-rank beta_hat pins
def lowrank_inputs(rng, B=2, H=3, T=7, dk=4, dv=6, r=5):
    x = rand_inputs(rng, B, H, T, dk, dv)
    x["g"] = rng.standard_normal(x["g"].shape) - 1.0   # pre-activations
    x["tau"] = rng.standard_normal(x["tau"].shape)
    u = rng.standard_normal((B, T, r))
    w_up = rng.standard_normal((H, r, dv)) / np.sqrt(r)
    return x, u, w_up


def check_lowrank_rank_one_outer_product(lib=None, seed=40):
    """Rank 1: u[b,t,0] = a[b,t] and w_up[h,0,j] = c[h,j] give the
    pre-activation a[b,t] c[h,j] (an outer product, formed here with
    numpy.multiply.outer); the forward equals the full-rank pre-activation
    forward on it.  All axis lengths differ, so a swapped index changes shapes
    or values."""
    rng = np.random.default_rng(seed)
    x, _, _ = lowrank_inputs(rng)
    B, H, T, _ = x["q"].shape
    dv = x["v"].shape[-1]
    a = rng.standard_normal((B, T))
    c = rng.standard_normal((H, dv))
    pre = np.moveaxis(np.multiply.outer(a, c), 2, 1)            # [B,H,T,dv]
    o_lr, S_lr = oracle.fwd_lowrank(x["q"], x["k"], x["v"], x["g"], x["tau"], a[..., None],
                                    c[:, None, :], x["S0"], lib=lib)
    o_fr, S_fr = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["tau"], pre, x["S0"], lib=lib,
                            preact=True)
    close(o_lr, o_fr, 1e-13, "rank-1 low-rank o")
    close(S_lr, S_fr, 1e-13, "rank-1 low-rank S_T")


def check_lowrank_finite_differences(lib=None, seed=41):
    """du and dw_up against central differences of the forward's loss
    sum(o * dO) + sum(S_T * dS_T)."""
    rng = np.random.default_rng(seed)
    x, u, w_up = lowrank_inputs(rng, T=5)
    dO = rng.standard_normal(x["v"].shape)
    dST = rng.standard_normal(x["S0"].shape)
    gr = oracle.bwd_lowrank(x["q"], x["k"], x["v"], x["g"], x["tau"], u, w_up, x["S0"], dO, dST,
                            lib=lib)

    def loss(uu, ww):
        o, ST = oracle.fwd_lowrank(x["q"], x["k"], x["v"], x["g"], x["tau"], uu, ww, x["S0"], lib=lib)
        return float(np.sum(o * dO) + np.sum(ST * dST))

    h = 1e-6
    for idx in ((0, 0, 0), (1, 4, 3), (0, 2, 4)):
        up, um = u.copy(), u.copy()
        up[idx] += h
        um[idx] -= h
        close(gr["du"][idx], (loss(up, w_up) - loss(um, w_up)) / (2 * h), 1e-7, f"du {idx}")
    for idx in ((0, 0, 0), (2, 4, 5), (1, 3, 2)):
        wp, wm = w_up.copy(), w_up.copy()
        wp[idx] += h
        wm[idx] -= h
        close(gr["dw_up"][idx], (loss(u, wp) - loss(u, wm)) / (2 * h), 1e-7, f"dw_up {idx}")


LOWRANK_PINS = [check_lowrank_rank_one_outer_product, check_lowrank_finite_differences]


# ------------------------------------------------------------------ SW-SKA pins
def ska_inputs(rng, B=2, H=3, T=13, dk=4, dv=5):
    return dict(q=rng.standard_normal((B, H, T, dk)), k=rng.standard_normal((B, T, dk)),
                v=rng.standard_normal((B, H, T, dv)))


def check_ska_hand_example(lib=None):
    """Worked by hand: d_k = d_v = 1, scale 1, window 2, q = 1, k = (0, ln 3, 0),
    v = (1, 2, 5).  Token 0 sees only itself: 1.  Token 1 weighs e^0 : e^{ln 3}
    = 1 : 3, so (1 + 3*2)/4 = 7/4.  Token 2 sees tokens 1, 2 with weights 3 : 1,
    so (3*2 + 5)/4 = 11/4."""
    q = np.ones((1, 1, 3, 1))
    k = np.array([0.0, math.log(3.0), 0.0]).reshape(1, 3, 1)
    v = np.array([1.0, 2.0, 5.0]).reshape(1, 1, 3, 1)
    o = oracle.ska_fwd(q, k, v, 2, scale=1.0, lib=lib)
    close(o[0, 0, :, 0], [1.0, 1.75, 2.75], 1e-15, "SW-SKA hand example")


def check_ska_window_one_and_uniform(lib=None, seed=30):
    """Window 1 returns v itself; with q = 0 every score is 0, so each token
    returns the plain mean of v over its window: a moving average, taken here
    from numpy prefix sums."""
    rng = np.random.default_rng(seed)
    x = ska_inputs(rng)
    close(oracle.ska_fwd(x["q"], x["k"], x["v"], 1, lib=lib), x["v"], 1e-15, "window 1")
    T = x["v"].shape[2]
    for w in (2, 5, 40):
        o = oracle.ska_fwd(np.zeros_like(x["q"]), x["k"], x["v"], w, lib=lib)
        c = np.concatenate([np.zeros_like(x["v"][:, :, :1]), np.cumsum(x["v"], 2)], 2)
        lo = np.maximum(np.arange(T) - w + 1, 0)
        n = (np.arange(T) - lo + 1)[None, None, :, None]
        close(o, (c[:, :, 1:] - c[:, :, lo]) / n, 1e-13, f"moving average window {w}")


def check_ska_matches_torch_sdpa(lib=None, seed=31):
    """Against torch's scaled_dot_product_attention in fp64 (its own softmax and
    1/sqrt(d_k) default scale), the shared key row repeated for every head: causal
    when the window covers the sequence, else with a boolean band mask that keeps
    keys t-w+1..t; plus an explicit scale."""
    import torch
    F = torch.nn.functional
    rng = np.random.default_rng(seed)
    x = ska_inputs(rng, T=17, dk=6, dv=3)
    q, v = torch.from_numpy(x["q"]), torch.from_numpy(x["v"])
    k = torch.from_numpy(x["k"])[:, None].expand(-1, q.shape[1], -1, -1)
    T = q.shape[2]
    close(oracle.ska_fwd(x["q"], x["k"], x["v"], T, lib=lib),
          F.scaled_dot_product_attention(q, k, v, is_causal=True).numpy(), 1e-13, "full causal")
    ti = torch.arange(T)
    for w in (2, 3, 8):
        band = (ti[None, :] <= ti[:, None]) & (ti[None, :] > ti[:, None] - w)
        close(oracle.ska_fwd(x["q"], x["k"], x["v"], w, lib=lib),
              F.scaled_dot_product_attention(q, k, v, attn_mask=band).numpy(), 1e-13,
              f"band window {w}")
        close(oracle.ska_fwd(x["q"], x["k"], x["v"], w, scale=0.3, lib=lib),
              F.scaled_dot_product_attention(q, k, v, attn_mask=band, scale=0.3).numpy(), 1e-13,
              f"band window {w} scale 0.3")


def check_ska_invariants(lib=None, seed=32):
    """Adding one vector c to every key shifts each token's scores by the same
    q.c, which softmax ignores; permuting the heads of q and v permutes the
    output's heads (the key is shared, nothing else couples heads)."""
    rng = np.random.default_rng(seed)
    x = ska_inputs(rng)
    o = oracle.ska_fwd(x["q"], x["k"], x["v"], 4, lib=lib)
    c = rng.standard_normal(x["k"].shape[-1])
    close(oracle.ska_fwd(x["q"], x["k"] + c, x["v"], 4, lib=lib), o, 1e-12, "key shift")
    perm = [2, 0, 1]
    close(oracle.ska_fwd(x["q"][:, perm], x["k"], x["v"][:, perm], 4, lib=lib), o[:, perm], 0.0,
          "head permutation")


def check_ska_decode_matches_forward(lib=None, seed=33):
    """Token-by-token decode against ring caches (position p in slot p mod w),
    from empty caches and past several wrap-arounds, reproduces the forward at
    every token; after the last step the caches hold the last w keys and values
    at their slots.  Sequences of one batch at different positions decode in
    one call."""
    rng = np.random.default_rng(seed)
    x = ska_inputs(rng, T=19)
    B, H, T, dk = x["q"].shape
    dv = x["v"].shape[-1]
    for w in (1, 4, 7, 30):
        o = oracle.ska_fwd(x["q"], x["k"], x["v"], w, lib=lib)
        kc, vc = np.zeros((B, w, dk)), np.zeros((B, H, w, dv))
        for t in range(T):
            od, kc, vc = oracle.ska_decode(x["q"][:, :, t], x["k"][:, t], x["v"][:, :, t], kc, vc,
                                           np.full(B, t), w, lib=lib)
            close(od, o[:, :, t], 1e-13, f"decode window {w} token {t}")
        for p in range(max(0, T - w), T):
            close(kc[:, p % w], x["k"][:, p], 0.0, f"k cache slot of position {p}")
            close(vc[:, :, p % w], x["v"][:, :, p], 0.0, f"v cache slot of position {p}")
    # ragged positions: batch 0 at its token 3, batch 1 at its token 11
    w = 5
    o = oracle.ska_fwd(x["q"], x["k"], x["v"], w, lib=lib)
    kc, vc = np.zeros((B, w, dk)), np.zeros((B, H, w, dv))
    for b, t in ((0, 3), (1, 11)):
        for p in range(max(0, t - w + 1), t):
            kc[b, p % w], vc[b, :, p % w] = x["k"][b, p], x["v"][b, :, p]
    sel = (np.array([0, 1]), np.array([3, 11]))
    od, _, _ = oracle.ska_decode(x["q"][sel[0], :, sel[1]], x["k"][sel], x["v"][sel[0], :, sel[1]],
                                 kc, vc, np.array([3, 11]), w, lib=lib)
    close(od[0], o[0, :, 3], 1e-13, "ragged batch 0")
    close(od[1], o[1, :, 11], 1e-13, "ragged batch 1")


SKA_PINS = [check_ska_hand_example, check_ska_window_one_and_uniform, check_ska_matches_torch_sdpa,
            check_ska_invariants, check_ska_decode_matches_forward]

FORWARD_PINS = [check_worked_example, check_T1_closed_form, check_g_zero, check_tau_zero,
                check_quadratic, check_linearity, check_split_and_decode]
BACKWARD_PINS = [check_bwd_finite_differences, check_bwd_autograd]
ALL_PINS = (FORWARD_PINS + BACKWARD_PINS + PREACT_PINS + FEED_PINS + CONV_PINS + SKA_PINS +
            LOWRANK_PINS)
