"""Mutation check of the oracle's pins: plant one plausible slip at a time in a
copy of the oracle's C source (on the CPU), build it, and require that at least
one pin fails.  A pin set that let a mutant through would not pin the oracle."""
import os
import subprocess

import numpy as np

import pytest

import oracle
from tests import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "rdm_oracle.c")

# (name, original text, planted slip, pins that must catch it)
MUTANTS = [
    ("decay sign", "return exp(-g * tau);", "return exp(g * tau);", P.FORWARD_PINS),
    ("decay uses g only", "return exp(-g * tau);", "return exp(-g);", P.FORWARD_PINS),
    ("write gate swapped pow", "return pow(g, tau);", "return pow(tau, g);", P.FORWARD_PINS),
    ("write gate dropped", "double kh = gate_alpha_hat(g[i], tau[i]) * k[i];",
     "double kh = k[i];", P.FORWARD_PINS),
    ("decay dropped", "row[j] = al * row[j] + kh * (beta[j] * v[j]);",
     "row[j] = row[j] + kh * (beta[j] * v[j]);", P.FORWARD_PINS),
    ("input gate dropped", "row[j] = al * row[j] + kh * (beta[j] * v[j]);",
     "row[j] = al * row[j] + kh * v[j];", P.FORWARD_PINS),
    ("readout with k", "acc += S[(size_t)i * dv + j] * q[i];",
     "acc += S[(size_t)i * dv + j] * k[i];", P.FORWARD_PINS),
    ("readout before update", "    if (o) {\n        for (int j = 0; j < dv; ++j) {",
     "    if (o && 0) {\n        for (int j = 0; j < dv; ++j) {", P.FORWARD_PINS),
    ("bwd readout with k", "dS[(size_t)i * dv + j] += q[i] * dO[j];",
     "dS[(size_t)i * dv + j] += k[i] * dO[j];", P.BACKWARD_PINS),
    ("bwd decay not propagated", "dS[(size_t)i * dv + j] *= al[i];",
     "dS[(size_t)i * dv + j] *= 1.0;", P.BACKWARD_PINS),
    ("bwd dalpha uses S_t", "a2 += dS[(size_t)i * dv + j] * Sp[(size_t)i * dv + j];",
     "a2 += dS[(size_t)i * dv + j] * St[(size_t)i * dv + j];", P.BACKWARD_PINS),
    ("bwd dg sign", "J->dg[ok + i] = dal[i] * (-tau[i] * al[i]) + dah * dah_dg;",
     "J->dg[ok + i] = dal[i] * (tau[i] * al[i]) + dah * dah_dg;", P.BACKWARD_PINS),
    ("bwd dtau log of tau", "ah[i] * log(g[i]);", "ah[i] * log(tau[i]);", P.BACKWARD_PINS),
    ("bwd dbeta with beta", "J->dbeta[ov + j] = v[j] * dvh[j];",
     "J->dbeta[ov + j] = beta[j] * dvh[j];", P.BACKWARD_PINS),
    ("bwd dk without gate", "J->dk_[ok + i] = ah[i] * dkh[i];",
     "J->dk_[ok + i] = dkh[i];", P.BACKWARD_PINS),
    ("bwd dq uses S_{t-1}", "acc += St[(size_t)i * dv + j] * dO[j];",
     "acc += Sp[(size_t)i * dv + j] * dO[j];", P.BACKWARD_PINS),
    ("bwd dv transposed gate", "J->dv_[ov + j] = beta[j] * dvh[j];",
     "J->dv_[ov + j] = v[j] * dvh[j];", P.BACKWARD_PINS),
    ("bwd upstream dS_T ignored", "if (J->dST) memcpy(dS, J->dST + ss, sizeof(double) * SS);",
     "if (0) memcpy(dS, J->dST + ss, sizeof(double) * SS);", P.BACKWARD_PINS),
    ("feedthrough on the gated input", "for (int j = 0; j < dv; ++j) o[j] += d[j] * v[j];",
     "for (int j = 0; j < dv; ++j) o[j] += d[j] * v[j] * 0.5;", P.FEED_PINS),
    ("feedthrough weight of another head",
     "J->dfeed + (size_t)(p % J->H) * dv,\n                                                  J->v + ov",
     "J->dfeed + (size_t)((p + 1) % J->H) * dv,\n                                                  J->v + ov",
     P.FEED_PINS),
    ("bwd feedthrough dv dropped", "J->dv_[ov + j] += d[j] * dO[j];", "J->dv_[ov + j] += 0.0;",
     P.FEED_PINS),
    ("bwd feedthrough dd with vhat", "J->ddfeed[(size_t)p * dv + j] += dO[j] * v[j];",
     "J->ddfeed[(size_t)p * dv + j] += dO[j] * v[j] * beta[j];", P.FEED_PINS),
    ("conv filter flipped",
     "z += w[((size_t)h * D + c) * W + i] * conv_input(xp, sp, T, D, W, t - i, c);\n                y[",
     "z += w[((size_t)h * D + c) * W + (W - 1 - i)] * conv_input(xp, sp, T, D, W, t - i, c);\n                y[",
     P.CONV_PINS),
    ("conv state newest first", "int s = W - 1 + t;", "int s = -1 - t;", P.CONV_PINS),
    ("conv silu derivative", "gz *= s * (1.0 + z * (1.0 - s));", "gz *= s;", P.CONV_PINS),
    ("conv weight grad off by one", "dw[((size_t)h * D + c) * W + i] += gz * conv_input(xp, sp, T, D, W, ti, c);",
     "dw[((size_t)h * D + c) * W + i] += gz * conv_input(xp, sp, T, D, W, ti - 1, c);", P.CONV_PINS),
    ("ska window one too wide", "const int u0 = t - w + 1 > 0 ? t - w + 1 : 0;",
     "const int u0 = t - w > 0 ? t - w : 0;", P.SKA_PINS),
    ("ska scale dropped", "p[u] = scale * a;", "p[u] = a;", P.SKA_PINS),
    ("ska unnormalised", "o[j] += (p[u] / sum) * vrow[u][j];", "o[j] += p[u] * vrow[u][j];",
     P.SKA_PINS),
    ("ska value of the next head", "vr[u - u0] = v + (bh * T + u) * dv;",
     "vr[u - u0] = v + (((bh + 1) % ((size_t)B * H)) * T + u) * dv;", P.SKA_PINS),
    ("ska key of the next token", "kr[u - u0] = k + ((size_t)b * T + u) * dk;",
     "kr[u - u0] = k + ((size_t)b * T + (u + 1 < T ? u + 1 : u)) * dk;", P.SKA_PINS),
    ("ska decode slot shifted", "const int slot = (int)(t % w);",
     "const int slot = (int)((t + 1) % w);", P.SKA_PINS),
    ("ska decode window one too narrow",
     "const long long t = pos[b], u0 = t - w + 1 > 0 ? t - w + 1 : 0;",
     "const long long t = pos[b], u0 = t - w + 2 > 0 ? t - w + 2 : 0;", P.SKA_PINS),
]


@pytest.mark.parametrize("name,orig,slip,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, orig, slip, pins):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"mutation anchor not unique/found: {orig!r}"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(orig, slip))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-shared",
                           "-fPIC", "-o", str(so), str(mpath), "-lm", "-lpthread"])
    lib = oracle.load_library(str(so))
    caught = []
    for check in pins:
        try:
            check(lib=lib)
        except (AssertionError, RuntimeError, FloatingPointError, ValueError):
            caught.append(check.__name__)
    assert caught, f"mutant '{name}' passed every pin"


# Slips in the oracle's Python-level low-rank beta_hat step (the C source is
# untouched): each replaces one function for the duration of the check.
def _lr_heads_reversed(u, w_up):
    return np.einsum("btr,hrj->bhtj", oracle._f64(u), oracle._f64(w_up)[::-1])


def _lr_bwd_one_head(q, k, v, g_pre, tau_pre, u, w_up, S0, dO, dST=None, nthreads=None, lib=None,
                     d=None):
    out = oracle.bwd(q, k, v, g_pre, tau_pre, oracle.lowrank_beta_pre(u, w_up), S0, dO, dST,
                     lib=lib, preact=True)
    db = out.pop("dbeta")
    w = oracle._f64(w_up)
    out["du"] = np.einsum("btj,rj->btr", db[:, 0], w[0]) * w.shape[0]
    out["dw_up"] = np.einsum("btr,bhtj->hrj", oracle._f64(u), db)
    return out


def _lr_bwd_no_sigmoid_grad(q, k, v, g_pre, tau_pre, u, w_up, S0, dO, dST=None, nthreads=None,
                            lib=None, d=None):
    pre = oracle.lowrank_beta_pre(u, w_up)
    out = oracle.bwd(q, k, v, g_pre, tau_pre, pre, S0, dO, dST, lib=lib, preact=True)
    s = oracle.sigmoid(pre)
    db = out.pop("dbeta") / (s * (1.0 - s))
    out["du"] = np.einsum("bhtj,hrj->btr", db, oracle._f64(w_up))
    out["dw_up"] = np.einsum("btr,bhtj->hrj", oracle._f64(u), db)
    return out


LOWRANK_SLIPS = [("lowrank_beta_pre", _lr_heads_reversed), ("bwd_lowrank", _lr_bwd_one_head),
                 ("bwd_lowrank", _lr_bwd_no_sigmoid_grad)]


@pytest.mark.parametrize("name,slip", LOWRANK_SLIPS, ids=[f.__name__ for _, f in LOWRANK_SLIPS])
def test_lowrank_pins_catch_python_slip(monkeypatch, name, slip):
    monkeypatch.setattr(oracle, name, slip)
    caught = []
    for check in P.LOWRANK_PINS:
        try:
            check()
        except (AssertionError, ValueError):
            caught.append(check.__name__)
    assert caught, f"no low-rank pin caught the slip {slip.__name__}"
