"""fp64 CPU oracle of the DDTS recurrence (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package; the CUDA library never does, and the two
share no code.  The arithmetic lives in ``rdm_oracle.c`` (plain C, double
precision, token by token); this module only builds it with gcc, marshals
numpy arrays and calls it.

Definition followed (Rodimus*, digest.lyk-ai.com summary, section "Method",
DDTS gates; paperhub.cn OpenReview rebuttal, "Efficient Parallelization"
bullet and Q2 on the fixed-size recurrent state):

    alpha_t = exp(-g_t * tau_t),  alpha_hat_t = g_t ** tau_t
    S_t = diag(alpha_t) S_{t-1} + (alpha_hat_t * k_t)(beta_hat_t * v_t)^T
    o_t = S_t^T q_t

With ``preact=True`` the gate inputs are taken before their activations (the
same page names a selection gate g_t, a temperature gate tau_t and a low-rank
beta_hat_t without printing the activations; the reading used here is
g = softplus(.), which keeps g >= 0, and tau = sigmoid(.), beta_hat =
sigmoid(.)): they are activated element-wise in fp64 around the same token
loop, and the backward applies the chain rule to the three gradients.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rdm_oracle.c")
_LIB = os.path.join(_HERE, "librdm_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile rdm_oracle.c into librdm_oracle.so next to it (gcc -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-shared",
                               "-fPIC", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str):
    """Open a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(ctypes.c_double)
    I = ctypes.c_int
    lib.rdm_oracle_fwd.argtypes = [I] * 5 + [P] * 10 + [I]
    lib.rdm_oracle_bwd.argtypes = [I] * 5 + [P] * 18 + [I]
    lib.rdm_oracle_decode_step.argtypes = [I] * 4 + [P] * 9 + [I]
    lib.rdm_oracle_shortconv_fwd.argtypes = [I] * 5 + [P] * 4 + [I] + [P] * 2
    lib.rdm_oracle_shortconv_bwd.argtypes = [I] * 5 + [P] * 4 + [I] + [P] * 6
    D = ctypes.c_double
    lib.rdm_oracle_ska_fwd.argtypes = [I] * 6 + [D] + [P] * 4
    lib.rdm_oracle_ska_decode.argtypes = [I] * 5 + [D, ctypes.POINTER(ctypes.c_longlong)] + [P] * 6
    for f in (lib.rdm_oracle_fwd, lib.rdm_oracle_bwd, lib.rdm_oracle_decode_step,
              lib.rdm_oracle_shortconv_fwd, lib.rdm_oracle_shortconv_bwd,
              lib.rdm_oracle_ska_fwd, lib.rdm_oracle_ska_decode):
        f.restype = I
    return lib


def _load(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def _f64(x):
    """Any array-like (numpy or torch, any float dtype) -> C-contiguous float64 numpy."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def softplus(x):
    """log(1 + exp(x)) in float64."""
    return np.logaddexp(0.0, x)


def sigmoid(x):
    """1 / (1 + exp(-x)) in float64 (each branch evaluated where it cannot overflow)."""
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def activate(g_pre, tau_pre, beta_pre):
    """Gate activations: g = softplus, tau = sigmoid, beta_hat = sigmoid."""
    return softplus(g_pre), sigmoid(tau_pre), sigmoid(beta_pre)


def fwd(q, k, v, g, tau, beta, S0=None, nthreads=None, lib=None, preact=False, d=None):
    """Token-by-token forward.  q,k,g,tau [B,H,T,dk]; v,beta [B,H,T,dv];
    S0 [B,H,dk,dv] or None (zeros).  Returns (o [B,H,T,dv], S_T [B,H,dk,dv]).
    preact: g, tau, beta are pre-activations (see the module docstring).
    d: feedthrough weights [H,dv] or None; o_t += d (.) v_t (the feedthrough of
    Eq. (11), paperhub.cn rebuttal answer to Q6; reading: one weight per head
    and value channel, applied to v_t)."""
    q, k, v, g, tau, beta, S0, d = map(_f64, (q, k, v, g, tau, beta, S0, d))
    if preact:
        g, tau, beta = activate(g, tau, beta)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, T, dv))
    ST = np.zeros((B, H, dk, dv))
    rc = _load(lib).rdm_oracle_fwd(B, H, T, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(tau), _p(beta),
                                _p(S0), _p(d), _p(o), _p(ST), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("rdm_oracle_fwd failed")
    return o, ST


def bwd(q, k, v, g, tau, beta, S0, dO, dST=None, nthreads=None, lib=None, preact=False, d=None):
    """Reverse mode of the token loop.  Returns dict dq, dk, dv, dg, dtau, dbeta, dS0
    (and dd [H,dv], the feedthrough gradient summed over the batch, when d is given).
    preact: g, tau, beta are pre-activations and dg, dtau, dbeta are the gradients
    with respect to them (d softplus = sigmoid, d sigmoid = s (1 - s))."""
    q, k, v, g, tau, beta, S0, dO, dST, d = map(_f64, (q, k, v, g, tau, beta, S0, dO, dST, d))
    if preact:
        g_pre = g
        g, tau, beta = activate(g, tau, beta)
        out = bwd(q, k, v, g, tau, beta, S0, dO, dST, nthreads=nthreads, lib=lib, d=d)
        out["dg"] *= sigmoid(g_pre)
        out["dtau"] *= tau * (1.0 - tau)
        out["dbeta"] *= beta * (1.0 - beta)
        return out
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    out = {n: np.zeros(q.shape) for n in ("dq", "dk", "dg", "dtau")}
    out.update({n: np.zeros(v.shape) for n in ("dv", "dbeta")})
    out["dS0"] = np.zeros((B, H, dk, dv))
    dd_pair = np.zeros((B, H, dv)) if d is not None else None
    rc = _load(lib).rdm_oracle_bwd(B, H, T, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(tau), _p(beta),
                                _p(S0), _p(dO), _p(dST), _p(d), _p(out["dq"]), _p(out["dk"]),
                                _p(out["dv"]), _p(out["dg"]), _p(out["dtau"]), _p(out["dbeta"]),
                                _p(out["dS0"]), _p(dd_pair), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("rdm_oracle_bwd failed")
    if d is not None:
        out["dd"] = dd_pair.sum(axis=0)
    return out


def lowrank_beta_pre(u, w_up):
    """beta_hat's pre-activation from its low-rank factorisation (Rodimus*,
    digest.lyk-ai.com summary, "Method": beta_hat is built from low-rank
    matrices to cut parameters and filter input noise).  The reading: the
    token's input projected down to rank r, u [B,T,r] (one row per token, shared
    by the heads), times an up-projection w_up [H,r,dv] gives the
    pre-activation [B,H,T,dv]; beta_hat = sigmoid of it."""
    return np.einsum("btr,hrj->bhtj", _f64(u), _f64(w_up))


def fwd_lowrank(q, k, v, g_pre, tau_pre, u, w_up, S0=None, nthreads=None, lib=None, d=None):
    """Forward with every gate passed before its activation and beta_hat's
    pre-activation given by its low-rank factors u [B,T,r], w_up [H,r,dv]."""
    return fwd(q, k, v, g_pre, tau_pre, lowrank_beta_pre(u, w_up), S0, nthreads=nthreads, lib=lib,
               preact=True, d=d)


def bwd_lowrank(q, k, v, g_pre, tau_pre, u, w_up, S0, dO, dST=None, nthreads=None, lib=None, d=None):
    """Reverse mode of fwd_lowrank: the gradient with respect to beta_hat's
    pre-activation, db [B,H,T,dv], is contracted into du[b,t,:] = sum_h
    w_up[h] db[b,h,t,:] and dw_up[h] = sum_{b,t} u[b,t,:]^T db[b,h,t,:]; the
    dict has du and dw_up in place of dbeta."""
    u, w_up = _f64(u), _f64(w_up)
    out = bwd(q, k, v, g_pre, tau_pre, lowrank_beta_pre(u, w_up), S0, dO, dST, nthreads=nthreads,
              lib=lib, preact=True, d=d)
    db = out.pop("dbeta")
    out["du"] = np.einsum("bhtj,hrj->btr", db, w_up)
    out["dw_up"] = np.einsum("btr,bhtj->hrj", u, db)
    return out


def decode_step(q, k, v, g, tau, beta, S, nthreads=None, lib=None, d=None):
    """One token per (b,h).  q,k,g,tau [B,H,dk]; v,beta [B,H,dv]; S [B,H,dk,dv]
    float64 numpy, updated in place; d feedthrough [H,dv] or None.  Returns o [B,H,dv]."""
    if not (isinstance(S, np.ndarray) and S.dtype == np.float64 and S.flags.c_contiguous):
        raise TypeError("S must be a C-contiguous float64 numpy array (updated in place)")
    q, k, v, g, tau, beta, d = map(_f64, (q, k, v, g, tau, beta, d))
    B, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, dv))
    rc = _load(lib).rdm_oracle_decode_step(B, H, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(tau),
                                        _p(beta), _p(d), _p(S), _p(o), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("rdm_oracle_decode_step failed")
    return o


def shortconv_fwd(x, w, bias=None, xs=None, silu=False, lib=None):
    """Causal depthwise short convolution along the tokens (the ShortConv of the
    Rodimus block; digest.lyk-ai.com summary, "Method"; width, activation and
    carried state are this library's reading):
        z[b,h,t,c] = bias[h,c] + sum_i w[h,c,i] x[b,h,t-i,c],   y = z or z*sigmoid(z)
    x [B,H,T,D]; w [H,D,W]; bias [H,D] or None; xs [B,H,W-1,D] the previous W-1
    inputs (oldest first) or None for zeros.  Returns (y [B,H,T,D], state after
    the sequence [B,H,W-1,D])."""
    x, w, bias, xs = map(_f64, (x, w, bias, xs))
    B, H, T, D = x.shape
    W = w.shape[-1]
    y = np.zeros((B, H, T, D))
    xs_out = np.zeros((B, H, W - 1, D))
    rc = _load(lib).rdm_oracle_shortconv_fwd(B, H, T, D, W, _p(x), _p(w), _p(bias), _p(xs),
                                             int(bool(silu)), _p(y), _p(xs_out))
    if rc != 0:
        raise RuntimeError("rdm_oracle_shortconv_fwd failed")
    return y, xs_out


def shortconv_bwd(x, w, bias, xs, dy, dxs_out=None, silu=False, lib=None):
    """Reverse mode of shortconv_fwd.  Returns dict dx, dw, dbias (None without
    bias) and dxs (None without a carried-in state)."""
    x, w, bias, xs, dy, dxs_out = map(_f64, (x, w, bias, xs, dy, dxs_out))
    B, H, T, D = x.shape
    W = w.shape[-1]
    out = dict(dx=np.zeros((B, H, T, D)), dw=np.zeros((H, D, W)),
               dbias=np.zeros((H, D)) if bias is not None else None,
               dxs=np.zeros((B, H, W - 1, D)) if xs is not None else None)
    rc = _load(lib).rdm_oracle_shortconv_bwd(B, H, T, D, W, _p(x), _p(w), _p(bias), _p(xs),
                                             int(bool(silu)), _p(dy), _p(dxs_out), _p(out["dx"]),
                                             _p(out["dw"]), _p(out["dbias"]), _p(out["dxs"]))
    if rc != 0:
        raise RuntimeError("rdm_oracle_shortconv_bwd failed")
    return out


def ska_fwd(q, k, v, window, scale=None, lib=None):
    """Sliding-window shared-key attention (SW-SKA of Rodimus+; digest.lyk-ai.com
    summary, "Method"; paperhub.cn rebuttal, Q1): token t of head h attends to
    tokens max(0, t-window+1)..t through the one key row per token that all heads
    share, scores scaled by ``scale`` (default 1/sqrt(d_k)), softmax over the
    window.  q [B,H,T,dk], k [B,T,dk], v [B,H,T,dv] -> o [B,H,T,dv] float64."""
    q, k, v = map(_f64, (q, k, v))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    sc = 1.0 / np.sqrt(dk) if scale is None else float(scale)
    o = np.zeros((B, H, T, dv))
    if _load(lib).rdm_oracle_ska_fwd(B, H, T, dk, dv, int(window), sc, _p(q), _p(k), _p(v),
                                     _p(o)) != 0:
        raise RuntimeError("rdm_oracle_ska_fwd failed")
    return o


def ska_decode(q, k, v, k_cache, v_cache, pos, window, scale=None, lib=None):
    """One SW-SKA decode step against ring caches of ``window`` slots (position p
    lives in slot p mod window).  q [B,H,dk], k [B,dk], v [B,H,dv], k_cache
    [B,window,dk], v_cache [B,H,window,dv], pos [B] the tokens seen before this
    one.  Returns (o [B,H,dv], new k_cache, new v_cache), all float64."""
    q, k, v, kc, vc = map(_f64, (q, k, v, k_cache, v_cache))
    kc, vc = kc.copy(), vc.copy()
    B, H, dk = q.shape
    dv = v.shape[-1]
    sc = 1.0 / np.sqrt(dk) if scale is None else float(scale)
    ps = np.ascontiguousarray(np.asarray(pos.cpu() if hasattr(pos, "cpu") else pos,
                                         dtype=np.int64))
    o = np.zeros((B, H, dv))
    rc = _load(lib).rdm_oracle_ska_decode(
        B, H, dk, dv, int(window), sc, ps.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)),
        _p(q), _p(k), _p(v), _p(kc), _p(vc), _p(o))
    if rc != 0:
        raise RuntimeError("rdm_oracle_ska_decode failed")
    return o, kc, vc
