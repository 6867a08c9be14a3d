"""Seeded synthetic inputs for the DDTS recurrence.

This module holds the workload shapes and the random draws only; it contains
none of the recurrence's arithmetic.  Both the CUDA path (tests, bench) and the
fp64 oracle consume the tensors it returns: bf16 workloads are rounded to bf16
once, here, and the oracle widens those same rounded values.

Value distributions (per token and channel):
    q, k ~ N(0,1)/sqrt(d_k)       v ~ N(0,1)
    g    = softplus(N(mu_g, 1))    (mu_g = -1; -2 for the long-memory workload)
    tau  = sigmoid(N(0,1))        beta_hat = sigmoid(N(0,1))
    dO   ~ N(0,1)                 S_0 ~ N(0, 0.1^2) where a workload has one
Draw order from one generator: q, k, v, g, tau, beta_hat, dO, S_0.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BASE_SEED = 20241009


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "fwd", "fwdbwd" or "decode"
    dtype: str           # "f32" or "bf16"
    B: int
    H: int
    T: int               # decode: number of steps
    dk: int
    dv: int
    mu_g: float = -1.0
    s0_std: float = 0.0  # 0 => S_0 = 0
    return_state: bool = False
    chunk: int = 64
    seed: int = BASE_SEED

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    0: Workload("fp32 fwd B1 H1 T128 dk16 dv32", "fwd", "f32", 1, 1, 128, 16, 32,
                seed=BASE_SEED + 0),
    1: Workload("bf16 fwd B8 H6 T2048 dk64 dv128 (130M-scale layer)", "fwd", "bf16",
                8, 6, 2048, 64, 128, seed=BASE_SEED + 1),
    2: Workload("bf16 fwd long-context B1 H16 T32768 dk128 dv128", "fwd", "bf16",
                1, 16, 32768, 128, 128, mu_g=-2.0, return_state=True, seed=BASE_SEED + 2),
    3: Workload("bf16 fwd+bwd B4 H16 T4096 dk64 dv128", "fwdbwd", "bf16",
                4, 16, 4096, 64, 128, s0_std=0.1, seed=BASE_SEED + 3),
    4: Workload("decode B256 H16 dk64 dv128, 1024 steps", "decode", "bf16",
                256, 16, 1024, 64, 128, seed=BASE_SEED + 4),
}


def _gen(device, seed):
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    return gen


def draw_sequence(B, H, T, dk, dv, dtype=torch.bfloat16, seed=BASE_SEED, mu_g=-1.0,
                  s0_std=0.0, with_dO=False, device="cpu", preact=False):
    """Inputs for one forward (and backward) call, layout [B,H,T,D].

    Returns a dict with q, k, g, tau [B,H,T,dk], v, beta [B,H,T,dv] in `dtype`,
    optionally dO [B,H,T,dv] in `dtype`, and S0 [B,H,dk,dv] float32 (None when
    s0_std == 0).  With preact, g, tau and beta are the normal draws before
    their softplus / sigmoid (same random numbers as without)."""
    gen = _gen(device, seed)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    q = torch.randn(B, H, T, dk, **f32) / math.sqrt(dk)
    k = torch.randn(B, H, T, dk, **f32) / math.sqrt(dk)
    v = torch.randn(B, H, T, dv, **f32)
    g_pre = torch.randn(B, H, T, dk, **f32) + mu_g
    tau_pre = torch.randn(B, H, T, dk, **f32)
    beta_pre = torch.randn(B, H, T, dv, **f32)
    if preact:
        g, tau, beta = g_pre, tau_pre, beta_pre
    else:
        g = torch.nn.functional.softplus(g_pre)
        tau = torch.sigmoid(tau_pre)
        beta = torch.sigmoid(beta_pre)
    out = dict(q=q, k=k, v=v, g=g, tau=tau, beta=beta)
    out = {n: t.to(dtype).contiguous() for n, t in out.items()}
    if with_dO:
        out["dO"] = torch.randn(B, H, T, dv, **f32).to(dtype).contiguous()
    out["S0"] = (torch.randn(B, H, dk, dv, **f32) * s0_std).contiguous() if s0_std else None
    return out


def draw_workload(w: Workload, device="cpu", **over):
    """Inputs of a sequence workload (kinds "fwd" and "fwdbwd")."""
    args = dict(B=w.B, H=w.H, T=w.T, dk=w.dk, dv=w.dv, dtype=w.torch_dtype, seed=w.seed,
                mu_g=w.mu_g, s0_std=w.s0_std, with_dO=(w.kind == "fwdbwd"), device=device)
    args.update(over)
    return draw_sequence(**args)


def draw_decode(B, H, dk, dv, steps, dtype=torch.bfloat16, seed=BASE_SEED + 4, mu_g=-1.0,
                device="cpu"):
    """Per-step decode inputs, layout [steps,B,H,D] (one token per (b,h) per step)."""
    gen = _gen(device, seed)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    q = torch.randn(steps, B, H, dk, **f32) / math.sqrt(dk)
    k = torch.randn(steps, B, H, dk, **f32) / math.sqrt(dk)
    v = torch.randn(steps, B, H, dv, **f32)
    g = torch.nn.functional.softplus(torch.randn(steps, B, H, dk, **f32) + mu_g)
    tau = torch.sigmoid(torch.randn(steps, B, H, dk, **f32))
    beta = torch.sigmoid(torch.randn(steps, B, H, dv, **f32))
    out = dict(q=q, k=k, v=v, g=g, tau=tau, beta=beta)
    return {n: t.to(dtype).contiguous() for n, t in out.items()}


# Sliding-window shared-key attention (the attention half of the Rodimus+ block;
# the pages give neither its window nor its head sizes): a forward on a
# 130M-scale layer, d_model 768 as 12 heads of 64 with one shared key head,
# window 512 -- (B, H, T, d, window) -- and batched decode at the 1.6B scale,
# d_model 2048 as 16 heads of 128, against full ring caches of 512 slots --
# (B, H, d, window, steps per timed graph).  q, k, v ~ N(0, 1) in bf16.
SKA_FWD = (8, 12, 2048, 64, 512)
SKA_DEC = (256, 16, 128, 512, 64)


def draw_lowrank(B, H, T, dv, r, dtype=torch.bfloat16, seed=BASE_SEED + 40, device="cpu"):
    """Factors of a low-rank beta_hat: u [B,T,r] ~ N(0, 1) in `dtype` (one row
    per token, shared by the heads) and w_up [H,r,dv] ~ N(0, 1/r) float32."""
    gen = _gen(device, seed)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    u = torch.randn(B, T, r, **f32).to(dtype).contiguous()
    w_up = (torch.randn(H, r, dv, **f32) / math.sqrt(r)).contiguous()
    return u, w_up
