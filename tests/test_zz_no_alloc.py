"""rdm_ddts_bwd_noalloc: the backward for callers that cannot allocate device
memory when they call it (a process that fixed its device-memory budget at
start-up, or a callback that must not call cudaMalloc / cudaFree because those
can synchronise the device).  It uses a fixed 16 MiB scratch array inside the
library instead of a workspace from the caller.

Collected last on purpose: it must pass both in a fresh process and after every
other test has run on the same device.  It compares, through the C ABI, the
no-allocation entry point against the existing workspace-taking entry point on
two calls in a row (the shared scratch keeps the first call's contents)."""
import ctypes

import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
from gated_linear_attention_ddts_b200 import _binding
from gated_linear_attention_ddts_b200.workloads import draw_sequence
from tests.parity import TOL, assert_close

pytestmark = pytest.mark.gpu
SEQ = ("q", "k", "v", "g", "tau", "beta")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_noalloc_backward_matches_workspace_backward(cuda_ok, dtype):
    for call, (T, seed) in enumerate(((150, 31), (97, 32))):
        x = draw_sequence(2, 3, T, 64, 128, dtype, seed=seed, s0_std=0.1, with_dO=True)
        d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
        dST = (0.1 * torch.randn(2, 3, 64, 128, generator=torch.Generator().manual_seed(seed))).cuda()
        ref = rdm.rdm_ddts_bwd(*(d[n] for n in SEQ), d["S0"], d["dO"], dST, impl="simt")
        got = rdm.rdm_ddts_bwd_noalloc(*(d[n] for n in SEQ), d["S0"], d["dO"], dST)
        torch.cuda.synchronize()
        assert rdm.rdm_ddts_sync_status() == rdm.RDM_OK
        for n in ("dq", "dk", "dv", "dg", "dtau", "dbeta", "dS0"):
            assert_close(got[n], ref[n], TOL[dtype], f"call {call}: {n}")


def test_noalloc_rejects_problems_larger_than_its_scratch(cuda_ok):
    fake = 1 << 20  # aligned placeholder; the size check refuses before any launch
    # q, k, v, g, tau, beta, S0, grad_o | grad_ST, saved | 6 gradients | grad_S0, workspace, bytes
    a = _binding.BwdArgs(64, 64, 4096, 64, 64, 0, _binding.RDM_BF16, 0, *([fake] * 8), None, None,
                         *([fake] * 6), None, None, 0)
    assert _binding.load().rdm_ddts_bwd_noalloc(ctypes.byref(a), None) == rdm.RDM_ERR_WORKSPACE
