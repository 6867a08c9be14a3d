"""The C-ABI library builds, loads and exports every symbol include/rdm_ddts.h
declares; host-side validation refuses bad arguments without launching (these
run without a GPU: each call fails before touching the device)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from gated_linear_attention_ddts_b200 import _binding, build
    build.build()
    return _binding.load()


def declared_functions():
    hdr = open(os.path.join(ROOT, "include", "rdm_ddts.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(rdm_[a-z_0-9]+)\s*\(", hdr)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("rdm_ddts_fwd", "rdm_ddts_bwd", "rdm_ddts_decode_step"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from gated_linear_attention_ddts_b200 import _binding
    out = subprocess.run(["nm", "-D", "--defined-only", _binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\S+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lib, n)


def test_binding_uses_the_same_names():
    import gated_linear_attention_ddts_b200 as m
    for n in declared_functions():
        assert callable(getattr(m, n)), n


def test_status_strings(lib):
    for s in range(6):
        assert lib.rdm_status_string(s)
    assert lib.rdm_ddts_version() >= 100


def _fwd_args(**kw):
    from gated_linear_attention_ddts_b200._binding import FwdArgs
    fake = 1 << 20  # aligned non-null placeholder; validation rejects before use
    base = dict(B=1, H=1, T=8, dk=64, dv=64, chunk=0, dtype=1, impl=0, q=fake, k=fake, v=fake,
                g=fake, tau=fake, beta=fake, S0=None, o=fake, ST=None, saved_states=None)
    base.update(kw)
    return FwdArgs(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), 1), (dict(H=-1), 1), (dict(T=-1), 1), (dict(dk=0), 1),
    (dict(dk=48), 2), (dict(dv=256), 2), (dict(chunk=48), 2), (dict(chunk=-2), 1),
    (dict(dtype=7), 1), (dict(impl=9), 1), (dict(q=None), 1), (dict(o=None), 1),
    (dict(k=(1 << 20) + 8), 1), (dict(S0=(1 << 20) + 4), 1), (dict(gate_inputs=7), 1),
    # low-rank beta_hat: rank 8 or 16, pre-activation gates, factors given and aligned
    (dict(beta_rank=-1), 1), (dict(beta_rank=4, gate_inputs=1, beta_u=1 << 20, beta_w=1 << 20), 2),
    (dict(beta_rank=16, gate_inputs=0, beta_u=1 << 20, beta_w=1 << 20), 1),
    (dict(beta_rank=16, gate_inputs=1, beta_u=None, beta_w=1 << 20), 1),
    (dict(beta_rank=8, gate_inputs=1, beta_u=1 << 20, beta_w=(1 << 20) + 4), 1),
])
def test_fwd_validation(lib, kw, status):
    a = _fwd_args(**kw)
    assert lib.rdm_ddts_fwd(ctypes.byref(a), None) == status


def _bwd_args(**kw):
    from gated_linear_attention_ddts_b200._binding import BwdArgs
    fake = 1 << 20
    base = dict(B=1, H=1, T=8, dk=64, dv=64, chunk=0, dtype=1, impl=0, q=fake, k=fake, v=fake,
                g=fake, tau=fake, beta=fake, S0=None, grad_o=fake, grad_ST=None,
                saved_states=None, grad_q=fake, grad_k=fake, grad_v=fake, grad_g=fake,
                grad_tau=fake, grad_beta=fake, grad_S0=None, workspace=None, workspace_bytes=0,
                gate_inputs=0)
    base.update(kw)
    return BwdArgs(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), 1), (dict(T=-3), 1), (dict(dk=48), 2), (dict(dv=256), 2), (dict(dtype=5), 1),
    (dict(impl=9), 1), (dict(gate_inputs=2), 1), (dict(grad_o=None), 1), (dict(q=None), 1),
    (dict(grad_q=(1 << 20) + 8), 1), (dict(grad_beta=None), 1), (dict(S0=(1 << 20) + 4), 1),
    (dict(saved_states=(1 << 20) + 4), 1), (dict(workspace=(1 << 20) + 2), 1),
    (dict(beta_rank=32, gate_inputs=1, beta_u=1 << 20, beta_w=1 << 20), 2),
    (dict(beta_rank=8, gate_inputs=1, beta_u=1 << 20, beta_w=1 << 20, grad_beta_w=1 << 20), 1),
    (dict(beta_rank=8, gate_inputs=1, beta_u=1 << 20, beta_w=1 << 20, grad_beta_u=1 << 20,
          grad_beta_w=(1 << 20) + 8), 1),
])
def test_bwd_validation(lib, kw, status):
    """Host-side checks of the backward reject before touching the device."""
    a = _bwd_args(**kw)
    assert lib.rdm_ddts_bwd(ctypes.byref(a), None) == status


def test_workspace_size_of_invalid_sizes(lib):
    size_max = ctypes.c_size_t(-1).value
    assert lib.rdm_ddts_fwd_workspace_size(ctypes.byref(_fwd_args(B=0))) == size_max
    assert lib.rdm_ddts_bwd_workspace_size(ctypes.byref(_bwd_args(dk=-1))) == size_max


def test_decode_validation(lib):
    fake = 1 << 20
    args = [fake] * 6 + [fake, fake]
    assert lib.rdm_ddts_decode_step(0, 1, 64, 64, 1, *args, None) == 1
    assert lib.rdm_ddts_decode_step(1, 1, 40, 64, 1, *args, None) == 2
    bad = list(args)
    bad[6] = fake + 4  # misaligned state
    assert lib.rdm_ddts_decode_step(1, 1, 64, 64, 1, *bad, None) == 1
    assert lib.rdm_ddts_decode_step(1, 1, 64, 64, 1, *([None] + args[1:]), None) == 1


def test_sizes(lib):
    assert lib.rdm_ddts_saved_states_size(2, 3, 130, 64, 128, 64) == 2 * 3 * 3 * 64 * 128 * 4
    assert lib.rdm_ddts_saved_states_size(2, 3, 130, 64, 100, 64) == 0


def test_test_hooks_validation(lib):
    from gated_linear_attention_ddts_b200._binding import RDM_ERR_INVALID_ARG, RDM_OK
    assert lib.rdm_ddts_set_test_hooks(-1, 0) == RDM_ERR_INVALID_ARG
    assert lib.rdm_ddts_set_test_hooks(0, 2) == RDM_ERR_INVALID_ARG
    assert lib.rdm_ddts_set_test_hooks(1000, 1) == RDM_OK
    assert lib.rdm_ddts_set_test_hooks(0, 0) == RDM_OK


def _ska_fwd(**kw):
    from gated_linear_attention_ddts_b200._binding import SkaFwdArgs
    fake = 1 << 20
    base = dict(B=1, H=2, T=8, dk=64, dv=64, window=4, scale=0.0, dtype=1, q=fake, k=fake, v=fake,
                o=fake, k_cache=None, v_cache=None, pos=None)
    base.update(kw)
    return SkaFwdArgs(**base)


def _ska_dec(**kw):
    from gated_linear_attention_ddts_b200._binding import SkaDecodeArgs
    fake = 1 << 20
    base = dict(B=1, H=2, dk=64, dv=64, window=4, scale=0.0, dtype=1, q=fake, k=fake, v=fake,
                k_cache=fake, v_cache=fake, pos=fake, advance_pos=1, o=fake)
    base.update(kw)
    return SkaDecodeArgs(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(window=0), 1), (dict(B=0), 1), (dict(T=-1), 1), (dict(scale=-1.0), 1),
    (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1), (dict(dtype=0), 2),
    (dict(dtype=5), 1), (dict(dk=32), 2), (dict(dv=16), 2), (dict(q=(1 << 20) + 8), 1),
    (dict(o=None), 1), (dict(k_cache=(1 << 20) + 2), 1), (dict(pos=(1 << 20) + 2), 1)])
def test_ska_fwd_validation(lib, kw, status):
    assert lib.rdm_ska_fwd(ctypes.byref(_ska_fwd(**kw)), None) == status


@pytest.mark.parametrize("kw,status", [
    (dict(window=0), 1), (dict(window=32769), 1), (dict(H=0), 1), (dict(scale=-2.0), 1),
    (dict(dtype=0), 2), (dict(dk=16), 2), (dict(k_cache=None), 1), (dict(pos=None), 1),
    (dict(v=(1 << 20) + 2), 1), (dict(o=None), 1)])
def test_ska_decode_validation(lib, kw, status):
    assert lib.rdm_ska_decode(ctypes.byref(_ska_dec(**kw)), None) == status


def _conv(**kw):
    from gated_linear_attention_ddts_b200._binding import RDM_BF16, ConvArgs
    a = dict(B=1, H=2, T=64, D=64, W=4, dtype=RDM_BF16, silu=1, x=4096, weight=8192, bias=None,
             state_in=None, y=12288, state_out=None)
    a.update(kw)
    return ConvArgs(a["B"], a["H"], a["T"], a["D"], a["W"], a["dtype"], a["silu"], a["x"], a["weight"],
                    a["bias"], a["state_in"], a["y"], a["state_out"])


def test_shortconv_many_validation(lib):
    """The batched ShortConv calls refuse n outside [1, 4], problems of
    different kinds (dtype, W, SiLU) and any problem that fails its own checks,
    before any CUDA call."""
    from gated_linear_attention_ddts_b200._binding import (RDM_ERR_INVALID_ARG, RDM_ERR_UNSUPPORTED,
                                                           ConvArgs)
    two = (ConvArgs * 2)(_conv(), _conv(D=128))
    assert lib.rdm_shortconv_fwd_many(two, 0, None) == RDM_ERR_INVALID_ARG
    assert lib.rdm_shortconv_fwd_many(two, 5, None) == RDM_ERR_INVALID_ARG
    assert lib.rdm_shortconv_fwd_many(None, 1, None) == RDM_ERR_INVALID_ARG
    for bad in (dict(W=3), dict(silu=0), dict(dtype=0)):
        mixed = (ConvArgs * 2)(_conv(), _conv(**bad))
        assert lib.rdm_shortconv_fwd_many(mixed, 2, None) == RDM_ERR_INVALID_ARG, bad
    assert lib.rdm_shortconv_fwd_many((ConvArgs * 2)(_conv(), _conv(D=48)), 2, None) == RDM_ERR_UNSUPPORTED
    assert lib.rdm_shortconv_fwd_many((ConvArgs * 2)(_conv(), _conv(y=12290)), 2, None) == RDM_ERR_INVALID_ARG


@pytest.mark.parametrize("B,H,T,dk,dv", [(1, 1, 8, 64, 64), (2, 3, 1000, 32, 128),
                                         (1, 2, 1024 + 37, 16, 32), (4, 16, 4096, 64, 128),
                                         (1, 1, 9000, 128, 16)])
def test_simt_workspace_size(lib, B, H, T, dk, dv):
    """The exact backward's scratch as the header states it: dq, one row a head,
    the flagged-head list and, from T = 1024 on, the maps of P = min(8, T/512)
    sequence segments (each part rounded up to 256 bytes)."""
    def up(x):
        return (x + 255) // 256 * 256
    P = min(8, T // 512) if T >= 1024 else 1
    if P > 1:  # segments of whole 16-token tiles; the count actually used
        tiles = (T + 15) // 16
        seg = -(-tiles // P) * 16
        P = -(-T // seg)
    rows = B * H * dk
    want = up(rows * T * 4) + up(rows * 4) + up((B * H + 1) * 4)
    if P > 1:
        want += up(rows * P * dv * 4) + 2 * up(rows * P * 4)
    a = _bwd_args(B=B, H=H, T=T, dk=dk, dv=dv, impl=1)
    assert lib.rdm_ddts_bwd_workspace_size(ctypes.byref(a)) == want
