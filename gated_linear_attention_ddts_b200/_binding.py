"""ctypes binding of librdm_ddts.so (include/rdm_ddts.h).

Argument marshalling only: torch tensors become device pointers, the current
torch stream becomes the cudaStream_t, statuses become exceptions.  Every step
of the computation runs in the library's CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librdm_ddts.so")

RDM_OK, RDM_ERR_INVALID_ARG, RDM_ERR_UNSUPPORTED, RDM_ERR_CUDA, RDM_ERR_TIMEOUT, \
    RDM_ERR_WORKSPACE = range(6)
RDM_F32, RDM_BF16 = 0, 1
IMPL = {"auto": 0, "simt": 1, "tc": 2, 0: 0, 1: 1, 2: 2}
# what g, tau, beta hold: the gates, or their pre-activations (softplus, sigmoid,
# sigmoid applied inside; gradients then refer to the pre-activations)
GATES = {"activated": 0, "preact": 1, 0: 0, 1: 1}

_VP = ctypes.c_void_p
_I = ctypes.c_int


class FwdArgs(ctypes.Structure):
    _fields_ = [("B", _I), ("H", _I), ("T", _I), ("dk", _I), ("dv", _I), ("chunk", _I),
                ("dtype", _I), ("impl", _I),
                ("q", _VP), ("k", _VP), ("v", _VP), ("g", _VP), ("tau", _VP), ("beta", _VP),
                ("S0", _VP), ("o", _VP), ("ST", _VP), ("saved_states", _VP),
                ("workspace", _VP), ("workspace_bytes", ctypes.c_size_t), ("gate_inputs", _I),
                ("feedthrough", _VP), ("beta_rank", _I), ("beta_u", _VP), ("beta_w", _VP)]


class BwdArgs(ctypes.Structure):
    _fields_ = [("B", _I), ("H", _I), ("T", _I), ("dk", _I), ("dv", _I), ("chunk", _I),
                ("dtype", _I), ("impl", _I),
                ("q", _VP), ("k", _VP), ("v", _VP), ("g", _VP), ("tau", _VP), ("beta", _VP),
                ("S0", _VP), ("grad_o", _VP), ("grad_ST", _VP), ("saved_states", _VP),
                ("grad_q", _VP), ("grad_k", _VP), ("grad_v", _VP), ("grad_g", _VP),
                ("grad_tau", _VP), ("grad_beta", _VP), ("grad_S0", _VP),
                ("workspace", _VP), ("workspace_bytes", ctypes.c_size_t), ("gate_inputs", _I),
                ("feedthrough", _VP), ("grad_feedthrough", _VP), ("beta_rank", _I),
                ("beta_u", _VP), ("beta_w", _VP), ("grad_beta_u", _VP), ("grad_beta_w", _VP)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("B", _I), ("H", _I), ("dk", _I), ("dv", _I), ("dtype", _I),
                ("q", _VP), ("k", _VP), ("v", _VP), ("g", _VP), ("tau", _VP), ("beta", _VP),
                ("S", _VP), ("o", _VP), ("feedthrough", _VP)]


class ConvArgs(ctypes.Structure):
    _fields_ = [("B", _I), ("H", _I), ("T", _I), ("D", _I), ("W", _I), ("dtype", _I), ("silu", _I),
                ("x", _VP), ("weight", _VP), ("bias", _VP), ("state_in", _VP), ("y", _VP),
                ("state_out", _VP)]


class ConvBwdArgs(ctypes.Structure):
    _fields_ = [("fwd", ConvArgs), ("grad_y", _VP), ("grad_state_out", _VP), ("grad_x", _VP),
                ("grad_weight", _VP), ("grad_bias", _VP), ("grad_state_in", _VP)]


class SkaFwdArgs(ctypes.Structure):
    _fields_ = [("B", _I), ("H", _I), ("T", _I), ("dk", _I), ("dv", _I), ("window", _I),
                ("scale", ctypes.c_float), ("dtype", _I), ("q", _VP), ("k", _VP), ("v", _VP),
                ("o", _VP), ("k_cache", _VP), ("v_cache", _VP), ("pos", _VP)]


class SkaDecodeArgs(ctypes.Structure):
    _fields_ = [("B", _I), ("H", _I), ("dk", _I), ("dv", _I), ("window", _I),
                ("scale", ctypes.c_float), ("dtype", _I), ("q", _VP), ("k", _VP), ("v", _VP),
                ("k_cache", _VP), ("v_cache", _VP), ("pos", _VP), ("advance_pos", _I), ("o", _VP)]


class RdmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None

EXPORTS = ["rdm_ddts_fwd", "rdm_ddts_fwd_workspace_size", "rdm_ddts_saved_states_size", "rdm_ddts_bwd",
           "rdm_ddts_bwd_workspace_size", "rdm_ddts_bwd_noalloc", "rdm_ddts_decode_step", "rdm_ddts_decode",
           "rdm_ddts_sync_status",
           "rdm_status_string", "rdm_ddts_set_test_hooks", "rdm_ddts_version", "rdm_shortconv_fwd",
           "rdm_shortconv_bwd", "rdm_shortconv_fwd_many", "rdm_shortconv_bwd_many", "rdm_ska_fwd",
           "rdm_ska_decode"]


def load():
    """Open librdm_ddts.so and declare its signatures.  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run "
                               "`python -m gated_linear_attention_ddts_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        lib.rdm_ddts_fwd.argtypes = [ctypes.POINTER(FwdArgs), _VP]
        lib.rdm_ddts_fwd.restype = _I
        lib.rdm_ddts_fwd_workspace_size.argtypes = [ctypes.POINTER(FwdArgs)]
        lib.rdm_ddts_fwd_workspace_size.restype = ctypes.c_size_t
        lib.rdm_ddts_saved_states_size.argtypes = [_I] * 6
        lib.rdm_ddts_saved_states_size.restype = ctypes.c_size_t
        lib.rdm_ddts_bwd.argtypes = [ctypes.POINTER(BwdArgs), _VP]
        lib.rdm_ddts_bwd.restype = _I
        lib.rdm_ddts_bwd_workspace_size.argtypes = [ctypes.POINTER(BwdArgs)]
        lib.rdm_ddts_bwd_workspace_size.restype = ctypes.c_size_t
        lib.rdm_ddts_bwd_noalloc.argtypes = [ctypes.POINTER(BwdArgs), _VP]
        lib.rdm_ddts_bwd_noalloc.restype = _I
        lib.rdm_ddts_decode_step.argtypes = [_I] * 5 + [_VP] * 9
        lib.rdm_ddts_decode_step.restype = _I
        lib.rdm_ddts_decode.argtypes = [ctypes.POINTER(DecodeArgs), _VP]
        lib.rdm_ddts_decode.restype = _I
        lib.rdm_ddts_sync_status.argtypes = [_VP]
        lib.rdm_ddts_sync_status.restype = _I
        lib.rdm_status_string.argtypes = [_I]
        lib.rdm_status_string.restype = ctypes.c_char_p
        lib.rdm_shortconv_fwd.argtypes = [ctypes.POINTER(ConvArgs), _VP]
        lib.rdm_shortconv_fwd.restype = _I
        lib.rdm_shortconv_bwd.argtypes = [ctypes.POINTER(ConvBwdArgs), _VP]
        lib.rdm_shortconv_bwd.restype = _I
        lib.rdm_shortconv_fwd_many.argtypes = [ctypes.POINTER(ConvArgs), _I, _VP]
        lib.rdm_shortconv_fwd_many.restype = _I
        lib.rdm_shortconv_bwd_many.argtypes = [ctypes.POINTER(ConvBwdArgs), _I, _VP]
        lib.rdm_shortconv_bwd_many.restype = _I
        lib.rdm_ska_fwd.argtypes = [ctypes.POINTER(SkaFwdArgs), _VP]
        lib.rdm_ska_fwd.restype = _I
        lib.rdm_ska_decode.argtypes = [ctypes.POINTER(SkaDecodeArgs), _VP]
        lib.rdm_ska_decode.restype = _I
        lib.rdm_ddts_set_test_hooks.argtypes = [ctypes.c_longlong, _I]
        lib.rdm_ddts_set_test_hooks.restype = _I
        lib.rdm_ddts_version.argtypes = []
        lib.rdm_ddts_version.restype = _I
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().rdm_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous CUDA tensors")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return RDM_BF16
    if t.dtype == torch.float32:
        return RDM_F32
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _check(status: int, where: str):
    if status != RDM_OK:
        raise RdmError(status, where)


def rdm_ddts_saved_states_size(B, H, T, dk, dv, chunk=0) -> int:
    return int(load().rdm_ddts_saved_states_size(B, H, T, dk, dv, chunk))


def _lowrank(beta_lowrank):
    """(rank, u, w) of a low-rank beta_hat given as (u [B,T,r], w_up [H,r,dv])."""
    if beta_lowrank is None:
        return 0, None, None
    u, w = beta_lowrank
    return int(u.shape[-1]), u, w


def _fwd_args(q, k, v, g, tau, beta, S0, o, ST, saved_states, ws, ws_bytes, chunk, impl,
              gates="activated", feedthrough=None, beta_lowrank=None):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    r, u, w = _lowrank(beta_lowrank)
    return FwdArgs(B, H, T, dk, dv, chunk, _dtype_code(q), IMPL[impl],
                   _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(tau), _ptr(beta), _ptr(S0), _ptr(o),
                   _ptr(ST), _ptr(saved_states), _ptr(ws), ws_bytes, GATES[gates],
                   _ptr(feedthrough), r, _ptr(u), _ptr(w))


def rdm_ddts_fwd_workspace_size(q, k, v, g, tau, beta, *, chunk=0, impl="auto",
                                gates="activated", beta_lowrank=None) -> int:
    a = _fwd_args(q, k, v, g, tau, beta, None, None, None, None, None, 0, chunk, impl, gates,
                  None, beta_lowrank)
    n = load().rdm_ddts_fwd_workspace_size(ctypes.byref(a))
    if n == ctypes.c_size_t(-1).value:
        raise RdmError(RDM_ERR_INVALID_ARG, "rdm_ddts_fwd_workspace_size")
    return int(n)


def rdm_ddts_fwd(q, k, v, g, tau, beta, S0=None, o=None, ST=None, saved_states=None, *,
                 workspace=None, chunk=0, impl="auto", return_state=False, stream=None,
                 gates="activated", feedthrough=None, beta_lowrank=None):
    """Forward over [B,H,T,D] sequences.  Allocates o (and S_T when
    return_state) with torch if not given, and the sequence-segment workspace
    when none is passed (workspace=False runs without one).  feedthrough: [H,dv]
    float32 weights d, o_t += d * v_t.  beta_lowrank: (u [B,T,r], w_up [H,r,dv]
    float32) for beta_hat = sigmoid(u . w_up) (gates="preact"; beta unused, may
    be None).  Returns (o, S_T or None)."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    if ST is None and return_state:
        ST = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    if workspace is None:
        need = rdm_ddts_fwd_workspace_size(q, k, v, g, tau, beta, chunk=chunk, impl=impl,
                                           gates=gates, beta_lowrank=beta_lowrank)
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device) if need else None
    elif workspace is False:
        workspace = None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    a = _fwd_args(q, k, v, g, tau, beta, S0, o, ST, saved_states, workspace, ws_bytes, chunk,
                  impl, gates, feedthrough, beta_lowrank)
    _check(load().rdm_ddts_fwd(ctypes.byref(a), _stream(stream)), "rdm_ddts_fwd")
    return o, ST


def _bwd_args(q, k, v, g, tau, beta, S0, grad_o, grad_ST, saved_states, grads, ws, ws_bytes,
              chunk, impl, gates="activated", feedthrough=None, beta_lowrank=None):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    r, u, w = _lowrank(beta_lowrank)
    return BwdArgs(B, H, T, dk, dv, chunk, _dtype_code(q), IMPL[impl],
                   _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(tau), _ptr(beta), _ptr(S0),
                   _ptr(grad_o), _ptr(grad_ST), _ptr(saved_states),
                   *(_ptr(grads.get(n)) for n in ("dq", "dk", "dv", "dg", "dtau", "dbeta",
                                                    "dS0")),
                   _ptr(ws), ws_bytes, GATES[gates], _ptr(feedthrough), _ptr(grads.get("dfeed")),
                   r, _ptr(u), _ptr(w), _ptr(grads.get("du")), _ptr(grads.get("dw_up")))


def _alloc_grads(grads, q, k, v, g, tau, beta, beta_lowrank):
    refs = [("dq", q), ("dk", k), ("dg", g), ("dtau", tau), ("dv", v)]
    if beta_lowrank is None:
        refs.append(("dbeta", beta))
    else:
        refs += [("du", beta_lowrank[0]), ("dw_up", beta_lowrank[1])]
    for n, ref in refs:
        if grads.get(n) is None:
            grads[n] = torch.empty_like(ref)


def rdm_ddts_bwd_workspace_size(q, k, v, g, tau, beta, S0=None, grad_o=None, grad_ST=None,
                                saved_states=None, *, chunk=0, impl="auto",
                                gates="activated", beta_lowrank=None) -> int:
    a = _bwd_args(q, k, v, g, tau, beta, S0, grad_o, grad_ST, saved_states, {}, None, 0,
                  chunk, impl, gates, None, beta_lowrank)
    n = load().rdm_ddts_bwd_workspace_size(ctypes.byref(a))
    if n == ctypes.c_size_t(-1).value:
        raise RdmError(RDM_ERR_INVALID_ARG, "rdm_ddts_bwd_workspace_size")
    return int(n)


def rdm_ddts_bwd(q, k, v, g, tau, beta, S0, grad_o, grad_ST=None, saved_states=None, *,
                 grads=None, workspace=None, chunk=0, impl="auto", want_dS0=True, stream=None,
                 gates="activated", feedthrough=None, beta_lowrank=None):
    """Backward.  `grads` may hold preallocated dq, dk, dv, dg, dtau, dbeta, dS0
    (and dfeed when feedthrough is given; du and dw_up in place of dbeta with
    beta_lowrank); missing ones are allocated with torch, as is the workspace.
    Returns the dict."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    grads = dict(grads or {})
    _alloc_grads(grads, q, k, v, g, tau, beta, beta_lowrank)
    if want_dS0 and grads.get("dS0") is None:
        grads["dS0"] = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    if feedthrough is not None and grads.get("dfeed") is None:
        grads["dfeed"] = torch.empty(H, dv, dtype=torch.float32, device=q.device)
    if workspace is None:
        need = rdm_ddts_bwd_workspace_size(q, k, v, g, tau, beta, S0, grad_o, grad_ST,
                                           saved_states, chunk=chunk, impl=impl, gates=gates,
                                           beta_lowrank=beta_lowrank)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    a = _bwd_args(q, k, v, g, tau, beta, S0, grad_o, grad_ST, saved_states, grads, workspace,
                  workspace.numel() * workspace.element_size(), chunk, impl, gates, feedthrough,
                  beta_lowrank)
    _check(load().rdm_ddts_bwd(ctypes.byref(a), _stream(stream)), "rdm_ddts_bwd")
    return grads


def rdm_ddts_bwd_noalloc(q, k, v, g, tau, beta, S0, grad_o, grad_ST=None, *, grads=None,
                         chunk=0, want_dS0=True, stream=None, gates="activated", beta_lowrank=None):
    """Backward through the library's own fixed scratch (no workspace
    argument).  Gradient tensors are allocated with torch if not given;
    returns the dict of gradients."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    grads = dict(grads or {})
    _alloc_grads(grads, q, k, v, g, tau, beta, beta_lowrank)
    if want_dS0 and grads.get("dS0") is None:
        grads["dS0"] = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    a = _bwd_args(q, k, v, g, tau, beta, S0, grad_o, grad_ST, None, grads, None, 0, chunk, "simt",
                  gates, None, beta_lowrank)
    _check(load().rdm_ddts_bwd_noalloc(ctypes.byref(a), _stream(stream)), "rdm_ddts_bwd_noalloc")
    return grads


def rdm_ddts_decode_step(q, k, v, g, tau, beta, S, o=None, *, stream=None):
    """One token per (b,h): q,k,g,tau [B,H,dk], v,beta [B,H,dv]; S [B,H,dk,dv]
    float32 updated in place.  Returns o [B,H,dv]."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    st = load().rdm_ddts_decode_step(B, H, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(g), _ptr(tau), _ptr(beta), _ptr(S), _ptr(o),
                                     _stream(stream))
    _check(st, "rdm_ddts_decode_step")
    return o


def rdm_ddts_decode(q, k, v, g, tau, beta, S, o=None, *, feedthrough=None, stream=None):
    """rdm_ddts_decode_step with the feedthrough: o = S^T q + d * v when
    feedthrough ([H,dv] float32) is given."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    a = DecodeArgs(B, H, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(tau),
                   _ptr(beta), _ptr(S), _ptr(o), _ptr(feedthrough))
    _check(load().rdm_ddts_decode(ctypes.byref(a), _stream(stream)), "rdm_ddts_decode")
    return o


def _conv_args(x, weight, bias, state_in, y, state_out, silu):
    B, H, T, D = x.shape
    return ConvArgs(B, H, T, D, weight.shape[-1], _dtype_code(x), int(bool(silu)), _ptr(x),
                    _ptr(weight), _ptr(bias), _ptr(state_in), _ptr(y), _ptr(state_out))


def rdm_shortconv_fwd(x, weight, bias=None, state_in=None, *, silu=False, y=None,
                      return_state=False, stream=None):
    """Causal depthwise short convolution along the tokens: x [B,H,T,D], weight
    [H,D,W] float32, bias [H,D] float32, state_in [B,H,W-1,D] (the previous
    W-1 inputs).  Returns (y, state_out or None)."""
    B, H, T, D = x.shape
    W = weight.shape[-1]
    if y is None:
        y = torch.empty_like(x)
    state_out = torch.empty(B, H, W - 1, D, dtype=x.dtype, device=x.device) if return_state else None
    a = _conv_args(x, weight, bias, state_in, y, state_out, silu)
    _check(load().rdm_shortconv_fwd(ctypes.byref(a), _stream(stream)), "rdm_shortconv_fwd")
    return y, state_out


def rdm_shortconv_bwd(x, weight, bias, state_in, grad_y, grad_state_out=None, *, silu=False,
                      out=None, stream=None):
    """Reverse mode of rdm_shortconv_fwd.  Returns dict dx, dw, dbias (None
    without bias) and dxs (None without state_in); `out` may hold them
    preallocated."""
    out = dict(out or {})
    if out.get("dx") is None:
        out["dx"] = torch.empty_like(x)
    if out.get("dw") is None:
        out["dw"] = torch.empty_like(weight)
    if out.get("dbias") is None:
        out["dbias"] = torch.empty_like(bias) if bias is not None else None
    if out.get("dxs") is None:
        out["dxs"] = torch.empty_like(state_in) if state_in is not None else None
    a = ConvBwdArgs(_conv_args(x, weight, bias, state_in, None, None, silu), _ptr(grad_y),
                    _ptr(grad_state_out), _ptr(out["dx"]), _ptr(out["dw"]), _ptr(out["dbias"]),
                    _ptr(out["dxs"]))
    _check(load().rdm_shortconv_bwd(ctypes.byref(a), _stream(stream)), "rdm_shortconv_bwd")
    return out


def rdm_shortconv_fwd_many(problems, *, silu=False, stream=None):
    """Several independent ShortConv forwards in one launch.  `problems` is a
    list (at most 4) of dicts with x, weight and optionally bias, state_in, y
    and return_state, as for rdm_shortconv_fwd (same dtype and W in all).
    Returns a list of (y, state_out or None)."""
    outs, args = [], []
    for pr in problems:
        x, weight = pr["x"], pr["weight"]
        B, H, T, D = x.shape
        W = weight.shape[-1]
        y = pr.get("y")
        if y is None:
            y = torch.empty_like(x)
        state_out = (torch.empty(B, H, W - 1, D, dtype=x.dtype, device=x.device)
                     if pr.get("return_state") else None)
        args.append(_conv_args(x, weight, pr.get("bias"), pr.get("state_in"), y, state_out, silu))
        outs.append((y, state_out))
    arr = (ConvArgs * len(args))(*args)
    _check(load().rdm_shortconv_fwd_many(arr, len(args), _stream(stream)), "rdm_shortconv_fwd_many")
    return outs


def rdm_shortconv_bwd_many(problems, *, silu=False, stream=None):
    """Several independent ShortConv backwards in one launch.  `problems` is a
    list (at most 4) of dicts with x, weight, grad_y and optionally bias,
    state_in, grad_state_out and out, as for rdm_shortconv_bwd.  Returns a list
    of dicts dx, dw, dbias, dxs."""
    outs, args = [], []
    for pr in problems:
        x, weight, bias, state_in = pr["x"], pr["weight"], pr.get("bias"), pr.get("state_in")
        out = dict(pr.get("out") or {})
        if out.get("dx") is None:
            out["dx"] = torch.empty_like(x)
        if out.get("dw") is None:
            out["dw"] = torch.empty_like(weight)
        if out.get("dbias") is None:
            out["dbias"] = torch.empty_like(bias) if bias is not None else None
        if out.get("dxs") is None:
            out["dxs"] = torch.empty_like(state_in) if state_in is not None else None
        args.append(ConvBwdArgs(_conv_args(x, weight, bias, state_in, None, None, silu),
                                _ptr(pr["grad_y"]), _ptr(pr.get("grad_state_out")), _ptr(out["dx"]),
                                _ptr(out["dw"]), _ptr(out["dbias"]), _ptr(out["dxs"])))
        outs.append(out)
    arr = (ConvBwdArgs * len(args))(*args)
    _check(load().rdm_shortconv_bwd_many(arr, len(args), _stream(stream)), "rdm_shortconv_bwd_many")
    return outs


def rdm_ska_fwd(q, k, v, window, *, scale=0.0, o=None, k_cache=None, v_cache=None, pos=None,
                stream=None):
    """Sliding-window shared-key attention: q [B,H,T,dk], k [B,T,dk] (one key
    row per token, shared by the heads), v [B,H,T,dv], all bf16; token t
    attends to tokens t-window+1..t.  scale 0 means 1/sqrt(dk).  With k_cache
    [B,window,dk] / v_cache [B,H,window,dv] / pos [B] int32 given, the last
    min(T, window) keys and values are written to slot (position mod window)
    and pos is set to T.  Returns o [B,H,T,dv]."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    a = SkaFwdArgs(B, H, T, dk, dv, int(window), float(scale), _dtype_code(q), _ptr(q), _ptr(k),
                   _ptr(v), _ptr(o), _ptr(k_cache), _ptr(v_cache), _ptr(pos))
    _check(load().rdm_ska_fwd(ctypes.byref(a), _stream(stream)), "rdm_ska_fwd")
    return o


def rdm_ska_decode(q, k, v, k_cache, v_cache, pos, *, scale=0.0, advance_pos=True, o=None,
                   stream=None):
    """One SW-SKA decode step against ring caches: q [B,H,dk], k [B,dk], v
    [B,H,dv] bf16; k_cache [B,window,dk], v_cache [B,H,window,dv] updated in
    place; pos [B] int32 tokens seen before this one (incremented when
    advance_pos).  Returns o [B,H,dv]."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    window = k_cache.shape[1]
    if o is None:
        o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    a = SkaDecodeArgs(B, H, dk, dv, int(window), float(scale), _dtype_code(q), _ptr(q), _ptr(k),
                      _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(pos), int(bool(advance_pos)),
                      _ptr(o))
    _check(load().rdm_ska_decode(ctypes.byref(a), _stream(stream)), "rdm_ska_decode")
    return o


def rdm_ddts_sync_status(stream=None) -> int:
    return int(load().rdm_ddts_sync_status(_stream(stream)))


def rdm_status_string(status: int) -> str:
    return status_string(status)


def rdm_ddts_set_test_hooks(wait_limit_cycles: int = 0, withhold_segment_flags: int = 0) -> None:
    """Test hooks of the bounded on-device waits (see include/rdm_ddts.h);
    (0, 0) restores the defaults."""
    _check(load().rdm_ddts_set_test_hooks(int(wait_limit_cycles), int(withhold_segment_flags)),
           "rdm_ddts_set_test_hooks")


def rdm_ddts_version() -> int:
    return int(load().rdm_ddts_version())
