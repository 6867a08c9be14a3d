"""GPU parity of the ShortConv kernels (causal depthwise convolution along the
tokens, the short convolution of the Rodimus block; digest.lyk-ai.com summary,
"Method") against the fp64 oracle, through the C ABI: widths 1-4, float32 and
bf16, with and without bias, SiLU and a carried-in state, ragged and tiny
sequences, sequences cut in two with the state carried across, and a
full-size tensor of the 130M-scale layer's shape."""
import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
import oracle
from tests.parity import TOL, assert_close

pytestmark = pytest.mark.gpu


def conv_inputs(B, H, T, D, W, dtype, seed, state=True, bias=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, H, T, D, generator=g).to(dtype)
    w = torch.randn(H, D, W, generator=g) / W
    b = torch.randn(H, D, generator=g) * 0.1 if bias else None
    xs = torch.randn(B, H, W - 1, D, generator=g).to(dtype) if state else None
    return x, w, b, xs


def cuda(t):
    return t.cuda() if t is not None else None


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("W", [1, 2, 3, 4])
@pytest.mark.parametrize("D,T", [(16, 1), (64, 2), (128, 37), (32, 300)])
@pytest.mark.parametrize("silu", [False, True])
def test_shortconv_fwd_bwd(cuda_ok, dtype, W, D, T, silu):
    B, H = 2, 3
    x, w, b, xs = conv_inputs(B, H, T, D, W, dtype, seed=T * 10 + W + D, state=(T % 2 == 1))
    y, so = rdm.rdm_shortconv_fwd(cuda(x), cuda(w), cuda(b), cuda(xs), silu=silu, return_state=True)
    gy = torch.randn(B, H, T, D, generator=torch.Generator().manual_seed(7)).to(dtype)
    gso = torch.randn(B, H, W - 1, D, generator=torch.Generator().manual_seed(8)).to(dtype)
    gr = rdm.rdm_shortconv_bwd(cuda(x), cuda(w), cuda(b), cuda(xs), cuda(gy), cuda(gso), silu=silu)
    torch.cuda.synchronize()
    y_ref, so_ref = oracle.shortconv_fwd(x, w, b, xs, silu=silu)
    ref = oracle.shortconv_bwd(x, w, b, xs, gy, gso, silu=silu)
    tol = TOL[dtype]
    assert_close(y, y_ref, tol, "shortconv y")
    assert_close(so, so_ref, tol, "shortconv state out")
    assert_close(gr["dx"], ref["dx"], tol, "shortconv dx")
    assert_close(gr["dw"], ref["dw"], tol, "shortconv dw")
    assert_close(gr["dbias"], ref["dbias"], tol, "shortconv dbias")
    if xs is not None and W > 1:
        assert_close(gr["dxs"], ref["dxs"], tol, "shortconv d state in")


@pytest.mark.parametrize("cut", [1, 3, 250])
def test_shortconv_state_carried_across_a_cut(cuda_ok, cut):
    x, w, b, xs = conv_inputs(1, 2, 517, 64, 4, torch.bfloat16, seed=cut)
    dx_, dw_, db_, ds_ = map(cuda, (x, w, b, xs))
    y, s = rdm.rdm_shortconv_fwd(dx_, dw_, db_, ds_, silu=True, return_state=True)
    y1, s1 = rdm.rdm_shortconv_fwd(dx_[:, :, :cut].contiguous(), dw_, db_, ds_, silu=True,
                                   return_state=True)
    y2, s2 = rdm.rdm_shortconv_fwd(dx_[:, :, cut:].contiguous(), dw_, db_, s1, silu=True,
                                   return_state=True)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([y1, y2], 2), y), "cut sequence output"
    assert torch.equal(s2, s), "cut sequence state"


def test_shortconv_full_size_layer_tensor(cuda_ok):
    """A q-shaped tensor of the 130M-scale layer (B8 H6 T2048 D64), width 4."""
    x, w, b, xs = conv_inputs(8, 6, 2048, 64, 4, torch.bfloat16, seed=99, state=False)
    y, s = rdm.rdm_shortconv_fwd(cuda(x), cuda(w), cuda(b), None, silu=True, return_state=True)
    gy = torch.randn(8, 6, 2048, 64, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    gr = rdm.rdm_shortconv_bwd(cuda(x), cuda(w), cuda(b), None, cuda(gy), None, silu=True)
    torch.cuda.synchronize()
    y_ref, s_ref = oracle.shortconv_fwd(x, w, b, None, silu=True)
    ref = oracle.shortconv_bwd(x, w, b, None, gy, None, silu=True)
    assert_close(y, y_ref, 2e-2, "workload 1 shortconv y")
    assert_close(s, s_ref, 2e-2, "workload 1 shortconv state")
    for n in ("dx", "dw", "dbias"):
        assert_close(gr[n], ref[n], 2e-2, f"workload 1 shortconv {n}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("silu", [False, True])
def test_shortconv_many_in_one_launch(cuda_ok, dtype, silu):
    """Problems of different shapes (D 16, 64, 128 and 32; ragged T; one
    without tokens; with and without bias and carried state) in one batched
    forward and one batched backward, each against the oracle, and equal to the
    single-problem calls."""
    W = 4
    shapes = [(2, 3, 37, 16, True, True), (1, 2, 300, 64, False, True), (2, 1, 129, 128, True, False),
              (1, 1, 0, 32, False, True)]
    probs, refs = [], []
    for i, (B, H, T, D, state, bias) in enumerate(shapes):
        x, w, b, xs = conv_inputs(B, H, T, D, W, dtype, seed=500 + i, state=state, bias=bias)
        gy = torch.randn(B, H, T, D, generator=torch.Generator().manual_seed(600 + i)).to(dtype)
        gso = torch.randn(B, H, W - 1, D, generator=torch.Generator().manual_seed(700 + i)).to(dtype)
        probs.append(dict(x=x, w=w, b=b, xs=xs, gy=gy, gso=gso))
        refs.append((oracle.shortconv_fwd(x, w, b, xs, silu=silu), oracle.shortconv_bwd(x, w, b, xs, gy, gso, silu=silu)))
    d = [{k: cuda(v) for k, v in pr.items()} for pr in probs]
    outs = rdm.rdm_shortconv_fwd_many(
        [dict(x=q["x"], weight=q["w"], bias=q["b"], state_in=q["xs"], return_state=True) for q in d], silu=silu)
    grads = rdm.rdm_shortconv_bwd_many(
        [dict(x=q["x"], weight=q["w"], bias=q["b"], state_in=q["xs"], grad_y=q["gy"], grad_state_out=q["gso"])
         for q in d], silu=silu)
    torch.cuda.synchronize()
    tol = TOL[dtype]
    for i, ((y, so), gr, ((y_ref, so_ref), ref)) in enumerate(zip(outs, grads, refs)):
        assert_close(y, y_ref, tol, f"batched shortconv y, problem {i}")
        assert_close(so, so_ref, tol, f"batched shortconv state out, problem {i}")
        assert_close(gr["dx"], ref["dx"], tol, f"batched shortconv dx, problem {i}")
        assert_close(gr["dw"], ref["dw"], tol, f"batched shortconv dw, problem {i}")
        if probs[i]["b"] is not None:
            assert_close(gr["dbias"], ref["dbias"], tol, f"batched shortconv dbias, problem {i}")
        if probs[i]["xs"] is not None:
            assert_close(gr["dxs"], ref["dxs"], tol, f"batched shortconv d state in, problem {i}")
        # the single-problem call gives the same forward bits
        q = d[i]
        y1, _ = rdm.rdm_shortconv_fwd(q["x"], q["w"], q["b"], q["xs"], silu=silu)
        torch.cuda.synchronize()
        assert torch.equal(y1, y), f"batched vs single forward, problem {i}"
