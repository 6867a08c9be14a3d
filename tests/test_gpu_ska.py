"""GPU parity of the sliding-window shared-key attention (SW-SKA of Rodimus+;
digest.lyk-ai.com summary, "Method"; paperhub.cn rebuttal, Q1) against the fp64
oracle, through the C ABI: the tensor-core forward over windows narrower than,
equal to and wider than a key tile and the sequence, ragged sequence ends and
every supported head size; the ring-cache fill after a prompt; decode steps
against the forward across ring wrap-arounds with sequences of one batch at
different positions; the full-size workloads on sampled heads; and a negative
position reported through the status word."""
import numpy as np
import pytest
import torch

import gated_linear_attention_ddts_b200 as rdm
import oracle
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

TOL = 2e-2  # bf16 inputs, bf16 softmax weights into the second product, bf16 output


def ska_inputs(B, H, T, dk, dv, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, T, dk, generator=g).to(torch.bfloat16)
    k = torch.randn(B, T, dk, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, T, dv, generator=g).to(torch.bfloat16)
    return q, k, v


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("T,window", [(1, 1), (37, 5), (128, 128), (300, 64), (300, 129),
                                      (517, 200), (260, 1000)])
def test_ska_fwd_parity(cuda_ok, dk, dv, T, window):
    B, H = 2, 3
    q, k, v = ska_inputs(B, H, T, dk, dv, seed=T + window + dk + dv)
    o = rdm.rdm_ska_fwd(q.cuda(), k.cuda(), v.cuda(), window)
    torch.cuda.synchronize()
    assert rdm.rdm_ddts_sync_status() == 0
    assert_close(o, oracle.ska_fwd(q, k, v, window), TOL, f"ska o T={T} w={window}")


def test_ska_fwd_explicit_scale_and_sharp_scores(cuda_ok):
    """A large scale makes the softmax nearly one-hot: the running maximum and
    the rescale of earlier tiles decide the result."""
    q, k, v = ska_inputs(1, 2, 400, 64, 64, seed=5)
    for scale in (0.02, 1.0):
        o = rdm.rdm_ska_fwd(q.cuda(), k.cuda(), v.cuda(), 300, scale=scale)
        torch.cuda.synchronize()
        assert_close(o, oracle.ska_fwd(q, k, v, 300, scale=scale), TOL, f"scale {scale}")


def test_ska_fwd_empty_sequence_sets_positions(cuda_ok):
    q, k, v = ska_inputs(2, 2, 0, 64, 64, seed=1)
    pos = torch.full((2,), 7, dtype=torch.int32, device="cuda")
    kc = torch.zeros(2, 4, 64, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros(2, 2, 4, 64, dtype=torch.bfloat16, device="cuda")
    o = rdm.rdm_ska_fwd(q.cuda(), k.cuda(), v.cuda(), 4, k_cache=kc, v_cache=vc, pos=pos)
    torch.cuda.synchronize()
    assert o.shape == (2, 2, 0, 64)
    assert pos.tolist() == [0, 0] and not kc.any() and not vc.any()


@pytest.mark.parametrize("T0,window,steps", [(1, 4, 9), (37, 16, 20), (200, 128, 70), (5, 300, 3)])
def test_ska_prompt_then_decode(cuda_ok, T0, window, steps):
    """Prompt through the forward (which fills the ring caches and positions),
    then token-by-token decode; every step equals the forward over the whole
    sequence at that token, and the caches match the oracle's."""
    B, H, dk, dv = 2, 3, 64, 128
    T = T0 + steps
    q, k, v = ska_inputs(B, H, T, dk, dv, seed=T0 * 7 + window)
    kc = torch.zeros(B, window, dk, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros(B, H, window, dv, dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    rdm.rdm_ska_fwd(q[:, :, :T0].contiguous().cuda(), k[:, :T0].contiguous().cuda(),
                    v[:, :, :T0].contiguous().cuda(), window, k_cache=kc, v_cache=vc, pos=pos)
    o_ref = oracle.ska_fwd(q, k, v, window)
    okc, ovc = np.zeros((B, window, dk)), np.zeros((B, H, window, dv))
    for p_ in range(max(0, T0 - window), T0):
        okc[:, p_ % window], ovc[:, :, p_ % window] = k[:, p_].double(), v[:, :, p_].double()
    torch.cuda.synchronize()
    assert pos.tolist() == [T0] * B
    assert_close(kc, okc, 0.0, "k cache after prompt")
    assert_close(vc, ovc, 0.0, "v cache after prompt")
    for s in range(steps):
        t = T0 + s
        od = rdm.rdm_ska_decode(q[:, :, t].contiguous().cuda(), k[:, t].contiguous().cuda(),
                                v[:, :, t].contiguous().cuda(), kc, vc, pos)
        torch.cuda.synchronize()
        assert_close(od, o_ref[:, :, t], TOL, f"decode token {t}")
    assert pos.tolist() == [T] * B
    for p_ in range(max(0, T - window), T):
        assert torch.equal(kc[:, p_ % window].cpu(), k[:, p_]), p_
        assert torch.equal(vc[:, :, p_ % window].cpu(), v[:, :, p_]), p_


def test_ska_decode_ragged_positions(cuda_ok):
    """Sequences of one batch at positions 0, 3 and 40 (window 16) in one call,
    caches filled per sequence by the forward on views of the batch."""
    B, H, dk, dv, w = 3, 2, 128, 64, 16
    q, k, v = ska_inputs(B, H, 41, dk, dv, seed=77)
    kc = torch.zeros(B, w, dk, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros(B, H, w, dv, dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    at = [0, 3, 40]
    for b, t in enumerate(at):
        rdm.rdm_ska_fwd(q[b:b + 1, :, :t].contiguous().cuda(), k[b:b + 1, :t].contiguous().cuda(),
                        v[b:b + 1, :, :t].contiguous().cuda(), w, k_cache=kc[b:b + 1],
                        v_cache=vc[b:b + 1], pos=pos[b:b + 1])
    idx = torch.tensor(at)
    ar = torch.arange(B)
    od = rdm.rdm_ska_decode(q[ar, :, idx].contiguous().cuda(), k[ar, idx].contiguous().cuda(),
                            v[ar, :, idx].contiguous().cuda(), kc, vc, pos)
    torch.cuda.synchronize()
    o_ref = oracle.ska_fwd(q, k, v, w)
    for b, t in enumerate(at):
        assert_close(od[b], o_ref[b, :, t], TOL, f"ragged batch {b} at {t}")
    assert pos.tolist() == [1, 4, 41]


def test_ska_decode_negative_position_reports_and_leaves_caches(cuda_ok):
    B, H, dk, dv, w = 2, 2, 64, 64, 8
    q, k, v = ska_inputs(B, H, 1, dk, dv, seed=3)
    kc = torch.randn(B, w, dk, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, H, w, dv, device="cuda").to(torch.bfloat16)
    kc0, vc0 = kc.clone(), vc.clone()
    pos = torch.tensor([-1, 2], dtype=torch.int32, device="cuda")
    rdm.rdm_ska_decode(q[:, :, 0].contiguous().cuda(), k[:, 0].contiguous().cuda(),
                       v[:, :, 0].contiguous().cuda(), kc, vc, pos, advance_pos=False)
    assert rdm.rdm_ddts_sync_status() == rdm.RDM_ERR_INVALID_ARG
    assert torch.equal(kc[0], kc0[0]) and torch.equal(vc[0], vc0[0])
    assert rdm.rdm_ddts_sync_status() == 0  # the word was cleared by the read


def test_ska_fwd_full_size_layer_sampled_heads(cuda_ok):
    """The 130M-scale SW-SKA layer (B8 H12 T2048 d_k=d_v=64, window 512), in
    the launch the benchmark times; every output of two (batch, head) pairs
    against the oracle run on those pairs alone."""
    B, H, T, d, w = 8, 12, 2048, 64, 512
    q, k, v = ska_inputs(B, H, T, d, d, seed=2024)
    o = rdm.rdm_ska_fwd(q.cuda(), k.cuda(), v.cuda(), w).cpu()
    assert rdm.rdm_ddts_sync_status() == 0
    for b, h in ((0, 0), (7, 11)):
        ref = oracle.ska_fwd(q[b:b + 1, h:h + 1], k[b:b + 1], v[b:b + 1, h:h + 1], w)
        assert_close(o[b:b + 1, h:h + 1], ref, TOL, f"full size b={b} h={h}")


def test_ska_decode_full_size_sampled(cuda_ok):
    """Batched decode at full size (B256 H16 d_k=d_v=128, window 512) with
    wrapped rings (positions 600 + b), one step; sampled sequences against the
    oracle, and every cache row written by the step."""
    B, H, d, w = 256, 16, 128, 512
    g = torch.Generator().manual_seed(4)
    kc = torch.randn(B, w, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, H, w, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    pos = torch.arange(600, 600 + B, dtype=torch.int32)
    kcd, vcd, posd = kc.cuda(), vc.cuda(), pos.cuda()
    od = rdm.rdm_ska_decode(q.cuda(), k.cuda(), v.cuda(), kcd, vcd, posd).cpu()
    assert rdm.rdm_ddts_sync_status() == 0
    assert torch.equal(posd.cpu(), pos + 1)
    slot = (pos % w).long()
    assert torch.equal(kcd.cpu()[torch.arange(B), slot], k)
    assert torch.equal(vcd.cpu()[torch.arange(B), :, slot], v)
    for b in (0, 77, 255):
        o_ref, _, _ = oracle.ska_decode(q[b:b + 1], k[b:b + 1], v[b:b + 1], kc[b:b + 1],
                                        vc[b:b + 1], pos[b:b + 1].numpy(), w)
        assert_close(od[b:b + 1], o_ref, TOL, f"decode full size b={b}")


@pytest.mark.parametrize("H", [1, 2, 4, 6, 8, 16])
def test_ska_decode_head_groups(cuda_ok, H):
    """Head counts that select every grouping of heads per CTA (8, 4, 2, 1
    heads sharing one pass over the key rows), with wrapped rings at different
    positions per sequence."""
    B, d, w = 3, 64, 24
    g = torch.Generator().manual_seed(H)
    kc = torch.randn(B, w, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, H, w, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    pos = torch.tensor([5, 23, 70], dtype=torch.int32)
    kcd, vcd = kc.cuda(), vc.cuda()
    od = rdm.rdm_ska_decode(q.cuda(), k.cuda(), v.cuda(), kcd, vcd, pos.cuda()).cpu()
    assert rdm.rdm_ddts_sync_status() == 0
    o_ref, kc_ref, vc_ref = oracle.ska_decode(q, k, v, kc, vc, pos.numpy(), w)
    assert_close(od, o_ref, TOL, f"decode H={H}")
    assert_close(kcd, kc_ref, 0.0, f"k cache H={H}")
    assert_close(vcd, vc_ref, 0.0, f"v cache H={H}")


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64)])
def test_ska_fwd_persistent_ctas_walk_several_tiles(cuda_ok, dk, dv):
    """Head sizes with one CTA per SM run persistent CTAs: with more query
    tiles than SMs (2 x 8 x 12 = 192 tiles of 128 queries), CTAs walk several
    tiles of different heads; sampled heads against the oracle."""
    B, H, T, w = 2, 8, 1500, 300
    q, k, v = ska_inputs(B, H, T, dk, dv, seed=dk + 2 * dv)
    o = rdm.rdm_ska_fwd(q.cuda(), k.cuda(), v.cuda(), w).cpu()
    assert rdm.rdm_ddts_sync_status() == 0
    for b, h in ((0, 0), (1, 5), (1, 7)):
        ref = oracle.ska_fwd(q[b:b + 1, h:h + 1], k[b:b + 1], v[b:b + 1, h:h + 1], w)
        assert_close(o[b:b + 1, h:h + 1], ref, TOL, f"persistent dk={dk} dv={dv} b={b} h={h}")
