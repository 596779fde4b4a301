"""Pins of the block mask (block-sparse attention) in the oracle: the
independent pure-Python brute force, reductions to independent sub-problems
and to the unmasked case, rows with no block, and the gradients' central
differences and fp64 autograd through torch's softmax with the mask expanded
element by element.

The pages name mask extensions as a direction without giving a form
(machinelearning.ru discussion page, the list of current directions); the
reading here is a 0/1 mask over blocks of block_m queries by block_n keys
that removes whole blocks, on top of the causal, length and window rules.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64)


def _mask(shape, density, seed):
    g = np.random.default_rng(seed)
    return (g.random(shape) < density).astype(np.uint8)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [(2, 2), (2, 3), (3, 1)])
@pytest.mark.parametrize("nq,nk", [(6, 6), (4, 7)])
def test_brute_force(causal, block, nq, nk):
    q, k, v = _rand((1, nq, 1, 4), 1), _rand((1, nk, 1, 4), 2), _rand((1, nk, 1, 4), 3)
    nqb, nkb = -(-nq // block[0]), -(-nk // block[1])
    m = _mask((1, 1, nqb, nkb), 0.6, seed=nq * 10 + nk + block[1])
    o, lse = oracle.attn_fwd(q, k, v, 0.5, causal, block_mask=m, block_size=block)
    bo, bl = brute.attention_rows(q[0, :, 0].tolist(), k[0, :, 0].tolist(), v[0, :, 0].tolist(),
                                  0.5, causal=causal, blocks=m[0, 0].tolist(), block=block)
    assert np.abs(o[0, :, 0] - np.array(bo)).max() < 1e-14
    bl = np.array(bl)
    fin = np.isfinite(bl)
    assert np.array_equal(np.isfinite(lse[0, 0]), fin)
    assert np.abs(lse[0, 0][fin] - bl[fin]).max(initial=0.0) < 1e-14


def test_all_ones_mask_is_no_mask():
    q, k, v = _rand((2, 20, 4, 8), 4), _rand((2, 27, 2, 8), 5), _rand((2, 27, 2, 8), 6)
    ones = np.ones((1, 1, 3, 4), np.uint8)
    for causal in (False, True):
        a = oracle.attn_fwd(q, k, v, 0.4, causal, seqlens_k=[27, 19], block_mask=ones,
                            block_size=8)
        b = oracle.attn_fwd(q, k, v, 0.4, causal, seqlens_k=[27, 19])
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("causal", [False, True])
def test_block_diagonal_is_independent_blocks(causal):
    # a block-diagonal mask cuts the problem into independent attentions of
    # 5 queries against their own 5 keys (causal inside each block when the
    # whole problem is causal and square)
    bs, nb = 5, 4
    n = bs * nb
    q, k, v = _rand((1, n, 2, 6), 7), _rand((1, n, 1, 6), 8), _rand((1, n, 1, 6), 9)
    diag = np.eye(nb, dtype=np.uint8)[None, None]
    o, lse = oracle.attn_fwd(q, k, v, 0.6, causal, block_mask=diag, block_size=bs)
    for t in range(nb):
        sl = slice(t * bs, (t + 1) * bs)
        ob, lb = oracle.attn_fwd(q[:, sl], k[:, sl], v[:, sl], 0.6, causal)
        assert np.abs(o[:, sl] - ob).max() < 1e-15
        assert np.abs(lse[:, :, sl] - lb).max() < 1e-14


def test_rows_without_a_block_give_zero_and_minus_inf():
    q, k, v = _rand((1, 12, 2, 4), 10), _rand((1, 12, 2, 4), 11), _rand((1, 12, 2, 4), 12)
    m = np.ones((1, 2, 3, 3), np.uint8)
    m[0, 1, 1, :] = 0  # head 1, queries 4..7: nothing
    o, lse = oracle.attn_fwd(q, k, v, 0.5, False, block_mask=m, block_size=4)
    assert not o[0, 4:8, 1].any()
    assert np.all(lse[0, 1, 4:8] == -math.inf)
    assert np.all(np.isfinite(lse[0, 0])) and np.all(np.isfinite(lse[0, 1, :4]))
    do = _rand((1, 12, 2, 4), 13)
    dq, _, _ = oracle.attn_bwd(q, k, v, do, 0.5, False, block_mask=m, block_size=4)
    assert not dq[0, 4:8, 1].any()


def test_per_head_and_per_batch_masks_and_sharing():
    B, H, n, bs = 2, 3, 16, 4
    q, k, v = _rand((B, n, H, 8), 14), _rand((B, n, 1, 8), 15), _rand((B, n, 1, 8), 16)
    full = _mask((B, H, 4, 4), 0.5, seed=17)
    full[:, :, :, 0] = 1
    o, lse = oracle.attn_fwd(q, k, v, 0.3, False, block_mask=full, block_size=bs)
    for b in range(B):
        for h in range(H):
            ob, lb = oracle.attn_fwd(q[b:b + 1, :, h:h + 1], k[b:b + 1], v[b:b + 1], 0.3, False,
                                     block_mask=full[b:b + 1, h:h + 1], block_size=bs)
            assert np.array_equal(o[b, :, h], ob[0, :, 0])
            assert np.array_equal(lse[b, h], lb[0, 0])
    # a [1, 1, ...] mask is shared by every batch and head
    shared = full[:1, :1]
    a = oracle.attn_fwd(q, k, v, 0.3, False, block_mask=shared, block_size=bs)
    b = oracle.attn_fwd(q, k, v, 0.3, False, block_mask=np.broadcast_to(shared, full.shape),
                        block_size=bs)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_masked_blocks_are_never_read():
    q, k, v = _rand((1, 16, 1, 4), 18), _rand((1, 16, 1, 4), 19), _rand((1, 16, 1, 4), 20)
    m = np.ones((1, 1, 4, 4), np.uint8)
    m[0, 0, :, 2] = 0  # keys 8..11 masked for every query
    clean = oracle.attn_fwd(q, k, v, 0.5, False, block_mask=m, block_size=4)
    k2, v2 = k.clone(), v.clone()
    k2[:, 8:12] = float("nan")
    v2[:, 8:12] = float("nan")
    dirty = oracle.attn_fwd(q, k2, v2, 0.5, False, block_mask=m, block_size=4)
    assert np.array_equal(clean[0], dirty[0]) and np.array_equal(clean[1], dirty[1])


def test_bad_mask_shapes_are_rejected():
    q, k, v = _rand((1, 9, 1, 4), 21), _rand((1, 9, 1, 4), 22), _rand((1, 9, 1, 4), 23)
    with pytest.raises(ValueError):  # 2 x 2 blocks of 4 do not cover 9 x 9
        oracle.attn_fwd(q, k, v, 0.5, False, block_mask=np.ones((1, 1, 2, 2)), block_size=4)
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k, v, 0.5, False, block_mask=np.ones((2, 1, 3, 3)), block_size=4)


def test_gradients_central_differences():
    q, k, v, do = (_rand((1, 6, 2, 3), 24), _rand((1, 7, 1, 3), 25), _rand((1, 7, 1, 3), 26),
                   _rand((1, 6, 2, 3), 27))
    m = np.array([[[[1, 0, 1], [0, 1, 1], [1, 1, 0]], [[0, 1, 0], [1, 0, 1], [1, 1, 1]]]],
                 np.uint8)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.7, True, block_mask=m, block_size=(2, 3))
    eps = 1e-5

    def loss():
        o, _ = oracle.attn_fwd(q, k, v, 0.7, True, block_mask=m, block_size=(2, 3))
        return float(np.sum(o * do.numpy()))
    for t, grad in ((q, dq), (k, dk), (v, dv)):
        flat = t.view(-1)
        for idx in range(flat.numel()):
            x0 = flat[idx].item()
            flat[idx] = x0 + eps
            lp = loss()
            flat[idx] = x0 - eps
            lm = loss()
            flat[idx] = x0
            assert abs(grad.reshape(-1)[idx] - (lp - lm) / (2 * eps)) < 2e-8


@pytest.mark.parametrize("causal", [False, True])
def test_gradients_torch_autograd(causal):
    B, Nq, Nk, Hq, Hkv, d, bs = 2, 33, 40, 4, 2, 16, 8
    q, k, v, do = (_rand((B, Nq, Hq, d), 28), _rand((B, Nk, Hkv, d), 29),
                   _rand((B, Nk, Hkv, d), 30), _rand((B, Nq, Hq, d), 31))
    m = _mask((B, Hq, 5, 5), 0.55, seed=32)
    seqlens = [40, 29]
    got = oracle.attn_bwd(q, k, v, do, 0.25, causal, seqlens_k=seqlens, block_mask=m,
                          block_size=bs)
    qq, kk, vv = (t.clone().requires_grad_(True) for t in (q, k, v))
    kr, vr = kk.repeat_interleave(2, dim=2), vv.repeat_interleave(2, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", qq, kr) * 0.25
    # the block mask expanded to elements, plus the length and causal rules
    el = torch.from_numpy(m.astype(bool)).repeat_interleave(bs, 2).repeat_interleave(bs, 3)
    vis = el[:, :, :Nq, :Nk].clone()
    for b in range(B):
        vis[b, :, :, seqlens[b]:] = False
        if causal:
            i = torch.arange(Nq)[:, None]
            j = torch.arange(Nk)[None, :]
            vis[b] &= (j <= i + seqlens[b] - Nq)
    p = torch.nan_to_num(torch.softmax(s.masked_fill(~vis, float("-inf")), dim=-1), nan=0.0)
    o = torch.einsum("bhij,bjhd->bihd", p, vr)
    (o * do).sum().backward()
    for name, a, r in zip(("dq", "dk", "dv"), got, (qq.grad, kk.grad, vv.grad)):
        assert np.abs(a - r.numpy()).max() < 1e-11, name
    # the forward through the same expanded mask
    of, _ = oracle.attn_fwd(q, k, v, 0.25, causal, seqlens_k=seqlens, block_mask=m,
                            block_size=bs)
    assert np.abs(of - o.detach().numpy()).max() < 1e-12


@pytest.mark.parametrize("nq,nk,causal", [(300, 500, True), (300, 500, False), (600, 200, True),
                                          (256, 256, True)])
def test_block_pair_counts_of_the_flop_accounting(nq, nk, causal):
    # the per-block visible pairs add up to the whole problem's, and a block
    # mask's count equals the element-by-element count of its visible pairs
    from io_aware_exact_29_b200 import accounting
    cnt = accounting.block_pair_counts(nq, nk, causal, block=128)
    assert cnt.sum() == accounting.visible_pairs(nq, nk, causal)
    m = _mask((2, 3) + cnt.shape, 0.5, seed=nq + nk)
    i = np.arange(nq)[:, None]
    j = np.arange(nk)[None, :]
    vis = (j <= i + nk - nq) if causal else np.ones((nq, nk), bool)
    el = m.repeat(128, 2).repeat(128, 3)[:, :, :nq, :nk].astype(bool) & vis
    assert accounting.blocksparse_flops(m, nq, nk, 64, causal, 2, 3) == 4 * 64 * int(el.sum())
