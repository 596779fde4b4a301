"""Pins of the backward oracle (oracle.attn_bwd) against things it does not
compute itself: finite differences of the forward oracle, torch autograd on
fp64 (a library routine), and invariants of the softmax.

The pages report training speed-ups (effectstory.com article,
"訓練性能量化提升" table) but print no backward algorithm; the oracle states
the plain derivative of L = sum(dO * O) (see attn_oracle.c).
"""
import numpy as np
import pytest
import torch

import oracle


def _inputs(B, Nq, Nk, Hq, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Nq, Hq, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, Nk, Hkv, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, Nk, Hkv, d, generator=g, dtype=torch.float64)
    do = torch.randn(B, Nq, Hq, d, generator=g, dtype=torch.float64)
    return q, k, v, do


def _loss(q, k, v, do, scale, causal, seqlens):
    o, _ = oracle.attn_fwd(q, k, v, scale, causal, seqlens_k=seqlens)
    return float(np.sum(o * do.numpy()))


@pytest.mark.parametrize("causal,seqlens", [(False, None), (True, None), (False, [4]),
                                            (True, [6]), (True, [3])])
def test_central_differences_of_the_forward_oracle(causal, seqlens):
    # every element of dq, dk, dv against (L(x + e) - L(x - e)) / 2e computed
    # with the forward oracle only; Nq != Nk exercises the bottom-right rule,
    # and causal with 3 keys for 5 queries leaves rows 0 and 1 with no key
    q, k, v, do = _inputs(1, 5, 6, 2, 1, 3, seed=1)
    scale = 0.7
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, scale, causal, seqlens_k=seqlens)
    eps = 1e-5
    for name, t, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        flat = t.view(-1)
        num = np.empty(flat.numel())
        for idx in range(flat.numel()):
            x0 = flat[idx].item()
            flat[idx] = x0 + eps
            lp = _loss(q, k, v, do, scale, causal, seqlens)
            flat[idx] = x0 - eps
            lm = _loss(q, k, v, do, scale, causal, seqlens)
            flat[idx] = x0
            num[idx] = (lp - lm) / (2 * eps)
        err = np.abs(grad.reshape(-1) - num).max()
        assert err < 2e-8, (name, err)


def _torch_reference(q, k, v, do, scale, causal, seqlens):
    """fp64 autograd through torch's own ops (softmax, matmul)."""
    q = q.clone().requires_grad_(True)
    k = k.clone().requires_grad_(True)
    v = v.clone().requires_grad_(True)
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    kr = k.repeat_interleave(G, dim=2)
    vr = v.repeat_interleave(G, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", q, kr) * scale
    mask = torch.zeros(B, 1, Nq, Nk, dtype=torch.bool)
    for b in range(B):
        lk = Nk if seqlens is None else seqlens[b]
        mask[b, :, :, lk:] = True
        if causal:
            i = torch.arange(Nq)[:, None]
            j = torch.arange(Nk)[None, :]
            mask[b, 0] |= j > i + (lk - Nq)
    s = s.masked_fill(mask, float("-inf"))
    p = torch.softmax(s, dim=-1)
    p = torch.nan_to_num(p, nan=0.0)  # rows with no visible key
    o = torch.einsum("bhij,bjhd->bihd", p, vr)
    (o * do).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (6, 1)])
@pytest.mark.parametrize("seqlens", [[50, 41], [50, 20]])
def test_matches_torch_autograd_fp64(causal, hq, hkv, seqlens):
    # with 20 keys for 37 causal queries, rows 0..16 of batch 1 see no key
    q, k, v, do = _inputs(2, 37, 50, hq, hkv, 16, seed=2)
    got = oracle.attn_bwd(q, k, v, do, 0.25, causal, seqlens_k=seqlens)
    ref = _torch_reference(q, k, v, do, 0.25, causal, seqlens)
    for name, a, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.abs(a - r).max() < 1e-11, name


def test_key_gradients_sum_to_zero():
    # adding one vector to every key shifts each score row by a constant,
    # which the softmax ignores: sum_j dK[j] = 0 for any mask
    q, k, v, do = _inputs(2, 33, 40, 4, 2, 8, seed=3)
    for causal in (False, True):
        _, dk, _ = oracle.attn_bwd(q, k, v, do, 0.3, causal, seqlens_k=[40, 29])
        assert np.abs(dk.sum(axis=1)).max() < 1e-12


def test_zero_upstream_gradient_gives_zero():
    q, k, v, do = _inputs(1, 9, 9, 2, 2, 4, seed=4)
    dq, dk, dv = oracle.attn_bwd(q, k, v, torch.zeros_like(do), 0.5, True)
    assert not dq.any() and not dk.any() and not dv.any()


def test_padded_keys_get_no_gradient_and_are_never_read():
    q, k, v, do = _inputs(1, 8, 12, 2, 1, 4, seed=5)
    clean = oracle.attn_bwd(q, k, v, do, 0.5, False, seqlens_k=[7])
    k2, v2 = k.clone(), v.clone()
    k2[:, 7:] = float("nan")
    v2[:, 7:] = float("nan")
    dirty = oracle.attn_bwd(q, k2, v2, do, 0.5, False, seqlens_k=[7])
    for a, b in zip(clean, dirty):
        assert np.array_equal(a, b)
    assert not clean[1][:, 7:].any() and not clean[2][:, 7:].any()


def test_grouped_heads_sum_the_per_head_gradients():
    # one kv head shared by 3 query heads == three copies of it, summed
    q, k, v, do = _inputs(1, 10, 11, 3, 1, 4, seed=6)
    dq_g, dk_g, dv_g = oracle.attn_bwd(q, k, v, do, 0.4, True)
    dq_r, dk_r, dv_r = oracle.attn_bwd(q, k.repeat(1, 1, 3, 1), v.repeat(1, 1, 3, 1), do, 0.4,
                                       True)
    assert np.abs(dq_g - dq_r).max() < 1e-14
    assert np.abs(dk_g[:, :, 0] - dk_r.sum(axis=2)).max() < 1e-13
    assert np.abs(dv_g[:, :, 0] - dv_r.sum(axis=2)).max() < 1e-13


def test_uniform_attention_value_gradient_closed_form():
    # q = 0: every visible key gets weight 1/count, so dV[j] is the sum over
    # the rows that see key j of dO[i] / (number of keys row i sees)
    _, k, v, do = _inputs(1, 6, 6, 1, 1, 3, seed=7)
    q = torch.zeros(1, 6, 1, 3, dtype=torch.float64)
    _, _, dv = oracle.attn_bwd(q, k, v, do, 1.0, True)
    expect = np.zeros((6, 3))
    for i in range(6):
        for j in range(i + 1):
            expect[j] += do[0, i, 0].numpy() / (i + 1)
    assert np.abs(dv[0, :, 0] - expect).max() < 1e-14
