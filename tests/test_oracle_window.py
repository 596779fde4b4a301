"""Pins of the sliding-window mask in the oracle (window_left): the
independent pure-Python brute force, closed forms and reductions to the
unwindowed case, and the gradients' central differences and fp64 autograd."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("w", [0, 1, 3])
@pytest.mark.parametrize("nq,nk", [(5, 5), (3, 7)])
def test_brute_force(causal, w, nq, nk):
    q, k, v = _rand((1, nq, 1, 4), 1), _rand((1, nk, 1, 4), 2), _rand((1, nk, 1, 4), 3)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, causal, window_left=w)
    bo, bl = brute.attention_rows(q[0, :, 0].tolist(), k[0, :, 0].tolist(), v[0, :, 0].tolist(),
                                  0.5, causal=causal, window_left=w)
    assert np.abs(o[0, :, 0] - np.array(bo)).max() < 1e-14
    assert np.abs(lse[0, 0] - np.array(bl)).max() < 1e-14


def test_window_zero_causal_selects_the_own_key():
    # each query sees exactly the key at its own position: O = V there,
    # LSE = its score
    q, k, v = _rand((2, 6, 2, 8), 4), _rand((2, 9, 1, 8), 5), _rand((2, 9, 1, 8), 6)
    o, lse = oracle.attn_fwd(q, k, v, 0.3, True, window_left=0)
    for b in range(2):
        for h in range(2):
            for i in range(6):
                j = i + 3
                assert np.array_equal(o[b, i, h], v[b, j, 0].numpy())
                s = 0.3 * float(np.dot(q[b, i, h].numpy(), k[b, j, 0].numpy()))
                assert abs(lse[b, h, i] - s) < 1e-14


def test_wide_window_is_no_window():
    q, k, v = _rand((1, 20, 2, 8), 7), _rand((1, 30, 2, 8), 8), _rand((1, 30, 2, 8), 9)
    for causal in (False, True):
        a = oracle.attn_fwd(q, k, v, 0.4, causal, seqlens_k=[25], window_left=40)
        b = oracle.attn_fwd(q, k, v, 0.4, causal, seqlens_k=[25])
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_window_gradients_central_differences():
    q, k, v, do = (_rand((1, 5, 2, 3), 10), _rand((1, 6, 1, 3), 11), _rand((1, 6, 1, 3), 12),
                   _rand((1, 5, 2, 3), 13))
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.7, True, window_left=2)
    eps = 1e-5

    def loss():
        o, _ = oracle.attn_fwd(q, k, v, 0.7, True, window_left=2)
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


def test_window_gradients_torch_autograd():
    q, k, v, do = (_rand((2, 33, 4, 16), 14), _rand((2, 40, 2, 16), 15), _rand((2, 40, 2, 16), 16),
                   _rand((2, 33, 4, 16), 17))
    W = 9
    got = oracle.attn_bwd(q, k, v, do, 0.25, True, seqlens_k=[40, 35], window_left=W)
    qq, kk, vv = (t.clone().requires_grad_(True) for t in (q, k, v))
    kr, vr = kk.repeat_interleave(2, dim=2), vv.repeat_interleave(2, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", qq, kr) * 0.25
    mask = torch.zeros(2, 1, 33, 40, dtype=torch.bool)
    for b, lk in enumerate([40, 35]):
        i = torch.arange(33)[:, None]
        j = torch.arange(40)[None, :]
        pos = i + lk - 33
        mask[b, 0] = (j >= lk) | (j > pos) | (j < pos - W)
    p = torch.nan_to_num(torch.softmax(s.masked_fill(mask, -math.inf), dim=-1), nan=0.0)
    (torch.einsum("bhij,bjhd->bihd", p, vr) * do).sum().backward()
    for a, r in zip(got, (qq.grad, kk.grad, vv.grad)):
        assert np.abs(a - r.numpy()).max() < 1e-11
