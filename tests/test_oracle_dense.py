"""Pins of the matrix-product fp64 oracle (``oracle/dense.py``), no GPU.

It is checked against the C oracle, an independent implementation that is
itself pinned to brute force, closed forms and torch's fp64 SDPA, on shapes
that cover every rule it states (causal bottom-right, key lengths, grouped
heads, rows with no key, NaN behind the length, ragged sizes), and directly
against closed forms: Q = 0 gives prefix means and LSE = log(count), V = 1
gives rows of ones (the softmax row sums to 1), causal row 0 is V[0], and a
shift of all keys leaves the softmax unchanged (so sum_j dK_j = 0).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import dense
from io_aware_exact_29_b200.workloads import (DecodeCase, FwdCase, fwd_inputs, kvcache_inputs,
                                              paged_from_packed, upstream_grad)

TOL = 1e-12


def _close(a, b, tol=TOL):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape
    both_inf = np.isneginf(a) & np.isneginf(b)
    assert np.array_equal(np.isnan(a), np.isnan(b))
    with np.errstate(invalid="ignore"):
        err = np.where(both_inf | np.isnan(a), 0.0, np.abs(a - b))
    assert float(err.max(initial=0.0)) <= tol, float(err.max(initial=0.0))


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal", [
    (1, 2, 2, 64, 64, 64, False), (2, 4, 2, 37, 90, 64, True), (1, 8, 2, 90, 37, 128, True),
    (2, 3, 1, 1, 129, 128, False), (1, 2, 2, 130, 1, 64, True), (3, 2, 2, 50, 50, 128, True)])
def test_fwd_equals_c_oracle(B, Hq, Hkv, Nq, Nk, d, causal):
    c = FwdCase("p", B, Hq, Hkv, Nq, Nk, d, causal)
    inp = fwd_inputs(c, seed=B + Nq + Nk)
    a = dense.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, causal)
    b = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, causal)
    _close(a[0], b[0])
    _close(a[1], b[1])


def test_fwd_key_lengths_nan_padding_and_rows():
    c = FwdCase("k", 4, 4, 2, 70, 120, 64, True, kpad_range=(1, 120))
    inp = fwd_inputs(c, seed=3)
    inp["seqlens_k"] = torch.tensor([120, 5, 69, 1], dtype=torch.int32)
    ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, True, seqlens_k=inp["seqlens_k"])
    for b, L in enumerate(inp["seqlens_k"].tolist()):
        inp["k"][b, L:] = float("nan")
        inp["v"][b, L:] = float("nan")
    got = dense.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, True, seqlens_k=inp["seqlens_k"])
    _close(got[0], ref[0])
    _close(got[1], ref[1])
    # rows with no visible key (bottom-right, Lk < Nq): O = 0, LSE = -inf
    assert np.all(got[0][1, :65] == 0) and np.all(np.isneginf(got[1][1, :, :65]))
    rows = [0, 3, 64, 69]
    sub = dense.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, True,
                         seqlens_k=inp["seqlens_k"], rows=rows)
    _close(sub[0][:, rows], got[0][:, rows])
    assert np.isnan(sub[0][:, 1]).all()


def test_fwd_closed_forms():
    g = torch.Generator().manual_seed(1)
    N, d = 200, 64
    q = torch.zeros(1, N, 2, d, dtype=torch.float64)
    k = torch.randn(1, N, 2, d, generator=g, dtype=torch.float64)
    v = torch.randn(1, N, 2, d, generator=g, dtype=torch.float64)
    o, lse = dense.attn_fwd(q, k, v, 0.125, True)
    means = torch.cumsum(v[0], 0) / torch.arange(1, N + 1, dtype=torch.float64)[:, None, None]
    assert np.abs(o[0] - means.numpy()).max() <= 1e-13
    assert np.abs(lse[0] - np.log(np.arange(1, N + 1))[None]).max() <= 1e-13
    q = torch.randn(1, N, 2, d, generator=g, dtype=torch.float64)
    o, lse = dense.attn_fwd(q, k, torch.ones_like(v), 0.125, False)
    assert np.abs(o - 1.0).max() <= TOL  # each softmax row sums to 1
    o, lse = dense.attn_fwd(q, k, v, 0.125, True)
    assert np.array_equal(o[0, 0], v[0, 0].numpy())
    s00 = 0.125 * float((q[0, 0, 0] * k[0, 0, 0]).sum())
    assert abs(lse[0, 0, 0] - s00) <= 1e-13


@pytest.mark.parametrize("nq,causal", [(1, False), (16, True), (5, True)])
def test_kvcache_equals_c_oracle(nq, causal):
    lens = [nq, 1, 300, 129, 2] if causal else [1, 300, 129, 0, 64]
    c = DecodeCase("kv", len(lens), 16, 2, nq, 128, (0, 300), causal, slack=7)
    clean = kvcache_inputs(c, seed=nq, seqlens=lens)
    dirty = kvcache_inputs(c, seed=nq, seqlens=lens, slack_fill=float("nan"))
    ref = oracle.attn_kvcache(clean["q"], clean["k_cache"], clean["v_cache"],
                              clean["cu_seqlens_k"], clean["seqlens_k"], c.scale, causal)
    got = dense.attn_kvcache(dirty["q"], dirty["k_cache"], dirty["v_cache"],
                             dirty["cu_seqlens_k"], dirty["seqlens_k"], c.scale, causal)
    _close(got[0], ref[0])
    _close(got[1], ref[1])


@pytest.mark.parametrize("block_size", [1, 16, 64])
def test_paged_equals_packed(block_size):
    c = DecodeCase("pg", 4, 8, 2, 3, 64, (3, 200), True)
    inp = kvcache_inputs(c, seed=5)
    pg = paged_from_packed(inp, block_size, seed=9)
    a = dense.attn_paged(inp["q"], pg["k_cache"], pg["v_cache"], pg["block_table"],
                         pg["seqlens_k"], c.scale, True)
    b = oracle.attn_kvcache(inp["q"], inp["k_cache"], inp["v_cache"], inp["cu_seqlens_k"],
                            inp["seqlens_k"], c.scale, True)
    _close(a[0], b[0])
    _close(a[1], b[1])


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,lens", [
    (2, 4, 2, 40, 70, 64, True, None), (1, 2, 1, 70, 40, 128, True, None),
    (3, 2, 2, 33, 50, 64, False, [50, 7, 1]), (2, 4, 4, 48, 48, 64, True, [48, 20])])
def test_bwd_equals_c_oracle(B, Hq, Hkv, Nq, Nk, d, causal, lens):
    c = FwdCase("b", B, Hq, Hkv, Nq, Nk, d, causal)
    inp = fwd_inputs(c, seed=Nq)
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32)
    dout = upstream_grad(inp["q"], seed=Nq)
    got = dense.attn_bwd(inp["q"], inp["k"], inp["v"], dout, c.scale, causal, seqlens_k=sl)
    ref = oracle.attn_bwd(inp["q"], inp["k"], inp["v"], dout, c.scale, causal, seqlens_k=sl)
    for x, y in zip(got, ref):
        _close(x, y, 1e-11)
    # a shift of every key leaves each softmax row unchanged: sum_j dK_j = 0
    assert np.abs(got[1].sum(axis=1)).max() <= 1e-10


def test_bwd_head_subset_matches_full():
    c = FwdCase("s", 2, 4, 2, 40, 40, 64, True)
    inp = fwd_inputs(c, seed=2)
    dout = upstream_grad(inp["q"], seed=2)
    full = dense.attn_bwd(inp["q"], inp["k"], inp["v"], dout, c.scale, True)
    # kv head 1 of batch 1 collects query heads 2 and 3
    sub = dense.attn_bwd(inp["q"], inp["k"], inp["v"], dout, c.scale, True,
                         heads=[(1, 2), (1, 3)])
    assert np.array_equal(sub[0][1, :, 2:4], full[0][1, :, 2:4])
    _close(sub[1][1, :, 1], full[1][1, :, 1], 1e-14)
    _close(sub[2][1, :, 1], full[2][1, :, 1], 1e-14)
    assert np.isnan(sub[0][0]).all()


def test_bwd_central_differences():
    # an independent check of the chain rule: d/dq of sum(dout * O) by
    # central differences of the forward
    c = FwdCase("cd", 1, 1, 1, 6, 9, 64, True)
    inp = fwd_inputs(c, seed=4)
    q, k, v = (inp[n].double() for n in ("q", "k", "v"))
    dout = upstream_grad(inp["q"], seed=4).double()
    dq, dk, dv = dense.attn_bwd(q, k, v, dout, c.scale, True)
    eps = 1e-6

    def loss(qq, kk, vv):
        o, _ = dense.attn_fwd(qq, kk, vv, c.scale, True)
        return float((o * dout.numpy()).sum())

    for name, t, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0, 0, 0), (0, 5, 0, 17), (0, 3, 0, 63)]:
            if name != "q" and idx[1] >= 9:
                continue
            tp, tm = t.clone(), t.clone()
            tp[idx] += eps
            tm[idx] -= eps
            args_p = {"q": (tp, k, v), "k": (q, tp, v), "v": (q, k, tp)}[name]
            args_m = {"q": (tm, k, v), "k": (q, tm, v), "v": (q, k, tm)}[name]
            num = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert math.isclose(num, grad[idx], rel_tol=1e-6, abs_tol=1e-8), (name, idx)
