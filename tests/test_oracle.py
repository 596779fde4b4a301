"""Pins of the fp64 CPU oracle to facts fixed outside itself (no GPU).

Each test checks the oracle against something the pages or the mathematics
fix: a library routine computing the same definition (torch's fp64 SDPA and
logsumexp), an independent term-by-term brute force, closed forms (Q = 0,
V = 1, causal row 0, one-hot selection), an invariance (joint permutation of
keys and values), the merge identity of partial softmax results, and the
worked size of S printed on the ai6s.net page.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import brute
from io_aware_exact_29_b200 import accounting
from io_aware_exact_29_b200.workloads import (DECODE_CASES, FWD_CASES, DecodeCase, FwdCase,
                                              default_scale, fwd_inputs, kvcache_inputs)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype)


def _sdpa_ref(q, k, v, scale, causal, seqlens=None):
    """torch fp64 SDPA on [B, N, H, d] tensors (a library routine)."""
    qd = q.double().permute(0, 2, 1, 3)
    kd = k.double().permute(0, 2, 1, 3)
    vd = v.double().permute(0, 2, 1, 3)
    B, H, Nq, d = qd.shape
    Nk = kd.shape[2]
    mask = torch.ones(B, 1, Nq, Nk, dtype=torch.bool)
    if seqlens is not None:
        for b in range(B):
            mask[b, :, :, int(seqlens[b]):] = False
    if causal:
        i = torch.arange(Nq)[:, None]
        j = torch.arange(Nk)[None, :]
        for b in range(B):
            lk = Nk if seqlens is None else int(seqlens[b])
            mask[b, 0] &= j <= i + (lk - Nq)
    o = F.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask, scale=scale,
                                       enable_gqa=(kd.shape[1] != H))
    G = H // kd.shape[1]
    s = torch.einsum("bhid,bhjd->bhij", qd, kd.repeat_interleave(G, 1)) * scale
    s = s.masked_fill(~mask, -math.inf)
    lse = torch.logsumexp(s, dim=-1)
    return o.permute(0, 2, 1, 3).numpy(), lse.numpy()


# --------------------------------------------------------------------------
# 1. library routine: torch's SDPA in fp64
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d", [(1, 2, 2, 37, 37, 64), (2, 4, 2, 19, 45, 128),
                                             (1, 8, 1, 5, 70, 64), (2, 3, 3, 64, 64, 16)])
def test_matches_torch_sdpa(causal, B, Hq, Hkv, Nq, Nk, d):
    q = _rand((B, Nq, Hq, d), 1)
    k = _rand((B, Nk, Hkv, d), 2)
    v = _rand((B, Nk, Hkv, d), 3)
    scale = default_scale(d)
    o, lse = oracle.attn_fwd(q, k, v, scale, causal)
    o_ref, lse_ref = _sdpa_ref(q, k, v, scale, causal)
    np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=0)


def test_key_padding_matches_torch_sdpa():
    B, H, N, d = 3, 2, 40, 64
    q, k, v = _rand((B, N, H, d), 4), _rand((B, N, H, d), 5), _rand((B, N, H, d), 6)
    sl = torch.tensor([40, 17, 1], dtype=torch.int32)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, 0.125, causal, seqlens_k=sl)
        o_ref, lse_ref = _sdpa_ref(q, k, v, 0.125, causal, seqlens=sl)
        np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=0)


# --------------------------------------------------------------------------
# 2. independent brute force, term by term with math.exp
def _as_lists(t):
    return t.double().tolist()


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_4x4(causal):
    q, k, v = _rand((1, 4, 1, 4), 7), _rand((1, 4, 1, 4), 8), _rand((1, 4, 1, 4), 9)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, causal)
    bo, bl = brute.attention_rows(_as_lists(q[0, :, 0]), _as_lists(k[0, :, 0]),
                                  _as_lists(v[0, :, 0]), 0.5, causal)
    np.testing.assert_allclose(o[0, :, 0], np.array(bo), atol=1e-14, rtol=0)
    np.testing.assert_allclose(lse[0, 0], np.array(bl), atol=1e-14, rtol=0)


def test_brute_force_gqa_and_padding():
    B, Hq, Hkv, Nq, Nk, d = 2, 4, 2, 3, 6, 8
    q, k, v = _rand((B, Nq, Hq, d), 10), _rand((B, Nk, Hkv, d), 11), _rand((B, Nk, Hkv, d), 12)
    sl = torch.tensor([6, 4], dtype=torch.int32)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, 0.3, causal, seqlens_k=sl)
        for b in range(B):
            for h in range(Hq):
                g = h // (Hq // Hkv)
                bo, bl = brute.attention_rows(_as_lists(q[b, :, h]), _as_lists(k[b, :, g]),
                                              _as_lists(v[b, :, g]), 0.3, causal,
                                              lk=int(sl[b]))
                np.testing.assert_allclose(o[b, :, h], np.array(bo), atol=1e-14, rtol=0)
                np.testing.assert_allclose(lse[b, h], np.array(bl), atol=1e-14, rtol=0)


def test_brute_force_kvcache_bottom_right():
    case = DecodeCase("t", 3, 4, 2, 3, 8, (1, 9), True, slack=2)
    inp = kvcache_inputs(case, seed=3, seqlens=[9, 3, 1])
    o, lse = oracle.attn_kvcache(inp["q"], inp["k_cache"], inp["v_cache"], inp["cu_seqlens_k"],
                                 inp["seqlens_k"], 0.4, True)
    cu = inp["cu_seqlens_k"].tolist()
    for b in range(3):
        lk = int(inp["seqlens_k"][b])
        kc = inp["k_cache"][cu[b]:cu[b] + lk]
        vc = inp["v_cache"][cu[b]:cu[b] + lk]
        for h in range(4):
            g = h // 2
            bo, bl = brute.attention_rows(_as_lists(inp["q"][b, :, h]), _as_lists(kc[:, g]),
                                          _as_lists(vc[:, g]), 0.4, True)
            np.testing.assert_allclose(o[b, :, h], np.array(bo), atol=1e-14, rtol=0)
            np.testing.assert_allclose(lse[b, h], np.array(bl), atol=1e-14, rtol=0)
    # Lk = 1 with 3 new tokens: only the last token sees the single key, the
    # other two see nothing (O = 0, LSE = -inf)
    assert np.all(o[2, :2] == 0.0) and np.all(np.isneginf(lse[2, :, :2]))


# --------------------------------------------------------------------------
# 3. closed forms
def test_rows_sum_to_one_over_32k_keys():
    # V = 1 makes O[i] = sum_j P[i][j]
    Nk, d = 32768, 16
    q = _rand((1, 4, 1, d), 13) * 3
    k = _rand((1, Nk, 1, d), 14)
    v = torch.ones((1, Nk, 1, d), dtype=torch.bfloat16)
    o, _ = oracle.attn_fwd(q, k, v, 0.25, False)
    assert np.max(np.abs(o - 1.0)) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_values(causal):
    N, d = 50, 64
    q = torch.zeros((1, N, 2, d), dtype=torch.bfloat16)
    k, v = _rand((1, N, 2, d), 15), _rand((1, N, 2, d), 16)
    o, lse = oracle.attn_fwd(q, k, v, 0.125, causal)
    vd = v.double().numpy()
    for i in range(N):
        cnt = i + 1 if causal else N
        np.testing.assert_allclose(o[0, i], vd[0, :cnt].mean(axis=0), atol=1e-14, rtol=0)
        np.testing.assert_allclose(lse[0, :, i], math.log(cnt), atol=1e-14, rtol=0)


def test_causal_first_row_is_first_value():
    q, k, v = _rand((2, 30, 3, 64), 17), _rand((2, 30, 3, 64), 18), _rand((2, 30, 3, 64), 19)
    o, lse = oracle.attn_fwd(q, k, v, 0.125, True)
    assert np.array_equal(o[:, 0], v[:, 0].double().numpy())
    s00 = 0.125 * (q[:, 0].double() * k[:, 0].double()).sum(-1).numpy()  # [B, H]
    np.testing.assert_allclose(lse[:, :, 0], s00, atol=1e-14, rtol=0)


def test_one_hot_key_selects_its_value():
    d = 64
    N = d
    alpha = 16.0
    k = torch.zeros((1, N, 1, d), dtype=torch.bfloat16)
    for j in range(N):
        k[0, j, 0, j] = alpha
    v = _rand((1, N, 1, d), 20)
    sel = [5, 0, 63, 31]
    q = torch.zeros((1, len(sel), 1, d), dtype=torch.bfloat16)
    for i, j in enumerate(sel):
        q[0, i, 0, j] = alpha
    # score of the matching key is alpha^2 * scale = 64, all others 0: margin 64
    o, lse = oracle.attn_fwd(q, k, v, 0.25, False)
    for i, j in enumerate(sel):
        np.testing.assert_allclose(o[0, i, 0], v[0, j, 0].double().numpy(), atol=N * math.exp(-60), rtol=0)
        np.testing.assert_allclose(lse[0, 0, i], 64.0, atol=N * math.exp(-60))


def test_joint_key_value_permutation_invariance():
    q, k, v = _rand((2, 33, 2, 64), 21), _rand((2, 77, 2, 64), 22), _rand((2, 77, 2, 64), 23)
    perm = torch.randperm(77, generator=torch.Generator().manual_seed(24))
    o1, l1 = oracle.attn_fwd(q, k, v, 0.125, False)
    o2, l2 = oracle.attn_fwd(q, k[:, perm], v[:, perm], 0.125, False)
    np.testing.assert_allclose(o1, o2, atol=1e-14, rtol=0)
    np.testing.assert_allclose(l1, l2, atol=1e-13, rtol=0)
    # a permutation of K alone must change the result (catches a K/V mix-up)
    o3, _ = oracle.attn_fwd(q, k[:, perm], v, 0.125, False)
    assert np.max(np.abs(o3 - o1)) > 1e-2


# --------------------------------------------------------------------------
# 4. merge of partial results over disjoint key sets equals the unsplit result
@pytest.mark.parametrize("cuts", [[64], [1, 2, 3], [100, 101], [10, 50, 90, 150]])
def test_partial_merge_equals_unsplit(cuts):
    q, k, v = _rand((1, 6, 2, 32), 25), _rand((1, 160, 2, 32), 26), _rand((1, 160, 2, 32), 27)
    o, lse = oracle.attn_fwd(q, k, v, 0.2, False)
    bounds = [0] + cuts + [160]
    parts_o, parts_l = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        po, pl = oracle.attn_fwd(q, k[:, a:b], v[:, a:b], 0.2, False)
        parts_o.append(po[0].transpose(1, 0, 2).reshape(-1, 32))  # rows = (h, i)
        parts_l.append(pl[0].reshape(-1))
    mo, ml = oracle.lse_combine(np.stack(parts_o), np.stack(parts_l))
    np.testing.assert_allclose(mo, o[0].transpose(1, 0, 2).reshape(-1, 32), atol=1e-14, rtol=0)
    np.testing.assert_allclose(ml, lse[0].reshape(-1), atol=1e-13, rtol=0)


def test_partial_merge_with_empty_parts():
    o_parts = np.array([[[1.0, 2.0]], [[5.0, 7.0]], [[0.0, 0.0]]])
    lse_parts = np.array([[0.0], [math.log(3.0)], [-math.inf]])
    o, lse = oracle.lse_combine(o_parts, lse_parts)
    # weights 1/4 and 3/4
    np.testing.assert_allclose(o[0], [0.25 * 1 + 0.75 * 5, 0.25 * 2 + 0.75 * 7], atol=1e-15)
    np.testing.assert_allclose(lse[0], math.log(4.0), atol=1e-15)
    o, lse = oracle.lse_combine(np.zeros((2, 1, 2)), np.full((2, 1), -math.inf))
    assert np.all(o == 0) and np.isneginf(lse[0])


# --------------------------------------------------------------------------
# 5. variable-length cache: unfilled slots never matter, rows outside are empty
def test_kvcache_sentinels_and_reduction_to_dense():
    case = DecodeCase("t", 4, 8, 2, 2, 64, (1, 70), True, slack=5)
    clean = kvcache_inputs(case, seed=5)
    dirty = kvcache_inputs(case, seed=5, slack_fill=float("nan"))
    oc, lc = oracle.attn_kvcache(clean["q"], clean["k_cache"], clean["v_cache"],
                                 clean["cu_seqlens_k"], clean["seqlens_k"], 0.125, True)
    od, ld = oracle.attn_kvcache(dirty["q"], dirty["k_cache"], dirty["v_cache"],
                                 dirty["cu_seqlens_k"], dirty["seqlens_k"], 0.125, True)
    assert np.array_equal(oc, od, equal_nan=True) and np.array_equal(lc, ld, equal_nan=True)
    assert not np.isnan(od).any()
    # each sequence equals dense attention over its filled keys
    cu = clean["cu_seqlens_k"].tolist()
    for b in range(case.B):
        lk = int(clean["seqlens_k"][b])
        kb = clean["k_cache"][cu[b]:cu[b] + lk].unsqueeze(0)
        vb = clean["v_cache"][cu[b]:cu[b] + lk].unsqueeze(0)
        o1, l1 = oracle.attn_fwd(clean["q"][b:b + 1], kb, vb, 0.125, True)
        o_ref, l_ref = _sdpa_ref(clean["q"][b:b + 1], kb, vb, 0.125, True)
        np.testing.assert_allclose(oc[b], o_ref[0], atol=1e-12, rtol=0)
        np.testing.assert_allclose(lc[b], l_ref[0], atol=1e-12, rtol=0)


def test_row_subset_matches_full():
    q, k, v = _rand((2, 300, 2, 64), 28), _rand((2, 300, 2, 64), 29), _rand((2, 300, 2, 64), 30)
    o, lse = oracle.attn_fwd(q, k, v, 0.125, True)
    rows = [0, 1, 127, 128, 299, 77]
    os_, ls_ = oracle.attn_fwd(q, k, v, 0.125, True, rows=rows)
    assert np.array_equal(os_[:, rows], o[:, rows])
    assert np.array_equal(ls_[:, :, rows], lse[:, :, rows])
    assert np.isnan(os_[:, 2]).all()


def test_oracle_rejects_bad_arguments():
    q = _rand((1, 4, 3, 8), 31)
    k = _rand((1, 4, 2, 8), 32)
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k, k, 0.1, False)  # Hq % Hkv != 0
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k[:, :, :1], k[:, :, :1], 0.1, False,
                        seqlens_k=torch.tensor([5], dtype=torch.int32))  # length > Nk


# --------------------------------------------------------------------------
# 6. the page's worked size of S and the bench's accounting
def test_worked_score_matrix_size():
    with open(os.path.join(GOLDEN, "score_matrix_size.json")) as f:
        g = json.load(f)
    assert accounting.score_matrix_elements(g["N"]) == g["elements"] == 64 * 2 ** 20
    assert accounting.score_matrix_bytes(g["N"], 2) == g["bytes_fp16"] == 128 * 2 ** 20


@pytest.mark.parametrize("nq,lk", [(1, 1), (5, 5), (7, 3), (3, 7), (128, 4096), (16, 16)])
def test_visible_pair_count(nq, lk):
    i = np.arange(nq)[:, None]
    j = np.arange(lk)[None, :]
    assert accounting.visible_pairs(nq, lk, True) == int((j <= i + lk - nq).sum())
    assert accounting.visible_pairs(nq, lk, False) == nq * lk
    if nq == lk:
        assert accounting.visible_pairs(nq, lk, True) == nq * (nq + 1) // 2


# --------------------------------------------------------------------------
# 7. workloads: the configured shapes and a deterministic generator
def test_workload_shapes_and_determinism():
    c = FWD_CASES["bert_large_varlen"]
    a = fwd_inputs(FwdCase("x", 2, 2, 2, 8, 8, 64, False, kpad_range=(256, 512)), seed=0)
    b = fwd_inputs(FwdCase("x", 2, 2, 2, 8, 8, 64, False, kpad_range=(256, 512)), seed=0)
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["seqlens_k"], b["seqlens_k"])
    assert (c.B, c.Hq, c.Nq, c.d) == (16, 16, 512, 64)
    dc = DECODE_CASES["llama70b_decode"]
    assert (dc.B, dc.Hq, dc.Hkv, dc.d, dc.lk_range) == (32, 64, 8, 128, (1, 32768))
    assert default_scale(64) == 0.125
    assert len([n for n in FWD_CASES if n.startswith("sweep_")]) == 20
