"""fp64 attention written with whole-matrix library steps -- TEST INFRASTRUCTURE.

A second statement of the same definition as ``attn_oracle.c`` (ai6s.net
"ops-transformer FlashAttention" article, section "标准注意力的致命伤不在算力，
在搬运": S = Q·Kᵀ, scale, softmax, ·V), in plain PyTorch CPU ops on float64:
one (batch, head) at a time it forms the whole score block S with a matrix
product, applies the additive 0/-inf mask, takes the row softmax and
multiplies by V with a second matrix product.  The matrix products are library
steps; nothing is blocked, fused or reordered beyond the definition.

It exists so that the GPU parity tests can compare every output element of
the configured workloads at their full sizes (the long-sequence sweep up to
4K, the Llama2-70B-shaped decode, the backward at the bench shape) in seconds:
the C oracle's compensated scalar loops take minutes there.  It is pinned
against the C oracle (an independent implementation, itself pinned to brute
force, closed forms and torch's fp64 SDPA) and to closed forms of its own in
``tests/test_oracle_dense.py``.

Readings (the same as the C oracle's): the mask is additive 0/-inf; causal
alignment is bottom-right (query i sees key j iff j <= i + Lk - Nq); a row
with no visible key gives O = 0 and LSE = -inf; grouped-query heads map
contiguously (kv head h // (Hq / Hkv)); keys at or past a sequence's length
are never read.

Only ``tests/``, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg
may import this module.
"""
from __future__ import annotations

import numpy as np
import torch

_F64 = torch.float64


def _t64(x) -> torch.Tensor:
    """Stored bf16/fp16/fp32 bits widened exactly to a float64 CPU tensor."""
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", _F64)
    return torch.as_tensor(np.asarray(x), dtype=_F64)


def _ints(x) -> list[int]:
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu()
    return [int(v) for v in np.asarray(x).reshape(-1)]


def _visible(row_index: torch.Tensor, Lk: int, Nq: int, causal: bool) -> torch.Tensor | None:
    """Bool [rows, Lk]: key j visible to query i (None: every key is)."""
    if not causal:
        return None
    j = torch.arange(Lk)[None, :]
    return j <= (row_index[:, None] + (Lk - Nq))


def _softmax_rows(S: torch.Tensor, vis: torch.Tensor | None):
    """Masked row softmax of scores S [r, Lk]: (P, m, l) with P = e / l.

    Rows without a visible key give P = 0, m = -inf, l = 0."""
    if vis is not None:
        S = S.masked_fill(~vis, float("-inf"))
    if S.shape[1] == 0:
        r = S.shape[0]
        return S, torch.full((r,), float("-inf"), dtype=_F64), torch.zeros(r, dtype=_F64)
    m = S.max(dim=1).values
    empty = torch.isneginf(m)
    e = torch.exp(S - torch.where(empty, torch.zeros_like(m), m)[:, None])
    if vis is not None:
        e = e.masked_fill(~vis, 0.0)
    l = e.sum(dim=1)
    P = e / torch.where(empty, torch.ones_like(l), l)[:, None]
    return P, m, l


def _attend(Q, K, V, scale, row_index, Nq, causal):
    """One query head against one key/value head: Q [r, d], K, V [Lk, d]."""
    Lk = K.shape[0]
    S = scale * (Q @ K.T)
    P, m, l = _softmax_rows(S, _visible(row_index, Lk, Nq, causal))
    O = P @ V
    lse = torch.where(torch.isneginf(m), m, m + torch.log(torch.where(l > 0, l,
                                                                      torch.ones_like(l))))
    return O, lse


def attn_fwd(q, k, v, scale: float, causal: bool, seqlens_k=None, rows=None):
    """O, LSE of dense attention, as ``oracle.attn_fwd`` (no window or block mask).

    q [B, Nq, Hq, d], k/v [B, Nk, Hkv, d]; seqlens_k optional [B]; rows:
    optional query-row indices (the other rows of the result are NaN).
    Returns float64 numpy arrays o [B, Nq, Hq, d], lse [B, Hq, Nq].
    """
    qd, kd, vd = _t64(q), _t64(k), _t64(v)
    B, Nq, Hq, d = qd.shape
    _, Nk, Hkv, _ = kd.shape
    G = Hq // Hkv
    lens = [Nk] * B if seqlens_k is None else _ints(seqlens_k)
    ridx = torch.arange(Nq) if rows is None else torch.as_tensor(_ints(rows), dtype=torch.long)
    o = np.full((B, Nq, Hq, d), np.nan)
    lse = np.full((B, Hq, Nq), np.nan)
    for b in range(B):
        Lk = lens[b]
        for h in range(Hq):
            g = h // G
            O, L = _attend(qd[b, ridx, h], kd[b, :Lk, g], vd[b, :Lk, g], scale, ridx, Nq,
                           causal)
            o[b, ridx.numpy(), h] = O.numpy()
            lse[b, h, ridx.numpy()] = L.numpy()
    return o, lse


def attn_kvcache(q, k_cache, v_cache, cu_seqlens_k, seqlens_k, scale: float, causal: bool):
    """O, LSE of new tokens against a packed cache, as ``oracle.attn_kvcache``.

    q [B, Nq, Hq, d]; k_cache/v_cache [slots, Hkv, d]; sequence b's keys are
    slots cu_seqlens_k[b] .. cu_seqlens_k[b] + seqlens_k[b] - 1; token t of
    the chunk is query row t (causal: bottom-right against the length).
    """
    qd, kd, vd = _t64(q), _t64(k_cache), _t64(v_cache)
    B, Nq, Hq, d = qd.shape
    Hkv = kd.shape[1]
    G = Hq // Hkv
    cu, lens = _ints(cu_seqlens_k), _ints(seqlens_k)
    o = np.full((B, Nq, Hq, d), np.nan)
    lse = np.full((B, Hq, Nq), np.nan)
    ridx = torch.arange(Nq)
    for b in range(B):
        s0, Lk = cu[b], lens[b]
        for h in range(Hq):
            g = h // G
            O, L = _attend(qd[b, :, h], kd[s0:s0 + Lk, g], vd[s0:s0 + Lk, g], scale, ridx, Nq,
                           causal)
            o[b, :, h] = O.numpy()
            lse[b, h] = L.numpy()
    return o, lse


def gather_paged(k_cache, v_cache, block_table, seqlens_k):
    """The logical cache of a paged layout as a packed one (a plain copy).

    k_cache/v_cache [num_blocks, block_size, Hkv, d]; logical key j of
    sequence b is row j % block_size of block block_table[b][j // block_size].
    Returns (k, v [sum(seqlens), Hkv, d] float64, cu_seqlens [B + 1]).
    """
    kc, vc = _t64(k_cache), _t64(v_cache)
    bs = kc.shape[1]
    bt = block_table.detach().cpu() if isinstance(block_table, torch.Tensor) else \
        torch.as_tensor(np.asarray(block_table))
    lens = _ints(seqlens_k)
    ks, vs, cu = [], [], [0]
    for b, L in enumerate(lens):
        j = torch.arange(L)
        blk = bt[b, j // bs].to(torch.long)
        ks.append(kc[blk, j % bs])
        vs.append(vc[blk, j % bs])
        cu.append(cu[-1] + L)
    return torch.cat(ks), torch.cat(vs), cu


def attn_paged(q, k_cache, v_cache, block_table, seqlens_k, scale: float, causal: bool):
    """O, LSE against a paged cache, as ``oracle.attn_paged`` (no append)."""
    k, v, cu = gather_paged(k_cache, v_cache, block_table, seqlens_k)
    return attn_kvcache(q, k, v, cu, seqlens_k, scale, causal)


def attn_bwd(q, k, v, dout, scale: float, causal: bool, seqlens_k=None, heads=None):
    """Gradients of L = sum(dout * O), as ``oracle.attn_bwd`` (no window or mask).

    The chain rule through the row softmax, per (batch, query head):
    dV += Pᵀ dO, dP = dO Vᵀ, dS = P ∘ (dP - rowsum(P ∘ dP)), dQ = scale dS K,
    dK += scale dSᵀ Q; dk, dv are summed over the heads of a kv head and are
    zero behind a sequence's length.  heads: optional list of (b, h) pairs to
    evaluate (dq rows of other pairs are NaN; dk, dv then hold only the
    listed pairs' contributions).
    Returns float64 numpy arrays (dq, dk, dv).
    """
    qd, kd, vd, dod = _t64(q), _t64(k), _t64(v), _t64(dout)
    B, Nq, Hq, d = qd.shape
    _, Nk, Hkv, _ = kd.shape
    G = Hq // Hkv
    lens = [Nk] * B if seqlens_k is None else _ints(seqlens_k)
    pairs = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else list(heads)
    dq = torch.full((B, Nq, Hq, d), float("nan"), dtype=_F64)
    dk = torch.zeros((B, Nk, Hkv, d), dtype=_F64)
    dv = torch.zeros((B, Nk, Hkv, d), dtype=_F64)
    ridx = torch.arange(Nq)
    for b, h in pairs:
        g, Lk = h // G, lens[b]
        Q, K, V, dO = qd[b, :, h], kd[b, :Lk, g], vd[b, :Lk, g], dod[b, :, h]
        S = scale * (Q @ K.T)
        P, _, _ = _softmax_rows(S, _visible(ridx, Lk, Nq, causal))
        dP = dO @ V.T
        Dr = (P * dP).sum(dim=1, keepdim=True)
        dS = P * (dP - Dr)
        dq[b, :, h] = scale * (dS @ K)
        dk[b, :Lk, g] += scale * (dS.T @ Q)
        dv[b, :Lk, g] += P.T @ dO
    return dq.numpy(), dk.numpy(), dv.numpy()


__all__ = ["attn_fwd", "attn_kvcache", "attn_paged", "gather_paged", "attn_bwd"]
