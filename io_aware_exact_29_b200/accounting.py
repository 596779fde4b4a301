"""Algorithmic work and traffic of the attention path (what the bench divides by).

Forward FLOPs count the two dense contractions only, exactly over the
unmasked (query, key) pairs: 4·d per pair (2·d for the score, 2·d for the
P·V product).  Forward bytes are one read of Q, K, V and one write of O (the
element size each) plus the fp32 LSE: the single-pass schedule of the
effectstory.com article "FlashAttention：IO 感知的精確注意力演算法...", section
"什麼是 FlashAttention？核心概念與 IO 感知機制" (load Q, K, V once, write back
once).  Decode bytes are the filled K and V cache rows read once plus the
query, the output and the LSE.
"""
from __future__ import annotations

import numpy as np


def score_matrix_elements(n: int) -> int:
    """Entries of one head's N×N score matrix S."""
    return n * n


def score_matrix_bytes(n: int, elem_bytes: int = 2) -> int:
    """Bytes of one head's S at ``elem_bytes`` per entry (fp16 = 2).

    The ai6s.net article's worked size (section "标准注意力的致命伤不在算力，
    在搬运"): N = 8192 gives 64M fp16 entries, 128 MB per head.
    """
    return score_matrix_elements(n) * elem_bytes


def visible_pairs(nq: int, lk: int, causal: bool) -> int:
    """Number of (query, key) pairs that the mask leaves visible for one head.

    Causal is bottom-right aligned: query i sees keys j <= i + lk - nq.
    """
    if not causal:
        return nq * lk
    total = 0
    off = lk - nq
    # rows whose visible prefix is clipped to [0, lk)
    for i in range(nq):
        c = i + off + 1
        if c > 0:
            total += min(c, lk)
    return total


def fwd_flops(B, Hq, Nq, Nk, d, causal, seqlens_k=None) -> int:
    if seqlens_k is None:
        return 4 * d * B * Hq * visible_pairs(Nq, Nk, causal)
    return sum(4 * d * Hq * visible_pairs(Nq, int(l), causal) for l in seqlens_k)


def block_pair_counts(Nq: int, Nk: int, causal: bool, block: int = 128) -> np.ndarray:
    """[nqb, nkb] int64: visible (query, key) pairs inside each block of a
    block mask, under the causal rule (bottom-right) when causal."""
    nqb, nkb = -(-Nq // block), -(-Nk // block)
    out = np.zeros((nqb, nkb), dtype=np.int64)
    off = Nk - Nq
    for qb in range(nqb):
        rows = np.arange(qb * block, min(Nq, (qb + 1) * block))
        for kb in range(nkb):
            lo, hi = kb * block, min(Nk, (kb + 1) * block)
            if causal:
                top = np.minimum(hi, rows + off + 1)
                out[qb, kb] = int(np.maximum(0, top - lo).sum())
            else:
                out[qb, kb] = len(rows) * (hi - lo)
    return out


def blocksparse_flops(mask, Nq: int, Nk: int, d: int, causal: bool, B: int, Hq: int,
                      block: int = 128) -> int:
    """4 d x (visible pairs) summed over batches and heads for a block mask
    [1|B, 1|Hq, nqb, nkb] (a size-1 dimension is shared)."""
    m = np.asarray(mask) != 0
    cnt = block_pair_counts(Nq, Nk, causal, block)
    per = (m * cnt[None, None]).sum(axis=(2, 3))  # [Bm, Hm]
    per = np.broadcast_to(per, (B, Hq))
    return int(4 * d * per.sum())


def fwd_bytes(B, Hq, Hkv, Nq, Nk, d, elem_bytes=2) -> int:
    q = B * Nq * Hq * d * elem_bytes
    kv = 2 * B * Nk * Hkv * d * elem_bytes
    o = B * Nq * Hq * d * elem_bytes
    lse = B * Hq * Nq * 4
    return q + kv + o + lse


def decode_bytes(seqlens_k, B, Hq, Hkv, Nq, d, elem_bytes=2) -> int:
    kv = 2 * sum(int(l) for l in seqlens_k) * Hkv * d * elem_bytes
    q = B * Nq * Hq * d * elem_bytes
    o = B * Nq * Hq * d * elem_bytes
    lse = B * Hq * Nq * 4
    return kv + q + o + lse


def decode_flops(seqlens_k, Hq, Nq, d, causal) -> int:
    return sum(4 * d * Hq * visible_pairs(Nq, int(l), causal) for l in seqlens_k)
