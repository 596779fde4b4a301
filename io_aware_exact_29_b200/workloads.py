"""Seeded synthetic workloads shared by the tests, the bench and the smoke run.

This module draws inputs only; it holds none of attention's arithmetic, so both
the CUDA path and the CPU oracle may be fed from it.

Recipe (one ``torch.Generator`` per call, ``manual_seed(seed)``, seed 0 by
default): first the per-sequence lengths (``randint`` with inclusive bounds),
then Q, K and V as float32 ``randn`` (i.i.d. N(0, 1)), then a round-to-nearest
cast to bf16 or fp16.  Both sides consume the same stored bits.  The shapes
mirror the workloads named by the pages: BERT-large at sequence length 512,
GPT-2 at 1K, the long-range sweep up to 16K and Llama2-70B decoding
(effectstory.com "FlashAttention：IO 感知的精確注意力演算法..." training table;
ai6s.net article, section "跑出来的数据比道理有说服力").  No dataset or trained
weight is involved.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}


def default_scale(d: int) -> float:
    """The fp32 value of 1/sqrt(d), passed identically to the kernel and the oracle."""
    return float(torch.tensor(1.0, dtype=torch.float32) / torch.sqrt(
        torch.tensor(float(d), dtype=torch.float32)))


@dataclass
class FwdCase:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    dtype: str = "bf16"
    kpad_range: tuple | None = None  # (lo, hi) inclusive key-length range, or None

    @property
    def scale(self) -> float:
        return default_scale(self.d)


@dataclass
class DecodeCase:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int  # new tokens per sequence
    d: int
    lk_range: tuple  # inclusive
    causal: bool
    dtype: str = "bf16"
    slack: int = 0  # pre-allocated unused slots after each sequence

    @property
    def scale(self) -> float:
        return default_scale(self.d)


def _cases():
    fwd = [
        FwdCase("tiny", 1, 2, 2, 128, 128, 64, False),
        FwdCase("tiny_causal", 1, 2, 2, 128, 128, 64, True),
        FwdCase("bert_large", 16, 16, 16, 512, 512, 64, False),
        FwdCase("bert_large_varlen", 16, 16, 16, 512, 512, 64, False, kpad_range=(256, 512)),
        FwdCase("gpt2", 8, 12, 12, 1024, 1024, 64, True),
        FwdCase("gpt2_fp16", 8, 12, 12, 1024, 1024, 64, True, dtype="fp16"),
    ]
    for d in (64, 128):
        for n in (1024, 2048, 4096, 8192, 16384):
            for causal in (False, True):
                fwd.append(FwdCase(f"sweep_d{d}_n{n}{'_causal' if causal else ''}",
                                   16384 // n, 16, 16, n, n, d, causal))
    dec = [
        DecodeCase("llama70b_decode", 32, 64, 8, 1, 128, (1, 32768), False),
        DecodeCase("llama70b_chunk16", 32, 64, 8, 16, 128, (16, 32768), True),
    ]
    return {c.name: c for c in fwd}, {c.name: c for c in dec}


FWD_CASES, DECODE_CASES = _cases()


@dataclass
class BlockSparseCase:
    """A forward problem plus a seeded block mask of 128 x 128 blocks."""
    name: str
    fwd: FwdCase
    density: float  # probability that an off-diagonal block is kept


# the long-sequence sweep's N = 8192, d = 128 point with a quarter of the
# blocks kept per head (the pages give no block-sparse workload; this is the
# dense sweep point thinned out)
BLOCKSPARSE_CASES = {
    "blocksparse_d128_n8192_25pct": BlockSparseCase(
        "blocksparse_d128_n8192_25pct", FwdCase("bs", 2, 16, 16, 8192, 8192, 128, False), 0.25),
    "blocksparse_d128_n8192_causal_25pct": BlockSparseCase(
        "blocksparse_d128_n8192_causal_25pct", FwdCase("bsc", 2, 16, 16, 8192, 8192, 128, True),
        0.25),
}


def block_mask_inputs(case: BlockSparseCase, seed: int = 0, device: str = "cpu",
                      block: int = 128) -> torch.Tensor:
    """uint8 [B, H, ceil(Nq/block), ceil(Nk/block)]: each block kept with
    probability case.density, and the block on the diagonal of the query's
    own position always kept (so that no causal row is left without keys)."""
    c = case.fwd
    g = torch.Generator(device="cpu").manual_seed(seed + 7_000_003)
    nqb, nkb = -(-c.Nq // block), -(-c.Nk // block)
    m = (torch.rand((c.B, c.Hq, nqb, nkb), generator=g) < case.density).to(torch.uint8)
    for qb in range(nqb):
        kb = min(nkb - 1, (qb * block + c.Nk - c.Nq) // block) if c.Nk > 0 else -1
        if kb >= 0:
            m[:, :, qb, kb] = 1
    return m.to(device)


def fwd_inputs(case: FwdCase, seed: int = 0, device: str = "cpu"):
    """Q [B,Nq,Hq,d], K/V [B,Nk,Hkv,d] in the case's dtype, and the optional
    per-batch key lengths [B] int32."""
    g = torch.Generator(device=device).manual_seed(seed)
    seqlens = None
    if case.kpad_range is not None:
        lo, hi = case.kpad_range
        seqlens = torch.randint(lo, hi + 1, (case.B,), generator=g, device=device,
                                dtype=torch.int32)
    dt = DTYPES[case.dtype]
    q = torch.randn((case.B, case.Nq, case.Hq, case.d), generator=g, device=device).to(dt)
    k = torch.randn((case.B, case.Nk, case.Hkv, case.d), generator=g, device=device).to(dt)
    v = torch.randn((case.B, case.Nk, case.Hkv, case.d), generator=g, device=device).to(dt)
    return dict(q=q, k=k, v=v, seqlens_k=seqlens)


def upstream_grad(like: torch.Tensor, seed: int = 0, device: str = "cpu") -> torch.Tensor:
    """dO for the backward pass: N(0, 1) values of q's shape and dtype, from
    its own generator (seed + 1_000_003) so that the forward's inputs are the
    same with or without it."""
    g = torch.Generator(device=device).manual_seed(seed + 1_000_003)
    return torch.randn(tuple(like.shape), generator=g, device=device).to(like.dtype)


def kvcache_inputs(case: DecodeCase, seed: int = 0, device: str = "cpu",
                   slack_fill: float | None = None, seqlens=None):
    """Packed variable-length KV cache.

    Sequence b owns slots cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1 of
    k_cache/v_cache [slots, Hkv, d]; the first seqlens_k[b] of them are filled
    and ``case.slack`` pre-allocated slots follow.  ``slack_fill`` (e.g. NaN)
    overwrites the unfilled slots with a sentinel.  ``seqlens`` overrides the
    drawn lengths (edge-case tests).
    """
    g = torch.Generator(device=device).manual_seed(seed)
    lo, hi = case.lk_range
    drawn = torch.randint(lo, hi + 1, (case.B,), generator=g, device=device, dtype=torch.int32)
    if seqlens is not None:
        drawn = torch.as_tensor(seqlens, dtype=torch.int32, device=device)
    caps = drawn.to(torch.int64) + case.slack
    cu = torch.zeros(case.B + 1, dtype=torch.int64, device=device)
    cu[1:] = torch.cumsum(caps, 0)
    total = int(cu[-1].item())
    dt = DTYPES[case.dtype]
    q = torch.randn((case.B, case.Nq, case.Hq, case.d), generator=g, device=device).to(dt)
    k_cache = torch.randn((total, case.Hkv, case.d), generator=g, device=device).to(dt)
    v_cache = torch.randn((total, case.Hkv, case.d), generator=g, device=device).to(dt)
    if slack_fill is not None and case.slack > 0:
        for b in range(case.B):
            s0 = int(cu[b].item()) + int(drawn[b].item())
            s1 = int(cu[b + 1].item())
            k_cache[s0:s1] = slack_fill
            v_cache[s0:s1] = slack_fill
    return dict(q=q, k_cache=k_cache, v_cache=v_cache, cu_seqlens_k=cu.to(torch.int32),
                seqlens_k=drawn)


def paged_from_packed(inp, block_size: int, seed: int = 0, spare_blocks: int = 2,
                      fill: float = float("nan"), new_tokens: int = 0):
    """The same logical cache as ``kvcache_inputs`` laid out in blocks.

    Sequence b's first seqlens_k[b] rows go, in order, into ceil(L/block_size)
    physical blocks drawn from a seeded permutation; every other row (block
    tails, spare blocks) holds ``fill``.  With ``new_tokens`` = n > 0 the last
    n filled rows of each sequence are left as ``fill`` too and returned as
    k_new/v_new [B, n, Hkv, d] (the rows an append would write).
    Returns dict(k_cache, v_cache [num_blocks, block_size, Hkv, d],
    block_table int32 [B, max_blocks] (-1 past a sequence's blocks),
    seqlens_k, and k_new/v_new when requested).
    """
    kc, vc = inp["k_cache"], inp["v_cache"]
    cu = inp["cu_seqlens_k"].tolist()
    lens = inp["seqlens_k"].tolist()
    B = len(lens)
    nblk = [(L + block_size - 1) // block_size for L in lens]
    total = sum(nblk) + spare_blocks
    g = torch.Generator().manual_seed(seed + 7)
    perm = torch.randperm(total, generator=g).tolist()
    Hkv, d = kc.shape[1], kc.shape[2]
    kp = torch.full((total, block_size, Hkv, d), fill, dtype=kc.dtype)
    vp = torch.full((total, block_size, Hkv, d), fill, dtype=vc.dtype)
    table = torch.full((B, max(1, max(nblk))), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        for i in range(nblk[b]):
            blk = perm[nxt]
            nxt += 1
            table[b, i] = blk
            r0 = i * block_size
            r1 = min(lens[b], r0 + block_size)
            kp[blk, : r1 - r0] = kc[cu[b] + r0: cu[b] + r1]
            vp[blk, : r1 - r0] = vc[cu[b] + r0: cu[b] + r1]
    out = dict(k_cache=kp, v_cache=vp, block_table=table, seqlens_k=inp["seqlens_k"].clone())
    if new_tokens:
        n = new_tokens
        kn = torch.zeros((B, n, Hkv, d), dtype=kc.dtype)
        vn = torch.zeros((B, n, Hkv, d), dtype=vc.dtype)
        for b in range(B):
            for t in range(n):
                pos = lens[b] - n + t
                if pos < 0:
                    continue
                kn[b, t] = kc[cu[b] + pos]
                vn[b, t] = vc[cu[b] + pos]
                blk = int(table[b, pos // block_size])
                kp[blk, pos % block_size] = fill
                vp[blk, pos % block_size] = fill
        out["k_new"], out["v_new"] = kn, vn
    return out
