"""Seeded random shapes against the matrix-product fp64 oracle.

Each case draws its sizes from a generator seeded by the case number: batch,
heads and their grouping, query and key lengths (ragged against the 128-row
tiles, more queries than keys or fewer), head dim, causal or not, bf16 or
fp16, and per-sequence key lengths with NaN behind them.  The decode cases
add token counts 1..16, empty sequences, unfilled slots holding NaN and split
sizes (both the tensor-core and the mma.sync instance), the paged ones block
sizes 16..256 with NaN in every unused row (and the fused append of the new
tokens' K/V), the backward cases the gradients of all three inputs, and the
masked cases sliding windows and block masks in the forward and backward
(against the C oracle, which takes both).  The softmax scale is 1/sqrt(d) in most cases
and otherwise small (nearly uniform rows) or large (nearly one-hot rows, many
moves of the running maximum).  Every output element is compared, through
guarded, NaN-prefilled buffers.
"""
from types import SimpleNamespace

import pytest
import torch

from oracle import dense
from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import (DecodeCase, FwdCase, fwd_inputs, kvcache_inputs,
                                              paged_from_packed, upstream_grad)
from tests.parity import (GRAD_FEW_KEYS, GRAD_MEAN_REL, GRAD_MEAN_REL_FEW_KEYS, compare,
                          compare_grads, run_fwd)
from tests.test_bwd_gpu import _run as run_bwd
from tests.test_decode_gpu import _run as run_decode
from tests.test_paged_gpu import _run as run_paged

pytestmark = pytest.mark.gpu

NAN = float("nan")


class _Draw:
    """Integers and choices from one seeded generator."""

    def __init__(self, seed):
        self.g = torch.Generator().manual_seed(7919 * (seed + 1))

    def int(self, lo, hi):
        return int(torch.randint(lo, hi + 1, (1,), generator=self.g).item())

    def pick(self, options):
        return options[self.int(0, len(options) - 1)]


def _nan_behind(inp, lens):
    for b, L in enumerate(lens):
        inp["k"][b, L:] = NAN
        inp["v"][b, L:] = NAN


@pytest.mark.parametrize("seed", range(48))
def test_forward_random_shapes(seed):
    r = _Draw(seed)
    B, Hkv, G = r.int(1, 4), r.pick([1, 2, 4]), r.pick([1, 2, 4, 8])
    Nq, Nk, d = r.int(1, 700), r.int(1, 900), r.pick([64, 128])
    causal, dtype, kpad = bool(r.int(0, 1)), r.pick(["bf16", "fp16"]), r.int(0, 2) == 0
    c = FwdCase("fz", B, Hkv * G, Hkv, Nq, Nk, d, causal, dtype=dtype)
    scale = r.pick([c.scale, c.scale, c.scale, 0.02, 0.3, 1.0])
    inp = fwd_inputs(c, seed=seed)
    what = (f"B{B} Hq{Hkv * G} Hkv{Hkv} Nq{Nq} Nk{Nk} d{d} causal {causal} {dtype} "
            f"kpad {kpad} scale {scale}")
    if kpad:
        lens = [r.int(0, Nk) for _ in range(B)]
        inp["seqlens_k"] = torch.tensor(lens, dtype=torch.int32)
        _nan_behind(inp, lens)
    o, lse = run_fwd(inp, causal, scale)
    o_ref, lse_ref = dense.attn_fwd(inp["q"], inp["k"], inp["v"], scale, causal,
                                    seqlens_k=inp.get("seqlens_k"))
    compare(o, lse, o_ref, lse_ref, what=what)


@pytest.mark.parametrize("seed", range(32))
def test_decode_random_shapes(seed):
    r = _Draw(100 + seed)
    B, Hkv, G = r.int(1, 40), r.pick([1, 2, 8]), r.pick([1, 2, 4, 8, 16])
    Nq = r.pick([1, r.int(2, 16)])
    d, dtype = r.pick([64, 128]), r.pick(["bf16", "fp16"])
    causal = Nq > 1 and bool(r.int(0, 1))
    split = r.pick([0, 0, 64, 128, 1024])
    lo = Nq if causal else 0
    lens = [r.pick([lo, r.int(lo, 3000), r.int(lo, 3000)]) for _ in range(B)]
    c = DecodeCase("fzd", B, Hkv * G, Hkv, Nq, d, (lo, 3000), causal, dtype=dtype,
                   slack=r.int(0, 9))
    scale = r.pick([c.scale, c.scale, c.scale, 0.02, 0.3, 1.0])
    inp = kvcache_inputs(c, seed=seed, seqlens=lens, slack_fill=NAN)
    o, lse = run_decode(inp, SimpleNamespace(scale=scale, causal=causal, Hkv=Hkv),
                        split_keys=split)
    o_ref, lse_ref = dense.attn_kvcache(inp["q"], inp["k_cache"], inp["v_cache"],
                                        inp["cu_seqlens_k"], inp["seqlens_k"], scale, causal)
    compare(o, lse, o_ref, lse_ref, what=f"decode B{B} G{G} Hkv{Hkv} Nq{Nq} d{d} {dtype} "
                                         f"causal {causal} split {split} scale {scale}")


@pytest.mark.parametrize("seed", range(16))
def test_paged_random_shapes(seed):
    r = _Draw(200 + seed)
    block = r.pick([16, 32, 64, 128, 256])
    B, Hkv, G = r.int(1, 24), r.pick([1, 2, 8]), r.pick([1, 2, 4, 8, 16])
    Nq = r.int(1, min(16, 128 // G))
    d, dtype = r.pick([64, 128]), r.pick(["bf16", "fp16"])
    causal = Nq > 1 and bool(r.int(0, 1))
    lo = Nq if causal else 0
    lens = [r.int(lo, 3000) for _ in range(B)]
    c = DecodeCase("fzp", B, Hkv * G, Hkv, Nq, d, (lo, 3000), causal, dtype=dtype)
    inp = kvcache_inputs(c, seed=seed, seqlens=lens)
    pg = paged_from_packed(inp, block, seed=seed)
    scale = r.pick([c.scale, c.scale, 0.3, 1.0])
    o, lse, _ = run_paged(inp, pg, SimpleNamespace(scale=scale, causal=causal, Hkv=Hkv))
    o_ref, lse_ref = dense.attn_kvcache(inp["q"], inp["k_cache"], inp["v_cache"],
                                        inp["cu_seqlens_k"], inp["seqlens_k"], scale, causal)
    compare(o, lse, o_ref, lse_ref, what=f"paged bs{block} B{B} G{G} Hkv{Hkv} Nq{Nq} d{d} "
                                         f"{dtype} causal {causal} scale {scale}")


@pytest.mark.parametrize("seed", range(16))
def test_backward_random_shapes(seed):
    r = _Draw(300 + seed)
    B, Hkv, G = r.int(1, 3), r.pick([1, 2]), r.pick([1, 2, 4])
    Nq, Nk, d = r.int(1, 400), r.int(1, 500), r.pick([64, 128])
    causal, dtype, kpad = bool(r.int(0, 1)), r.pick(["bf16", "fp16"]), r.int(0, 2) == 0
    c = FwdCase("fzb", B, Hkv * G, Hkv, Nq, Nk, d, causal, dtype=dtype)
    inp = fwd_inputs(c, seed=seed)
    if kpad:
        lens = [r.int(1, Nk) for _ in range(B)]
        inp["seqlens_k"] = torch.tensor(lens, dtype=torch.int32)
        _nan_behind(inp, lens)
    scale = r.pick([c.scale, c.scale, 0.02, 0.3])
    dout = upstream_grad(inp["q"], seed=seed)
    got = run_bwd(inp, SimpleNamespace(scale=scale, causal=causal), dout)
    ref = dense.attn_bwd(inp["q"], inp["k"], inp["v"], dout, scale, causal,
                         seqlens_k=inp.get("seqlens_k"))
    # keys each row sees (bottom-right causal), averaged over rows that see any
    seen = []
    for b in range(B):
        L = lens[b] if kpad else Nk
        for i in range(Nq):
            n = max(0, min(L, i + L - Nq + 1)) if causal else L
            if n > 0:
                seen.append(n)
    few = not seen or sum(seen) / len(seen) < GRAD_FEW_KEYS
    compare_grads(got, ref, what=f"bwd B{B} Hq{Hkv * G} Hkv{Hkv} Nq{Nq} Nk{Nk} d{d} "
                                 f"causal {causal} {dtype} kpad {kpad} scale {scale}",
                  mean_rel=GRAD_MEAN_REL_FEW_KEYS if few else GRAD_MEAN_REL)


@pytest.mark.parametrize("seed", range(16))
def test_masked_forward_and_backward_random_shapes(seed):
    # sliding windows and block masks (against the C oracle, which takes both)
    import numpy as np

    import oracle

    r = _Draw(400 + seed)
    B, Hkv, G = r.int(1, 2), r.pick([1, 2]), r.pick([1, 2, 4])
    Nq, Nk, d = r.int(1, 400), r.int(1, 500), r.pick([64, 128])
    causal, dtype = bool(r.int(0, 1)), r.pick(["bf16", "fp16"])
    window = r.pick([-1, r.int(0, 300)])
    sparse = r.int(0, 1) == 1 or window < 0
    c = FwdCase("fzm", B, Hkv * G, Hkv, Nq, Nk, d, causal, dtype=dtype)
    inp = fwd_inputs(c, seed=seed)
    what = f"masked B{B} Hq{Hkv * G} Nq{Nq} Nk{Nk} d{d} causal {causal} window {window}"
    mask = None
    if sparse:
        blk = attn.MASK_BLOCK
        rng = np.random.default_rng(seed)
        shape = (r.pick([1, B]), r.pick([1, Hkv * G]), -(-Nq // blk), -(-Nk // blk))
        mask = (rng.random(shape) < r.pick([0.3, 0.6, 0.9])).astype(np.uint8)
        what += f" block mask {shape}"
    dev = {n: inp[n].cuda() for n in ("q", "k", "v")}
    m = None if mask is None else torch.from_numpy(mask).cuda()
    o, lse = attn.attn_fwd(dev["q"], dev["k"], dev["v"], scale=c.scale, causal=causal,
                           window_left=window, block_mask=m)
    dout = upstream_grad(inp["q"], seed=seed)
    dq, dk, dv = attn.attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dout.cuda(),
                               scale=c.scale, causal=causal, window_left=window, block_mask=m)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    kw = dict(window_left=window)
    if mask is not None:
        kw.update(block_mask=mask, block_size=attn.MASK_BLOCK)
    o_ref, lse_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, causal, **kw)
    compare(o, lse, o_ref, lse_ref, what=what)
    ref = oracle.attn_bwd(inp["q"], inp["k"], inp["v"], dout, c.scale, causal, **kw)
    # keys each (batch, head, row) sees under causal, window and block mask,
    # averaged over the rows that see any (the mean bound depends on it)
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    vis = np.ones((Nq, Nk), dtype=bool)
    if causal:
        vis &= j <= i + Nk - Nq
    if window >= 0:
        vis &= j >= i + Nk - Nq - window
    seen = []
    for b in range(B):
        for h in range(Hkv * G):
            v_bh = vis
            if mask is not None:
                mb = mask[min(b, mask.shape[0] - 1), min(h, mask.shape[1] - 1)]
                v_bh = vis & mb[i // attn.MASK_BLOCK, j // attn.MASK_BLOCK].astype(bool)
            n = v_bh.sum(axis=1)
            seen.extend(n[n > 0].tolist())
    few = not seen or sum(seen) / len(seen) < GRAD_FEW_KEYS
    compare_grads((dq, dk, dv), ref, what=what,
                  mean_rel=GRAD_MEAN_REL_FEW_KEYS if few else GRAD_MEAN_REL)


@pytest.mark.parametrize("seed", range(8))
def test_paged_append_random_shapes(seed):
    # the fused append writes the new tokens' K/V into the paged cache, then
    # the decode reads them with the rest of each sequence
    import oracle

    r = _Draw(500 + seed)
    block = r.pick([16, 32, 64, 256])
    B, Hkv, G = r.int(1, 12), r.pick([1, 2, 8]), r.pick([1, 2, 4, 8])
    Nq = r.int(1, min(16, 128 // G))
    d, dtype = r.pick([64, 128]), r.pick(["bf16", "fp16"])
    causal = Nq > 1 and bool(r.int(0, 1))
    lens = [r.int(Nq, 3000) for _ in range(B)]
    c = DecodeCase("fza", B, Hkv * G, Hkv, Nq, d, (Nq, 3000), causal, dtype=dtype)
    inp = kvcache_inputs(c, seed=seed, seqlens=lens)
    full = paged_from_packed(inp, block, seed=seed)
    holes = paged_from_packed(inp, block, seed=seed, new_tokens=Nq)
    o, lse, dev = run_paged(inp, holes, c, with_new=True)
    o_ref, lse_ref = oracle.attn_kvcache(inp["q"], inp["k_cache"], inp["v_cache"],
                                         inp["cu_seqlens_k"], inp["seqlens_k"], c.scale, causal)
    compare(o, lse, o_ref, lse_ref, what=f"append bs{block} B{B} G{G} Nq{Nq} d{d} {dtype}")
    for name in ("k_cache", "v_cache"):
        assert torch.equal(dev[name].cpu().view(torch.int16), full[name].view(torch.int16))
