"""Block-sparse attention (attn_fwd_blocksparse, attn_bwd_blocksparse)
against the fp64 oracle with the same block mask: random masks of several
densities, per-head, per-batch and shared masks, causal and not, ragged
sizes, key padding, a window on top, rows with no block, skipped key blocks
holding NaN, and the gradients under the same masks."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import FwdCase, fwd_inputs, upstream_grad
from tests.parity import compare, compare_grads

pytestmark = pytest.mark.gpu

BLK = attn.MASK_BLOCK


def _mask(shape, density, seed):
    g = np.random.default_rng(seed)
    return (g.random(shape) < density).astype(np.uint8)


def _fwd(inp, c, mask, window_left=-1):
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    m = torch.from_numpy(np.ascontiguousarray(mask)).cuda() if isinstance(mask, np.ndarray) \
        else mask
    o, lse = attn.attn_fwd(dev["q"], dev["k"], dev["v"], scale=c.scale, causal=c.causal,
                           seqlens_k=dev["seqlens_k"], window_left=window_left, block_mask=m)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    return o, lse, dev


def _nb(c):
    return -(-c.Nq // BLK), -(-c.Nk // BLK)


@pytest.mark.parametrize("density", [0.2, 0.5, 0.9])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_random_masks_per_head(density, causal, d):
    c = FwdCase("bs", 2, 4, 2, 600, 700, d, causal)
    inp = fwd_inputs(c, seed=200 + int(density * 10))
    nqb, nkb = _nb(c)
    m = _mask((c.B, c.Hq, nqb, nkb), density, seed=int(density * 100) + d + causal)
    o, lse, _ = _fwd(inp, c, m)
    o_ref, l_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, c.causal,
                                   block_mask=m, block_size=BLK)
    compare(o, lse, o_ref, l_ref, what=f"block-sparse {density} causal {causal} d{d}")


@pytest.mark.parametrize("shape", ["shared", "per_batch", "per_head"])
def test_mask_sharing(shape):
    c = FwdCase("bss", 3, 4, 1, 512, 640, 128, False)
    inp = fwd_inputs(c, seed=210)
    nqb, nkb = _nb(c)
    dims = {"shared": (1, 1), "per_batch": (c.B, 1), "per_head": (1, c.Hq)}[shape]
    m = _mask(dims + (nqb, nkb), 0.5, seed=211)
    o, lse, _ = _fwd(inp, c, m)
    o_ref, l_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, False, block_mask=m,
                                   block_size=BLK)
    compare(o, lse, o_ref, l_ref, what=f"mask {shape}")


def test_padded_mask_rows():
    # the mask is a view into a wider array: its row stride exceeds the key-block count
    c = FwdCase("bsp", 2, 2, 2, 300, 500, 64, True)
    inp = fwd_inputs(c, seed=212)
    nqb, nkb = _nb(c)
    wide = _mask((c.B, c.Hq, nqb, nkb + 5), 0.6, seed=213)
    view = torch.from_numpy(wide).cuda()[..., :nkb]
    assert view.stride(2) == nkb + 5
    o, lse, _ = _fwd(inp, c, view)
    o_ref, l_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, True,
                                   block_mask=wide[..., :nkb], block_size=BLK)
    compare(o, lse, o_ref, l_ref, what="strided mask")


def test_all_ones_is_the_dense_result():
    c = FwdCase("bs1", 2, 4, 2, 520, 777, 128, True)
    inp = fwd_inputs(c, seed=214)
    nqb, nkb = _nb(c)
    o, lse, dev = _fwd(inp, c, np.ones((1, 1, nqb, nkb), np.uint8))
    a = attn.attn_fwd(dev["q"], dev["k"], dev["v"], scale=c.scale, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o, a[0]) and torch.equal(lse, a[1])


def test_rows_without_blocks_and_empty_mask():
    c = FwdCase("bs0", 1, 2, 2, 384, 384, 128, False)
    inp = fwd_inputs(c, seed=215)
    m = np.ones((1, 2, 3, 3), np.uint8)
    m[0, 0, 1, :] = 0  # head 0, rows 128..255: no key block at all
    o, lse, _ = _fwd(inp, c, m)
    assert not o[0, 128:256, 0].any()
    assert torch.isneginf(lse[0, 0, 128:256]).all()
    o_ref, l_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, False, block_mask=m,
                                   block_size=BLK)
    compare(o, lse, o_ref, l_ref, what="rows without blocks")
    o, lse, _ = _fwd(inp, c, np.zeros((1, 1, 3, 3), np.uint8))
    assert not o.any() and torch.isneginf(lse).all()


def test_skipped_blocks_are_not_read():
    # key block 2 is masked for every query block: NaN stored there stays out
    c = FwdCase("bsn", 2, 4, 2, 512, 640, 128, False)
    inp = fwd_inputs(c, seed=216)
    nqb, nkb = _nb(c)
    m = _mask((c.B, c.Hq, nqb, nkb), 0.7, seed=217)
    m[..., 2] = 0
    m[..., 0] = 1
    clean = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, False, block_mask=m,
                            block_size=BLK)
    inp["k"][:, 2 * BLK:3 * BLK] = float("nan")
    inp["v"][:, 2 * BLK:3 * BLK] = float("nan")
    o, lse, _ = _fwd(inp, c, m)
    compare(o, lse, clean[0], clean[1], what="NaN in skipped blocks")


def test_with_key_padding_and_window():
    c = FwdCase("bsw", 3, 4, 4, 400, 900, 128, True)
    inp = fwd_inputs(c, seed=218)
    inp["seqlens_k"] = torch.tensor([900, 555, 260], dtype=torch.int32)
    for b, L in enumerate(inp["seqlens_k"].tolist()):
        inp["k"][b, L:] = float("nan")
        inp["v"][b, L:] = float("nan")
    nqb, nkb = _nb(c)
    m = _mask((c.B, c.Hq, nqb, nkb), 0.6, seed=219)
    for w in (-1, 300):
        o, lse, _ = _fwd(inp, c, m, window_left=w)
        o_ref, l_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, True,
                                       seqlens_k=inp["seqlens_k"], window_left=w, block_mask=m,
                                       block_size=BLK)
        compare(o, lse, o_ref, l_ref, what=f"block-sparse + key padding, window {w}")


def test_fp16_and_long_rows_sampled():
    # a longer problem checked on sampled rows: 16 key blocks, ~30% kept
    c = FwdCase("bsl", 1, 2, 1, 2048, 2048, 128, True, dtype="fp16")
    inp = fwd_inputs(c, seed=220)
    m = _mask((1, c.Hq, 16, 16), 0.3, seed=221)
    m[..., 0] = 1
    o, lse, _ = _fwd(inp, c, m)
    rows = sorted({0, 1, 127, 128, 1000, 2047} | set(range(300, 2048, 97)))
    o_ref, l_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, True, rows=rows,
                                   block_mask=m, block_size=BLK)
    compare(o, lse, o_ref, l_ref, rows=rows, what="fp16 block-sparse, sampled rows")


def _bwd(inp, c, m, window_left=-1, seed=0):
    o, lse, dev = _fwd(inp, c, m, window_left)
    mt = torch.from_numpy(np.ascontiguousarray(m)).cuda()
    dout = upstream_grad(inp["q"], seed=seed)
    got = attn.attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dout.cuda(), scale=c.scale,
                        causal=c.causal, seqlens_k=dev["seqlens_k"], window_left=window_left,
                        block_mask=mt)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    ref = oracle.attn_bwd(inp["q"], inp["k"], inp["v"], dout, c.scale, c.causal,
                          seqlens_k=inp["seqlens_k"], window_left=window_left, block_mask=m,
                          block_size=BLK)
    return got, ref


@pytest.mark.parametrize("density", [0.3, 0.7])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_backward_random_masks(density, causal, d):
    # GQA: the four query heads of a kv head carry different masks, so dK and
    # dV sum over differently masked heads
    c = FwdCase("bsb", 2, 8, 2, 448, 520, d, causal)
    inp = fwd_inputs(c, seed=230 + d)
    nqb, nkb = _nb(c)
    m = _mask((c.B, c.Hq, nqb, nkb), density, seed=231 + int(density * 10) + causal)
    got, ref = _bwd(inp, c, m, seed=232)
    compare_grads(got, ref, what=f"bwd block-sparse {density} causal {causal} d{d}")


def test_backward_empty_rows_and_columns():
    c = FwdCase("bse", 1, 2, 1, 384, 512, 128, False)
    inp = fwd_inputs(c, seed=233)
    m = np.ones((1, 2, 3, 4), np.uint8)
    m[0, :, :, 1] = 0  # key block 1 masked for every query: dK, dV = 0 there
    m[0, 0, 2, :] = 0  # head 0, query block 2: no key: dQ = 0 there
    got, ref = _bwd(inp, c, m, seed=234)
    dq, dk, dv = (t.float().cpu() for t in got)
    assert not dk[0, 128:256].any() and not dv[0, 128:256].any()
    assert not dq[0, 256:384, 0].any()
    compare_grads(got, ref, what="bwd empty rows and columns")


def test_backward_with_key_padding_and_window():
    c = FwdCase("bsbw", 2, 4, 2, 384, 700, 128, True)
    inp = fwd_inputs(c, seed=235)
    inp["seqlens_k"] = torch.tensor([700, 333], dtype=torch.int32)
    for b, L in enumerate(inp["seqlens_k"].tolist()):
        inp["k"][b, L:] = float("nan")
        inp["v"][b, L:] = float("nan")
    nqb, nkb = _nb(c)
    m = _mask((1, c.Hq, nqb, nkb), 0.6, seed=236)
    for w in (-1, 250):
        got, ref = _bwd(inp, c, m, window_left=w, seed=237)
        compare_grads(got, ref, what=f"bwd block-sparse + key padding, window {w}")


@pytest.mark.parametrize("nq,nk", [(300, 900), (640, 384)])
def test_rectangular_causal_bottom_right(nq, nk):
    # fewer queries than keys (a chunk at the end of a long prefix) and more
    # queries than keys (rows before the first key see nothing), causal
    c = FwdCase("bsr", 2, 4, 2, nq, nk, 128, True)
    inp = fwd_inputs(c, seed=240 + nq)
    nqb, nkb = _nb(c)
    m = _mask((c.B, c.Hq, nqb, nkb), 0.6, seed=241 + nk)
    o, lse, _ = _fwd(inp, c, m)
    o_ref, l_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, True, block_mask=m,
                                   block_size=BLK)
    compare(o, lse, o_ref, l_ref, what=f"block-sparse causal {nq}x{nk}")


def test_d64_fp16_with_key_padding():
    c = FwdCase("bs64", 3, 6, 2, 520, 600, 64, False, dtype="fp16")
    inp = fwd_inputs(c, seed=242)
    inp["seqlens_k"] = torch.tensor([600, 333, 129], dtype=torch.int32)
    for b, L in enumerate(inp["seqlens_k"].tolist()):
        inp["k"][b, L:] = float("nan")
        inp["v"][b, L:] = float("nan")
    nqb, nkb = _nb(c)
    m = _mask((c.B, c.Hq, nqb, nkb), 0.5, seed=243)
    o, lse, _ = _fwd(inp, c, m)
    o_ref, l_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, False,
                                   seqlens_k=inp["seqlens_k"], block_mask=m, block_size=BLK)
    compare(o, lse, o_ref, l_ref, what="block-sparse d64 fp16 key padding")


def test_backward_d64_fp16_causal_rectangular():
    c = FwdCase("bsb64", 2, 4, 1, 300, 520, 64, True, dtype="fp16")
    inp = fwd_inputs(c, seed=244)
    nqb, nkb = _nb(c)
    m = _mask((c.B, c.Hq, nqb, nkb), 0.6, seed=245)
    got, ref = _bwd(inp, c, m, seed=246)
    compare_grads(got, ref, what="bwd block-sparse d64 fp16 causal 300x520")
