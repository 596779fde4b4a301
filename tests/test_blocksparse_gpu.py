"""Block-sparse forward (attn_fwd_blocksparse) against the fp64 oracle with
the same block mask: random masks of several densities, per-head, per-batch
and shared masks, causal and not, ragged sizes, key padding, a window on
top, rows with no block, and skipped key blocks holding NaN."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import FwdCase, fwd_inputs
from tests.parity import compare

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
