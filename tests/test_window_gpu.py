"""Sliding-window mask (attn_fwd_window, attn_bwd_window) against the fp64
oracle with the same window: windows inside one key tile, across tile edges
and wider than the keys, causal and not, ragged sizes, key padding, GQA and
both head sizes."""
import pytest
import torch

import oracle
from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import FwdCase, fwd_inputs, upstream_grad
from tests.parity import compare, compare_grads

pytestmark = pytest.mark.gpu


def _fwd(inp, c, w):
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o, lse = attn.attn_fwd(dev["q"], dev["k"], dev["v"], scale=c.scale, causal=c.causal,
                           seqlens_k=dev["seqlens_k"], window_left=w)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    return o, lse, dev


@pytest.mark.parametrize("w", [0, 1, 100, 127, 128, 300, 5000])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_forward_windows(w, causal, d):
    c = FwdCase("w", 2, 4, 2, 600, 700, d, causal)
    inp = fwd_inputs(c, seed=100 + w)
    o, lse, _ = _fwd(inp, c, w)
    o_ref, l_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, c.causal,
                                   window_left=w)
    compare(o, lse, o_ref, l_ref, what=f"window {w} causal {causal} d{d}")


def test_forward_window_with_key_padding():
    c = FwdCase("wp", 3, 4, 4, 384, 512, 128, True)
    inp = fwd_inputs(c, seed=110)
    inp["seqlens_k"] = torch.tensor([512, 300, 130], dtype=torch.int32)
    for b, L in enumerate(inp["seqlens_k"].tolist()):
        inp["k"][b, L:] = float("nan")
        inp["v"][b, L:] = float("nan")
    o, lse, _ = _fwd(inp, c, 200)
    o_ref, l_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, True,
                                   seqlens_k=inp["seqlens_k"], window_left=200)
    compare(o, lse, o_ref, l_ref, what="window + key padding")


def test_no_window_is_bit_identical():
    c = FwdCase("wn", 2, 4, 2, 300, 300, 128, True)
    inp = fwd_inputs(c, seed=111)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    a = attn.attn_fwd(dev["q"], dev["k"], dev["v"], scale=c.scale, causal=True)
    b = attn.attn_fwd(dev["q"], dev["k"], dev["v"], scale=c.scale, causal=True, window_left=1000)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("w,causal", [(0, True), (64, True), (200, True), (150, False)])
@pytest.mark.parametrize("d", [64, 128])
def test_backward_windows(w, causal, d):
    c = FwdCase("wb", 2, 8, 2, 384, 448, d, causal)
    inp = fwd_inputs(c, seed=120 + w)
    o, lse, dev = _fwd(inp, c, w)
    dout = upstream_grad(inp["q"], seed=120 + w)
    got = attn.attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dout.cuda(), scale=c.scale,
                        causal=causal, window_left=w)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    ref = oracle.attn_bwd(inp["q"], inp["k"], inp["v"], dout, c.scale, causal, window_left=w)
    compare_grads(got, ref, what=f"bwd window {w} causal {causal} d{d}")
