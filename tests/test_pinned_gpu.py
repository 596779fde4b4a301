"""The pipelined pinned-host forward (attn.PinnedForward) against the device
call and the fp64 oracle.

Each piece of the batch is one attn_fwd launch on a sub-batch, and a work
unit's arithmetic does not depend on which CTA runs it, so the host results
equal the device call's bit for bit.  Two back-to-back calls on different
inputs check that a call's copies in wait for the previous call's forward of
the same piece, and its forward for the previous call's copies out.
"""
import pytest
import torch

from oracle import dense
from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import FwdCase, fwd_inputs
from tests.parity import compare

pytestmark = pytest.mark.gpu


def _pinned(t):
    return t.contiguous().pin_memory()


@pytest.mark.parametrize("pieces,causal,d", [(3, False, 64), (4, True, 128), (1, False, 128),
                                             (8, False, 64)])
def test_pinned_forward_equals_device_call(pieces, causal, d):
    c = FwdCase("pin", 5, 4, 2, 300, 333, d, causal)
    pf = attn.PinnedForward(c.B, c.Nq, c.Hq, c.Nk, c.Hkv, c.d, pieces=pieces)
    outs = []
    for seed in (1, 2):
        inp = fwd_inputs(c, seed=seed)
        h = {n: _pinned(inp[n]) for n in ("q", "k", "v")}
        ho = torch.full(tuple(inp["q"].shape), float("nan"), dtype=inp["q"].dtype).pin_memory()
        hl = torch.full((c.B, c.Hq, c.Nq), float("nan"), dtype=torch.float32).pin_memory()
        pf(h["q"], h["k"], h["v"], ho, hl, scale=c.scale, causal=causal)
        outs.append((inp, ho, hl))
    pf.join()
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    for inp, ho, hl in outs:
        o, lse = attn.attn_fwd(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), scale=c.scale,
                               causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(ho, o.cpu()) and torch.equal(hl, lse.cpu())
        o_ref, lse_ref = dense.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, causal)
        compare(ho, hl, o_ref, lse_ref, what=f"pinned forward pieces {pieces}")


def test_pinned_forward_rejects_device_or_pageable_tensors():
    c = FwdCase("pin", 2, 2, 2, 64, 64, 64, False)
    pf = attn.PinnedForward(c.B, c.Nq, c.Hq, c.Nk, c.Hkv, c.d, pieces=2)
    inp = fwd_inputs(c, seed=3)
    ho = torch.empty(tuple(inp["q"].shape), dtype=inp["q"].dtype).pin_memory()
    hl = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32).pin_memory()
    with pytest.raises(ValueError):
        pf(inp["q"], inp["k"], inp["v"], ho, hl)  # pageable inputs
    with pytest.raises(ValueError):
        pf(inp["q"].cuda(), _pinned(inp["k"]), _pinned(inp["v"]), ho, hl)
    with pytest.raises(ValueError):
        pf(_pinned(inp["q"][:1]), _pinned(inp["k"]), _pinned(inp["v"]), ho, hl)
