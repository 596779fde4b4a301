"""Backward pass (attn_bwd: dQ, dK, dV) against the fp64 oracle's gradients.

The GPU forward provides O and LSE (as in training); the oracle recomputes
everything from the same stored q, k, v, dO bits."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import FWD_CASES, FwdCase, fwd_inputs, upstream_grad
from tests.parity import compare_grads

pytestmark = pytest.mark.gpu


def _run(inp, case, dout):
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o, lse = attn.attn_fwd(dev["q"], dev["k"], dev["v"], scale=case.scale, causal=case.causal,
                           seqlens_k=dev["seqlens_k"])
    dq, dk, dv = attn.attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dout.cuda(),
                               scale=case.scale, causal=case.causal, seqlens_k=dev["seqlens_k"])
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    return dq, dk, dv


def _check(case, seed=0, seqlens=None, what="", nan_pad=False):
    inp = fwd_inputs(case, seed=seed)
    if seqlens is not None:
        inp["seqlens_k"] = torch.tensor(seqlens, dtype=torch.int32)
    if nan_pad:
        for b, L in enumerate(inp["seqlens_k"].tolist()):
            inp["k"][b, L:] = float("nan")
            inp["v"][b, L:] = float("nan")
    dout = upstream_grad(inp["q"], seed=seed)
    got = _run(inp, case, dout)
    ref = oracle.attn_bwd(inp["q"], inp["k"], inp["v"], dout, case.scale, case.causal,
                          seqlens_k=inp["seqlens_k"])
    errs = compare_grads(got, ref, what=what or case.name)
    print(what or case.name, {k: f"{a:.2e}/{b:.2e}" for k, (a, b) in errs.items()})
    return got, ref


@pytest.mark.parametrize("name", ["tiny", "tiny_causal"])
def test_tiny(name):
    _check(FWD_CASES[name])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
def test_tiles_heads_and_groups(d, causal, hq, hkv):
    c = FwdCase("g", 2, hq, hkv, 256, 384, d, causal)
    _check(c, seed=3, what=f"d{d} causal {causal} {hq}/{hkv}")


@pytest.mark.parametrize("nq,nk", [(200, 300), (300, 200), (1, 130), (129, 129), (77, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_sizes(nq, nk, causal):
    c = FwdCase("r", 2, 4, 2, nq, nk, 128, causal)
    _check(c, seed=4, what=f"ragged {nq}x{nk} causal {causal}")


def test_key_padding_with_nan_behind_the_length():
    c = FwdCase("p", 3, 4, 2, 256, 320, 64, False)
    got, _ = _check(c, seed=5, seqlens=[320, 200, 1], nan_pad=True, what="kpad NaN")
    dk, dv = got[1].float().cpu(), got[2].float().cpu()
    assert torch.all(dk[1, 200:] == 0) and torch.all(dv[2, 1:] == 0)


def test_fp16():
    c = FwdCase("h", 2, 4, 4, 256, 256, 64, True, dtype="fp16")
    _check(c, seed=6, what="fp16")


def test_bert_shape_sampled_batches():
    # the BERT-large shape; the oracle checks two of the 16 batch entries
    c = FWD_CASES["bert_large"]
    inp = fwd_inputs(c, seed=0)
    dout = upstream_grad(inp["q"], seed=0)
    got = _run(inp, c, dout)
    for b in (0, 11):
        ref = oracle.attn_bwd(inp["q"][b:b + 1], inp["k"][b:b + 1], inp["v"][b:b + 1],
                              dout[b:b + 1], c.scale, c.causal)
        compare_grads(tuple(t[b:b + 1] for t in got), ref, what=f"bert batch {b}")


def test_long_sequence_one_head():
    # the bench's forward shape (B=4, H=16, N=4096, d=128); heads are
    # independent (Hq = Hkv), so the oracle checks batch 1, head 5 alone
    c = FWD_CASES["sweep_d128_n4096"]
    inp = fwd_inputs(c, seed=0)
    dout = upstream_grad(inp["q"], seed=0)
    got = _run(inp, c, dout)
    sl = (slice(1, 2), slice(None), slice(5, 6))
    ref = oracle.attn_bwd(inp["q"][sl], inp["k"][sl], inp["v"][sl], dout[sl], c.scale,
                          c.causal)
    compare_grads(tuple(t[sl] for t in got), ref, what="N=4096 d=128 b1 h5")


def test_repeatable_bit_for_bit():
    c = FwdCase("det", 2, 8, 2, 384, 384, 128, True)
    inp = fwd_inputs(c, seed=7)
    dout = upstream_grad(inp["q"], seed=7)
    a = _run(inp, c, dout)
    b = _run(inp, c, dout)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
