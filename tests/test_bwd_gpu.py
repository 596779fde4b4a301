"""Backward pass (attn_bwd: dQ, dK, dV) against the fp64 oracle's gradients.

The GPU forward provides O and LSE (as in training); the oracle recomputes
everything from the same stored q, k, v, dO bits.  Gradients and the
workspace are guarded and NaN/junk-filled (tests/parity.py); the BERT-large
shape is compared in full and the bench's shape (B=4, H=16, N=4096, d=128)
on 16 of its 64 (batch, head) pairs, against the matrix-product oracle."""
import pytest
import torch

import oracle
from oracle import dense
from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import FWD_CASES, FwdCase, fwd_inputs, upstream_grad
from tests.parity import Guarded, check_defined, compare_grads

pytestmark = pytest.mark.gpu


def _run(inp, case, dout):
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o, lse = attn.attn_fwd(dev["q"], dev["k"], dev["v"], scale=case.scale, causal=case.causal,
                           seqlens_k=dev["seqlens_k"])
    B, Nq, Hq, _ = inp["q"].shape
    gq = Guarded(tuple(inp["q"].shape), inp["q"].dtype)
    gk = Guarded(tuple(inp["k"].shape), inp["k"].dtype)
    gv = Guarded(tuple(inp["v"].shape), inp["v"].dtype)
    gw = Guarded((attn.bwd_workspace_bytes(B, Hq, Nq),), torch.uint8)
    dq, dk, dv = attn.attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dout.cuda(),
                               scale=case.scale, causal=case.causal, seqlens_k=dev["seqlens_k"],
                               workspace=gw.t, dq=gq.t, dk=gk.t, dv=gv.t)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    for g, n in ((gq, "dq"), (gk, "dk"), (gv, "dv"), (gw, "workspace")):
        g.check(n)
    check_defined("backward", dq, dk, dv)
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


@pytest.mark.parametrize("name", ["bert_large", "bert_large_varlen", "gpt2"])
def test_workload_shapes_in_full(name):
    # every batch entry and head of the BERT-large (and its key-padded
    # variant) and GPT-2 shapes against the matrix-product oracle
    c = FWD_CASES[name]
    inp = fwd_inputs(c, seed=0)
    dout = upstream_grad(inp["q"], seed=0)
    got = _run(inp, c, dout)
    ref = dense.attn_bwd(inp["q"], inp["k"], inp["v"], dout, c.scale, c.causal,
                         seqlens_k=inp["seqlens_k"])
    errs = compare_grads(got, ref, what=name)
    print(name, {k: f"{a:.2e}/{b:.2e}" for k, (a, b) in errs.items()})


@pytest.mark.parametrize("causal", [False, True])
def test_long_sequence_sixteen_heads(causal):
    # the bench's forward shape (B=4, H=16, N=4096, d=128): heads are
    # independent (Hq = Hkv), so the oracle checks 16 of the 64 (batch, head)
    # pairs in full -- every batch entry, four heads each
    c = FWD_CASES["sweep_d128_n4096_causal" if causal else "sweep_d128_n4096"]
    inp = fwd_inputs(c, seed=0)
    dout = upstream_grad(inp["q"], seed=0)
    got = _run(inp, c, dout)
    heads = (0, 5, 10, 15)
    ref = dense.attn_bwd(inp["q"], inp["k"], inp["v"], dout, c.scale, c.causal,
                         heads=[(b, h) for b in range(c.B) for h in heads])
    sl = (slice(None), slice(None), list(heads))
    errs = compare_grads(tuple(t[sl] for t in got), tuple(r[sl] for r in ref),
                         what=f"N=4096 d=128 causal {causal}")
    print(f"N=4096 causal {causal}", {k: f"{a:.2e}/{b:.2e}" for k, (a, b) in errs.items()})


def test_repeatable_bit_for_bit():
    c = FwdCase("det", 2, 8, 2, 384, 384, 128, True)
    inp = fwd_inputs(c, seed=7)
    dout = upstream_grad(inp["q"], seed=7)
    a = _run(inp, c, dout)
    b = _run(inp, c, dout)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
