"""Decode against a paged KV cache (attn_fwd_paged_kvcache) against the fp64
oracle: block sizes below, at and above the 128-key tile, shuffled physical
blocks with NaN in every unused row, and the fused append of the new tokens'
K/V.  Outputs and the workspace are guarded and NaN/junk-filled (tests/parity.py)."""
import pytest
import torch

import oracle
from oracle import dense
from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import DecodeCase, kvcache_inputs, paged_from_packed
from tests.parity import Guarded, check_defined, compare

pytestmark = pytest.mark.gpu

LENS = [0, 1, 16, 127, 128, 129, 1000, 2049, 5000]


def _run(inp, pg, c, with_new=False, split_keys=0):
    dev = {k: v.cuda() for k, v in pg.items()}
    ml = int(inp["seqlens_k"].max().item())
    B, Nq, Hq, d = inp["q"].shape
    go = Guarded((B, Nq, Hq, d), inp["q"].dtype)
    gl = Guarded((B, Hq, Nq), torch.float32)
    need = attn.decode_workspace_bytes(B, Hq, c.Hkv, Nq, d, ml, split_keys)
    gw = Guarded((max(need, 1),), torch.uint8)
    o, lse = attn.attn_fwd_paged_kvcache(
        inp["q"].cuda(), dev["k_cache"], dev["v_cache"], dev["block_table"], dev["seqlens_k"], ml,
        scale=c.scale, causal=c.causal, k_new=dev.get("k_new") if with_new else None,
        v_new=dev.get("v_new") if with_new else None, split_keys=split_keys, workspace=gw.t,
        out=go.t, lse=gl.t)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    for g, n in ((go, "O"), (gl, "LSE"), (gw, "workspace")):
        g.check(n)
    check_defined("paged decode", o, lse)
    return o, lse, dev


def _ref(inp, c):
    return oracle.attn_kvcache(inp["q"], inp["k_cache"], inp["v_cache"], inp["cu_seqlens_k"],
                               inp["seqlens_k"], c.scale, c.causal)


@pytest.mark.parametrize("block_size", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("nq,causal", [(1, False), (16, True)])
def test_block_sizes(block_size, nq, causal):
    lens = [max(L, nq) if causal else L for L in LENS]
    c = DecodeCase("pg", len(lens), 16, 2, nq, 128, (0, 5000), causal)
    inp = kvcache_inputs(c, seed=50 + block_size, seqlens=lens)
    pg = paged_from_packed(inp, block_size, seed=block_size)
    o, lse, _ = _run(inp, pg, c)
    o_ref, l_ref = _ref(inp, c)
    compare(o, lse, o_ref, l_ref, what=f"paged bs {block_size} nq {nq}")


@pytest.mark.parametrize("split", [128, 1024])
def test_split_sizes(split):
    c = DecodeCase("pgs", len(LENS), 16, 2, 16, 128, (0, 5000), True)
    lens = [max(L, 16) for L in LENS]
    inp = kvcache_inputs(c, seed=60, seqlens=lens)
    pg = paged_from_packed(inp, 32, seed=61)
    o, lse, _ = _run(inp, pg, c, split_keys=split)
    o_ref, l_ref = _ref(inp, c)
    compare(o, lse, o_ref, l_ref, what=f"paged split {split}")


@pytest.mark.parametrize("block_size,nq", [(16, 1), (64, 16), (256, 4)])
def test_fused_append(block_size, nq):
    lens = [nq, 200, 1000, 3000]
    c = DecodeCase("pga", len(lens), 16, 2, nq, 128, (nq, 3000), nq > 1)
    inp = kvcache_inputs(c, seed=70, seqlens=lens)
    full = paged_from_packed(inp, block_size, seed=71)
    holes = paged_from_packed(inp, block_size, seed=71, new_tokens=nq)
    o, lse, dev = _run(inp, holes, c, with_new=True)
    o_ref, l_ref = _ref(inp, c)
    compare(o, lse, o_ref, l_ref, what=f"append bs {block_size} nq {nq}")
    # the appended rows are in the cache, every other row untouched
    for name in ("k_cache", "v_cache"):
        assert torch.equal(dev[name].cpu().view(torch.int16), full[name].view(torch.int16))


def test_d64_fp16():
    c = DecodeCase("pgh", 5, 32, 4, 8, 64, (8, 3000), True, dtype="fp16")
    inp = kvcache_inputs(c, seed=80)
    pg = paged_from_packed(inp, 16, seed=81)
    o, lse, _ = _run(inp, pg, c)
    o_ref, l_ref = _ref(inp, c)
    compare(o, lse, o_ref, l_ref, what="paged d64 fp16")


def test_unsupported_group_size():
    c = DecodeCase("pgu", 2, 24, 2, 1, 128, (1, 300), False)
    inp = kvcache_inputs(c, seed=90)
    pg = paged_from_packed(inp, 16, seed=90)
    with pytest.raises(attn.AttnError) as e:
        _run(inp, pg, c)
    assert e.value.status == -2


def test_bad_table_entry_is_reported():
    c = DecodeCase("pgb", 2, 16, 2, 1, 128, (1, 500), False)
    inp = kvcache_inputs(c, seed=91, seqlens=[500, 300])
    pg = paged_from_packed(inp, 64, seed=91)
    pg["block_table"][1, 2] = pg["k_cache"].shape[0] + 5  # past the last block
    dev = {k: v.cuda() for k, v in pg.items()}
    attn.get_device_error()
    attn.attn_fwd_paged_kvcache(inp["q"].cuda(), dev["k_cache"], dev["v_cache"],
                                dev["block_table"], dev["seqlens_k"], 500, scale=c.scale)
    torch.cuda.synchronize()
    assert attn.get_device_error() == attn.ERR_DECODE_BASE + 8


def test_llama70b_shape_paged_bs16_in_full():
    # the bench's paged decode at full size (B=32, Hq=64, Hkv=8, d=128, lengths
    # up to 32768, 16-row blocks, shuffled table, NaN in every unused row);
    # every sequence against the matrix-product oracle on the paged layout
    from io_aware_exact_29_b200.workloads import DECODE_CASES
    c = DECODE_CASES["llama70b_decode"]
    inp = kvcache_inputs(c, seed=0)
    pg = paged_from_packed(inp, 16, seed=0)
    o, lse, _ = _run(inp, pg, c)
    o_ref, lse_ref = dense.attn_paged(inp["q"], pg["k_cache"], pg["v_cache"], pg["block_table"],
                                      pg["seqlens_k"], c.scale, c.causal)
    compare(o, lse, o_ref, lse_ref, what="paged bs16 Llama2-70B shape")
