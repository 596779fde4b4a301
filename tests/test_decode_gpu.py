"""KV-cache decode kernel (split-K over a packed variable-length cache)
against the fp64 oracle."""
import pytest
import torch

import oracle
from oracle import dense
from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import DECODE_CASES, DecodeCase, kvcache_inputs
from tests.parity import Guarded, check_defined, compare

pytestmark = pytest.mark.gpu


def _run(inp, case, split_keys=0, max_seqlen=None):
    """The decode on guarded, NaN-prefilled outputs and a guarded workspace
    of exactly the size the library asks for, filled with junk bytes."""
    dev = {k: v.cuda() for k, v in inp.items()}
    ml = int(inp["seqlens_k"].max().item()) if max_seqlen is None else max_seqlen
    B, Nq, Hq, d = inp["q"].shape
    go = Guarded((B, Nq, Hq, d), inp["q"].dtype)
    gl = Guarded((B, Hq, Nq), torch.float32)
    need = attn.decode_workspace_bytes(B, Hq, case.Hkv, Nq, d, ml, split_keys)
    gw = Guarded((max(need, 1),), torch.uint8)
    o, lse = attn.attn_fwd_varlen_kvcache(dev["q"], dev["k_cache"], dev["v_cache"],
                                          dev["cu_seqlens_k"], dev["seqlens_k"], ml,
                                          scale=case.scale, causal=case.causal,
                                          split_keys=split_keys, workspace=gw.t, out=go.t,
                                          lse=gl.t)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    for g, n in ((go, "O"), (gl, "LSE"), (gw, "workspace")):
        g.check(n)
    check_defined("decode", o, lse)
    return o, lse


def _check(inp, case, split_keys=0, what=""):
    o, lse = _run(inp, case, split_keys)
    o_ref, lse_ref = oracle.attn_kvcache(inp["q"], inp["k_cache"], inp["v_cache"],
                                         inp["cu_seqlens_k"], inp["seqlens_k"], case.scale,
                                         case.causal)
    return compare(o, lse, o_ref, lse_ref, what=what), o, lse


def test_tiny_decode():
    c = DecodeCase("t", 3, 8, 2, 1, 128, (1, 200), False)
    inp = kvcache_inputs(c, seed=1, seqlens=[1, 64, 200])
    _check(inp, c, what="tiny decode")


@pytest.mark.parametrize("split", [0, 64, 256, 1024, 8192])
def test_tile_and_split_boundaries(split):
    lens = [1, 63, 64, 65, 127, 128, 129, 1023, 1024, 1025, 4097, 0]
    c = DecodeCase("b", len(lens), 16, 2, 1, 128, (0, 4097), False, slack=3)
    inp = kvcache_inputs(c, seed=2, seqlens=lens)
    _check(inp, c, split_keys=split, what=f"split {split}")


def test_split_results_agree():
    c = DecodeCase("s", 4, 8, 1, 1, 128, (1, 3000), False)
    inp = kvcache_inputs(c, seed=3, seqlens=[3000, 1500, 777, 64])
    (_, o1, l1) = _check(inp, c, split_keys=64, what="split 64")
    (_, o2, l2) = _check(inp, c, split_keys=4096, what="one split")
    assert (o1.float() - o2.float()).abs().max().item() <= 1.6e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_unfilled_slots_hold_nan():
    c = DecodeCase("n", 6, 8, 2, 1, 128, (1, 700), False, slack=40)
    clean = kvcache_inputs(c, seed=4)
    dirty = kvcache_inputs(c, seed=4, slack_fill=float("nan"))
    (_, o1, l1) = _check(clean, c, split_keys=256, what="clean")
    (_, o2, l2) = _check(dirty, c, split_keys=256, what="NaN in unfilled slots")
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("nq", [1, 16])
def test_largest_batch_decode(nq):
    # B = 65535 sequences, the largest batch the C ABI takes, 8 query heads
    # on one kv head (the tensor-core path: its plan covers every sequence),
    # short lengths; compared on 64 seeded sequences including the first and
    # the last
    c = DecodeCase("maxb", 65535, 8, 1, nq, 128, (nq, 40), nq > 1, slack=2)
    inp = kvcache_inputs(c, seed=8)
    o, lse = _run(inp, c)
    g = torch.Generator().manual_seed(7)
    sel = sorted(set([0, 1, c.B - 1] + torch.randperm(c.B, generator=g)[:61].tolist()))
    cu, lens = inp["cu_seqlens_k"], inp["seqlens_k"]
    o_ref, lse_ref = dense.attn_kvcache(inp["q"][sel], inp["k_cache"], inp["v_cache"], cu[sel],
                                        lens[sel], c.scale, c.causal)
    compare(o[sel], lse[sel], o_ref, lse_ref, what=f"B=65535 Nq={nq}")


@pytest.mark.parametrize("d,dtype", [(64, "bf16"), (128, "fp16"), (64, "fp16")])
def test_head_dims_and_fp16(d, dtype):
    c = DecodeCase("h", 5, 12, 3, 1, d, (1, 2500), False, dtype=dtype)
    _check(kvcache_inputs(c, seed=5), c, what=f"d{d} {dtype}")


@pytest.mark.parametrize("nq", [2, 5, 16])
def test_chunk_causal_bottom_right(nq):
    lens = [nq, nq + 1, 100, 2000, 3]  # the last one: some tokens see no key
    c = DecodeCase("c", len(lens), 16, 2, nq, 128, (1, 2000), True)
    inp = kvcache_inputs(c, seed=6, seqlens=lens)
    _, o, lse = _check(inp, c, split_keys=256, what=f"chunk {nq}")
    if nq > 3:
        # last sequence has 3 keys: tokens 0..nq-4 see nothing
        assert torch.all(o[4, : nq - 3] == 0)
        assert torch.all(torch.isneginf(lse[4, :, : nq - 3]))


# Shapes whose G query heads per kv head divide 128 and whose Nq * G query
# rows fit 128 run on the tensor-core decode kernel (one 128-row tile, 128-key
# tiles, stream-K ranges); the rest, and split sizes that are not a multiple
# of 128, on the mma.sync one.
TC_LENS = [0, 1, 15, 16, 17, 127, 128, 129, 511, 512, 513, 2047, 2048, 2049, 5000]


@pytest.mark.parametrize("hq,hkv,nq", [(16, 2, 16), (16, 2, 8), (32, 2, 8), (8, 2, 16),
                                       (64, 2, 4), (128, 1, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_tensor_core_chunk_shapes(hq, hkv, nq, causal):
    c = DecodeCase("tc", len(TC_LENS), hq, hkv, nq, 128, (0, 5000), causal, slack=5)
    inp = kvcache_inputs(c, seed=20 + nq, seqlens=TC_LENS)
    _check(inp, c, split_keys=0, what=f"tc {hq}/{hkv} nq {nq} causal {causal}")


@pytest.mark.parametrize("split", [128, 384, 1024, 8192])
def test_tensor_core_split_sizes(split):
    c = DecodeCase("tcs", len(TC_LENS), 16, 2, 16, 128, (0, 5000), True, slack=3)
    inp = kvcache_inputs(c, seed=31, seqlens=TC_LENS)
    _check(inp, c, split_keys=split, what=f"tc split {split}")


@pytest.mark.parametrize("d,dtype", [(64, "bf16"), (64, "fp16"), (128, "fp16")])
def test_tensor_core_head_dims_and_fp16(d, dtype):
    c = DecodeCase("tch", 7, 32, 4, 16, d, (1, 3000), True, dtype=dtype)
    _check(kvcache_inputs(c, seed=32), c, split_keys=512, what=f"tc d{d} {dtype}")


def test_tensor_core_unfilled_slots_hold_nan():
    c = DecodeCase("tcn", 6, 16, 2, 16, 128, (1, 700), True, slack=40)
    clean = kvcache_inputs(c, seed=33)
    dirty = kvcache_inputs(c, seed=33, slack_fill=float("nan"))
    (_, o1, l1) = _check(clean, c, split_keys=256, what="tc clean")
    (_, o2, l2) = _check(dirty, c, split_keys=256, what="tc NaN in unfilled slots")
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_tensor_core_and_mma_sync_paths_agree():
    c = DecodeCase("tca", 5, 16, 2, 16, 128, (1, 4000), True)
    inp = kvcache_inputs(c, seed=34)
    (_, o1, l1) = _check(inp, c, split_keys=64, what="mma.sync path")   # 64: not a 128 multiple
    (_, o2, l2) = _check(inp, c, split_keys=1024, what="tensor-core path")
    assert (o1.float() - o2.float()).abs().max().item() <= 1.6e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


@pytest.mark.parametrize("name", ["llama70b_decode", "llama70b_chunk16"])
def test_llama70b_shape_in_full(name):
    # full-size launch (B=32, Hq=64, Hkv=8, d=128, lengths up to 32768) in the
    # configuration the bench times; every sequence, head and token against
    # the matrix-product oracle
    c = DECODE_CASES[name]
    inp = kvcache_inputs(c, seed=0)
    o, lse = _run(inp, c)
    o_ref, lse_ref = dense.attn_kvcache(inp["q"], inp["k_cache"], inp["v_cache"],
                                        inp["cu_seqlens_k"], inp["seqlens_k"], c.scale, c.causal)
    compare(o, lse, o_ref, lse_ref, what=name)


def test_max_seqlen_too_small_is_reported():
    c = DecodeCase("e", 2, 8, 2, 1, 128, (1, 3000), False)
    inp = kvcache_inputs(c, seed=8, seqlens=[3000, 10])
    attn.get_device_error()
    _run_ok = True
    dev = {k: v.cuda() for k, v in inp.items()}
    attn.attn_fwd_varlen_kvcache(dev["q"], dev["k_cache"], dev["v_cache"], dev["cu_seqlens_k"],
                                 dev["seqlens_k"], 1000, scale=c.scale, split_keys=256)
    torch.cuda.synchronize()
    assert attn.get_device_error() == attn.ERR_DECODE_BASE + 1


# The mma.sync kernel: query heads per kv head that do not divide 128, more
# than 128 query rows per kv head, or split sizes that are not a multiple of
# 128.
@pytest.mark.parametrize("hq,hkv,nq,split", [(24, 2, 1, 0), (24, 2, 11, 0), (12, 2, 5, 256),
                                             (32, 2, 16, 0), (16, 2, 1, 64), (16, 2, 16, 320)])
@pytest.mark.parametrize("causal", [False, True])
def test_mma_sync_path_shapes(hq, hkv, nq, split, causal):
    lens = [0, 1, 63, 64, 65, 129, 1000, 2500]
    c = DecodeCase("ms", len(lens), hq, hkv, nq, 128, (0, 2500), causal, slack=2)
    inp = kvcache_inputs(c, seed=40 + nq, seqlens=lens)
    _check(inp, c, split_keys=split, what=f"mma.sync {hq}/{hkv} nq {nq} split {split}")


def test_tensor_core_max_seqlen_too_small_is_reported():
    c = DecodeCase("tce", 2, 16, 2, 16, 128, (16, 3000), True)
    inp = kvcache_inputs(c, seed=35, seqlens=[3000, 20])
    attn.get_device_error()
    dev = {k: v.cuda() for k, v in inp.items()}
    attn.attn_fwd_varlen_kvcache(dev["q"], dev["k_cache"], dev["v_cache"], dev["cu_seqlens_k"],
                                 dev["seqlens_k"], 1000, scale=c.scale, causal=True,
                                 split_keys=256)
    torch.cuda.synchronize()
    assert attn.get_device_error() == attn.ERR_DECODE_BASE + 1
