"""Forward kernel (tcgen05) against the fp64 oracle, element by element.

Full comparisons on shapes the oracle finishes in seconds (several 128-row
tiles and ragged tails), the tiny / BERT-large / GPT-2 workloads in full, the
long-sequence sweep in full up to N = 4096 (every query row of every head,
against the matrix-product oracle), and at N = 8192 and 16384 on 256 seeded
random rows per head plus rows 0, 1, 127, 128 and N - 1, in the launch
configuration the bench times.  Outputs are written into guarded, NaN-filled
buffers (tests/parity.py: run_fwd).
"""

import numpy as np
import pytest
import torch

from oracle import dense
from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import FWD_CASES, FwdCase, default_scale, fwd_inputs
from tests.parity import check_fwd, compare, compare_selected, run_fwd, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
def test_tiny(causal):
    c = FWD_CASES["tiny_causal" if causal else "tiny"]
    check_fwd(fwd_inputs(c), c.causal, c.scale, what=c.name)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk", [(1, 1, 1, 128, 128), (2, 3, 3, 200, 333),
                                            (1, 8, 2, 257, 257), (2, 4, 1, 77, 300),
                                            (1, 2, 2, 300, 77), (3, 2, 1, 1, 129),
                                            (1, 2, 2, 513, 1), (4, 2, 2, 200, 300),
                                            (1, 2, 1, 256, 256)])
def test_ragged_and_grouped(B, Hq, Hkv, Nq, Nk, d, causal):
    c = FwdCase("r", B, Hq, Hkv, Nq, Nk, d, causal)
    check_fwd(fwd_inputs(c, seed=Nq + Nk + d), causal, c.scale,
              what=f"B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nk{Nk} d{d} causal{causal}")


@pytest.mark.parametrize("name", ["bert_large", "bert_large_varlen", "gpt2", "gpt2_fp16"])
def test_workloads_in_full(name):
    c = FWD_CASES[name]
    check_fwd(fwd_inputs(c), c.causal, c.scale, what=name)


SWEEP = sorted(n for n in FWD_CASES if n.startswith("sweep_"))


@pytest.mark.parametrize("name", [n for n in SWEEP if FWD_CASES[n].Nq <= 4096])
def test_long_sequence_sweep_in_full(name):
    c = FWD_CASES[name]
    inp = fwd_inputs(c)
    o, lse = run_fwd(inp, c.causal, c.scale)
    o_ref, lse_ref = dense.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, c.causal)
    compare(o, lse, o_ref, lse_ref, what=name)


@pytest.mark.parametrize("name", [n for n in SWEEP if FWD_CASES[n].Nq > 4096])
def test_long_sequence_sweep_sampled_rows(name):
    # 256 seeded random rows per (batch, head), drawn per head, plus the
    # tile-edge rows; each row is exact on its own
    c = FWD_CASES[name]
    inp = fwd_inputs(c)
    o, lse = run_fwd(inp, c.causal, c.scale)
    sel = np.zeros((c.B, c.Hq, c.Nq), dtype=bool)
    o_ref = np.full((c.B, c.Nq, c.Hq, c.d), np.nan)
    lse_ref = np.full((c.B, c.Hq, c.Nq), np.nan)
    G = c.Hq // c.Hkv
    for b in range(c.B):
        for h in range(c.Hq):
            g = h // G
            rows = sample_rows(c.Nq, 256, seed=c.Nq + 97 * b + h)
            ob, lb = dense.attn_fwd(inp["q"][b:b + 1, :, h:h + 1], inp["k"][b:b + 1, :, g:g + 1],
                                    inp["v"][b:b + 1, :, g:g + 1], c.scale, c.causal, rows=rows)
            o_ref[b, rows, h] = ob[0, rows, 0]
            lse_ref[b, h, rows] = lb[0, 0, rows]
            sel[b, h, rows] = True
    compare_selected(o, lse, o_ref, lse_ref, sel, what=name)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("kpad", [False, True])
def test_persistent_units_more_than_sms_ragged(d, kpad):
    # the persistent forward (non-causal, at most 4096 keys): 300 units of
    # 256 query rows for 148 CTAs, the last row tile of every head only
    # partly filled (Nq = 300), grouped heads, optionally key lengths
    c = FwdCase("pu", 3, 50, 10, 300, 700, d, False, kpad_range=(1, 700) if kpad else None)
    check_fwd(fwd_inputs(c, seed=d + kpad), False, c.scale,
              what=f"persistent units d{d} kpad {kpad}")


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_d64_units_key_lengths_at_tile_edges(dtype):
    # the d = 64 forward without masks (persistent units of 256 query rows):
    # Nq = 600 leaves a unit with one partly filled Q tile; 9 x 20 heads give
    # 540 units for 148 CTAs; the key lengths sit at and around the half-tile
    # (64) and tile (128) edges, including none at all, and the keys behind
    # each length hold NaN
    c = FwdCase("u64", 9, 20, 4, 600, 333, 64, False, dtype=dtype)
    inp = fwd_inputs(c, seed=21)
    inp["seqlens_k"] = torch.tensor([0, 1, 63, 64, 65, 127, 128, 129, 333], dtype=torch.int32)
    o_ref, lse_ref = dense.attn_fwd(inp["q"], inp["k"], inp["v"], c.scale, False,
                                    seqlens_k=inp["seqlens_k"])
    o, lse = run_fwd(inp, False, c.scale)
    clean = compare(o, lse, o_ref, lse_ref, what=f"d64 units {dtype}")
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))  # no keys
    for b, L in enumerate(inp["seqlens_k"].tolist()):
        inp["k"][b, L:] = float("nan")
        inp["v"][b, L:] = float("nan")
    o2, lse2 = run_fwd(inp, False, c.scale)
    assert torch.equal(o2, o) and torch.equal(lse2, lse)
    assert clean == compare(o2, lse2, o_ref, lse_ref, what=f"d64 units {dtype} NaN padding")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_largest_batch(d, causal):
    # B = 65535, the largest batch the C ABI takes: one work unit per
    # sequence (the persistent kernel strides each CTA over about 443 of
    # them, the causal grid has 65535 CTAs); compared on 64 seeded sequences
    # including the first and the last
    c = FwdCase("maxb", 65535, 1, 1, 3, 5, d, causal)
    inp = fwd_inputs(c, seed=31)
    o, lse = run_fwd(inp, causal, c.scale)
    g = torch.Generator().manual_seed(5)
    sel = sorted(set([0, 1, c.B - 1] + torch.randperm(c.B, generator=g)[:61].tolist()))
    o_ref, lse_ref = dense.attn_fwd(inp["q"][sel], inp["k"][sel], inp["v"][sel], c.scale, causal)
    compare(o[sel], lse[sel], o_ref, lse_ref, what=f"B=65535 d{d} causal {causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_largest_head_count(causal):
    # Hq = 65535 query heads on 5 kv heads (13107 per group), the largest
    # head count the C ABI takes; compared on 64 seeded heads, each against
    # its own kv head
    c = FwdCase("maxh", 1, 65535, 5, 2, 3, 64, causal)
    inp = fwd_inputs(c, seed=32)
    o, lse = run_fwd(inp, causal, c.scale)
    g = torch.Generator().manual_seed(6)
    sel = sorted(set([0, 13106, 13107, c.Hq - 1] + torch.randperm(c.Hq, generator=g)[:60].tolist()))
    kv = [h // (c.Hq // c.Hkv) for h in sel]
    o_ref, lse_ref = dense.attn_fwd(inp["q"][:, :, sel], inp["k"][:, :, kv], inp["v"][:, :, kv],
                                    c.scale, causal)
    compare(o[:, :, sel], lse[:, sel], o_ref, lse_ref, what=f"Hq=65535 causal {causal}")


def test_fp16_head128_causal_gqa():
    c = FwdCase("h", 2, 8, 2, 384, 384, 128, True, dtype="fp16")
    check_fwd(fwd_inputs(c, seed=3), True, c.scale, what="fp16 d128 gqa causal")


def test_key_padding_ignores_nan_behind_the_length():
    c = FwdCase("k", 4, 2, 2, 200, 300, 128, False, kpad_range=(1, 300))
    inp = fwd_inputs(c, seed=11)
    inp["seqlens_k"] = torch.tensor([300, 129, 128, 1], dtype=torch.int32)
    clean = check_fwd(inp, False, c.scale, what="kpad clean")
    for b, L in enumerate(inp["seqlens_k"].tolist()):
        inp["k"][b, L:] = float("nan")
        inp["v"][b, L:] = float("nan")
    dirty = check_fwd(inp, False, c.scale, what="kpad with NaN padding")
    assert dirty == clean
    for causal in (True,):
        check_fwd(inp, causal, c.scale, what="kpad causal with NaN padding")


def test_zero_query_gives_prefix_means():
    # closed form on the GPU: Q = 0 makes every visible key equally likely
    c = FwdCase("z", 1, 2, 2, 300, 300, 64, True)
    inp = fwd_inputs(c, seed=5)
    inp["q"].zero_()
    o, lse = run_fwd(inp, True, c.scale)
    v = inp["v"].double()
    means = torch.cumsum(v[0], 0) / torch.arange(1, 301, dtype=torch.float64)[:, None, None]
    assert (o[0].double().cpu() - means).abs().max().item() <= 1e-2
    expect = torch.log(torch.arange(1, 301, dtype=torch.float64))
    assert (lse[0].double().cpu() - expect).abs().max().item() <= 1e-3
    # causal row 0 is V[0] up to the output rounding
    assert torch.equal(o[0, 0].cpu(), inp["v"][0, 0])


def test_no_keys_and_fully_masked_rows():
    c = FwdCase("m", 1, 2, 2, 256, 100, 64, True)
    inp = fwd_inputs(c, seed=9)
    o, lse = run_fwd(inp, True, c.scale)  # rows i < 156 see no key (bottom-right)
    assert torch.all(o[0, :156] == 0)
    assert torch.all(torch.isneginf(lse[0, :, :156]))
    check_fwd(inp, True, c.scale, what="causal Nq > Nk")
    inp0 = dict(inp)
    inp0["k"] = inp["k"][:, :0].contiguous()
    inp0["v"] = inp["v"][:, :0].contiguous()
    # no keys at all: pass any valid pointer for k/v
    q = inp["q"].cuda()
    kv = torch.empty((1, 0, 2, 64), dtype=torch.bfloat16, device="cuda")
    o, lse = attn.attn_fwd(q, kv, kv, causal=False)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_repeatable_bit_for_bit():
    c = FWD_CASES["gpt2"]
    inp = fwd_inputs(FwdCase("d", 2, 4, 4, 1024, 1024, 128, True), seed=1)
    o1, l1 = run_fwd(inp, True, default_scale(128))
    o2, l2 = run_fwd(inp, True, default_scale(128))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bounded_wait_reports_instead_of_hanging():
    # the loader is told to skip its work: every consumer wait runs out after
    # 100 ms, the kernel records the site, frees tensor memory and returns
    q = torch.randn(1, 128, 1, 64, device="cuda").to(torch.bfloat16)
    o = torch.empty_like(q)
    lse = torch.empty(1, 1, 128, device="cuda")
    attn.get_device_error()  # clear
    attn.selftest_watchdog(q, q, q, o, lse, limit_ms=100)
    code = attn.get_device_error()
    assert code // 16 == 1 and code % 16 != 0, code
    # the context is still usable and the word is clear again
    check_fwd(fwd_inputs(FWD_CASES["tiny"]), False, 0.125, what="after watchdog")
    assert attn.get_device_error() == 0
