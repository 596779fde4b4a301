"""The bench's accounting and its committed DRAM-traffic records, no GPU.

The roofline line divides algorithmic work by measured time, so the
accounting must equal its closed forms: 4·B·H·N²·d FLOP for the non-causal
forward, 4·B·H·d·N(N+1)/2 causal, and one read of the filled cache rows plus
q, o and LSE for the decode.  The `traffic` figure comes from
`profiles/dram_traffic.json` only while the record was taken on the current
kernel source; a record of an earlier version says so and is not reported;
every record must add up and stay within what one pass over the operands
allows.
"""
import json
import os

import pytest

import bench
from io_aware_exact_29_b200 import accounting

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_forward_flops_closed_forms():
    B, H, N, d = 4, 16, 4096, 128
    assert accounting.fwd_flops(B, H, N, N, d, False) == 4 * B * H * N * N * d == 549755813888
    assert accounting.fwd_flops(B, H, N, N, d, True) == 4 * B * H * d * N * (N + 1) // 2
    # key lengths: the sum over sequences of their own pair counts
    lens = [1, 300, 4096, 0]
    assert accounting.fwd_flops(4, H, N, N, d, False, lens) == sum(4 * d * H * N * L for L in lens)


def test_forward_bytes_closed_form():
    B, Hq, Hkv, N, d = 4, 16, 16, 4096, 128
    per = B * N * Hq * d * 2
    assert accounting.fwd_bytes(B, Hq, Hkv, N, N, d) == 4 * per + B * Hq * N * 4
    assert accounting.fwd_bytes(B, Hq, Hkv, N, N, d) == 269484032


def test_decode_bytes_closed_form():
    lens, B, Hq, Hkv, Nq, d = [5, 0, 17], 3, 8, 2, 1, 128
    kv = sum(lens) * Hkv * d * 2 * 2
    q = o = B * Nq * Hq * d * 2
    lse = B * Hq * Nq * 4
    assert accounting.decode_bytes(lens, B, Hq, Hkv, Nq, d) == kv + q + o + lse


# record name -> kernel source file
SOURCES = {
    "fwd": "attn_fwd_persist_sm100a.cu",
    "decode": "attn_decode_tc_sm100a.cu",
    "decode_chunk16": "attn_decode_tc_sm100a.cu",
    "decode_paged_bs16": "attn_decode_tc_sm100a.cu",
    "bwd_dkdv": "attn_bwd_sm100a.cu",
    "bwd_dq": "attn_bwd_sm100a.cu",
}


def _records():
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as fh:
        return json.load(fh)


def _current(name):
    src = os.path.join(ROOT, "io_aware_exact_29_b200", "csrc", SOURCES[name])
    return _records()[name]["source_sha256_16"] == bench.source_hash(src)


@pytest.mark.parametrize("name", sorted(SOURCES))
def test_traffic_record_is_current_or_not_reported(name):
    rec = _records()[name]
    if not _current(name):
        # a record of an earlier version of the kernel stays for reference
        # only: it says so, and the bench reports no traffic from it
        assert rec.get("superseded"), (
            f"{name}: the record was taken on another version of {SOURCES[name]}")
        if name in bench.KERNEL_SOURCES:
            assert bench.load_traffic(name) is None
    assert rec["bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    # the capture leaves the clocks alone (the dQ record shares the dK/dV
    # kernel's capture, which counted both kernels' launches)
    cmd = rec["command"]
    if cmd == "(the same capture)":
        cmd = _records()["bwd_dkdv"]["command"]
    assert "--clock-control none" in cmd and "ncu" in cmd


@pytest.mark.parametrize("name", ["fwd", "bwd_dkdv", "bwd_dq"])
def test_headline_kernels_have_current_records(name):
    # the roofline line's traffic (the forward) and the backward's summary
    assert _current(name), f"{name}: the record was taken on another version of {SOURCES[name]}"


def test_bench_reads_the_records_it_reports():
    assert bench.KERNEL_SOURCES["fwd"].endswith(SOURCES["fwd"])
    assert bench.KERNEL_SOURCES["decode"].endswith(SOURCES["decode"])
    for name in ("fwd", "decode"):
        expect = _records()[name]["bytes_per_launch"] if _current(name) else None
        assert bench.load_traffic(name) == expect


@pytest.mark.parametrize("name", ["fwd", "decode_chunk16", "decode_paged_bs16"])
def test_traffic_is_one_pass_over_the_operands(name):
    # at most the algorithmic bytes and a little (split partials, tile
    # rounding); below them only by the part of the output still in L2 when
    # the kernel ends
    rec = _records()[name]
    ratio = rec["bytes_per_launch"] / rec["algorithmic_bytes"]
    assert 0.5 <= ratio <= 1.05, ratio
    if name == "fwd":
        # the reads alone: Q, K and V once (the bench's forward, 201.3 MB)
        assert abs(rec["dram_bytes_read"] / (3 * 4 * 4096 * 16 * 128 * 2) - 1) < 0.01
