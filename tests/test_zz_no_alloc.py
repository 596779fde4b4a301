"""The decode entry point that allocates nothing (attn_fwd_varlen_kvcache_noalloc).

It serves callers that cannot allocate device memory themselves (a host
program that owns all device memory without exposing an allocator, or a
decode loop that must not call cudaMalloc because it can synchronise the
device): the library's built-in static scratch replaces the workspace.  These
tests call it through the C ABI and compare it with the ordinary entry point
that takes a caller-allocated workspace, on two different calls in a row, so
that anything a call leaves behind in the shared scratch would show in the
next one.  The file is named to be collected last.
"""
import ctypes

import pytest
import torch

from io_aware_exact_29_b200 import attn
from io_aware_exact_29_b200.workloads import DecodeCase, kvcache_inputs
from tests.parity import LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS

SCRATCH_BYTES = 32 << 20


def _noalloc_fn():
    lib = attn.load_library()
    fn = lib.attn_fwd_varlen_kvcache_noalloc
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [vp, vp, vp, vp, vp, i, i, vp, vp, i, i, i, i, i, f, i, i, i, vp]
    fn.restype = i
    return fn


def test_declared_and_exported():
    assert "attn_fwd_varlen_kvcache_noalloc" in attn.header_functions()
    assert hasattr(attn.load_library(), "attn_fwd_varlen_kvcache_noalloc")
    with open(attn.HEADER_PATH) as fh:
        assert "#define ATTN_NOALLOC_SCRATCH_BYTES (32u << 20)" in fh.read()


def test_rejects_sizes_beyond_the_scratch_before_any_work():
    fn = _noalloc_fn()
    P = 1 << 20
    # 12 query heads per kv head (the mma.sync decode) at the Llama2-70B
    # batch and lengths, automatic 1024-key split: ~68 MB
    need = attn.decode_workspace_bytes(32, 96, 8, 1, 128, 32768)
    assert need > SCRATCH_BYTES
    rc = fn(P, P, P, P, P, 32768, 1 << 20, P, P, 32, 96, 8, 1, 128, 0.088, 0, 0, 0, None)
    assert rc == -4  # ATTN_ERR_WORKSPACE
    # the tensor-core decode with ranges of 128 keys: far beyond the scratch
    assert attn.decode_workspace_bytes(32, 64, 8, 1, 128, 32768, split_keys=128) > SCRATCH_BYTES
    rc = fn(P, P, P, P, P, 32768, 1 << 20, P, P, 32, 64, 8, 1, 128, 0.088, 0, 0, 128, None)
    assert rc == -4
    # invalid sizes are reported as such
    rc = fn(P, P, P, P, P, 100, 100, P, P, 2, 8, 2, 17, 128, 0.088, 0, 0, 0, None)
    assert rc == -1


def test_same_status_codes_as_the_workspace_entry_point():
    # the argument checks run before the size check, so a head dim or dtype
    # the decode does not take is reported as unsupported, as by the
    # workspace entry point, and oversized batches as invalid
    fn = _noalloc_fn()
    lib = attn.load_library()
    P = 1 << 20
    cases = [
        (96, 0, 32),      # d = 96: ATTN_ERR_UNSUPPORTED
        (128, 7, 32),     # unknown dtype: ATTN_ERR_UNSUPPORTED
        (128, 0, 70000),  # B > 65535: ATTN_ERR_INVALID_ARG
    ]
    for d, dtype, B in cases:
        a = fn(P, P, P, P, P, 4096, 1 << 20, P, P, B, 64, 8, 1, d, 0.088, 0, dtype, 0, None)
        b = lib.attn_fwd_varlen_kvcache(P, P, P, P, P, 4096, 1 << 20, P, P, B, 64, 8, 1, d,
                                        0.088, 0, dtype, P, 1 << 30, 0, None)
        assert a == b, (d, dtype, B, a, b)
    assert fn(P, P, P, P, P, 4096, 1 << 20, P, P, 32, 64, 8, 1, 96, 0.088, 0, 0, 0, None) == -2
    assert fn(P, P, P, P, P, 4096, 1 << 20, P, P, 70000, 64, 8, 1, 128, 0.088, 0, 0, 0,
              None) == -1


def _call_noalloc(fn, dev, case, max_len, split):
    o = torch.empty_like(dev["q"])
    lse = torch.empty((case.B, case.Hq, case.Nq), dtype=torch.float32, device="cuda")
    dtype_code = 0 if dev["q"].dtype == torch.bfloat16 else 1
    rc = fn(dev["q"].data_ptr(), dev["k_cache"].data_ptr(), dev["v_cache"].data_ptr(),
            dev["cu_seqlens_k"].data_ptr(), dev["seqlens_k"].data_ptr(), max_len,
            dev["k_cache"].shape[0], o.data_ptr(), lse.data_ptr(), case.B, case.Hq, case.Hkv,
            case.Nq, case.d, case.scale, int(case.causal), dtype_code, split,
            torch.cuda.current_stream().cuda_stream)
    assert rc == 0, rc
    return o, lse


def _close(a, b, la, lb):
    err = (a.float() - b.float()).abs()
    assert err.max().item() <= O_MAX_ABS and err.mean().item() <= O_MEAN_ABS
    both = torch.isneginf(la) & torch.isneginf(lb)
    lerr = torch.where(both, torch.zeros_like(la), (la - lb).abs())
    assert lerr.max().item() <= LSE_MAX_ABS


@pytest.mark.gpu
def test_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    fn = _noalloc_fn()
    cases = [
        (DecodeCase("a", 16, 32, 4, 1, 128, (1, 6000), False), 0, 11),
        (DecodeCase("b", 6, 16, 2, 4, 128, (4, 3000), True), 256, 12),
        (DecodeCase("c", 5, 24, 2, 1, 128, (1, 3000), False), 0, 13),  # mma.sync decode
    ]
    for case, split, seed in cases:
        inp = kvcache_inputs(case, seed=seed)
        dev = {k: v.cuda() for k, v in inp.items()}
        max_len = int(inp["seqlens_k"].max())
        assert attn.decode_workspace_bytes(case.B, case.Hq, case.Hkv, case.Nq, case.d, max_len,
                                           split) <= SCRATCH_BYTES
        o_ref, lse_ref = attn.attn_fwd_varlen_kvcache(
            dev["q"], dev["k_cache"], dev["v_cache"], dev["cu_seqlens_k"], dev["seqlens_k"],
            max_len, scale=case.scale, causal=case.causal, split_keys=split)
        o, lse = _call_noalloc(fn, dev, case, max_len, split)
        torch.cuda.synchronize()
        assert attn.get_device_error() == 0
        _close(o, o_ref, lse, lse_ref)
