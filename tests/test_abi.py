"""The C-ABI library loads without a GPU and exports what include/attn.h
declares; host-side validation rejects bad arguments before any CUDA call."""
import os
import subprocess

import pytest

from io_aware_exact_29_b200 import attn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_header_declares_the_boundary():
    names = attn.header_functions()
    for n in ("attn_fwd", "attn_fwd_kpad", "attn_fwd_varlen_kvcache",
              "attn_decode_workspace_bytes", "attn_status_string", "attn_get_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = attn.load_library()
    for n in attn.header_functions():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", attn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(attn.header_functions()) <= exported


def test_library_is_built_for_sm100a():
    # the build passes exactly one gencode, for sm_100a
    from io_aware_exact_29_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings():
    lib = attn.load_library()
    assert lib.attn_status_string(0) == b"ok"
    assert b"invalid" in lib.attn_status_string(-1)
    assert lib.attn_status_string(-5)
    assert attn.version().startswith("attn-b200")


P = 1 << 20  # a fake, 16-byte aligned address: validation fails before it is used


@pytest.mark.parametrize("args,expect", [
    # (q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype)
    ((0, P, P, P, P, 1, 1, 1, 1, 1, 64, 0.125, 0, 0), -1),   # null q
    ((P + 2, P, P, P, P, 1, 1, 1, 1, 1, 64, 0.125, 0, 0), -1),  # misaligned q
    ((P, P, P, P, P, 1, 3, 2, 1, 1, 64, 0.125, 0, 0), -1),   # Hq % Hkv != 0
    ((P, P, P, P, P, 0, 1, 1, 1, 1, 64, 0.125, 0, 0), -1),   # B = 0
    ((P, P, P, P, P, 1, 1, 1, 0, 1, 64, 0.125, 0, 0), -1),   # Nq = 0
    ((P, P, P, P, P, 1, 1, 1, 1, -1, 64, 0.125, 0, 0), -1),  # Nk < 0
    ((P, P, P, P, P, 1, 1, 1, 1, 1, 96, 0.125, 0, 0), -2),   # d = 96
    ((P, P, P, P, P, 1, 1, 1, 1, 1, 64, 0.125, 0, 7), -2),   # dtype
    ((P, P, P, P, P, 1, 1, 1, 1, 1, 64, -1.0, 0, 0), -1),    # scale <= 0
    ((P, P, P, P, P, 1, 1, 1, 1, 1, 64, float("nan"), 0, 0), -1),
])
def test_fwd_rejects_bad_arguments(args, expect):
    lib = attn.load_library()
    assert lib.attn_fwd(*args, None) == expect


@pytest.mark.parametrize("mask,sb,sh,srow", [
    (0, 0, 0, 8),       # no mask
    (P, -1, 0, 8),      # negative batch stride
    (P, 0, -16, 8),     # negative head stride
    (P, 0, 0, 7),       # a row of the mask shorter than ceil(1000 / 128) = 8 key blocks
])
def test_blocksparse_rejects_bad_masks(mask, sb, sh, srow):
    lib = attn.load_library()
    rc = lib.attn_fwd_blocksparse(P, P, P, P, P, 1, 2, 1, 300, 1000, 128, 0.09, 0, -1, 0, None,
                                  mask or None, sb, sh, srow, None)
    assert rc == -1


@pytest.mark.parametrize("sb,sh,srow", [(-1, 0, 8), (0, -16, 8), (0, 0, 7)])
def test_bwd_blocksparse_rejects_bad_masks(sb, sh, srow):
    lib = attn.load_library()
    ws = attn.bwd_workspace_bytes(1, 2, 300)
    rc = lib.attn_bwd_blocksparse(P, P, P, P, P, P, P, P, P, 1, 2, 1, 300, 1000, 128, 0.09, 0,
                                  -1, 0, None, P, sb, sh, srow, P, ws, None)
    assert rc == -1


def test_decode_rejects_bad_arguments():
    lib = attn.load_library()
    base = dict(q=P, k=P, v=P, cu=P, sl=P, maxl=100, slots=100, o=P, lse=P, B=2, Hq=8, Hkv=2,
                Nq=1, d=128, scale=0.088, causal=0, dtype=0, ws=P, wsb=1 << 30, split=0)

    def call(**kw):
        a = dict(base, **kw)
        return lib.attn_fwd_varlen_kvcache(a["q"], a["k"], a["v"], a["cu"], a["sl"], a["maxl"],
                                           a["slots"], a["o"], a["lse"], a["B"], a["Hq"],
                                           a["Hkv"], a["Nq"], a["d"], a["scale"], a["causal"],
                                           a["dtype"], a["ws"], a["wsb"], a["split"], None)

    assert call(Nq=17) == -1         # at most 16 new tokens
    assert call(Nq=0) == -1
    assert call(Hq=6, Hkv=4) == -1
    assert call(split=100) == -1     # split not a multiple of 64
    assert call(slots=0) == -1
    assert call(cu=P + 2) == -1
    assert call(d=80) == -2
    # host-only size query (no GPU needed)
    need = attn.decode_workspace_bytes(2, 8, 2, 1, 128, 100)
    assert need > 0
    assert attn.decode_workspace_bytes(2, 8, 2, 17, 128, 100) == 0
    assert attn.decode_workspace_bytes(2, 8, 2, 1, 128, 100, split_keys=96) == 0


def test_decode_workspace_accounting():
    # mma.sync decode (12 query heads per kv head do not divide 128): B=32,
    # Hkv=8, one row group (12 query rows), auto split of 1024 keys over
    # 32768 keys: 32 splits x 16 padded rows x (128 + 1) floats + counters
    n = attn.decode_workspace_bytes(32, 96, 8, 1, 128, 32768)
    units, splits = 32 * 8, 32
    expect = units * splits * 16 * 128 * 4 + units * splits * 16 * 4 + units * 4
    assert expect <= n <= expect + 3 * 256


def test_decode_workspace_accounting_tensor_core_layout():
    # 16 new tokens x 8 query heads per kv head = 128 rows: the tensor-core
    # decode.  Automatic mode cuts the work into at most 192 ranges, each
    # owning two 128-row partial slots of (128 + 1) floats; plus the weight
    # prefix over sequences (int64), each range's first and last unit and the
    # plan header.  Independent of the lengths.
    n = attn.decode_workspace_bytes(32, 64, 8, 16, 128, 32768)
    ranges = 192
    expect = (2 * ranges * 128 * 128 * 4 + 2 * ranges * 128 * 4 + 33 * 8 + ranges * 8 + 24)
    assert expect <= n <= expect + 5 * 256
    assert n < 32 << 20  # fits the no-alloc entry point's scratch
    # small problems need fewer ranges (at least 8 tiles of weight each)
    n_small = attn.decode_workspace_bytes(2, 16, 2, 16, 128, 1000)
    r_small = (4 * (8 + 2) + 7) // 8
    assert n_small >= 2 * r_small * 128 * 128 * 4
    assert n_small < 2 * (r_small + 1) * 128 * 128 * 4
    # with split_keys, ranges of split_keys / 128 tiles of weight
    n_split = attn.decode_workspace_bytes(2, 16, 2, 16, 128, 1000, split_keys=256)
    r_split = (4 * (8 + 2) + 1) // 2
    assert 2 * r_split * 128 * 128 * 4 <= n_split < 2 * (r_split + 1) * 128 * 128 * 4
    # a split that is not a multiple of 128 keeps the mma.sync layout
    n64 = attn.decode_workspace_bytes(32, 64, 8, 16, 128, 32768, split_keys=64)
    expect64 = 32 * 8 * 8 * 512 * 16 * 128 * 4 + 32 * 8 * 8 * 512 * 16 * 4 + 32 * 8 * 8 * 4
    assert expect64 <= n64 <= expect64 + 3 * 256


def test_python_binding_fails_loudly_without_cuda_tensors():
    import torch
    q = torch.zeros(1, 128, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, q, q)


def test_paged_decode_argument_checks():
    lib = attn.load_library()
    P = 1 << 20
    f = lib.attn_fwd_paged_kvcache
    base = dict(q=P, kc=P, vc=P, bt=P, mb=4, bs=16, nb=8, sl=P, ml=64, kn=None, vn=None, o=P,
                lse=P, B=2, Hq=16, Hkv=2, Nq=1, d=128, scale=0.088, causal=0, dtype=0, ws=P,
                wsb=1 << 30, split=0, st=None)

    def call(**kw):
        a = dict(base, **kw)
        return f(a["q"], a["kc"], a["vc"], a["bt"], a["mb"], a["bs"], a["nb"], a["sl"], a["ml"],
                 a["kn"], a["vn"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["d"],
                 a["scale"], a["causal"], a["dtype"], a["ws"], a["wsb"], a["split"], a["st"])
    assert call(bs=24) == -1          # not a power of two
    assert call(bs=8) == -1           # below 16
    assert call(ml=65) == -1          # max_blocks * block_size < max_seqlen_k
    assert call(kn=P) == -1           # k_new without v_new
    assert call(Nq=17) == -1
    assert call(d=80) == -2
    assert call(Hq=24) == -2          # 12 heads per kv head: not the tensor-core decode
