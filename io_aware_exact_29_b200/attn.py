"""ctypes binding of libattn.so (argument marshalling only).

Every step of the attention path runs in the CUDA library; this module only
allocates outputs with PyTorch, passes ``data_ptr()`` values and the current
stream, and turns status codes into exceptions.  There is no CPU fallback: if
the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "attn.h")

ATTN_BF16, ATTN_FP16 = 0, 1
STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported", -3: "CUDA error",
          -4: "workspace", -5: "timeout"}
ERR_FWD_BASE, ERR_DECODE_BASE, ERR_BWD_BASE = 16, 32, 48

_lock = threading.Lock()
_lib = None


class AttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status})")
        self.status = status


def load_library():
    """Load libattn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m io_aware_exact_29_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp]
            lib.attn_fwd.restype = i
            lib.attn_fwd_kpad.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp, vp]
            lib.attn_fwd_kpad.restype = i
            lib.attn_fwd_window.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp,
                                            vp]
            lib.attn_fwd_window.restype = i
            ll = ctypes.c_longlong
            lib.attn_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i,
                                                 vp, vp, ll, ll, i, vp]
            lib.attn_fwd_blocksparse.restype = i
            lib.attn_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i,
                                                 i, i, f, i, i, i, vp, vp, ll, ll, i, vp, sz, vp]
            lib.attn_bwd_blocksparse.restype = i
            lib.attn_bwd_window.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i,
                                            f, i, i, i, vp, vp, sz, vp]
            lib.attn_bwd_window.restype = i
            lib.attn_decode_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
            lib.attn_decode_workspace_bytes.restype = sz
            lib.attn_fwd_varlen_kvcache.argtypes = [vp, vp, vp, vp, vp, i, i, vp, vp, i, i, i, i,
                                                    i, f, i, i, vp, sz, i, vp]
            lib.attn_fwd_varlen_kvcache.restype = i
            lib.attn_fwd_paged_kvcache.argtypes = [vp, vp, vp, vp, i, i, i, vp, i, vp, vp, vp,
                                                   vp, i, i, i, i, i, f, i, i, vp, sz, i, vp]
            lib.attn_fwd_paged_kvcache.restype = i
            lib.attn_bwd_workspace_bytes.argtypes = [i, i, i]
            lib.attn_bwd_workspace_bytes.restype = sz
            lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i,
                                     i, vp, vp, sz, vp]
            lib.attn_bwd.restype = i
            lib.attn_status_string.argtypes = [i]
            lib.attn_status_string.restype = ctypes.c_char_p
            lib.attn_get_device_error.argtypes = [ctypes.POINTER(i), vp]
            lib.attn_get_device_error.restype = i
            lib.attn_selftest_watchdog.argtypes = [vp, vp, vp, vp, vp, i, vp]
            lib.attn_selftest_watchdog.restype = i
            lib.attn_version.restype = ctypes.c_char_p
            lib.attn_hbm_read_probe.argtypes = [vp, sz, vp, i, vp]
            lib.attn_hbm_read_probe.restype = i
            ip = ctypes.POINTER(i)
            lib.attn_schedule_band_unit.argtypes = [ctypes.c_uint, i, i, i, ip, ip]
            lib.attn_schedule_band_unit.restype = i
            lib.attn_schedule_sparse_steps.argtypes = [vp, vp, i, i, i, i, i, ip]
            lib.attn_schedule_sparse_steps.restype = i
            _lib = lib
    return _lib


def header_functions():
    """Names of the functions that include/attn.h declares."""
    with open(HEADER_PATH) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"^ATTN_API\s+[A-Za-z_][\w \*]*?\b(attn_\w+)\s*\(", text, re.M)))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    if t.dtype == torch.float16:
        return ATTN_FP16
    raise TypeError(f"unsupported dtype {t.dtype}: bf16 or fp16")


def _stream_ptr(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _check(fn: str, status: int):
    if status != 0:
        raise AttnError(fn, status)


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


MASK_BLOCK = 128  # queries and keys per block-mask entry


def block_mask_args(block_mask, B, Hq, Nq, Nk):
    """(pointer, stride_b, stride_h, stride_row) of a block mask tensor.

    block_mask: uint8 or bool CUDA tensor [1|B, 1|Hq, nqb, nkb] with
    nqb >= ceil(Nq / 128), nkb >= ceil(Nk / 128) and unit stride along key
    blocks; a size-1 batch or head dimension is shared (stride 0).
    """
    if not block_mask.is_cuda:  # strided views are fine: only the key-block stride must be 1
        raise ValueError("block_mask must be a CUDA tensor")
    if block_mask.dtype not in (torch.uint8, torch.bool):
        raise TypeError("block_mask must be uint8 or bool")
    if block_mask.dim() != 4 or block_mask.shape[0] not in (1, B) or \
            block_mask.shape[1] not in (1, Hq):
        raise ValueError(f"block_mask shape {tuple(block_mask.shape)} is not [1|B, 1|Hq, nqb, nkb]")
    nqb, nkb = -(-Nq // MASK_BLOCK), -(-Nk // MASK_BLOCK)
    if block_mask.shape[2] < nqb or block_mask.shape[3] < nkb or block_mask.stride(3) != 1:
        raise ValueError("block_mask does not cover the (query, key) blocks")
    sb = 0 if block_mask.shape[0] == 1 else block_mask.stride(0)
    sh = 0 if block_mask.shape[1] == 1 else block_mask.stride(1)
    return block_mask.data_ptr(), sb, sh, block_mask.stride(2)


def attn_fwd(q, k, v, scale=None, causal=False, seqlens_k=None, out=None, lse=None,
             stream=None, window_left=-1, block_mask=None):
    """Exact attention forward.

    q [B, Nq, Hq, d], k/v [B, Nk, Hkv, d] (bf16/fp16, CUDA, contiguous);
    seqlens_k: optional int32 [B] key lengths; window_left: -1 or the
    sliding window; block_mask: optional [1|B, 1|Hq, ceil(Nq/128),
    ceil(Nk/128)] uint8/bool, 0 removes a 128 x 128 block (see
    block_mask_args).  Returns (o, lse) with o [B, Nq, Hq, d] and
    lse [B, Hq, Nq] float32.
    """
    lib = load_library()
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    if scale is None:
        scale = float(d) ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    st = _stream_ptr(stream)
    if block_mask is not None:
        sl = 0
        if seqlens_k is not None:
            _dev(seqlens_k, "seqlens_k")
            if seqlens_k.dtype != torch.int32:
                raise TypeError("seqlens_k must be int32")
            sl = seqlens_k.data_ptr()
        mp, sb, sh, sr = block_mask_args(block_mask, B, Hq, Nq, Nk)
        rc = lib.attn_fwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale),
                                      int(bool(causal)), int(window_left), _dtype_code(q),
                                      sl or None, mp, sb, sh, sr, st)
        _check("attn_fwd_blocksparse", rc)
    elif window_left >= 0:
        sl = 0
        if seqlens_k is not None:
            _dev(seqlens_k, "seqlens_k")
            if seqlens_k.dtype != torch.int32:
                raise TypeError("seqlens_k must be int32")
            sl = seqlens_k.data_ptr()
        rc = lib.attn_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale),
                                 int(bool(causal)), int(window_left), _dtype_code(q), sl or None,
                                 st)
        _check("attn_fwd_window", rc)
    elif seqlens_k is None:
        rc = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                          lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)),
                          _dtype_code(q), st)
        _check("attn_fwd", rc)
    else:
        _dev(seqlens_k, "seqlens_k")
        if seqlens_k.dtype != torch.int32:
            raise TypeError("seqlens_k must be int32")
        rc = lib.attn_fwd_kpad(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale),
                               int(bool(causal)), _dtype_code(q), seqlens_k.data_ptr(), st)
        _check("attn_fwd_kpad", rc)
    return out, lse


class PinnedForward:
    """attn_fwd on pinned host tensors, pipelined over pieces of the batch.

    Every call copies all of q, k, v host -> device and all of o, lse
    device -> host.  The batch is cut into `pieces` contiguous pieces so that
    the copy of piece i + 1 in, the forward of piece i (one attn_fwd launch on
    the sub-batch) and the copy of piece i - 1 out run at the same time on
    three CUDA streams; the copies in and out also overlap across calls.  The
    device buffers, streams and events live as long as the object: a piece's
    input buffers are refilled only after the previous call's forward of that
    piece has read them, and its output buffers rewritten only after the
    previous call's copy out has read them.  Call `join(stream)` before
    reading the host outputs or timing on `stream`.
    """

    def __init__(self, B, Nq, Hq, Nk, Hkv, d, dtype=torch.bfloat16, pieces=4, device=None):
        dev = torch.device("cuda") if device is None else torch.device(device)
        self.pieces = max(1, min(int(pieces), B))
        bounds = [B * i // self.pieces for i in range(self.pieces + 1)]
        self.ranges = [(a, b) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]
        self.q = torch.empty((B, Nq, Hq, d), dtype=dtype, device=dev)
        self.k = torch.empty((B, Nk, Hkv, d), dtype=dtype, device=dev)
        self.v = torch.empty((B, Nk, Hkv, d), dtype=dtype, device=dev)
        self.o = torch.empty((B, Nq, Hq, d), dtype=dtype, device=dev)
        self.lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
        self.s_in = torch.cuda.Stream(dev)
        self.s_run = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        n = len(self.ranges)
        self.ev_in = [torch.cuda.Event() for _ in range(n)]
        self.ev_run = [torch.cuda.Event() for _ in range(n)]
        self.ev_out = [torch.cuda.Event() for _ in range(n)]
        self.used = False  # events recorded by an earlier call

    def __call__(self, q_h, k_h, v_h, o_h, lse_h, scale=None, causal=False):
        for t, n in ((q_h, "q"), (k_h, "k"), (v_h, "v"), (o_h, "o"), (lse_h, "lse")):
            if t.is_cuda or not t.is_pinned() or not t.is_contiguous():
                raise ValueError(f"{n} must be a contiguous pinned host tensor")
        if q_h.shape != self.q.shape or k_h.shape != self.k.shape or v_h.shape != self.v.shape:
            raise ValueError("input shapes differ from the ones this object was built for")
        if o_h.shape != self.o.shape or lse_h.shape != self.lse.shape:
            raise ValueError("output shapes differ from the ones this object was built for")
        if q_h.dtype != self.q.dtype or o_h.dtype != self.o.dtype or lse_h.dtype != torch.float32:
            raise TypeError("dtype differs from the one this object was built for")
        # work queued on the caller's stream before this call comes first
        self.s_in.wait_stream(torch.cuda.current_stream())
        for i, (a, b) in enumerate(self.ranges):
            with torch.cuda.stream(self.s_in):
                if self.used:
                    self.s_in.wait_event(self.ev_run[i])  # the last forward read them
                self.q[a:b].copy_(q_h[a:b], non_blocking=True)
                self.k[a:b].copy_(k_h[a:b], non_blocking=True)
                self.v[a:b].copy_(v_h[a:b], non_blocking=True)
                self.ev_in[i].record(self.s_in)
            self.s_run.wait_event(self.ev_in[i])
            if self.used:
                self.s_run.wait_event(self.ev_out[i])  # the last copy out read them
            attn_fwd(self.q[a:b], self.k[a:b], self.v[a:b], scale=scale, causal=causal,
                     out=self.o[a:b], lse=self.lse[a:b], stream=self.s_run)
            self.ev_run[i].record(self.s_run)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.ev_run[i])
                o_h[a:b].copy_(self.o[a:b], non_blocking=True)
                lse_h[a:b].copy_(self.lse[a:b], non_blocking=True)
                self.ev_out[i].record(self.s_out)
        self.used = True
        return o_h, lse_h

    def join(self, stream=None):
        """Make `stream` (default: the current one) wait for every copy out."""
        s = stream if stream is not None else torch.cuda.current_stream()
        s.wait_stream(self.s_out)


def bwd_workspace_bytes(B, Hq, Nq) -> int:
    return int(load_library().attn_bwd_workspace_bytes(B, Hq, Nq))


def attn_bwd(q, k, v, o, lse, dout, scale=None, causal=False, seqlens_k=None, workspace=None,
             dq=None, dk=None, dv=None, stream=None, window_left=-1, block_mask=None):
    """Gradients of L = sum(dout * O) for O = attn_fwd(q, k, v, ...).

    o and lse are the forward's outputs for the same arguments (window_left
    and block_mask included).  Returns
    (dq [B, Nq, Hq, d], dk, dv [B, Nk, Hkv, d]) in the input dtype; dk and dv
    are summed over the query heads that share a kv head.
    """
    lib = load_library()
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (lse, "lse"), (dout, "dout")):
        _dev(t, n)
    if scale is None:
        scale = float(d) ** -0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(bwd_workspace_bytes(B, Hq, Nq), dtype=torch.uint8,
                                device=q.device)
    sl = 0
    if seqlens_k is not None:
        _dev(seqlens_k, "seqlens_k")
        if seqlens_k.dtype != torch.int32:
            raise TypeError("seqlens_k must be int32")
        sl = seqlens_k.data_ptr()
    if block_mask is not None:
        mp, sb, sh, sr = block_mask_args(block_mask, B, Hq, Nq, Nk)
        rc = lib.attn_bwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      lse.data_ptr(), dout.data_ptr(), dq.data_ptr(),
                                      dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq, Nk, d,
                                      float(scale), int(bool(causal)), int(window_left),
                                      _dtype_code(q), sl or None, mp, sb, sh, sr,
                                      workspace.data_ptr(), workspace.numel(),
                                      _stream_ptr(stream))
    else:
        rc = lib.attn_bwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                 dv.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale),
                                 int(bool(causal)), int(window_left), _dtype_code(q), sl or None,
                                 workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check("attn_bwd", rc)
    return dq, dk, dv


def decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_seqlen_k, split_keys=0) -> int:
    return int(load_library().attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_seqlen_k,
                                                           split_keys))


def attn_fwd_varlen_kvcache(q, k_cache, v_cache, cu_seqlens_k, seqlens_k, max_seqlen_k,
                            scale=None, causal=False, split_keys=0, workspace=None, out=None,
                            lse=None, stream=None):
    """Decode attention against a packed variable-length KV cache.

    q [B, Nq, Hq, d]; k_cache/v_cache [slots, Hkv, d]; cu_seqlens_k int32
    [B+1]; seqlens_k int32 [B]; max_seqlen_k (host int) >= every length.
    Returns (o [B, Nq, Hq, d], lse [B, Hq, Nq] float32).
    """
    lib = load_library()
    B, Nq, Hq, d = q.shape
    slots, Hkv, _ = k_cache.shape
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                 (cu_seqlens_k, "cu_seqlens_k"), (seqlens_k, "seqlens_k")):
        _dev(t, n)
    if scale is None:
        scale = float(d) ** -0.5
    need = decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_seqlen_k, split_keys)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    rc = lib.attn_fwd_varlen_kvcache(
        q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), cu_seqlens_k.data_ptr(),
        seqlens_k.data_ptr(), int(max_seqlen_k), int(slots), out.data_ptr(), lse.data_ptr(), B,
        Hq, Hkv, Nq, d, float(scale), int(bool(causal)), _dtype_code(q), workspace.data_ptr(),
        workspace.numel(), int(split_keys), _stream_ptr(stream))
    _check("attn_fwd_varlen_kvcache", rc)
    return out, lse


def attn_fwd_paged_kvcache(q, k_cache, v_cache, block_table, seqlens_k, max_seqlen_k,
                           scale=None, causal=False, k_new=None, v_new=None, split_keys=0,
                           workspace=None, out=None, lse=None, stream=None):
    """Decode attention against a paged KV cache.

    q [B, Nq, Hq, d]; k_cache/v_cache [num_blocks, block_size, Hkv, d];
    block_table int32 [B, max_blocks]; seqlens_k int32 [B] (lengths including
    the new tokens); k_new/v_new optional [B, Nq, Hkv, d], written into the
    cache before the attention.  Returns (o, lse).
    """
    lib = load_library()
    B, Nq, Hq, d = q.shape
    num_blocks, block_size, Hkv, _ = k_cache.shape
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                 (block_table, "block_table"), (seqlens_k, "seqlens_k")):
        _dev(t, n)
    if block_table.dtype != torch.int32 or seqlens_k.dtype != torch.int32:
        raise TypeError("block_table and seqlens_k must be int32")
    if scale is None:
        scale = float(d) ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_seqlen_k, split_keys),
                                dtype=torch.uint8, device=q.device)
    kn = vn = None
    if k_new is not None:
        _dev(k_new, "k_new")
        _dev(v_new, "v_new")
        kn, vn = k_new.data_ptr(), v_new.data_ptr()
    rc = lib.attn_fwd_paged_kvcache(
        q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_table.data_ptr(),
        block_table.shape[1], block_size, num_blocks, seqlens_k.data_ptr(), int(max_seqlen_k),
        kn, vn, out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, d, float(scale),
        int(bool(causal)), _dtype_code(q), workspace.data_ptr(), workspace.numel(),
        int(split_keys), _stream_ptr(stream))
    _check("attn_fwd_paged_kvcache", rc)
    return out, lse


def get_device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    _check("attn_get_device_error",
           load_library().attn_get_device_error(ctypes.byref(code), _stream_ptr(stream)))
    return code.value


def selftest_watchdog(q, k, v, out, lse, limit_ms=200, stream=None):
    rc = load_library().attn_selftest_watchdog(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                               out.data_ptr(), lse.data_ptr(), int(limit_ms),
                                               _stream_ptr(stream))
    _check("attn_selftest_watchdog", rc)


def hbm_read_probe(buf: torch.Tensor, out: torch.Tensor, n_ctas: int, stream=None):
    """Measurement helper: read `buf` (contiguous CUDA tensor, size a multiple
    of 16 bytes) once; `out` is an int32/uint32 CUDA tensor of >= n_ctas words."""
    _dev(buf, "buf")
    _dev(out, "out")
    if out.numel() * out.element_size() < 4 * n_ctas:
        raise ValueError("out holds fewer than n_ctas words")
    _check("attn_hbm_read_probe",
           load_library().attn_hbm_read_probe(buf.data_ptr(), buf.numel() * buf.element_size(),
                                              out.data_ptr(), int(n_ctas), _stream_ptr(stream)))


def schedule_band_unit(u: int, band: int, n_pairs: int, n_tiles: int):
    """(pair, tile rank) that block u of a banded causal grid runs (host only)."""
    pair, rank = ctypes.c_int(-1), ctypes.c_int(-1)
    _check("attn_schedule_band_unit",
           load_library().attn_schedule_band_unit(u, band, n_pairs, n_tiles, ctypes.byref(pair),
                                                  ctypes.byref(rank)))
    return pair.value, rank.value


def schedule_sparse_steps(m0, m1, nt0, nt1, j00=0, j01=0):
    """The block-sparse forward's lockstep steps (host only): a list of dicts
    with x0, x1, pos0, pos1, has0, has1, shared."""
    n = max(len(m0), len(m1), 1)
    a = (ctypes.c_ubyte * n)(*[1 if x else 0 for x in m0])
    b = (ctypes.c_ubyte * n)(*[1 if x else 0 for x in m1])
    out = (ctypes.c_int * (7 * n))()
    r = load_library().attn_schedule_sparse_steps(a, b, nt0, nt1, j00, j01, n, out)
    if r < 0:
        raise AttnError("attn_schedule_sparse_steps", r)
    keys = ("x0", "x1", "pos0", "pos1", "has0", "has1", "shared")
    return [{k: (bool(out[7 * i + c]) if c >= 4 else out[7 * i + c]) for c, k in enumerate(keys)}
            for i in range(r)]


def version() -> str:
    return load_library().attn_version().decode()
