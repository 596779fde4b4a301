"""fp64 CPU oracle for exact scaled dot-product attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it and the
two share no code.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over
(batch, head)); this module compiles it with gcc on first use, widens the
stored bf16/fp16 bits to fp64 exactly and marshals pointers.  ``brute.py`` holds
an independent pure-Python statement used to pin the C code on tiny inputs.

Definition (ai6s.net "ops-transformer FlashAttention" article, section
"标准注意力的致命伤不在算力，在搬运"): O = softmax(scale·Q·Kᵀ + mask)·V, with the
additive 0/-inf mask of the causal rule (adaptation point 2) and of the real
KV length (adaptation point 3), LSE = natural log of the row's sum of
exponentials.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_DP = ctypes.POINTER(ctypes.c_double)
_IP = ctypes.POINTER(ctypes.c_int)
_U8P = ctypes.POINTER(ctypes.c_ubyte)
# block_mask, mask_sb, mask_sh, mask_nqb, mask_nkb, block_m, block_n
_MASK_ARGS = [_U8P, ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int,
              ctypes.c_int]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (gcc, -O2, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            lib.oracle_attn_fwd.restype = ctypes.c_int
            lib.oracle_attn_fwd.argtypes = [
                _DP, _DP, _DP, _DP, _DP, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                _IP, _IP, ctypes.c_int, ctypes.c_int]
            lib.oracle_attn_kvcache.restype = ctypes.c_int
            lib.oracle_attn_kvcache.argtypes = [
                _DP, _DP, _DP, _IP, _IP, _DP, _DP, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int]
            lib.oracle_lse_combine.restype = ctypes.c_int
            lib.oracle_lse_combine.argtypes = [_DP, _DP, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, _DP, _DP]
            lib.oracle_attn_bwd.restype = ctypes.c_int
            lib.oracle_attn_bwd.argtypes = [
                _DP, _DP, _DP, _DP, _DP, _DP, _DP, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int, _IP,
                ctypes.c_int]
            lib.oracle_attn_fwd_mask.restype = ctypes.c_int
            lib.oracle_attn_fwd_mask.argtypes = lib.oracle_attn_fwd.argtypes + _MASK_ARGS
            lib.oracle_attn_bwd_mask.restype = ctypes.c_int
            lib.oracle_attn_bwd_mask.argtypes = lib.oracle_attn_bwd.argtypes + _MASK_ARGS
            lib.oracle_attn_paged.restype = ctypes.c_int
            lib.oracle_attn_paged.argtypes = [
                _DP, _DP, _DP, _IP, ctypes.c_int, ctypes.c_int, ctypes.c_int, _IP, _DP, _DP,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, ctypes.c_int]
            lib.oracle_max_threads.restype = ctypes.c_int
            lib.oracle_set_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def _f64(t) -> np.ndarray:
    """Widen stored bits to fp64 exactly (bf16/fp16/fp32 all embed in fp64)."""
    if isinstance(t, torch.Tensor):
        t = t.detach().to("cpu", torch.float64).contiguous().numpy()
    return np.ascontiguousarray(t, dtype=np.float64)


def _i32(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().to("cpu").numpy()
    return np.ascontiguousarray(t, dtype=np.int32)


def _dp(a: np.ndarray):
    return a.ctypes.data_as(_DP)


def _ip(a):
    return None if a is None else a.ctypes.data_as(_IP)


def _block_mask_args(block_mask, block_size, B, Hq):
    """(array kept alive, ctypes argument tuple) for an optional block mask.

    block_mask: [Bm, Hm, nqb, nkb] with Bm in {1, B} and Hm in {1, Hq} (a
    size-1 dimension is shared); nonzero = the block's keys take part.
    block_size: int or (block_m, block_n).
    """
    if block_mask is None:
        return None, (None, 0, 0, 0, 0, 1, 1)
    if isinstance(block_mask, torch.Tensor):
        block_mask = block_mask.detach().to("cpu").numpy()
    m = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
    if m.ndim != 4 or m.shape[0] not in (1, B) or m.shape[1] not in (1, Hq):
        raise ValueError(f"block_mask shape {m.shape} is not [1|B, 1|Hq, nqb, nkb]")
    bm, bn = (block_size, block_size) if isinstance(block_size, int) else block_size
    nqb, nkb = m.shape[2], m.shape[3]
    sh = 0 if m.shape[1] == 1 else nqb * nkb
    sb = 0 if m.shape[0] == 1 else m.shape[1] * nqb * nkb
    return m, (m.ctypes.data_as(_U8P), sb, sh, nqb, nkb, int(bm), int(bn))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def attn_fwd(q, k, v, scale: float, causal: bool, seqlens_k=None, rows=None, window_left=-1,
             block_mask=None, block_size=128):
    """O, LSE of dense attention.

    q [B, Nq, Hq, d], k/v [B, Nk, Hkv, d] (any float dtype; widened exactly).
    seqlens_k: optional [B] key lengths (keys at or past it are masked).
    window_left: -1, or the sliding window: keys more than window_left
    positions before the query's own position i + (Lk - Nq) are masked.
    block_mask: optional [1|B, 1|Hq, nqb, nkb]; a zero entry masks the keys
    of block (i // block_m, j // block_n) for those queries (block_size is
    block_m = block_n, or a pair).
    rows: optional list of query-row indices; only those rows are computed
    (the other entries of the returned arrays are NaN).
    Returns (o [B, Nq, Hq, d] float64, lse [B, Hq, Nq] float64) numpy arrays.
    """
    qd, kd, vd = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d = qd.shape
    _, Nk, Hkv, _ = kd.shape
    o = np.full((B, Nq, Hq, d), np.nan)
    lse = np.full((B, Hq, Nq), np.nan)
    sl = None if seqlens_k is None else _i32(seqlens_k)
    rw = None if rows is None else _i32(rows)
    keep, margs = _block_mask_args(block_mask, block_size, B, Hq)
    rc = _load().oracle_attn_fwd_mask(_dp(qd), _dp(kd), _dp(vd), _dp(o), _dp(lse), B, Hq, Hkv,
                                      Nq, Nk, d, float(scale), int(bool(causal)), _ip(sl),
                                      _ip(rw), 0 if rw is None else len(rw), int(window_left),
                                      *margs)
    del keep
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd rejected its arguments (rc={rc})")
    return o, lse


def attn_kvcache(q, k_cache, v_cache, cu_seqlens_k, seqlens_k, scale: float, causal: bool):
    """O, LSE of new query tokens against a packed variable-length KV cache.

    q [B, Nq, Hq, d]; k_cache/v_cache [slots, Hkv, d]; cu_seqlens_k [B+1] slot
    offsets; seqlens_k [B] filled lengths.  Returns float64 numpy arrays
    (o [B, Nq, Hq, d], lse [B, Hq, Nq]).
    """
    qd, kd, vd = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Nq, Hq, d = qd.shape
    Hkv = kd.shape[1]
    cu, sl = _i32(cu_seqlens_k), _i32(seqlens_k)
    o = np.full((B, Nq, Hq, d), np.nan)
    lse = np.full((B, Hq, Nq), np.nan)
    rc = _load().oracle_attn_kvcache(_dp(qd), _dp(kd), _dp(vd), _ip(cu), _ip(sl), _dp(o),
                                     _dp(lse), B, Hq, Hkv, Nq, d, float(scale),
                                     int(bool(causal)))
    if rc != 0:
        raise ValueError(f"oracle_attn_kvcache rejected its arguments (rc={rc})")
    return o, lse


def lse_combine(o_parts, lse_parts):
    """Merge partial results over disjoint key sets.

    o_parts [P, R, d], lse_parts [P, R] -> (o [R, d], lse [R]).
    """
    op, lp = _f64(o_parts), _f64(lse_parts)
    P, R, d = op.shape
    o = np.empty((R, d))
    lse = np.empty((R,))
    rc = _load().oracle_lse_combine(_dp(op), _dp(lp), P, R, d, _dp(o), _dp(lse))
    if rc != 0:
        raise ValueError("oracle_lse_combine rejected its arguments")
    return o, lse


def attn_bwd(q, k, v, dout, scale: float, causal: bool, seqlens_k=None, window_left=-1,
             block_mask=None, block_size=128):
    """Gradients (dq, dk, dv) of L = sum(dout * O) for O = attention(q, k, v).

    q, dout [B, Nq, Hq, d]; k, v [B, Nk, Hkv, d]; seqlens_k optional [B];
    window_left, block_mask, block_size as in attn_fwd.
    Returns float64 numpy arrays dq [B, Nq, Hq, d], dk and dv [B, Nk, Hkv, d]
    (dk, dv summed over the query heads that share a kv head; zero behind a
    sequence's real key length).
    """
    qd, kd, vd, dod = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Nq, Hq, d = qd.shape
    _, Nk, Hkv, _ = kd.shape
    dq = np.full((B, Nq, Hq, d), np.nan)
    dk = np.full((B, Nk, Hkv, d), np.nan)
    dv = np.full((B, Nk, Hkv, d), np.nan)
    sl = None if seqlens_k is None else _i32(seqlens_k)
    keep, margs = _block_mask_args(block_mask, block_size, B, Hq)
    rc = _load().oracle_attn_bwd_mask(_dp(qd), _dp(kd), _dp(vd), _dp(dod), _dp(dq), _dp(dk),
                                      _dp(dv), B, Hq, Hkv, Nq, Nk, d, float(scale),
                                      int(bool(causal)), _ip(sl), int(window_left), *margs)
    del keep
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd rejected its arguments (rc={rc})")
    return dq, dk, dv


def paged_append(k_cache, v_cache, block_table, seqlens_k, k_new, v_new):
    """The cache after writing the new tokens' rows (a plain copy, no arithmetic).

    k_cache/v_cache [num_blocks, block_size, Hkv, d]; k_new/v_new [B, Nq, Hkv, d];
    token t of sequence b goes to logical position seqlens_k[b] - Nq + t, i.e.
    block block_table[b][pos // block_size], row pos % block_size (positions
    below 0 are dropped).  Returns float64 copies (k, v).
    """
    kc, vc = _f64(k_cache).copy(), _f64(v_cache).copy()
    kn, vn = _f64(k_new), _f64(v_new)
    bt, sl = _i32(block_table), _i32(seqlens_k)
    bs = kc.shape[1]
    B, Nq = kn.shape[0], kn.shape[1]
    for b in range(B):
        for t in range(Nq):
            pos = int(sl[b]) - Nq + t
            if pos < 0:
                continue
            blk, r = int(bt[b, pos // bs]), pos % bs
            kc[blk, r] = kn[b, t]
            vc[blk, r] = vn[b, t]
    return kc, vc


def attn_paged(q, k_cache, v_cache, block_table, seqlens_k, scale: float, causal: bool,
               k_new=None, v_new=None):
    """O, LSE against a paged KV cache (optionally after appending k_new/v_new).

    q [B, Nq, Hq, d]; k_cache/v_cache [num_blocks, block_size, Hkv, d];
    block_table [B, max_blocks] int; seqlens_k [B] (lengths after the append).
    Returns float64 numpy arrays (o [B, Nq, Hq, d], lse [B, Hq, Nq]).
    """
    if k_new is not None:
        kd, vd = paged_append(k_cache, v_cache, block_table, seqlens_k, k_new, v_new)
    else:
        kd, vd = _f64(k_cache), _f64(v_cache)
    qd = _f64(q)
    bt, sl = _i32(block_table), _i32(seqlens_k)
    B, Nq, Hq, d = qd.shape
    num_blocks, bs, Hkv, _ = kd.shape
    o = np.full((B, Nq, Hq, d), np.nan)
    lse = np.full((B, Hq, Nq), np.nan)
    rc = _load().oracle_attn_paged(_dp(qd), _dp(kd), _dp(vd), _ip(bt), bt.shape[1], bs,
                                   num_blocks, _ip(sl), _dp(o), _dp(lse), B, Hq, Hkv, Nq, d,
                                   float(scale), int(bool(causal)))
    if rc != 0:
        raise ValueError(f"oracle_attn_paged rejected its arguments (rc={rc})")
    return o, lse


__all__ = ["build", "attn_fwd", "attn_kvcache", "lse_combine", "attn_bwd", "attn_paged",
           "paged_append", "max_threads", "set_threads"]
