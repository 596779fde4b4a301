"""Shared helpers for the GPU parity tests: run the CUDA path, run the oracle
on the same stored bits, compare element by element."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from io_aware_exact_29_b200 import attn

# Tolerances for bf16/fp16 inputs drawn from N(0, 1) with fp32 accumulation.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3


def compare(o_gpu, lse_gpu, o_ref, lse_ref, rows=None, what=""):
    """o_* [B, Nq, H, d], lse_* [B, H, Nq]; rows restricts the query rows."""
    og = o_gpu.float().cpu().numpy().astype(np.float64)
    lg = lse_gpu.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        og, o_ref = og[:, rows], o_ref[:, rows]
        lg, lse_ref = lg[:, :, rows], lse_ref[:, :, rows]
    assert np.isfinite(og).all(), f"{what}: non-finite output"
    assert not np.isnan(lg).any(), f"{what}: NaN in LSE"
    err = np.abs(og - o_ref)
    max_err, mean_err = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    both_inf = np.isneginf(lg) & np.isneginf(lse_ref)
    with np.errstate(invalid="ignore"):
        lerr = np.where(both_inf, 0.0, np.abs(lg - lse_ref))
    lse_err = float(np.nan_to_num(lerr, nan=np.inf).max(initial=0.0))
    worst = np.unravel_index(np.argmax(err), err.shape) if err.size else None
    msg = (f"{what}: O max {max_err:.3e} (at {worst}) mean {mean_err:.3e}, "
           f"LSE max {lse_err:.3e}")
    assert max_err <= O_MAX_ABS, msg
    assert mean_err <= O_MEAN_ABS, msg
    assert lse_err <= LSE_MAX_ABS, msg
    return max_err, mean_err, lse_err


def compare_selected(o_gpu, lse_gpu, o_ref, lse_ref, sel, what=""):
    """As compare, on the query rows selected per (batch, head): sel is a
    bool array [B, H, Nq] (the reference may hold NaN elsewhere)."""
    og = o_gpu.float().cpu().numpy().astype(np.float64)
    lg = lse_gpu.float().cpu().numpy().astype(np.float64)
    ob, ib, hb = np.nonzero(np.transpose(sel, (0, 2, 1)))  # [B, Nq, H] order
    return compare(torch.from_numpy(og[ob, ib, hb][None, :, None]),
                   torch.from_numpy(lg[ob, hb, ib][None, None, :]),
                   o_ref[ob, ib, hb][None, :, None], lse_ref[ob, hb, ib][None, None, :],
                   what=what)


# Gradients (no tolerance is stated for them): errors normalised by the
# reference tensor's own magnitude.  Rounding the output to bf16 alone gives
# about 2^-10 (1e-3) mean and 2^-9 max relative error; P and dS are rounded to
# bf16 for the tensor-core products and D comes from the bf16 forward output,
# each adding errors of the same order that partly average out over the sums,
# so the mean bound is a few times 2^-10 (measured: about 2.3e-3 at every
# shape, d = 64 and 128, causal or not, bf16 and fp16).
# The normalisers have a floor of GRAD_FLOOR: where the exact gradient is 0
# (one key: P = 1, so dS = dP - D = 0) the test is an absolute one, and with
# N(0, 1) inputs the gradients of every real case are well above it.
# With fewer than 64 visible keys per row nothing shrinks |O| by averaging,
# so the error D inherits from the bf16 output (about sqrt(d) 2^-9 |dO| |O|)
# is no longer small against dP - D: for a two-key row dS_0 = -dS_1 =
# P_0 P_1 (dP_0 - dP_1) and the relative error of dq grows as 1 / P_1, up to
# about 1% for a peaked row.  Such shapes get the looser mean bound.
GRAD_MAX_REL = 2e-2   # max |err| / max(max |ref|, floor)
GRAD_MEAN_REL = 5e-3  # mean |err| / max(mean |ref|, floor)
GRAD_MEAN_REL_FEW_KEYS = 1e-2  # the same, rows with fewer than 64 visible keys
GRAD_FEW_KEYS = 64
GRAD_FLOOR = 1e-3


# ---------------------------------------------------------------- canaries
# The sanitizer is not available, so outputs and workspaces are placed inside
# larger device buffers whose margins hold a byte pattern; after the run the
# margins must be unchanged (no write past either end), and outputs are
# prefilled with NaN so that an element the kernel never wrote shows up.
GUARD_BYTES = 4096
GUARD_BYTE = 0xA5


class Guarded:
    """A device tensor of `shape`/`dtype` at a 256-byte aligned offset inside a
    buffer with GUARD_BYTES of pattern on each side; `t` is the tensor."""

    def __init__(self, shape, dtype, fill=float("nan"), device="cuda"):
        elem = torch.empty((), dtype=dtype).element_size()
        self.nbytes = math.prod(shape) * elem
        span = -(-self.nbytes // 256) * 256
        self.raw = torch.full((2 * GUARD_BYTES + span,), GUARD_BYTE, dtype=torch.uint8,
                              device=device)
        self.t = self.raw[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype).view(shape)
        if dtype == torch.uint8:
            self.t.fill_(0x5A if fill != fill else int(fill))  # NaN -> a junk byte
        else:
            self.t.fill_(fill)

    def check(self, what=""):
        torch.cuda.synchronize()
        front = self.raw[:GUARD_BYTES]
        back = self.raw[GUARD_BYTES + self.nbytes:]
        assert bool((front == GUARD_BYTE).all()), f"{what}: write before the start"
        assert bool((back == GUARD_BYTE).all()), f"{what}: write past the end"


def check_defined(what, *tensors):
    """No NaN left in outputs that the kernels define everywhere."""
    for t in tensors:
        assert not bool(torch.isnan(t.float()).any()), f"{what}: NaN left in an output"


def compare_grads(gpu, ref, what="", key_rows=None, mean_rel=GRAD_MEAN_REL):
    """gpu: (dq, dk, dv) tensors; ref: the oracle's float64 arrays.
    key_rows: optional slice of key rows that dk/dv are compared on;
    mean_rel: the mean bound (GRAD_MEAN_REL_FEW_KEYS for few-key shapes)."""
    out = {}
    for name, g, r in zip(("dq", "dk", "dv"), gpu, ref):
        a = g.float().cpu().numpy().astype(np.float64)
        if key_rows is not None and name != "dq":
            a, r = a[:, key_rows], r[:, key_rows]
        assert np.isfinite(a).all(), f"{what} {name}: non-finite"
        err = np.abs(a - r)
        scale_max = max(float(np.abs(r).max(initial=0.0)), GRAD_FLOOR)
        scale_mean = max(float(np.abs(r).mean()) if r.size else 0.0, GRAD_FLOOR)
        emax = float(err.max(initial=0.0)) / scale_max
        emean = (float(err.mean()) if err.size else 0.0) / scale_mean
        out[name] = (emax, emean)
        msg = f"{what} {name}: max rel {emax:.3e} mean rel {emean:.3e}"
        assert emax <= GRAD_MAX_REL, msg
        assert emean <= mean_rel, msg
    return out


def run_fwd(inp, causal, scale=None):
    """The forward on guarded, NaN-prefilled outputs; checks the guards and
    that every output element was written."""
    q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
    sl = inp.get("seqlens_k")
    sl = None if sl is None else sl.cuda()
    B, Nq, Hq, _ = q.shape
    go = Guarded(tuple(q.shape), q.dtype)
    gl = Guarded((B, Hq, Nq), torch.float32)
    o, lse = attn.attn_fwd(q, k, v, scale=scale, causal=causal, seqlens_k=sl, out=go.t,
                           lse=gl.t)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    go.check("O")
    gl.check("LSE")
    check_defined("forward", o, lse)
    return o, lse


def check_fwd(inp, causal, scale, rows=None, what=""):
    o, lse = run_fwd(inp, causal, scale)
    o_ref, lse_ref = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], scale, causal,
                                     seqlens_k=inp.get("seqlens_k"), rows=rows)
    return compare(o, lse, o_ref, lse_ref, rows=rows, what=what)


def sample_rows(n, count, seed=0):
    fixed = [r for r in (0, 1, 127, 128, n - 1) if 0 <= r < n]
    g = torch.Generator().manual_seed(seed)
    extra = torch.randperm(n, generator=g)[:count].tolist()
    return sorted(set(fixed + extra))
