"""Shared helpers for the GPU parity tests: run the CUDA path, run the oracle
on the same stored bits, compare element by element."""
from __future__ import annotations

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


# Gradients (no tolerance is stated for them): errors normalised by the
# reference tensor's own magnitude.  Rounding the output to bf16 alone gives
# about 2^-10 mean and 2^-9 max relative error; P and dS are rounded to bf16
# for the tensor-core products and D comes from the bf16 forward output, each
# adding errors of the same order that average out over the sums.
# The normalisers have a floor of GRAD_FLOOR: where the exact gradient is 0
# (one key: P = 1, so dS = dP - D = 0) the test is an absolute one, and with
# N(0, 1) inputs the gradients of every real case are well above it.
GRAD_MAX_REL = 2e-2   # max |err| / max(max |ref|, floor)
GRAD_MEAN_REL = 1e-2  # mean |err| / max(mean |ref|, floor)
GRAD_FLOOR = 1e-3


def compare_grads(gpu, ref, what="", key_rows=None):
    """gpu: (dq, dk, dv) tensors; ref: the oracle's float64 arrays.
    key_rows: optional slice of key rows that dk/dv are compared on."""
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
        assert emean <= GRAD_MEAN_REL, msg
    return out


def run_fwd(inp, causal, scale=None):
    q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
    sl = inp.get("seqlens_k")
    sl = None if sl is None else sl.cuda()
    o, lse = attn.attn_fwd(q, k, v, scale=scale, causal=causal, seqlens_k=sl)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
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
