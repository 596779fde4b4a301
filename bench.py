"""Throughput of the attention path on B200: one JSON line on rank 0.

A step is one pass of the whole path over one batch of synthetic inputs:
  forward  : B=4, H=16, N=4096, d=128, bf16, non-causal (the long-sequence
             sweep point at which the forward target is stated), then
  backward : dQ, dK, dV of that forward for a seeded dO, then
  decode   : Llama2-70B shape, B=32, Hq=64, Hkv=8, d=128, one new token per
             sequence, packed bf16 KV cache with lengths ~ U[1, 32768], then
  decode16 : the same shape with a causal chunk of 16 new tokens per sequence
             (its own cache of the same size), then
  paged    : the one-token decode again, its cache in 16-row blocks.
`value` is the forward's TFLOP/s (algorithmic FLOPs / device time of the
forward launches, summed over ranks); the decodes' GB/s are reported beside
it.
All inputs are larger than L2 (126 MB), so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs the same per-rank workload on its own GPU with
no collective on the data path (weak scaling); the timed region is bracketed
by a barrier and a device synchronisation, and the max over ranks is taken.
Started without a launcher, `--gpus N` (N > 1) re-runs itself as N ranks under
torch.distributed.run on 127.0.0.1; under a launcher whose WORLD_SIZE differs
from N it refuses to run.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from io_aware_exact_29_b200 import accounting  # noqa: E402
from io_aware_exact_29_b200.workloads import (BLOCKSPARSE_CASES, DECODE_CASES,  # noqa: E402
                                              FWD_CASES, block_mask_inputs, fwd_inputs,
                                              kvcache_inputs, paged_from_packed,
                                              upstream_grad)

FWD_CASE = FWD_CASES["sweep_d128_n4096"]
DEC_CASE = DECODE_CASES["llama70b_decode"]
DEC16_CASE = DECODE_CASES["llama70b_chunk16"]
METRIC = "attn fwd TFLOP/s & % of BF16 TC peak; KV-cache decode GB/s & % of HBM peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    # the bench's forward (no mask, 4096 keys) runs on the persistent kernel
    "fwd": os.path.join(ROOT, "io_aware_exact_29_b200", "csrc", "attn_fwd_persist_sm100a.cu"),
    "decode": os.path.join(ROOT, "io_aware_exact_29_b200", "csrc", "attn_decode_tc_sm100a.cu"),
}
L2_BYTES = 126 * 2 ** 20


def source_hash(path: str) -> str:
    with open(path, "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; None otherwise."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh).get(kernel)
    if not rec or rec.get("source_sha256_16") != source_hash(KERNEL_SOURCES[kernel]):
        return None
    return rec.get("bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock, power and throttle reasons sampled while the timed region runs.

    NVML is read from a thread every 10 ms (reading only; no setting is
    touched), so that a region of under a second still gets tens of samples;
    where NVML cannot be loaded, nvidia-smi is polled every 200 ms instead."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index: int, period_s: float = 0.01):
        # the CUDA device's PCI address names the same GPU to NVML and
        # nvidia-smi whatever CUDA_VISIBLE_DEVICES does to the numbering
        self.index = index
        self.pci = None
        try:
            pr = torch.cuda.get_device_properties(index)
            self.pci = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
        except Exception:
            pass
        self.period_s = period_s
        self.proc = None
        self.lines = []
        self.samples = []  # (sm_mhz, max_mhz, set of reasons)
        self.source = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByPciBusId(self.pci) if self.pci else
                 pynvml.nvmlDeviceGetHandleByIndex(self.index))
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            mx = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def poll():
                while not self._stop.is_set():
                    try:
                        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((sm, mx, {n for n, b in bits.items() if r & b}))
                    except Exception:  # pragma: no cover - a failed read is skipped
                        pass
                    self._stop.wait(self.period_s)

            self.source = "nvml 10 ms"
            self._t = threading.Thread(target=poll, daemon=True)
            self._t.start()
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.pci or self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi 200 ms"
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self._t is not None:
            self._t.join(timeout=5)

    def summary(self):
        samples = list(self.samples)
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            samples.append((sm, mx, {n for n, v in zip(self.REASONS, parts[5:9])
                                     if v.lower() == "active"}))
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": self.source}
        reasons = set().union(*(r for _, _, r in samples))
        return {"sm_mhz": statistics.median(s for s, _, _ in samples),
                "sm_max_mhz": samples[-1][1], "reasons": sorted(reasons),
                "samples": len(samples), "source": self.source}


# ------------------------------------------------------------------ helpers
def launch_plan(n_gpus: int, env) -> str:
    """What main() does for `--gpus n_gpus` in environment `env`: "run" (this
    process is the only rank, or one of the torchrun ranks), "spawn" (start
    n_gpus ranks under torch.distributed.run), or an error message when a
    launcher already set a different world size."""
    if n_gpus < 1:
        return "error: --gpus must be >= 1"
    if "WORLD_SIZE" in env:
        world = int(env["WORLD_SIZE"])
        if world != n_gpus:
            return f"error: --gpus {n_gpus} but WORLD_SIZE={world}"
        return "run"
    return "spawn" if n_gpus > 1 else "run"


def spawn_ranks(n_gpus: int, argv) -> int:
    """Re-run this script as n_gpus ranks, one per GPU, on this node."""
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n_gpus}", "--master-addr=127.0.0.1", f"--master-port={port}",
           os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def job_rate(units_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: the units every rank processed in `steps` steps
    divided by the slowest rank's time (units per second)."""
    return units_per_step * steps * world / (max_ms * 1e-3)


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def reduce_max(values, world: int, device=None):
    """Element-wise max of a list of floats over all ranks (timing only)."""
    if world <= 1:
        return list(values)
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def fwd_work(case):
    return accounting.fwd_flops(case.B, case.Hq, case.Nq, case.Nk, case.d, case.causal)


# ------------------------------------------------------------------ our arm
def measure_read_peak(attn, dev, stream, gib: int = 4, reps: int = 10):
    """Read-only device-memory bandwidth on this GPU, in GB/s: the library's
    read probe over a `gib` GiB buffer (far above L2), CUDA events around each
    pass, best pass of the best of three grid sizes."""
    n = gib << 30
    buf = torch.zeros(n, dtype=torch.uint8, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out = torch.empty(sms * 8, dtype=torch.int32, device=dev)
    best_ms, best_ctas = float("inf"), 0
    for ctas in (sms * 2, sms * 4, sms * 8):
        for _ in range(2):
            attn.hbm_read_probe(buf, out, ctas, stream=stream)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        for a, b in evs:
            a.record(stream)
            attn.hbm_read_probe(buf, out, ctas, stream=stream)
            b.record(stream)
        torch.cuda.synchronize()
        ms = min(a.elapsed_time(b) for a, b in evs)
        if ms < best_ms:
            best_ms, best_ctas = ms, ctas
    del buf, out
    return {"gbs": round(n / (best_ms * 1e-3) / 1e9, 1), "bytes": n, "ctas": best_ctas,
            "how": (f"attn_hbm_read_probe over {gib} GiB, 16-byte loads, best of {reps} "
                    "passes and of 2/4/8 CTAs per SM, CUDA events")}


def run_ours(args, rank, world, local):
    from io_aware_exact_29_b200 import attn

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    # inputs, seeded per rank (independent problems), generated on the device
    fc, dc = FWD_CASE, DEC_CASE
    fin = fwd_inputs(fc, seed=1000 * rank, device=str(dev))
    q, k, v = fin["q"], fin["k"], fin["v"]
    o = torch.empty_like(q)
    lse = torch.empty((fc.B, fc.Hq, fc.Nq), dtype=torch.float32, device=dev)
    din = kvcache_inputs(dc, seed=1000 * rank, device=str(dev))
    dq, kc, vc = din["q"], din["k_cache"], din["v_cache"]
    cu, sl = din["cu_seqlens_k"], din["seqlens_k"]
    max_len = int(sl.max().item())
    do = torch.empty_like(dq)
    dlse = torch.empty((dc.B, dc.Hq, dc.Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(attn.decode_workspace_bytes(dc.B, dc.Hq, dc.Hkv, dc.Nq, dc.d, max_len),
                     dtype=torch.uint8, device=dev)
    # the one-token decode's cache in 16-row blocks behind a shuffled block table
    pg = paged_from_packed({k: t.cpu() for k, t in din.items()}, 16, seed=1000 * rank + 3,
                           fill=0.0)
    pgd = {k: t.to(dev) for k, t in pg.items()}
    del pg
    do_pg = torch.empty_like(dq)
    dl_pg = torch.empty_like(dlse)
    # the 16-token chunk variant of the decode (same cache shape, causal chunk)
    c16 = DEC16_CASE
    din16 = kvcache_inputs(c16, seed=1000 * rank + 1, device=str(dev))
    max16 = int(din16["seqlens_k"].max().item())
    o16 = torch.empty_like(din16["q"])
    l16 = torch.empty((c16.B, c16.Hq, c16.Nq), dtype=torch.float32, device=dev)
    ws16 = torch.empty(attn.decode_workspace_bytes(c16.B, c16.Hq, c16.Hkv, c16.Nq, c16.d, max16),
                       dtype=torch.uint8, device=dev)
    # the backward of the same forward (training step): dO seeded, O and LSE
    # from the step's own forward launch
    dout = upstream_grad(q, seed=1000 * rank + 2, device=str(dev))
    dq_b, dk_b, dv_b = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_b = torch.empty(attn.bwd_workspace_bytes(fc.B, fc.Hq, fc.Nq), dtype=torch.uint8,
                       device=dev)
    fflops = fwd_work(fc)
    bflops = 2.5 * fflops  # five tile products of the forward's size (S, dP, dV, dK, dQ)
    dbytes = accounting.decode_bytes(sl.tolist(), dc.B, dc.Hq, dc.Hkv, dc.Nq, dc.d)
    dbytes16 = accounting.decode_bytes(din16["seqlens_k"].tolist(), c16.B, c16.Hq, c16.Hkv,
                                       c16.Nq, c16.d)

    def step(ev):
        ev[0].record(stream)
        attn.attn_fwd(q, k, v, scale=fc.scale, causal=fc.causal, out=o, lse=lse, stream=stream)
        ev[1].record(stream)
        attn.attn_bwd(q, k, v, o, lse, dout, scale=fc.scale, causal=fc.causal, workspace=ws_b,
                      dq=dq_b, dk=dk_b, dv=dv_b, stream=stream)
        ev[4].record(stream)
        attn.attn_fwd_varlen_kvcache(dq, kc, vc, cu, sl, max_len, scale=dc.scale,
                                     causal=dc.causal, workspace=ws, out=do, lse=dlse,
                                     stream=stream)
        ev[2].record(stream)
        attn.attn_fwd_varlen_kvcache(din16["q"], din16["k_cache"], din16["v_cache"],
                                     din16["cu_seqlens_k"], din16["seqlens_k"], max16,
                                     scale=c16.scale, causal=c16.causal, workspace=ws16, out=o16,
                                     lse=l16, stream=stream)
        ev[3].record(stream)
        attn.attn_fwd_paged_kvcache(dq, pgd["k_cache"], pgd["v_cache"], pgd["block_table"],
                                    pgd["seqlens_k"], max_len, scale=dc.scale, causal=dc.causal,
                                    workspace=ws, out=do_pg, lse=dl_pg, stream=stream)
        ev[5].record(stream)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for _ in range(args.warmup):
        step(evs[0])
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0

    with ClockSampler(local) as clk:
        time.sleep(0.3)
        barrier(world)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    total_ms = t0.elapsed_time(t1)
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = sum(e[1].elapsed_time(e[4]) for e in evs)
    dec_ms = sum(e[4].elapsed_time(e[2]) for e in evs)
    dec16_ms = sum(e[2].elapsed_time(e[3]) for e in evs)
    pg_ms = sum(e[3].elapsed_time(e[5]) for e in evs)
    total_ms, fwd_ms, bwd_ms, dec_ms, dec16_ms, pg_ms = reduce_max(
        [total_ms, fwd_ms, bwd_ms, dec_ms, dec16_ms, pg_ms], world, dev)
    assert attn.get_device_error() == 0

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(args, attn, fin, din, max_len, stream, dev)
    e2e_fwd_ms, e2e_dec_ms = reduce_max([e2e["fwd_ms"], e2e["dec_ms"]], world, dev)

    read_peak = measure_read_peak(attn, dev, stream)
    read_gbs = reduce_max([-read_peak["gbs"]], world, dev)[0] * -1  # the slowest rank's
    peaks, peak_src = load_peaks()
    fwd_tflops = job_rate(fflops, args.steps, world, fwd_ms) / 1e12
    dec_gbs = job_rate(dbytes, args.steps, world, dec_ms) / 1e9
    per_launch_ms = fwd_ms / args.steps
    achieved = fflops / (per_launch_ms * 1e-3) / 1e12
    # the timed region is well under a second at full clocks, so the burst
    # cuBLAS figure is the peak that matches it; the sustained one (a 4 s
    # GEMM under the power cap) is reported beside it
    peak_t = peaks["bf16_tflops"]
    peak_ts = peaks["bf16_tflops_sustained"]
    dec_launch_ms = dec_ms / args.steps
    dec_achieved = dbytes / (dec_launch_ms * 1e-3) / 1e9
    dec16_call_ms = dec16_ms / args.steps
    dec16_achieved = dbytes16 / (dec16_call_ms * 1e-3) / 1e9

    out = {
        "metric": METRIC,
        "value": round(fwd_tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16; decode lengths ~U[1,32768])",
        "config": {
            "workload": ("fwd: long-sequence sweep point B=4 H=16 N=4096 d=128 non-causal; "
                         "decode: Llama2-70B shape B=32 Hq=64 Hkv=8 d=128 Nq=1 "
                         "lengths U[1,32768] packed bf16 cache"),
            "fwd": {"B": fc.B, "H": fc.Hq, "N": fc.Nq, "d": fc.d, "causal": fc.causal},
            "decode": {"B": dc.B, "Hq": dc.Hq, "Hkv": dc.Hkv, "d": dc.d, "Nq": dc.Nq,
                       "sum_len": int(sl.sum().item()), "max_len": max_len},
            "decode_chunk16": {"B": c16.B, "Hq": c16.Hq, "Hkv": c16.Hkv, "d": c16.d,
                               "Nq": c16.Nq, "causal": c16.causal,
                               "sum_len": int(din16["seqlens_k"].sum().item()),
                               "max_len": max16},
            "l2": "inputs larger than L2 (fwd 268 MB, each decode cache 2.1 GB); no flush",
            "parallelism": f"replicas x{world} (independent problems per GPU, no collective)",
        },
        "roofline": {
            "bound": "tensor",
            "kernel": "attn_fwd_persist_kernel<128, bf16>",
            "achieved": round(achieved, 2),
            "peak": peak_t,
            "unit": "TFLOP/s",
            "frac": round(achieved / peak_t, 4),
            "peak_source": (f"{peak_src} bf16_tflops (burst cuBLAS 8192^3): the timed region "
                            "is under a second at full clocks"),
            "frac_of_sustained_peak": round(achieved / peak_ts, 4),
            "sustained_peak": peak_ts,
            "flops_per_launch": fflops,
            "ms_per_launch": round(per_launch_ms, 4),
            "traffic": load_traffic("fwd"),
        },
        "decode": {
            "value": round(dec_gbs, 1),
            "unit": "GB/s",
            "achieved_per_call": round(dec_achieved, 1),
            "peak": peaks["hbm_gbs"],
            "frac": round(dec_achieved / peaks["hbm_gbs"], 4),
            "peak_source": f"{peak_src} hbm_gbs (1 GiB copy, read + write bytes)",
            "read_peak": read_gbs,
            "frac_read_peak": round(dec_achieved / read_gbs, 4),
            "read_peak_how": read_peak["how"],
            "bytes_per_call": dbytes,
            "ms_per_call": round(dec_launch_ms, 4),
            "kernels_per_call": "plan + attn_decode_tc_kernel + merge",
            "bound": "hbm",
            "traffic": load_traffic("decode"),
            "e2e": {"value": round(job_rate(dbytes, 1, world, e2e_dec_ms) / 1e9, 1),
                    "unit": "GB/s", "h2d_bytes_per_step": e2e["dec_h2d"],
                    "d2h_bytes_per_step": e2e["dec_d2h"]},
        },
        "bwd": {
            "value": round(job_rate(bflops, args.steps, world, bwd_ms) / 1e12, 2),
            "unit": "TFLOP/s",
            "flops_per_call": bflops,
            "flop_count": "2.5 x the forward's (S, dP, dV, dK, dQ tile products); the kernels "
                          "recompute S and dP once more for dQ, which is not counted",
            "ms_per_call": round(bwd_ms / args.steps, 4),
            "frac": round(bflops / (bwd_ms / args.steps * 1e-3) / 1e12 / peak_t, 4),
            "peak": peak_t,
            "frac_of_sustained_peak": round(bflops / (bwd_ms / args.steps * 1e-3) / 1e12 /
                                            peak_ts, 4),
            "kernels_per_call": "attn_bwd_pre + attn_bwd_dkdv + attn_bwd_dq",
            "bound": "tensor",
        },
        "decode_paged_bs16": {
            "value": round(job_rate(dbytes, args.steps, world, pg_ms) / 1e9, 1),
            "unit": "GB/s",
            "ms_per_call": round(pg_ms / args.steps, 4),
            "frac": round(dbytes / (pg_ms / args.steps * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "frac_read_peak": round(dbytes / (pg_ms / args.steps * 1e-3) / 1e9 / read_gbs, 4),
            "bytes_per_call": dbytes,
            "layout": "the one-token decode's cache in 16-row blocks, shuffled block table",
            "kernels_per_call": "plan + attn_decode_tc_kernel + merge",
            "bound": "hbm",
        },
        "decode_chunk16": {
            "value": round(job_rate(dbytes16, args.steps, world, dec16_ms) / 1e9, 1),
            "unit": "GB/s",
            "achieved_per_call": round(dec16_achieved, 1),
            "peak": peaks["hbm_gbs"],
            "frac": round(dec16_achieved / peaks["hbm_gbs"], 4),
            "frac_read_peak": round(dec16_achieved / read_gbs, 4),
            "bytes_per_call": dbytes16,
            "ms_per_call": round(dec16_call_ms, 4),
            "kernels_per_call": "plan + attn_decode_tc_kernel + merge",
            "bound": "hbm",
        },
        "e2e": {"value": round(job_rate(fflops, 1, world, e2e_fwd_ms) / 1e12, 2),
                "unit": "TFLOP/s", "h2d_bytes_per_step": e2e["fwd_h2d"],
                "d2h_bytes_per_step": e2e["fwd_d2h"]},
        # per step: the forward kernel, the three backward kernels, and
        # plan + decode + merge for each of the three decodes
        "gpu_launches": 13 * args.steps,
        "clocks": clk.summary(),
        "fwd_ms_per_launch": round(per_launch_ms, 4),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_budget)
    return out


def run_e2e(args, attn, fin, din, max_len, stream, dev):
    """Same workload through the public calls with pinned host buffers: every
    step copies its inputs host->device and its outputs device->host."""
    fc, dc = FWD_CASE, DEC_CASE
    h = {n: fin[n].cpu().pin_memory() for n in ("q", "k", "v")}
    hq = din["q"].cpu().pin_memory()
    hcu = din["cu_seqlens_k"].cpu().pin_memory()
    hsl = din["seqlens_k"].cpu().pin_memory()
    ho = torch.empty(tuple(fin["q"].shape), dtype=fin["q"].dtype).pin_memory()
    hl = torch.empty((fc.B, fc.Hq, fc.Nq), dtype=torch.float32).pin_memory()
    kc, vc = din["k_cache"], din["v_cache"]  # resident cache (built on device by prefill)
    ddq = torch.empty_like(din["q"])
    dcu = torch.empty_like(din["cu_seqlens_k"])
    dsl = torch.empty_like(din["seqlens_k"])
    do = torch.empty_like(din["q"])
    dl = torch.empty((dc.B, dc.Hq, dc.Nq), dtype=torch.float32, device=dev)
    hdo = torch.empty(do.shape, dtype=do.dtype).pin_memory()
    hdl = torch.empty(dl.shape, dtype=dl.dtype).pin_memory()
    ws = torch.empty(attn.decode_workspace_bytes(dc.B, dc.Hq, dc.Hkv, dc.Nq, dc.d, max_len),
                     dtype=torch.uint8, device=dev)
    steps = max(3, min(args.steps, 10))

    # the forward through the pinned-host call: the batch in four pieces, the
    # copy in of one piece, the forward of the previous one and the copy out
    # of the one before on three streams (every byte still crosses every step)
    pf = attn.PinnedForward(fc.B, fc.Nq, fc.Hq, fc.Nk, fc.Hkv, fc.d, dtype=fin["q"].dtype,
                            pieces=4, device=dev)

    def fwd_step():
        pf(h["q"], h["k"], h["v"], ho, hl, scale=fc.scale, causal=fc.causal)

    def dec_step():
        ddq.copy_(hq, non_blocking=True)
        dcu.copy_(hcu, non_blocking=True)
        dsl.copy_(hsl, non_blocking=True)
        attn.attn_fwd_varlen_kvcache(ddq, kc, vc, dcu, dsl, max_len, scale=dc.scale,
                                     causal=dc.causal, workspace=ws, out=do, lse=dl,
                                     stream=stream)
        hdo.copy_(do, non_blocking=True)
        hdl.copy_(dl, non_blocking=True)

    res = {}
    for name, fn in (("fwd", fwd_step), ("dec", dec_step)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        pf.join(stream)
        b.record(stream)
        torch.cuda.synchronize()
        res[name + "_ms"] = a.elapsed_time(b) / steps
    res["fwd_h2d"] = sum(t.numel() * t.element_size() for t in h.values())
    res["fwd_d2h"] = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    res["dec_h2d"] = sum(t.numel() * t.element_size() for t in (hq, hcu, hsl))
    res["dec_d2h"] = hdo.numel() * hdo.element_size() + hdl.numel() * hdl.element_size()
    return res


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(rows_per_head: int, seed: int = 0):
    """A bounded sample of the forward workload: every (batch, head), a seeded
    subset of query rows against all keys."""
    fc = FWD_CASE
    inp = fwd_inputs(fc, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    rows = sorted(torch.randperm(fc.Nq, generator=g)[:rows_per_head].tolist())
    flops = 4 * fc.d * fc.B * fc.Hq * len(rows) * fc.Nk  # non-causal: every key visible
    return inp, rows, flops


def cpu_baseline(budget_s: float = 15.0):
    import oracle

    fc = FWD_CASE
    rows_per_head = 16
    inp, rows, flops = oracle_sample(rows_per_head)
    t = time.perf_counter()
    oracle.attn_fwd(inp["q"], inp["k"], inp["v"], fc.scale, fc.causal, rows=rows)
    dt = time.perf_counter() - t
    # grow the sample to fill about `budget_s` of CPU time, then time it once
    scale = max(1, min(int(budget_s / max(dt, 1e-3)), fc.Nq // rows_per_head))
    if scale > 1:
        inp, rows, flops = oracle_sample(rows_per_head * scale)
        t = time.perf_counter()
        oracle.attn_fwd(inp["q"], inp["k"], inp["v"], fc.scale, fc.causal, rows=rows)
        dt = time.perf_counter() - t
    cores = oracle.max_threads()
    out = {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s",
           "cores": cores, "kind": "oracle",
           "sample": (f"fwd workload B=4 H=16 N=4096 d=128: {len(rows)} seeded query rows "
                      f"per head x all 64 heads x all 4096 keys, fp64 ({dt:.1f} s)")}
    # the tiny configuration (B=1 H=2 N=128 d=64, non-causal and causal) on one core
    tc = FWD_CASES["tiny"]
    tin = fwd_inputs(tc, seed=0)
    oracle.set_threads(1)
    try:
        per = {}
        for causal in (False, True):
            reps, t = 0, time.perf_counter()
            while reps < 3 or time.perf_counter() - t < 0.5:
                oracle.attn_fwd(tin["q"], tin["k"], tin["v"], tc.scale, causal)
                reps += 1
            per["causal" if causal else "non_causal"] = round(
                (time.perf_counter() - t) / reps * 1e3, 3)
    finally:
        oracle.set_threads(cores)
    out["tiny_one_core_ms"] = per
    return out


def run_reference(args, rank, world):
    """The oracle arm: the fp64 CPU oracle on the host cores, each step a
    bounded sample of the forward workload."""
    import oracle

    fc = FWD_CASE
    inp, rows, flops = oracle_sample(args.ref_rows)
    for _ in range(args.warmup):
        oracle.attn_fwd(inp["q"], inp["k"], inp["v"], fc.scale, fc.causal, rows=rows[:4])
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.attn_fwd(inp["q"], inp["k"], inp["v"], fc.scale, fc.causal, rows=rows)
    dt = time.perf_counter() - t
    value = flops * args.steps / dt / 1e12
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 inputs widened to fp64)",
        "config": {"workload": ("fwd: long-sequence sweep point B=4 H=16 N=4096 d=128 "
                                "non-causal (the value: the forward TFLOP/s, as in the "
                                "kernel arm; the oracle takes a sample of query rows per step)"),
                   "fwd": {"B": fc.B, "H": fc.Hq, "N": fc.Nq, "d": fc.d, "causal": fc.causal},
                   "parallelism": "rank 0 only, host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                         "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": f"{len(rows)} query rows per head x 64 heads x 4096 keys"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_profile_case(kernel: str, launches: int):
    """Small, self-contained launches for ncu captures: the forward of the
    bench workload (268 MB of inputs), or a decode of the Llama2-70B shape with
    lengths up to 8192 (about 0.5 GB of cache; one new token, or a causal
    chunk of 16); all larger than L2."""
    from io_aware_exact_29_b200 import attn
    from io_aware_exact_29_b200.workloads import DecodeCase

    dev = torch.device("cuda", 0)
    if kernel == "bwd":
        # backward of the bench's forward shape (inputs and gradients ~0.5 GB)
        fc = FWD_CASE
        fin = fwd_inputs(fc, seed=0, device="cuda")
        o, lse = attn.attn_fwd(fin["q"], fin["k"], fin["v"], scale=fc.scale, causal=fc.causal)
        dout = upstream_grad(fin["q"], seed=0, device="cuda")
        for _ in range(2 + launches):
            attn.attn_bwd(fin["q"], fin["k"], fin["v"], o, lse, dout, scale=fc.scale,
                          causal=fc.causal)
    elif kernel.startswith("fwd"):
        # fwd: the bench's forward; fwd_d64: the N=4096 d=64 sweep point
        # (134 MB of inputs); fwd_gpt2 / fwd_bert: those workloads
        fc = {"fwd": FWD_CASE, "fwd_d64": FWD_CASES["sweep_d64_n4096"],
              "fwd_gpt2": FWD_CASES["gpt2"], "fwd_bert": FWD_CASES["bert_large"]}[kernel]
        fin = fwd_inputs(fc, seed=0, device="cuda")
        for _ in range(2 + launches):
            attn.attn_fwd(fin["q"], fin["k"], fin["v"], scale=fc.scale, causal=fc.causal)
    else:
        nq = 16 if kernel == "decode_chunk16" else 1
        dc = DecodeCase("profile", 32, 64, 8, nq, 128, (nq, 8192), nq > 1)
        din = kvcache_inputs(dc, seed=0, device="cuda")
        ml = int(din["seqlens_k"].max().item())
        ws = torch.empty(attn.decode_workspace_bytes(dc.B, dc.Hq, dc.Hkv, dc.Nq, dc.d, ml),
                         dtype=torch.uint8, device=dev)
        if kernel == "decode_paged":
            # the same cache in 16-row blocks behind a shuffled table
            pg = paged_from_packed({k: t.cpu() for k, t in din.items()}, 16, seed=3, fill=0.0)
            pgd = {k: t.to(dev) for k, t in pg.items()}
            for _ in range(2 + launches):
                attn.attn_fwd_paged_kvcache(din["q"], pgd["k_cache"], pgd["v_cache"],
                                            pgd["block_table"], pgd["seqlens_k"], ml,
                                            scale=dc.scale, causal=dc.causal, workspace=ws)
        for _ in range(2 + launches if kernel != "decode_paged" else 0):
            attn.attn_fwd_varlen_kvcache(din["q"], din["k_cache"], din["v_cache"],
                                         din["cu_seqlens_k"], din["seqlens_k"], ml,
                                         scale=dc.scale, causal=dc.causal, workspace=ws)
        lens = din["seqlens_k"].tolist()
        print("decode profile case: sum_len", sum(lens), "algorithmic bytes per launch",
              accounting.decode_bytes(lens, dc.B, dc.Hq, dc.Hkv, dc.Nq, dc.d))
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    print(f"profile case {kernel}: {2 + launches} launches ok")


def run_sweep(reps: int = 20):
    """One JSON line per configured workload (forward TFLOP/s, decode GB/s),
    each timed with CUDA events over `reps` back-to-back launches after 3
    warm-ups; inputs seeded on the device.  Separate from the one JSON line of the default run."""
    from io_aware_exact_29_b200 import attn

    peaks, _ = load_peaks()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    for name, c in FWD_CASES.items():
        fin = fwd_inputs(c, seed=0, device="cuda")
        sl = fin["seqlens_k"]
        o = torch.empty_like(fin["q"])
        lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)
        ms = timed(lambda: attn.attn_fwd(fin["q"], fin["k"], fin["v"], scale=c.scale,
                                         causal=c.causal, seqlens_k=sl, out=o, lse=lse))
        flops = accounting.fwd_flops(c.B, c.Hq, c.Nq, c.Nk, c.d, c.causal,
                                     None if sl is None else sl.tolist())
        tf = flops / (ms * 1e-3) / 1e12
        print(json.dumps({"sweep": name, "kind": "fwd", "dtype": c.dtype, "causal": c.causal,
                          "B": c.B, "H": c.Hq, "N": c.Nq, "d": c.d, "ms": round(ms, 4),
                          "TFLOP/s": round(tf, 1),
                          "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 3),
                          "frac_burst": round(tf / peaks["bf16_tflops"], 3)}), flush=True)
        # the backward of the same forward (five tile products counted)
        dout = upstream_grad(fin["q"], seed=0, device="cuda")
        ws_b = torch.empty(attn.bwd_workspace_bytes(c.B, c.Hq, c.Nq), dtype=torch.uint8, device=dev)
        grads = (torch.empty_like(fin["q"]), torch.empty_like(fin["k"]), torch.empty_like(fin["v"]))
        ms_b = timed(lambda: attn.attn_bwd(fin["q"], fin["k"], fin["v"], o, lse, dout, scale=c.scale,
                                           causal=c.causal, seqlens_k=sl, workspace=ws_b,
                                           dq=grads[0], dk=grads[1], dv=grads[2]))
        tb = 2.5 * flops / (ms_b * 1e-3) / 1e12
        print(json.dumps({"sweep": name, "kind": "bwd", "dtype": c.dtype, "causal": c.causal,
                          "B": c.B, "H": c.Hq, "N": c.Nq, "d": c.d, "ms": round(ms_b, 4),
                          "TFLOP/s": round(tb, 1),
                          "frac_sustained": round(tb / peaks["bf16_tflops_sustained"], 3)}),
              flush=True)
        del fin, o, lse, dout, ws_b, grads
    for name, bc in BLOCKSPARSE_CASES.items():
        c = bc.fwd
        fin = fwd_inputs(c, seed=0, device="cuda")
        m = block_mask_inputs(bc, seed=0, device="cuda")
        o = torch.empty_like(fin["q"])
        lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)
        ms = timed(lambda: attn.attn_fwd(fin["q"], fin["k"], fin["v"], scale=c.scale,
                                         causal=c.causal, out=o, lse=lse, block_mask=m))
        flops = accounting.blocksparse_flops(m.cpu().numpy(), c.Nq, c.Nk, c.d, c.causal, c.B,
                                             c.Hq)
        dense = accounting.fwd_flops(c.B, c.Hq, c.Nq, c.Nk, c.d, c.causal)
        tf = flops / (ms * 1e-3) / 1e12
        print(json.dumps({"sweep": name, "kind": "fwd", "dtype": c.dtype, "causal": c.causal,
                          "B": c.B, "H": c.Hq, "N": c.Nq, "d": c.d,
                          "kept": round(flops / dense, 4), "ms": round(ms, 4),
                          "TFLOP/s": round(tf, 1),
                          "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 3)}),
              flush=True)
        dout = upstream_grad(fin["q"], seed=0, device="cuda")
        ws_b = torch.empty(attn.bwd_workspace_bytes(c.B, c.Hq, c.Nq), dtype=torch.uint8, device=dev)
        grads = (torch.empty_like(fin["q"]), torch.empty_like(fin["k"]), torch.empty_like(fin["v"]))
        ms_b = timed(lambda: attn.attn_bwd(fin["q"], fin["k"], fin["v"], o, lse, dout, scale=c.scale,
                                           causal=c.causal, workspace=ws_b, dq=grads[0],
                                           dk=grads[1], dv=grads[2], block_mask=m))
        tb = 2.5 * flops / (ms_b * 1e-3) / 1e12
        print(json.dumps({"sweep": name, "kind": "bwd", "dtype": c.dtype, "causal": c.causal,
                          "B": c.B, "H": c.Hq, "N": c.Nq, "d": c.d,
                          "kept": round(flops / dense, 4), "ms": round(ms_b, 4),
                          "TFLOP/s": round(tb, 1),
                          "frac_sustained": round(tb / peaks["bf16_tflops_sustained"], 3)}),
              flush=True)
        del fin, m, o, lse, dout, ws_b, grads
    for name, c in DECODE_CASES.items():
        din = kvcache_inputs(c, seed=0, device="cuda")
        ml = int(din["seqlens_k"].max().item())
        ws = torch.empty(attn.decode_workspace_bytes(c.B, c.Hq, c.Hkv, c.Nq, c.d, ml),
                         dtype=torch.uint8, device=dev)
        o = torch.empty_like(din["q"])
        lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)
        ms = timed(lambda: attn.attn_fwd_varlen_kvcache(
            din["q"], din["k_cache"], din["v_cache"], din["cu_seqlens_k"], din["seqlens_k"], ml,
            scale=c.scale, causal=c.causal, workspace=ws, out=o, lse=lse))
        lens = din["seqlens_k"].tolist()
        by = accounting.decode_bytes(lens, c.B, c.Hq, c.Hkv, c.Nq, c.d)
        fl = accounting.decode_flops(lens, c.Hq, c.Nq, c.d, c.causal)
        gbs = by / (ms * 1e-3) / 1e9
        print(json.dumps({"sweep": name, "kind": "decode", "Nq": c.Nq, "ms": round(ms, 4),
                          "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 3),
                          "TFLOP/s": round(fl / (ms * 1e-3) / 1e12, 1)}), flush=True)
        del din, ws, o, lse
    assert attn.get_device_error() == 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--profile", choices=["fwd", "fwd_d64", "fwd_gpt2", "fwd_bert", "bwd", "decode",
                                          "decode_chunk16", "decode_paged"],
                    default=None,
                    help="run a small case of one kernel for an ncu capture and exit")
    ap.add_argument("--profile-launches", type=int, default=3)
    ap.add_argument("--sweep", action="store_true",
                    help="time every configured workload, one JSON line each, and exit")
    args = ap.parse_args(argv)
    if args.sweep:
        run_sweep()
        return 0
    if args.profile:
        run_profile_case(args.profile, args.profile_launches)
        return 0
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    plan = launch_plan(args.gpus, os.environ)
    if plan.startswith("error"):
        ap.error(plan[len("error: "):])
    if args.impl == "reference":
        # the oracle arm runs on rank 0's host cores only; other ranks leave
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0
    if plan == "spawn":
        # one process per GPU: re-run this script under torch.distributed.run
        return spawn_ranks(args.gpus, sys.argv[1:] if argv is None else argv)
    rank, world, local = dist_setup(args.gpus)
    try:
        out = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
        return 0
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
