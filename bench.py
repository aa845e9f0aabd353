"""Benchmark of the pooled block-sparse attention hot path on B200.

One step = the whole path for one batch of synthetic video-shaped input:
the block mask (pool, score + softmax, hybrid Top-k/Top-p select) followed by
block-sparse attention; for the SLA2 workloads also the per-head linear
summaries and the sparse + linear mix.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints ONE JSON line (rank 0). Under torchrun every rank runs its own copy of
the workload (independent problems, no collective on the data path: weak
scaling); only the timing uses the process group.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_pooled_b200 import synth  # noqa: E402

METRIC = "ms/call, effective TFLOPS & tensor-pipe % of bf16 peak at 32K/75K-token shapes"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="480p", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--variant", default="bf16", choices=["bf16", "q8", "bwd"],
                    help="q8: the low-bit sparse branch (int8 Q/K codes, e4m3 P and V), no linear branch; "
                         "bwd: a training step (mask, forward, backward; the sparse + linear mix on SLA2 "
                         "workloads, whose backward recomputes its forward pieces)")
    ap.add_argument("--router", type=int, default=0, choices=[0, 64, 128],
                    help="score the mask through a learnt router of this width (seeded stand-in projections)")
    ap.add_argument("--sparse-only", action="store_true",
                    help="on an SLA2 workload, run the sparse branch alone (sparge_attn_fwd)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=0,
                    help="run only the first H heads of batch 0 of the workload (a smaller case of the same "
                         "shape, for profiler captures); 0 = all")
    ap.add_argument("--report", choices=["regimes"], default=None,
                    help="regimes: kept fraction and error against dense attention of Top-k alone, Top-p alone "
                         "and the hybrid on the flat and peaked sweep workloads (one GPU; prints a table)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other headline shapes (720p sparse and SLA2, sla2_480p) timed after the 480p line")
    return ap.parse_args()


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(value: float, world: int, device=None) -> float:
    """The maximum of a per-rank scalar over all ranks (identity when world == 1)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- work accounting
def kept_flops(kv_idx: torch.Tensor, kv_cnt: torch.Tensor, N: int, d: int, bq: int, bk: int) -> float:
    """4*d * sum over kept (query block, key block) pairs of valid rows x valid keys."""
    B, H, nqb, nkb = kv_idx.shape
    rows = torch.clamp(N - torch.arange(nqb, device=kv_idx.device) * bq, max=bq).to(torch.float64)
    keys_of_block = torch.clamp(N - torch.arange(nkb, device=kv_idx.device) * bk, max=bk).to(torch.float64)
    valid = torch.arange(nkb, device=kv_idx.device)[None, None, None, :] < kv_cnt[..., None]
    keys = torch.where(valid, keys_of_block[kv_idx.long().clamp(0, nkb - 1)], torch.zeros((), dtype=torch.float64,
                                                                                          device=kv_idx.device))
    per_row = keys.sum(-1) * rows[None, None, :]
    return float(4.0 * d * per_row.sum().item())


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples during the timed region (clocks and throttle reasons)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


class NvmlClockSampler:
    """SM clock and clock-event reasons read in-process through NVML (read-only
    queries) every few milliseconds during the timed region, so that even a
    timed region of a few tens of milliseconds gets samples. Falls back to the
    nvidia-smi sampler when NVML cannot be opened."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, gpu_id: str, period_s: float = 0.002):
        self.gpu_id = gpu_id
        self.period = period_s
        self.samples = []  # (sm_mhz, max_mhz, reasons bitmask)
        self._stop = threading.Event()
        self._nvml = None
        self._fallback = None

    def __enter__(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu_id) if self.gpu_id.isdigit() else 0)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            self._max = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._nvml = (pynvml, h, get_reasons)
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception:
            self._nvml = None
            self._fallback = ClockSampler(self.gpu_id).__enter__()
        return self

    def _sample(self):
        pynvml, h, get_reasons = self._nvml
        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        reasons = get_reasons(h) if get_reasons is not None else 0
        self.samples.append((float(sm), float(self._max), int(reasons)))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                break
            self._stop.wait(self.period)

    def __exit__(self, *exc):
        if self._nvml is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            try:
                self._sample()  # one sample at the end of the region
                self._nvml[0].nvmlShutdown()
            except Exception:
                pass
        if self._fallback is not None:
            self._fallback.__exit__(*exc)

    def summary(self):
        if self._fallback is not None:
            out = self._fallback.summary()
            out["source"] = "nvidia-smi -lms 200"
            return out
        sm = [x[0] for x in self.samples]
        reasons = sorted({n for _, _, r in self.samples for n, bit in self.REASONS if r & bit})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": self.samples[0][1] if self.samples else None,
                "sm_mhz_min": min(sm) if sm else None, "reasons": reasons, "samples": len(sm),
                "source": f"NVML in-process, every {self.period * 1e3:.0f} ms"}


def clocks_at_max(clocks) -> bool:
    """True when the sampled SM clock held >= 95% of its maximum, or when there
    are no samples (unknown: the burst peak, the larger denominator, applies)."""
    if not clocks.get("samples") or clocks.get("sm_mhz") is None or not clocks.get("sm_max_mhz"):
        return True
    return clocks["sm_mhz"] >= 0.95 * clocks["sm_max_mhz"]


def _smi_id(dev) -> str:
    """nvidia-smi --id for a torch device: its UUID when torch exposes it."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        cvd = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [x for x in cvd.split(",") if x.strip()]
        return ids[dev.index].strip() if dev.index < len(ids) else str(dev.index)


# Source files each timed kernel is built from (its own header and the PTX helpers).
KERNEL_SOURCES = {"attn_fwd_kernel": ("attn.cuh", "ptx.cuh"), "attn_q8_kernel": ("attn_q8.cuh", "ptx.cuh")}


def kernel_source_sha(kernel: str) -> str:
    """Digest of the CUDA sources of one kernel, to tell whether stored counters still apply."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_attention_pooled_b200", "csrc")
    for name in KERNEL_SOURCES[kernel.split("<")[0]]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def _capture(workload: str, kernel: str):
    """The committed ncu capture of the dominant kernel on this workload, or
    None when there is none or the kernel's sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        entry = json.load(f).get(workload)
    if not entry or entry.get("kernel") != kernel or entry.get("csrc_sha") != kernel_source_sha(kernel):
        return None
    return entry


def dram_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    capture, or None when there is none or the kernel changed since."""
    entry = _capture(workload, kernel)
    return None if entry is None else entry["dram_bytes_per_launch"]


def tensor_pipe_pct(workload: str, kernel: str):
    """ncu's sm__pipe_tensor_cycles_active (% of peak sustained, active cycles)
    from the same capture, or None."""
    entry = _capture(workload, kernel)
    return None if entry is None else entry.get("tensor_pipe_active_pct")


# ----------------------------------------------------------------------------- end-to-end timing
def e2e_serial_ms(k, step, io, host_ins, hosts, stream, cuda=None):
    """ms per step when each step copies its inputs in, runs, and copies its
    results out, all on the compute stream (the copies' time adds to the
    step's). io = (device inputs, device results) as step(io=...) takes them."""
    cuda = torch.cuda if cuda is None else cuda
    e0, e1 = cuda.Event(enable_timing=True), cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(k):
        for dst, src in zip(io[0], host_ins):
            dst.copy_(src, non_blocking=True)
        step(io=io)
        for h, t in zip(hosts, io[1]):
            h.copy_(t, non_blocking=True)
    e1.record(stream)
    cuda.synchronize()
    return e0.elapsed_time(e1) / k


def e2e_overlapped_ms(k, step, sets, host_ins, hosts, stream, s_in, s_out, cuda=None):
    """ms per step when step i copies its inputs in on s_in and its results
    out on s_out, through buffer set i % 2 (sets[b] = (device inputs, device
    results), hosts[b] = host result buffers), so that step i's work overlaps
    the copy-in of step i + 1 and the copy-out of step i - 1. Events order the
    reuse of a set: step i + 2's copy-in waits until step i has run, and step
    i + 2 waits until step i's results have been copied out. The timed region
    ends once every copy-out has finished."""
    cuda = torch.cuda if cuda is None else cuda
    in_ready = [cuda.Event() for _ in range(2)]
    ran = [cuda.Event() for _ in range(2)]
    out_done = [cuda.Event() for _ in range(2)]
    e0, e1 = cuda.Event(enable_timing=True), cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(k):
        b = i & 1
        ins, outs = sets[b]
        if i >= 2:
            s_in.wait_event(ran[b])
        with cuda.stream(s_in):
            for dst, src in zip(ins, host_ins):
                dst.copy_(src, non_blocking=True)
        in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        if i >= 2:
            stream.wait_event(out_done[b])
        step(io=sets[b])
        ran[b].record(stream)
        s_out.wait_event(ran[b])
        with cuda.stream(s_out):
            for h, t in zip(hosts[b], outs):
                h.copy_(t, non_blocking=True)
        out_done[b].record(s_out)
    for b in range(min(2, k)):
        stream.wait_event(out_done[b])
    e1.record(stream)
    cuda.synchronize()
    return e0.elapsed_time(e1) / k


# ----------------------------------------------------------------------------- peaks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ----------------------------------------------------------------------------- oracle (CPU) timing
def cpu_sample(w, Q, K, V, alpha, n_qblocks=4, heads=1, variant="bf16", router=None, dO=None):
    """Times the oracle on a bounded sample: the mask of `heads` head(s) and the
    attention of `n_qblocks` query blocks of the first head, and returns
    (effective FLOP/s, description, threads)."""
    import oracle

    oracle.build()
    Qh, Kh, Vh = Q[:1, :heads].contiguous(), K[:1, :heads].contiguous(), V[:1, :heads].contiguous()
    t0 = time.perf_counter()
    if router is None:
        idx, cnt, _ = oracle.mask(Qh, Kh, w.bq, w.bk, w.topk, w.topp)
    else:
        Wq, Wk = (W[:heads].numpy() for W in router)
        idx, cnt, _ = oracle.mask_router(Qh, Kh, w.bq, w.bk, Wq, Wk, w.topk, w.topp)
    t_mask = time.perf_counter() - t0
    qbs = np.linspace(0, w.nqb - 1, n_qblocks).astype(np.int64)
    rows = np.concatenate([np.arange(qb * w.bq, min(w.N, qb * w.bq + w.bq)) for qb in qbs]).astype(np.int64)
    mode = variant if variant in ("q8", "bwd") else ("sla2" if w.sla2 else "sparse")
    t0 = time.perf_counter()
    if mode == "bwd":
        # forward and backward of the sampled rows' dQ (the sparse + linear mix on SLA2 workloads)
        oracle.attention_bwd(Qh, Kh, Vh, dO[:1, :heads].contiguous(), w.bq, w.bk, idx, cnt,
                             alpha=alpha[:heads].numpy() if w.sla2 else None, mode="sla2" if w.sla2 else "sparse",
                             rows=rows, kblocks=np.zeros(0, np.int64))
    elif mode == "q8":
        oracle.attention_q8_rows(Qh, Kh, Vh, w.bq, w.bk, idx, cnt, rows)
    else:
        oracle.attention_rows(Qh, Kh, Vh, w.bq, w.bk, idx, cnt, alpha[:heads].numpy(), mode=mode, rows=rows)
    t_attn = time.perf_counter() - t0
    # Credit only the products the sample computes. The backward sample takes
    # dQ of its rows: the forward's two products plus the backward's S, dP and
    # dQ (its dK and dV products are not sampled), 2.5 times the forward's
    # kept-block FLOPs; the GPU step's 3.5 adds dV and dK.
    flops = 0.0
    for qb in qbs:
        nrows = min(w.bq, w.N - qb * w.bq)
        keys = sum(min(w.bk, w.N - int(J) * w.bk) for J in idx[0, 0, qb, : cnt[0, 0, qb]])
        flops += 4.0 * w.d * nrows * keys * (2.5 if mode == "bwd" else 1.0)
    # the mask's time is charged pro rata to the sampled query blocks
    t = t_attn + t_mask * (len(qbs) / (w.nqb * heads))
    desc = (f"oracle {'router ' if router is not None else ''}mask of {heads} head(s) ({t_mask:.2f} s, charged pro rata) + {mode} attention of "
            f"{len(qbs)} query blocks x {w.bq} rows ({t_attn:.2f} s); {w.name} workload")
    return flops / t, desc, 1


# ----------------------------------------------------------------------------- timing
L2_FLUSH_BYTES = 256 << 20  # written between timed steps: twice the 126 MB L2
NOMINAL_BF16_TFLOPS = 2250.0


def timed_steps(step, steps, stream, flush, cuda=None):
    """Runs `steps` steps, each bracketed by its own CUDA events on the
    launching stream, with the L2 flushed (a buffer larger than L2 written)
    before each step, outside its events. step(ev_a, ev_b) records ev_a / ev_b
    around the library call it times (the attention span). Returns the
    per-step and per-span milliseconds."""
    cuda = torch.cuda if cuda is None else cuda
    evs = [tuple(cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(steps)]
    for e0, ea, eb, e1 in evs:
        flush.zero_()
        e0.record(stream)
        step(ea, eb)
        e1.record(stream)
    cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, _, _, e1 in evs], [ea.elapsed_time(eb) for _, ea, eb, _ in evs]


def roofline_peak(achieved, clocks, ratio=1.0):
    """The measured bf16 peak a kernel timed alone is held to: the burst figure
    when the SM clock held its maximum (or was not sampled), the sustained
    (power-capped) one otherwise; both fractions and the nominal one are
    returned. ratio scales the bf16 peaks for another operand type."""
    peaks, peak_kind = measured_peaks()
    burst = float(peaks["bf16_tflops"]) * ratio
    sustained = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])) * ratio
    at_max = clocks_at_max(clocks)
    peak = burst if at_max else sustained
    desc = (f"{peak_kind} bf16 {'burst' if at_max else 'sustained'}"
            + (" (SM clock at max during the timed region)" if at_max and clocks.get("samples") else
               " (no clock samples: burst)" if at_max else " (SM clock below max during the timed region)")
            + (f" x {ratio:g} (nominal 8-bit / bf16 ratio)" if ratio != 1.0 else ""))
    fracs = {"frac_vs_burst": achieved / burst, "frac_vs_sustained": achieved / sustained,
             "frac_vs_nominal": achieved / (NOMINAL_BF16_TFLOPS * ratio)}
    return peak, fracs, desc


# The other shapes the metric is quoted at: (workload, library call).
OTHER_WORKLOADS = (("720p", "sparge_attn_fwd"), ("720p", "sla2_attn_fwd"), ("sla2_480p", "sla2_attn_fwd"))


def time_other_workloads(args, dev, stream, flush):
    """Mask + attention steps of the other headline shapes on this GPU, timed
    like the main line (per-step events, L2 flushed between steps)."""
    from block_sparse_attention_pooled_b200 import sparge

    out = {}
    cache = {}
    for name, call in OTHER_WORKLOADS:
        w = synth.WORKLOADS[name]
        if name not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            Qh, Kh, Vh, alpha_h = synth.make_workload(w)
            cache[name] = (Qh.to(dev), Kh.to(dev), Vh.to(dev), alpha_h.to(dev))
        Q, K, V, alpha = cache[name]
        shape = sparge.make_shape(Q, w.bq, w.bk)
        B, H, N, d = Q.shape
        ws_mask = torch.empty(sparge.workspace_bytes(sparge.OP_MASK, shape), dtype=torch.uint8, device=dev)
        op = sparge.OP_SLA2 if call == "sla2_attn_fwd" else sparge.OP_ATTN
        ws = torch.empty(max(1, sparge.workspace_bytes(op, shape)), dtype=torch.uint8, device=dev)
        kv_idx = torch.empty((B, H, w.nqb, w.nkb), dtype=torch.int32, device=dev)
        kv_cnt = torch.empty((B, H, w.nqb), dtype=torch.int32, device=dev)
        O = torch.empty_like(Q)

        def step(ev_a=None, ev_b=None):
            sparge.sparge_mask(Q, K, w.bq, w.bk, w.topk, w.topp, kv_idx=kv_idx, kv_cnt=kv_cnt, workspace=ws_mask)
            if ev_a is not None:
                ev_a.record(stream)
            if call == "sla2_attn_fwd":
                sparge.sla2_attn_fwd(Q, K, V, kv_idx, kv_cnt, alpha, w.bq, w.bk, O=O, workspace=ws)
            else:
                sparge.sparge_attn_fwd(Q, K, V, kv_idx, kv_cnt, w.bq, w.bk, O=O, workspace=ws)
            if ev_b is not None:
                ev_b.record(stream)

        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize()
        assert sparge.device_status() == 0, "a kernel gave up a bounded wait"
        flops = kept_flops(kv_idx, kv_cnt, N, d, w.bq, w.bk)
        with NvmlClockSampler(_smi_id(dev)) as clk:
            step_ms, attn_ms = timed_steps(step, args.steps, stream, flush)
        clocks = clk.summary()
        ms = sum(step_ms) / len(step_ms)
        span = sum(attn_ms) / len(attn_ms)
        achieved = flops / (span * 1e-3) / 1e12
        peak, fracs, desc = roofline_peak(achieved, clocks)
        kernel = f"attn_fwd_kernel<{d}, {1 if call == 'sla2_attn_fwd' else 0}>"
        capture_key = name + ("_sparse" if call == "sparge_attn_fwd" and w.sla2 else "")
        out[f"{name}:{call}"] = {
            "config": {"B": w.B, "H": w.H, "N": w.N, "d": w.d, "bq": w.bq, "bk": w.bk, "topk": w.topk,
                       "topp": w.topp, "alpha": "U[0.6,1] per head" if call == "sla2_attn_fwd" else 1.0},
            "ms_per_step": ms, "ms_per_step_median": statistics.median(step_ms),
            "kept_tflops": flops / (ms * 1e-3) / 1e12, "kept_fraction": flops / (4.0 * B * H * N * N * d),
            "mask_ms": ms - span, "attn_ms": span,
            "roofline": {"kernel": kernel, "timed_span": call, "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "peak_kind": desc, **fracs,
                         "ncu_tensor_pipe_active_pct": tensor_pipe_pct(capture_key, kernel),
                         "traffic": dram_traffic(capture_key, kernel)},
            "clocks": clocks,
        }
        del ws_mask, ws, kv_idx, kv_cnt, O
    cache.clear()
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- mask regimes
def regime_settings():
    """(rule, top-k, top-p) of the mask-regime sweep: Top-k alone, Top-p alone
    and the hybrid over the sweep grid."""
    out = [("top-k", k, 0.0) for k in synth.SWEEP_TOPK]
    out += [("top-p", 0.0, p) for p in synth.SWEEP_TOPP]
    out += [("hybrid", k, p) for k in synth.SWEEP_TOPK for p in synth.SWEEP_TOPP]
    return out


def regime_rows(w, Q, K, V, settings, dev, check_rows=64):
    """For each (rule, k, p): the kept fraction of the mask sparge_mask builds
    and the error of sparge_attn_fwd on it against dense attention (the same
    kernel with every block kept). The dense reference is first checked
    against the oracle's dense attention on sampled rows. Returns (rows,
    dense_check)."""
    import oracle
    from block_sparse_attention_pooled_b200 import sparge

    B, H, N, d = Q.shape
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    shape = sparge.make_shape(Qd, w.bq, w.bk)
    ws_mask = torch.empty(sparge.workspace_bytes(sparge.OP_MASK, shape), dtype=torch.uint8, device=dev)
    ws_attn = torch.empty(sparge.workspace_bytes(sparge.OP_ATTN, shape), dtype=torch.uint8, device=dev)
    all_idx = torch.arange(w.nkb, dtype=torch.int32, device=dev).expand(B, H, w.nqb, w.nkb).contiguous()
    all_cnt = torch.full((B, H, w.nqb), w.nkb, dtype=torch.int32, device=dev)
    Od = sparge.sparge_attn_fwd(Qd, Kd, Vd, all_idx, all_cnt, w.bq, w.bk, workspace=ws_attn)
    torch.cuda.synchronize()
    rng = np.random.default_rng(w.seed)
    rows = np.sort(rng.choice(B * H * N, size=check_rows, replace=False)).astype(np.int64)
    ref, _ = oracle.attention_rows(Q, K, V, w.bq, w.bk, mode="dense", rows=rows)
    got = Od.float().cpu().numpy().reshape(-1, d)[rows].astype(np.float64)
    err = np.abs(got - ref)
    dense_check = {"rows": int(len(rows)), "max_abs": float(err.max()),
                   "mean_rel_l1": float(err.sum() / np.abs(ref).sum())}
    Odf = Od.double()
    den_l1, den_l2 = float(Odf.abs().sum()), float(Odf.norm())
    dense_flops = 4.0 * B * H * N * N * d
    out = []
    for rule, k, p in settings:
        kv_idx, kv_cnt = sparge.sparge_mask(Qd, Kd, w.bq, w.bk, k, p, workspace=ws_mask)
        O = sparge.sparge_attn_fwd(Qd, Kd, Vd, kv_idx, kv_cnt, w.bq, w.bk, workspace=ws_attn)
        diff = O.double() - Odf
        out.append({"rule": rule, "topk": k, "topp": p,
                    "kept_fraction": kept_flops(kv_idx, kv_cnt, N, d, w.bq, w.bk) / dense_flops,
                    "mean_kept_blocks": float(kv_cnt.double().mean()),
                    "rel_l1_vs_dense": float(diff.abs().sum()) / den_l1,
                    "rel_l2_vs_dense": float(diff.norm()) / den_l2,
                    "max_abs_vs_dense": float(diff.abs().max()),
                    "cos_sim_vs_dense": float((O.double() * Odf).sum()) / (float(O.double().norm()) * den_l2)})
    assert sparge.device_status() == 0, "a kernel gave up a bounded wait"
    return out, dense_check


def run_regime_report(args):
    """The mask-regime report: for the flat and the peaked sweep workloads,
    the kept fraction and the error against dense attention of Top-k alone,
    Top-p alone and their union. Prints a markdown table and one JSON line."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    report = {"report": "mask regimes", "workloads": {}}
    lines = ["| distribution | rule | top-k | top-p | kept fraction | mean kept blocks | rel. L1 error | "
             "rel. L2 error | max abs error | cosine similarity |", "|---|---|---|---|---|---|---|---|---|---|"]
    for name in ("sweep_flat", "sweep_peaked"):
        w = synth.WORKLOADS[name]
        Q, K, V, _ = synth.make_workload(w)
        rows, check = regime_rows(w, Q, K, V, regime_settings(), dev)
        report["workloads"][name] = {"dense_check_vs_oracle": check, "rows": rows,
                                     "config": {"B": w.B, "H": w.H, "N": w.N, "d": w.d, "bq": w.bq, "bk": w.bk,
                                                "s": w.s}}
        for r in rows:
            lines.append(f"| {name.split('_')[1]} (s = {w.s}) | {r['rule']} | {r['topk']:.2f} | {r['topp']:.2f} | "
                         f"{r['kept_fraction']:.4f} | {r['mean_kept_blocks']:.1f} | {r['rel_l1_vs_dense']:.4f} | "
                         f"{r['rel_l2_vs_dense']:.4f} | {r['max_abs_vs_dense']:.3f} | {r['cos_sim_vs_dense']:.4f} |")
        del Q, K, V
        torch.cuda.empty_cache()
    print("\n".join(lines), flush=True)
    print(json.dumps(report), flush=True)


# ----------------------------------------------------------------------------- runs
def run_reference(args, w, rank, world):
    if rank != 0:
        return
    Q, K, V, alpha = synth.make_workload(w, heads=[(0, 0)])
    router = synth.make_router(w.H, w.d, args.router, seed=w.seed) if args.router else None
    dO = synth.make_dout(w.B, w.H, w.N, w.d, seed=w.seed, heads=[(0, 0)]) if args.variant == "bwd" else None
    vals = []
    for i in range(args.warmup + args.steps):
        v, desc, cores = cpu_sample(w, Q, K, V, alpha, n_qblocks=4, variant=args.variant, router=router, dO=dO)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "bq": w.bq, "bk": w.bk,
                   "topk": w.topk, "topp": w.topp,
                   "path": "oracle: low-bit sparse branch" if args.variant == "q8" else
                           "oracle: sparse branch forward + backward (dQ of the sampled rows)" if args.variant == "bwd" else
                           ("oracle: sparse + linear mix" if w.sla2 else "oracle: sparse branch"),
                   "router": args.router or None},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, w, rank, world, local_rank):
    from block_sparse_attention_pooled_b200 import sparge

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    seedw = synth.Workload(**{**w.__dict__, "seed": w.seed + rank})
    Qh, Kh, Vh, alpha_h = synth.make_workload(seedw)
    pin = lambda t: t.pin_memory()  # noqa: E731
    Qh, Kh, Vh = pin(Qh), pin(Kh), pin(Vh)
    Q, K, V, alpha = Qh.to(dev), Kh.to(dev), Vh.to(dev), alpha_h.to(dev)
    B, H, N, d = Q.shape
    shape = sparge.make_shape(Q, w.bq, w.bk)
    router_h = synth.make_router(H, d, args.router, seed=w.seed) if args.router else None
    mask_op = sparge.OP_MASK_ROUTER if router_h is not None else sparge.OP_MASK
    ws_mask = torch.empty(max(1, sparge.workspace_bytes(mask_op, shape)), dtype=torch.uint8, device=dev)
    Wq, Wk = (router_h[0].to(dev), router_h[1].to(dev)) if router_h is not None else (None, None)
    q8 = args.variant == "q8"
    bwd = args.variant == "bwd"
    sla2 = w.sla2 and not q8  # the low-bit variant runs the sparse branch alone
    n_sla2 = sparge.workspace_bytes(sparge.OP_SLA2, shape) if sla2 else 0
    ws_sla2 = torch.empty(max(1, n_sla2), dtype=torch.uint8, device=dev)
    n_q8 = sparge.workspace_bytes(sparge.OP_ATTN_Q8, shape) if q8 else 0
    ws_q8 = torch.empty(max(1, n_q8), dtype=torch.uint8, device=dev)
    kv_idx = torch.empty((B, H, w.nqb, w.nkb), dtype=torch.int32, device=dev)
    kv_cnt = torch.empty((B, H, w.nqb), dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    O_fwd = O
    ws_attn = torch.empty(sparge.workspace_bytes(sparge.OP_ATTN, shape), dtype=torch.uint8, device=dev)
    if bwd:
        dOh = pin(synth.make_dout(w.B, w.H, w.N, w.d, seed=w.seed + rank))
        dO = dOh.to(dev)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
        ws_bwd = torch.empty(sparge.workspace_bytes(sparge.OP_SLA2_BWD if sla2 else sparge.OP_ATTN_BWD, shape),
                             dtype=torch.uint8, device=dev)
        dalpha = torch.empty(H, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    # One set of device buffers: the step's inputs (read) and results (written).
    io0 = ([Q, K, V] + ([dO] if bwd else []), ([dQ, dK, dV] + ([dalpha] if sla2 else [])) if bwd else [O])

    def step(ev_a=None, ev_b=None, io=None):
        ins, outs = io0 if io is None else io
        Q, K, V = ins[0], ins[1], ins[2]
        if bwd:
            dO, (dQ, dK, dV) = ins[3], outs[:3]
            dalpha_ = outs[3] if sla2 else None
            O = O_fwd  # the forward's output feeds the backward only
        else:
            O = outs[0]
        if Wq is not None:
            sparge.sparge_mask_router(Q, K, Wq, Wk, w.bq, w.bk, w.topk, w.topp, kv_idx=kv_idx, kv_cnt=kv_cnt,
                                      workspace=ws_mask)
        else:
            sparge.sparge_mask(Q, K, w.bq, w.bk, w.topk, w.topp, kv_idx=kv_idx, kv_cnt=kv_cnt, workspace=ws_mask)
        if bwd:
            if sla2:
                sparge.sla2_attn_fwd(Q, K, V, kv_idx, kv_cnt, alpha, w.bq, w.bk, O=O, workspace=ws_sla2)
            else:
                sparge.sparge_attn_fwd(Q, K, V, kv_idx, kv_cnt, w.bq, w.bk, O=O, lse=lse, workspace=ws_attn)
            if ev_a is not None:
                ev_a.record(stream)
            if sla2:
                sparge.sla2_attn_bwd(Q, K, V, kv_idx, kv_cnt, alpha, dO, w.bq, w.bk, dQ, dK, dV, dalpha_,
                                     workspace=ws_bwd)
            else:
                sparge.sparge_attn_bwd(Q, K, V, kv_idx, kv_cnt, O, lse, dO, w.bq, w.bk, dQ, dK, dV, workspace=ws_bwd)
            if ev_b is not None:
                ev_b.record(stream)
            return
        if ev_a is not None:
            ev_a.record(stream)
        if q8:
            sparge.sparge_attn_fwd_q8(Q, K, V, kv_idx, kv_cnt, w.bq, w.bk, O=O, workspace=ws_q8)
        elif sla2:
            sparge.sla2_attn_fwd(Q, K, V, kv_idx, kv_cnt, alpha, w.bq, w.bk, O=O, workspace=ws_sla2)
        else:
            sparge.sparge_attn_fwd(Q, K, V, kv_idx, kv_cnt, w.bq, w.bk, O=O, workspace=ws_attn)
        if ev_b is not None:
            ev_b.record(stream)

    n_order = sparge.order_launches(shape)
    launches_per_step = ((sparge.ROUTER_LAUNCHES if Wq is not None else sparge.MASK_LAUNCHES) +
                         (sparge.Q8_LAUNCHES if q8 else sparge.SLA2_LAUNCHES if sla2 else sparge.ATTN_LAUNCHES) +
                         n_order + ((sparge.SLA2_BWD_LAUNCHES if sla2 else sparge.BWD_LAUNCHES) + n_order
                                    if bwd else 0))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert sparge.device_status() == 0, "a kernel gave up a bounded wait"
    flops = kept_flops(kv_idx, kv_cnt, N, d, w.bq, w.bk)
    dense_flops = 4.0 * B * H * N * N * d
    # A training step counts the forward's kept-block FLOPs once and the
    # backward's five products (S, dP, dV, dK, dQ) as 2.5 times them.
    step_flops = flops * (3.5 if bwd else 1.0)
    span_flops = flops * (2.5 if bwd else 1.0)

    # ---- device-timed region (inputs resident in HBM; L2 flushed between steps)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with NvmlClockSampler(_smi_id(dev)) as clk:
        step_ms, attn_ms = timed_steps(step, args.steps, stream, flush)
    if world > 1:
        torch.distributed.barrier()
    ms_step = max_over_ranks(sum(step_ms) / len(step_ms), world, dev)
    value = step_flops * world / (ms_step * 1e-3) / 1e12
    attn_avg = sum(attn_ms) / len(attn_ms)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        host_ins = [Qh, Kh, Vh] + ([dOh] if bwd else [])
        h2d = sum(t.numel() * t.element_size() for t in host_ins)
        d2h = sum(t.numel() * t.element_size() for t in io0[1])
        ksteps = max(3, args.steps // 4)
        hosts0 = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in io0[1]]

        e2e_serial_ms(2, step, io0, host_ins, hosts0, stream)
        e2e_serial = max_over_ranks(e2e_serial_ms(ksteps, step, io0, host_ins, hosts0, stream), world, dev)
        pipe, pipe_err = float("inf"), None
        try:
            sets = [io0, ([torch.empty_like(t) for t in io0[0]], [torch.empty_like(t) for t in io0[1]])]
            hosts = [hosts0, [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in io0[1]]]
            s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
            e2e_overlapped_ms(2, step, sets, host_ins, hosts, stream, s_in, s_out)
            pipe = e2e_overlapped_ms(ksteps, step, sets, host_ins, hosts, stream, s_in, s_out)
        except Exception as exc:  # the serial figure stands; the line says why
            torch.cuda.synchronize()
            pipe_err = f"{type(exc).__name__}: {exc}"[:300]
        pipe = max_over_ranks(pipe, world, dev)  # every rank takes this collective
        overlapped = math.isfinite(pipe)
        e2e_ms = pipe if overlapped else e2e_serial
        e2e = {"value": step_flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "copies": ("overlapped: each step's inputs copied in on one stream and its results out on another, "
                          "two buffer sets, while the neighbouring step runs" if overlapped else
                          "serial: copy in, step, copy out on one stream"),
               "serial_ms_per_step": e2e_serial,
               "serial_value": step_flops * world / (e2e_serial * 1e-3) / 1e12}
        if pipe_err is not None:
            e2e["overlap_error"] = pipe_err
    assert sparge.device_status() == 0, "a kernel gave up a bounded wait"

    if rank != 0:
        return
    clocks = clk.summary()
    achieved = span_flops / (attn_avg * 1e-3) / 1e12
    peak, fracs, peak_desc = roofline_peak(achieved, clocks, 2.0 if q8 else 1.0)
    # The timed span is one library call: tile order + attn_fwd_kernel for the
    # pure sparse path; tile order, linear summaries, linear_out and
    # attn_fwd_kernel<128, 1> for the sparse + linear mix.
    kernel_name = "attn_q8_kernel" if q8 else (f"attn_fwd_kernel<{d}, 1>" if sla2 else f"attn_fwd_kernel<{d}, 0>")
    if bwd:
        kernel_name = "attn_bwd_dq_kernel + attn_bwd_dkdv_kernel"
    span = (("sla2_attn_bwd (12-13 launches: forward pieces, row pass, gradient summaries, transposed mask, dQ, "
             "dK/dV sparse and linear parts)" if sla2 else
             "sparge_attn_bwd (D_i, transposed mask, tile order when used, dQ, dK/dV)") if bwd else
            "sparge_attn_fwd_q8 (codes, V codes, tile order when used, attention)" if q8 else
            "sla2_attn_fwd (4-5 launches)" if sla2 else "sparge_attn_fwd (tile order when used, attention)")
    # Counters were captured with the plain mask; a router mask keeps other tiles.
    # Captures are stored per workload and path: "<name>", "<name>_q8", and
    # "<name>_sparse" for the sparse branch alone on a sparse + linear workload.
    named = synth.WORKLOADS.get(w.name)
    key = w.name + ("_q8" if q8 else "_sparse" if named is not None and named.sla2 and not sla2 else "")
    partial = args.router or bwd or getattr(args, "heads", 0)  # captures were taken on the full plain path
    traffic = None if partial else dram_traffic(key, kernel_name)
    tensor_pct = None if partial else tensor_pipe_pct(key, kernel_name)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, desc, cores = cpu_sample(w, Qh, Kh, Vh, alpha_h, variant=args.variant, router=router_h,
                                    dO=dOh if bwd else None)
        cpu = {"value": v / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8+e4m3" if q8 else "bf16",
        "data": "synthetic (seeded video-shaped Q/K/V, see synth.py)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "bq": w.bq, "bk": w.bk,
                   "topk": w.topk, "topp": w.topp, "alpha": "U[0.6,1] per head" if sla2 else 1.0,
                   "path": "sparge_attn_fwd_q8" if q8 else
                           ("sla2_attn_fwd + sla2_attn_bwd" if sla2 else "sparge_attn_fwd + sparge_attn_bwd") if bwd else
                           ("sla2_attn_fwd" if sla2 else "sparge_attn_fwd"),
                   "flops": ("kept-block FLOPs x 3.5 (forward + backward; the linear branch's work is not counted)"
                             if bwd else "kept-block FLOPs"),
                   "mask": f"sparge_mask_router (dr {args.router})" if args.router else "sparge_mask",
                   "l2": (f"L2 flushed between steps (a {L2_FLUSH_BYTES >> 20} MB buffer written outside each "
                          f"step's events); inputs also larger than L2 ({3 * Q.numel() * 2 / 1e6:.0f} MB of Q/K/V "
                          f"per rank)"),
                   "parallelism": f"independent replicas x{world}"},
        "timing": ("CUDA events around each step on the launching stream; ms_per_step = mean over the timed "
                   "steps (max over ranks)"),
        "ms_per_step_median": statistics.median(step_ms),
        "kept_fraction": flops / dense_flops,
        "dense_equiv_tflops": dense_flops * world / (ms_step * 1e-3) / 1e12,
        "attn_ms": attn_avg,
        "attn_ms_median": statistics.median(attn_ms),
        "mask_ms": ms_step - attn_avg,
        "roofline": {"kernel": kernel_name, "timed_span": span, "bound": "tensor", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "peak_kind": peak_desc, **fracs,
                     "ncu_tensor_pipe_active_pct": tensor_pct, "traffic": traffic},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    if (w.name == "480p" and world == 1 and not getattr(args, "no_extra", False) and args.variant == "bf16"
            and not args.router):
        # The other headline shapes, timed in the same process (no e2e, no CPU leg).
        del Q, K, V, O, ws_mask, ws_sla2, ws_q8, ws_attn, io0
        torch.cuda.empty_cache()
        line["per_workload"] = time_other_workloads(args, dev, stream, flush)
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    w = synth.WORKLOADS[args.workload]
    if args.heads:
        # The first heads of batch 0: the generator seeds every (batch, head)
        # on its own, so these are the same tensors as in the full workload.
        w = synth.Workload(**{**w.__dict__, "B": 1, "H": min(args.heads, w.H)})
    if args.sparse_only:
        w = synth.Workload(**{**w.__dict__, "sla2": False})
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        backend = "gloo" if args.impl == "reference" else "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    if args.report == "regimes":
        run_regime_report(args)
        return
    try:
        if args.impl == "reference":
            run_reference(args, w, rank, world)
        else:
            run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
