"""Benchmark of the microscaling-FP4 attention forward on B200.

One step = one whole forward (K mean + quantization of Q, K, V + fused FP4 attention) over
one batch of the long-sequence workload (B=1, H=24, N=32768, D=128, bf16, non-causal).
Metric: attention TOPS = 4*B*H*N^2*D (halved when causal) per second, whole job over all
ranks. The inputs (576 MiB) exceed the 126 MB L2, so no flush runs between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Under torchrun the job is one problem of world x B*H (batch, head) pairs split across the
ranks by microscaling_fp4_quantized_b200.shard.head_slice: rank r holds and computes its
own contiguous slice (the workload's shape, drawn with the rank's own seed). The pairs are
independent, so there is no data-path collective (weak scaling: the work per GPU is
fixed); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from microscaling_fp4_quantized_b200 import workloads  # noqa: E402

METRIC = "FP4 attention fwd TOPS (4·B·H·N²·D/s) at N=32K D=128; % of B200 FP4 peak"
UNIT = "TOPS"
DEFAULT_WORKLOAD = workloads.LONG.name
FP4_NOMINAL_TFLOPS = 9000.0
FP4_PER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor throughput on B200 (9 : 2.25 PFLOP/s)


def fp4_peak(peaks: dict, basis: str, probe=None, b8: bool = False):
    """Roofline denominator of the attention kernel (timed per launch, in isolation: the
    burst figure). FP4: the measured bf16 burst rate x 4 (nominal FP4 : BF16), or the
    measured rate of the FP4 instruction itself (sage.mma_rate) when that is higher;
    8-bit: bf16 burst x 2. Returns (TFLOP/s, description)."""
    burst = peaks.get("bf16_tflops", peaks.get("bf16_tflops_sustained"))
    ratio = 2.0 if b8 else FP4_PER_BF16
    peak = ratio * burst
    how = f"{basis} bf16 burst {burst} TFLOP/s x {ratio:g} (nominal {'8-bit' if b8 else 'FP4'}:BF16)"
    if probe is not None and not b8 and probe["tflops"] > peak:
        peak = probe["tflops"]
        how = (f"measured FP4 tensor-core rate (tcgen05 mxf4nvf4 M128 N{probe['n']} K64, "
               f"{probe['ctas']} CTAs), above the bf16-derived {ratio * burst:.0f}")
    return peak, how


def quant_algorithmic_bytes(wl, b8=False):
    """Bytes the quantization of a dense problem with K smoothing must move: Q, K and V
    read once, K read again after its mean (8-bit: V again after its channel scales), and
    the quantized tensors written (FP4: half a byte per element plus one scale byte per 16
    elements; 8-bit: one byte per element, scales negligible). 2-byte inputs."""
    E = wl.B * wl.H * wl.N * wl.D
    if b8:
        return 5 * E * 2 + 3 * E
    return 4 * E * 2 + 3 * E * (0.5 + 1.0 / 16.0)


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return j, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi samples (200 ms) during the timed region."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = f"/tmp/sage_clocks_{os.getpid()}.csv"

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax.append(float(parts[1]))
                    power.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[4:8]):
                    if val.lower().startswith("active"):
                        reasons.add(nm)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


def _attn_traffic(wl, b8=False):
    """DRAM bytes per attention launch from the committed ncu capture, or None when the
    kernel sources (hashed in the record's order) have changed since the capture, or
    no capture exists."""
    import hashlib
    name = "attn8_fwd_kernel_traffic.json" if b8 else "attn_fp4_fwd_kernel_traffic.json"
    try:
        with open(os.path.join(ROOT, "profiles", name)) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for src in rec.get("sources") or [rec["source"]]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        sha = h.hexdigest()
    except Exception:
        return None, "no capture"
    if not sha.startswith(rec["source_sha256_prefix"]):
        return None, "kernel changed since the capture"
    cap = workloads.by_name(rec["captured_workload"])
    if cap.name == wl.name:
        return float(rec["dram_bytes_per_launch"]), f"ncu capture of {cap.name}"
    # attention traffic is the quantized inputs plus the output: it scales with B*H*N
    scale = (wl.B * wl.H * wl.N) / (cap.B * cap.H * cap.N)
    return float(rec["dram_bytes_per_launch"]) * scale, f"ncu capture of {cap.name}, scaled by B*H*N"


TRAFFIC_SOURCES = {
    False: ("attn_fp4_fwd_kernel", "attn_fp4_fwd_kernel_traffic.json",
            ["microscaling_fp4_quantized_b200/csrc/attn_fp4_kernel.cuh",
             "microscaling_fp4_quantized_b200/csrc/attn_common.cuh",
             "microscaling_fp4_quantized_b200/csrc/sm100_ptx.cuh",
             "microscaling_fp4_quantized_b200/csrc/sage_internal.h"]),
    True: ("attn8_fwd_kernel", "attn8_fwd_kernel_traffic.json",
           ["microscaling_fp4_quantized_b200/csrc/attn8_fwd.cu",
            "microscaling_fp4_quantized_b200/csrc/attn_common.cuh",
            "microscaling_fp4_quantized_b200/csrc/sm100_ptx.cuh",
            "microscaling_fp4_quantized_b200/csrc/sage_internal.h"]),
}

_BYTE_UNITS = {"byte": 1.0, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "tbyte": 1e12,
               "kibyte": 1024.0, "mibyte": 1024.0 ** 2, "gibyte": 1024.0 ** 3}


def write_traffic_record(csv_path: str, wl, b8: bool) -> dict:
    """Traffic record of the attention kernel from an ncu CSV of one launch
    (--metrics dram__bytes_read.sum,dram__bytes_write.sum --csv), hashed over the kernel's
    sources as they are now: run it right after the capture, on the same tree."""
    import csv
    import hashlib
    kernel, name, sources = TRAFFIC_SOURCES[b8]
    total, launches = {}, set()
    with open(csv_path, newline="") as f:
        rows = [r for r in csv.reader(f)]
    head = next(i for i, r in enumerate(rows) if "Metric Name" in r)
    cols = rows[head]
    ki, mi, ui, vi, ii = (cols.index(c) for c in ("Kernel Name", "Metric Name", "Metric Unit", "Metric Value", "ID"))
    for r in rows[head + 1:]:
        if len(r) <= vi or kernel not in r[ki] or r[mi] not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        launches.add(r[ii])
        total[r[ii]] = total.get(r[ii], 0.0) + float(r[vi].replace(",", "")) * _BYTE_UNITS[r[ui].strip().lower()]
    if not total:
        raise RuntimeError(f"no {kernel} DRAM metrics in {csv_path}")
    h = hashlib.sha256()
    for src in sources:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    rec = {"kernel": kernel, "sources": sources, "source_sha256_prefix": h.hexdigest()[:16],
           "captured_workload": wl.name, "launches_captured": len(launches),
           "dram_bytes_per_launch": statistics.mean(total.values()),
           "note": "dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture (per launch); "
                   "written by bench.py --write-traffic from that capture's CSV; reported only while the "
                   "hash of the sources matches"}
    with open(os.path.join(ROOT, "profiles", name), "w") as f:
        json.dump(rec, f, indent=1)
    return rec


def max_over_ranks(value: float, dist, device) -> float:
    """The largest of the ranks' values (device times are reduced with MAX)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(ops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput in TOPS: every rank computes its slice of ops_per_rank."""
    return world * ops_per_rank / (ms_per_step * 1e-3) / 1e12


def cpu_oracle_rate(wl, budget_s: float, q=None, k=None, v=None):
    """Time the CPU oracle (as it stands) on a bounded sample of the workload: one head's
    quantization plus as many query rows as fit the budget; extrapolate to TOPS."""
    import numpy as np
    import oracle
    oracle.build()
    if q is None:
        small = workloads.Workload(wl.name, 1, 1, wl.N, wl.D, wl.causal, wl.dtype, wl.seed, wl.bias_sigma,
                                   wl.outliers)
        q, k, v = workloads.make_inputs(small)
    qh = q.reshape(-1, wl.N, wl.D)[:1].float().numpy()
    kh = k.reshape(-1, wl.N, wl.D)[:1].float().numpy()
    vh = v.reshape(-1, wl.N, wl.D)[:1].float().numpy()
    t0 = time.perf_counter()
    qz = oracle.quantize_qkv(qh, kh, vh)
    t_quant = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    rows_done, t_rows, n = 0, 0.0, 8
    ops_rows = 0.0
    while t_rows < budget_s and rows_done < wl.N:
        n = min(n, wl.N - rows_done)
        idx = rng.choice(wl.N, size=n, replace=False)
        rows = np.stack([np.zeros(n, np.int64), idx], 1)
        t0 = time.perf_counter()
        oracle.attn_emulated(qz, wl.causal, wl.sm_scale, Bk=128, rows=rows)
        dt = time.perf_counter() - t0
        t_rows += dt
        rows_done += n
        keys = (idx + 1) if wl.causal else np.full(n, wl.N)
        ops_rows += float((4.0 * keys * wl.D).sum())
        n = int(min(4 * n, max(8, n * (budget_s - t_rows) / max(dt, 1e-6))))
    per_head_ops = 4.0 * wl.N * wl.N * wl.D / (2 if wl.causal else 1)
    # time of a whole head = quantization + rows extrapolated by op count
    t_head = t_quant + t_rows * per_head_ops / ops_rows
    value = per_head_ops / t_head / 1e12
    sample = (f"1 of {wl.B * wl.H} heads: quantize N={wl.N} x D={wl.D} ({t_quant:.2f} s) + "
              f"{rows_done} query rows over all keys ({t_rows:.2f} s); extrapolated to the whole forward")
    return value, t_quant + t_rows, sample, oracle.num_threads()


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    budget = 2.0
    for _ in range(args.warmup):
        cpu_oracle_rate(wl, 0.5)
    vals, times = [], []
    sample = ""
    cores = 1
    for _ in range(args.steps):
        v, t, sample, cores = cpu_oracle_rate(wl, budget)
        vals.append(v)
        times.append(t)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": wl.describe(),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_sweep(args):
    """Every named configuration once (tiny, medium, causal LLM, long, the 16-point sweep):
    whole-forward and attention-only TOPS (CUDA events, median of 10 after 3 warm-ups),
    parity against the oracle on sampled rows of the first and last head, and the
    oracle's own rate on a bounded sample. One JSON line per configuration."""
    import numpy as np
    import oracle
    import microscaling_fp4_quantized_b200 as sage
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks, basis = _peaks()
    probe = sage.mma_rate(n=128)
    peak_tflops, peak_how = fp4_peak(peaks, basis, probe)
    print(json.dumps({"fp4_mma_probe": probe, "peak_tflops": peak_tflops, "peak_basis": peak_how}), flush=True)
    for wl in [workloads.TINY, workloads.MEDIUM, workloads.LLM_CAUSAL, workloads.LONG] + workloads.SWEEP:
        q, k, v = workloads.make_inputs(wl)
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        out = torch.empty_like(qd)
        plan = sage.Plan(wl.B, wl.H, wl.N, wl.D, wl.dtype, dev)
        for _ in range(3):
            plan.quantize(qd, kd, vd)
            plan.attention(out, causal=wl.causal, sm_scale=wl.sm_scale)
        torch.cuda.synchronize()
        whole, attn = [], []
        for _ in range(10):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record(stream)
            plan.quantize(qd, kd, vd)
            e[1].record(stream)
            plan.attention(out, causal=wl.causal, sm_scale=wl.sm_scale)
            e[2].record(stream)
            whole.append(e)
        torch.cuda.synchronize()
        ms = statistics.median(a.elapsed_time(c) for a, _, c in whole)
        ms_attn = statistics.median(b.elapsed_time(c) for _, b, c in whole)
        err = sage.device_error()
        BH = wl.B * wl.H
        heads = sorted({0, BH - 1})
        kmean = plan.k_mean[: BH * wl.D].reshape(BH, wl.D).cpu().numpy()
        f = lambda t: t.float().reshape(BH, wl.N, wl.D)[heads].numpy()  # noqa: E731
        qh, kh, vh = f(q), f(k), f(v)
        rng = np.random.default_rng(wl.seed)
        nr = wl.N if wl.N <= 256 else 32
        rr = np.unique(np.concatenate([[0, wl.N - 1], rng.choice(wl.N, nr, replace=False)]))
        rows = np.array([(i, r) for i in range(len(heads)) for r in rr], np.int64)
        em, _ = oracle.attention(qh, kh, vh, wl.causal, wl.sm_scale, Bk=128, rows=rows,
                                 kmean_in=kmean[heads])
        ex = oracle.attn_exact(qh, kh, vh, wl.causal, wl.sm_scale, rows=rows)
        og = out.float().reshape(BH, wl.N, wl.D)[heads].cpu().numpy()
        got = og[rows[:, 0], rows[:, 1]]
        m_em, m_ex = oracle.metrics(got, em), oracle.metrics(got, ex)
        cpu_val, _, sample, cores = cpu_oracle_rate(wl, args.cpu_budget_s)
        print(json.dumps({
            "workload": wl.name, "ops": wl.ops, "tops": wl.ops / (ms * 1e-3) / 1e12, "ms": ms,
            "attn_tops": wl.ops / (ms_attn * 1e-3) / 1e12, "attn_ms": ms_attn,
            "pct_of_fp4_peak": 100.0 * wl.ops / (ms * 1e-3) / 1e12 / peak_tflops,
            "attn_pct_of_fp4_peak": 100.0 * wl.ops / (ms_attn * 1e-3) / 1e12 / peak_tflops,
            "pct_of_nominal_fp4": 100.0 * wl.ops / (ms * 1e-3) / 1e12 / FP4_NOMINAL_TFLOPS,
            "vs_emulated": {"cos": m_em["cos"], "max_abs_over_max_v": m_em["max_abs"] / float(np.abs(vh).max())},
            "vs_exact": {"cos": m_ex["cos"], "rel_l1": m_ex["rel_l1"], "rmse": m_ex["rmse"]},
            "sampled_rows": int(len(rows)), "device_error_word": err,
            "cpu_oracle": {"value": cpu_val, "unit": UNIT, "cores": cores, "sample": sample}}), flush=True)
        del qd, kd, vd, out, plan
        torch.cuda.empty_cache()
    return 0


def time_e2e(sage, wl, q, k, v, dev, stream, steps, dist, world, precision="fp4"):
    """End to end through the public API: every step copies its inputs from pinned host
    memory, runs sage.attn, and copies the output back to pinned host memory.
    Pipelined (the headline): a copy-in stream, the compute stream and a copy-out stream
    with two device buffer sets, so step i+1's inputs and step i-1's output move while
    step i computes -- a serving loop's schedule. Serial (reported beside it): the three
    stages of each step back to back on one stream."""
    hin = [(q.pin_memory(), k.pin_memory(), v.pin_memory()) for _ in range(2)]
    hout = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(2)]
    din = [tuple(torch.empty(q.shape, dtype=q.dtype, device=dev) for _ in range(3)) for _ in range(2)]
    dout = [torch.empty(q.shape, dtype=q.dtype, device=dev) for _ in range(2)]
    ws_bytes = sage.problem_sizes(sage.sageattn_problem(din[0][0], din[0][1], din[0][2], dout[0], "HND", wl.causal,
                                                        wl.sm_scale, precision=precision))["workspace"]
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    def forward(a, b, c, o):
        return sage.sageattn(a, b, c, is_causal=wl.causal, sm_scale=wl.sm_scale, out=o, workspace=ws,
                             precision=precision)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def pipelined(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_c = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        s_in.wait_event(t0)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_c[i - 2])          # buffer set b free again
                for d, h in zip(din[b], hin[b]):
                    d.copy_(h, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])           # output buffer b read back
            forward(*din[b], dout[b])
            ev_c[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[i])
                hout[b].copy_(dout[b], non_blocking=True)
                ev_out[i].record(s_out)
        stream.wait_event(ev_out[n - 1])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1) / n

    def serial(n):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(n):
            a, b, c = (h.to(dev, non_blocking=True) for h in hin[0])
            o = forward(a, b, c, torch.empty_like(a))
            hout[0].copy_(o, non_blocking=True)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1) / n

    pipelined(3)
    serial(2)
    if dist is not None:
        dist.barrier()
    ms_p = max_over_ranks(pipelined(steps), dist, dev)
    ms_s = max_over_ranks(serial(steps), dist, dev)
    if sage.device_error() != 0:
        raise RuntimeError("device error word set in the end-to-end run")
    nbytes = q.numel() * q.element_size()
    return {"value": job_value(wl.ops, world, ms_p), "unit": UNIT, "ms_per_step": ms_p,
            "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
            "schedule": "pipelined: copy-in / compute / copy-out streams, two buffer sets",
            "serial": {"value": job_value(wl.ops, world, ms_s), "ms_per_step": ms_s}}


# Kernels per step: quantizer pass A (K statistics, Q, V^T), K mean, quantizer pass B (K),
# attention.
LAUNCHES_PER_STEP = 4


def time_general(sage, gw, dev, stream, warmup, steps, inputs=None):
    """Whole forward of a general workload through sageattn / sageattn_varlen with a
    preallocated workspace: CUDA events on the launching stream, median per step."""
    if inputs is None:
        x = workloads.make_general_inputs(gw, dev)
    else:
        x = {"q": inputs[0], "k": inputs[1], "v": inputs[2]}
    out = torch.empty(x["q"].shape, dtype=x["q"].dtype, device=dev)
    if gw.packed:
        pr = sage.sageattn_varlen_problem(x["q"], x["k"], x["v"], out, x["cu_seqlens_q"],
                                          x["cu_seqlens_k"], max(gw.lens_q), max(gw.lens_k),
                                          gw.causal, None, True, gw.gscale, gw.smooth_q, gw.precision)
    else:
        pr = sage.sageattn_problem(x["q"], x["k"], x["v"], out, gw.layout, gw.causal, None, True,
                                   gw.gscale, gw.smooth_q, gw.precision)
    ws = torch.empty(sage.problem_sizes(pr)["workspace"], dtype=torch.uint8, device=dev)

    def run():
        if gw.packed:
            sage.sageattn_varlen(x["q"], x["k"], x["v"], x["cu_seqlens_q"], x["cu_seqlens_k"],
                                 max(gw.lens_q), max(gw.lens_k), is_causal=gw.causal,
                                 gscale=gw.gscale, out=out, workspace=ws, smooth_q=gw.smooth_q,
                                 precision=gw.precision)
        else:
            sage.sageattn(x["q"], x["k"], x["v"], tensor_layout=gw.layout, is_causal=gw.causal,
                          gscale=gw.gscale, out=out, workspace=ws, smooth_q=gw.smooth_q,
                          precision=gw.precision)

    for _ in range(max(warmup, 3)):
        run()
    torch.cuda.synchronize()
    if sage.device_error() != 0:
        raise RuntimeError(f"device error word set running {gw.name}")
    ts = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        ts.append((e0, e1))
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in ts)
    return {"ms_per_step": ms, "value": gw.ops / (ms * 1e-3) / 1e12, "unit": UNIT}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--variants", action="store_true",
                    help="also time the general-problem paths (second-level scales, packed "
                         "grouped-query batch) and report them under 'variants'")
    ap.add_argument("--precision", default="fp4", choices=["fp4", "8bit"],
                    help="the method's FP4 path (default) or its 8-bit path")
    ap.add_argument("--sweep", action="store_true",
                    help="measure every named configuration (one JSON line each) instead of "
                         "the single bench line")
    ap.add_argument("--write-traffic", metavar="CSV",
                    help="write the attention kernel's traffic record under profiles/ from the CSV of "
                         "an ncu capture of this workload and exit")
    ap.add_argument("--no-mma-probe", action="store_true",
                    help="skip the FP4 tensor-core rate probe that sets the roofline peak")
    args = ap.parse_args()
    if args.write_traffic:
        print(json.dumps(write_traffic_record(args.write_traffic, workloads.by_name(args.workload),
                                              args.precision == "8bit")))
        return 0
    if args.sweep:
        return run_sweep(args)
    wl = workloads.by_name(args.workload)
    if args.impl == "reference":
        return run_reference(args, wl)

    import microscaling_fp4_quantized_b200 as sage

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # This rank's slice of the global problem: the workload's shape, its own seed.
    q, k, v = workloads.make_inputs(dataclasses.replace(wl, seed=wl.seed + 1000 * rank) if rank else wl)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty_like(qd)
    plan = sage.ProblemPlan(sage.sageattn_problem(qd, kd, vd, out, "HND", wl.causal, wl.sm_scale,
                                                  precision=args.precision), dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev_mid=None, ev_end=None):
        plan.quantize(qd, kd, vd)
        if ev_mid is not None:
            ev_mid.record(stream)
        plan.attention(out)
        if ev_end is not None:
            ev_end.record(stream)

    probe = None
    if not args.no_mma_probe and args.precision == "fp4":
        probe = sage.mma_rate(n=128)       # the FP4 instruction's own measured rate

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if sage.device_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    sampler = ClockSampler(local)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_begin.record(stream)
    for i in range(args.steps):
        starts[i].record(stream)
        step(mids[i], ends[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if dist is not None:
        dist.barrier()
    elapsed_ms = t_begin.elapsed_time(t_end)
    attn_ms = [mids[i].elapsed_time(ends[i]) for i in range(args.steps)]
    quant_ms = [starts[i].elapsed_time(mids[i]) for i in range(args.steps)]
    elapsed_ms = max_over_ranks(elapsed_ms, dist, dev)
    ms_per_step = elapsed_ms / args.steps
    value = job_value(wl.ops, world, ms_per_step)
    err = sage.device_error()

    # --- end to end through the public API: pinned host inputs -> result on the host ---
    e2e = None
    if not args.no_e2e:
        e2e = time_e2e(sage, wl, q, k, v, dev, stream, max(3, args.steps), dist, world, args.precision)

    variants = None
    if args.variants:
        variants = {}
        for g in ("tensor", "head"):
            gw = workloads.general(f"{wl.name}_gscale_{g}", wl.H, wl.H, wl.D, (wl.N,) * wl.B,
                                   causal=wl.causal, packed=False, seed=wl.seed, gscale=g)
            variants[gw.name] = time_general(sage, gw, dev, stream, args.warmup, min(args.steps, 20),
                                             inputs=(qd, kd, vd))
        qw = workloads.general(f"{wl.name}_smooth_q", wl.H, wl.H, wl.D, (wl.N,) * wl.B, causal=wl.causal,
                               packed=False, seed=wl.seed, smooth_q=True)
        variants[qw.name] = time_general(sage, qw, dev, stream, args.warmup, min(args.steps, 20),
                                         inputs=(qd, kd, vd))
        ew = workloads.general(f"{wl.name}_8bit", wl.H, wl.H, wl.D, (wl.N,) * wl.B, causal=wl.causal,
                               packed=False, seed=wl.seed, precision="8bit")
        variants[ew.name] = time_general(sage, ew, dev, stream, args.warmup, min(args.steps, 20),
                                         inputs=(qd, kd, vd))
        gw = workloads.LLM_VARLEN_GQA
        variants[gw.name] = time_general(sage, gw, dev, stream, args.warmup, min(args.steps, 20))
        variants[gw.name]["config"] = gw.describe()

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, basis = _peaks()
    b8 = args.precision == "8bit"
    peak, peak_how = fp4_peak(peaks, basis, probe, b8)
    attn_avg_ms = statistics.mean(attn_ms)
    achieved = wl.ops / (attn_avg_ms * 1e-3) / 1e12
    traffic, traffic_src = _attn_traffic(wl, b8)
    nominal = FP4_NOMINAL_TFLOPS / 2 if b8 else FP4_NOMINAL_TFLOPS
    roofline = {
        "kernel": "attn8_fwd_kernel" if b8 else "attn_fp4_fwd_kernel", "bound": "tensor", "achieved": achieved,
        "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
        "traffic_source": traffic_src, "peak_basis": peak_how,
        "frac_of_nominal": achieved / nominal, "nominal_tflops": nominal,
        "fp4_mma_probe_tflops": None if probe is None else probe["tflops"],
        "attn_ms": attn_avg_ms, "quant_ms": statistics.mean(quant_ms),
    }
    # The quantization's own HBM roofline: algorithmic bytes over its CUDA-event time.
    qbytes = quant_algorithmic_bytes(wl, b8)
    qgbs = qbytes / (roofline["quant_ms"] * 1e-3) / 1e9 if roofline["quant_ms"] > 0 else None
    roofline["quant_bytes"] = qbytes
    roofline["quant_gbs"] = qgbs
    roofline["quant_frac_of_hbm"] = None if qgbs is None else qgbs / float(peaks.get("hbm_gbs", 6650.0))
    cpu = None
    if not args.no_cpu_baseline:
        val, _, sample, cores = cpu_oracle_rate(wl, args.cpu_budget_s)
        cpu = {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
    cfg = wl.describe()
    cfg["precision"] = args.precision
    cfg["l2"] = "inputs larger than L2 (no flush)"
    cfg["timing"] = "CUDA events on the launching stream, max over ranks"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8_e4m3" if b8 else "fp4_e2m1", "data": "synthetic",
        "config": cfg, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": LAUNCHES_PER_STEP * args.steps, "clocks": clocks, "device_error_word": err,
        "pct_of_fp4_peak": 100.0 * value / world / peak,
        "pct_of_nominal_fp4": 100.0 * value / world / nominal,
    }
    if variants is not None:
        line["variants"] = variants
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
