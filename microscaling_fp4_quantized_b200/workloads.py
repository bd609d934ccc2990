"""Seeded synthetic workloads for the FP4 attention forward.

This module holds no arithmetic of the method: it only names the workload shapes and
draws the random inputs. Both the tests (for the CPU oracle and the CUDA path) and
the benchmark take their inputs from here.

Recipe (the shapes stand in for the pages' video-diffusion and LLM workloads; no
dataset is involved):
  * One CPU ``torch.Generator`` seeded with the workload's seed draws, in this order,
    Q, K, V ~ N(0, 1) as float32 [B, H, N, D]; then the per-channel K bias
    ~ N(0, sigma^2) with shape [B, H, 1, D] (shared across tokens); then, for the
    outlier workload only, per head one channel index (max(1, round(0.01 * D))
    channels, drawn by ``randperm`` per head) that is multiplied by 20 in both Q and K.
  * The outlier scaling and the bias are applied in float32, then the three tensors
    are cast (round to nearest even) to the workload's dtype.
Because the generator runs on the CPU, the same seed gives the same tensors on any
machine, with or without a GPU.
"""
from __future__ import annotations

import dataclasses
import itertools
import math
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    D: int
    causal: bool
    dtype: torch.dtype
    seed: int
    bias_sigma: float
    outliers: bool = False

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def ops(self) -> float:
        """Attention operations per forward: 4*B*H*N^2*D, halved when causal."""
        o = 4.0 * self.B * self.H * self.N * self.N * self.D
        return o / 2 if self.causal else o

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "N": self.N, "D": self.D,
                "causal": self.causal, "dtype": str(self.dtype).replace("torch.", ""),
                "seed": self.seed, "k_bias_sigma": self.bias_sigma, "outlier_channels": self.outliers}


def _sweep() -> List[Workload]:
    out = []
    idx = 0
    for D in (64, 128):
        for N in (1024, 4096, 16384, 65536):
            for causal in (False, True):
                B = max(1, 65536 // N)
                out.append(Workload(f"sweep_D{D}_N{N}_{'causal' if causal else 'full'}", B, 32, N, D,
                                    causal, torch.bfloat16, 4 + idx, 2.0))
                idx += 1
    return out


TINY = Workload("tiny_B1_H2_N256_D64_fp16", 1, 2, 256, 64, False, torch.float16, 0, 2.0)
MEDIUM = Workload("B1_H16_N4096_D128", 1, 16, 4096, 128, False, torch.bfloat16, 1, 2.0)
LLM_CAUSAL = Workload("llm_causal_B4_H32_N8192_D128_outliers", 4, 32, 8192, 128, True,
                      torch.bfloat16, 2, 2.0, outliers=True)
LONG = Workload("video_long_B1_H24_N32768_D128", 1, 24, 32768, 128, False, torch.bfloat16, 3, 4.0)
SWEEP = _sweep()
# Profiling size: inputs (192 MiB) larger than the 126 MB L2, a few GB on the device at most.
PROFILE = Workload("profile_B1_H16_N16384_D128", 1, 16, 16384, 128, False, torch.bfloat16, 7, 2.0)

ALL = [TINY, MEDIUM, LLM_CAUSAL, LONG, PROFILE] + SWEEP


def by_name(name: str) -> Workload:
    for w in ALL:
        if w.name == name:
            return w
    raise KeyError(name)


def custom(B: int, H: int, N: int, D: int, causal: bool = False, dtype=torch.bfloat16,
           seed: int = 123, bias_sigma: float = 2.0, outliers: bool = False) -> Workload:
    return Workload(f"custom_B{B}_H{H}_N{N}_D{D}_{'causal' if causal else 'full'}", B, H, N, D,
                    causal, dtype, seed, bias_sigma, outliers)


def make_inputs(w: Workload, device: Optional[str] = None):
    """Draw (q, k, v) as [B, H, N, D] tensors of ``w.dtype`` (on ``device`` if given)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.D)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    bias = torch.randn((w.B, w.H, 1, w.D), generator=g, dtype=torch.float32) * w.bias_sigma
    if w.outliers:
        count = max(1, int(round(0.01 * w.D)))
        for b in range(w.B):
            for h in range(w.H):
                ch = torch.randperm(w.D, generator=g)[:count]
                q[b, h, :, ch] *= 20.0
                k[b, h, :, ch] *= 20.0
    k += bias
    q, k, v = q.to(w.dtype), k.to(w.dtype), v.to(w.dtype)
    if device is not None:
        q, k, v = q.to(device), k.to(device), v.to(device)
    return q, k, v


# ----------------------------------------------------------- general problems --
#
# Recipe: one CPU generator seeded with the workload's seed draws, in this order,
# Q [Tq, Hq, D], K [Tk, Hkv, D], V [Tk, Hkv, D] ~ N(0, 1) in float32 (Tq, Tk = the summed
# lengths; sequence b owns the next lens[b] tokens), then one K bias per (sequence, key
# head) ~ N(0, sigma^2) [B, Hkv, D] added to that sequence's keys, then (only when
# q_bias_sigma > 0) one query offset per (sequence, query head) ~ N(0, q_bias_sigma^2)
# [B, Hq, D] added to that sequence's queries. Q, K and V are then
# multiplied by q_scale, k_scale and v_scale (to reach the one-level format's range
# limits) and cast to the dtype. Dense workloads view the same draws as [B, H, N, D]
# ("HND") or [B, N, H, D] ("NHD") tensors.

@dataclasses.dataclass(frozen=True)
class GeneralWorkload:
    name: str
    Hq: int
    Hkv: int
    D: int
    lens_q: tuple
    lens_k: tuple
    causal: bool
    packed: bool
    layout: str = "HND"
    dtype: torch.dtype = torch.bfloat16
    seed: int = 0
    bias_sigma: float = 2.0
    q_scale: float = 1.0
    k_scale: float = 1.0
    v_scale: float = 1.0
    gscale: str = "none"
    smooth_q: bool = False
    q_bias_sigma: float = 0.0
    precision: str = "fp4"

    @property
    def B(self) -> int:
        return len(self.lens_q)

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def ops(self) -> float:
        """4 * Hq * Lq * Lk * D per sequence, halved when causal (the square-problem
        convention of the dense workloads)."""
        o = sum(4.0 * self.Hq * lq * lk * self.D for lq, lk in zip(self.lens_q, self.lens_k))
        return o / 2 if self.causal else o

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "Hq": self.Hq, "Hkv": self.Hkv, "D": self.D,
                "lens_q": list(self.lens_q) if len(self.lens_q) <= 16 else f"{len(self.lens_q)} sequences",
                "total_q": sum(self.lens_q), "total_k": sum(self.lens_k), "causal": self.causal,
                "packed": self.packed, "layout": self.layout,
                "dtype": str(self.dtype).replace("torch.", ""), "seed": self.seed,
                "gscale": self.gscale, "smooth_q": self.smooth_q, "q_bias_sigma": self.q_bias_sigma,
                "precision": self.precision}


def general(name: str, Hq: int, Hkv: int, D: int, lens_q, lens_k=None, causal: bool = False,
            packed: bool = True, **kw) -> GeneralWorkload:
    lens_q = tuple(int(x) for x in lens_q)
    lens_k = lens_q if lens_k is None else tuple(int(x) for x in lens_k)
    return GeneralWorkload(name, Hq, Hkv, D, lens_q, lens_k, causal, packed, **kw)


def length_mix(count: int, lo: int, hi: int, seed: int) -> tuple:
    """Sequence lengths drawn uniformly from [lo, hi] by a seeded CPU generator."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (count,), generator=g))


# An LLM-serving batch: 16 packed prompts of mixed length, grouped-query heads (32 query
# heads sharing 8 key/value heads), causal.
LLM_VARLEN_GQA = general("llm_varlen_gqa_Hq32_Hkv8_D128_16seq", 32, 8, 128,
                         length_mix(16, 256, 16384, seed=41), causal=True, seed=41)


def make_general_inputs(w: GeneralWorkload, device: Optional[str] = None) -> dict:
    """Draw the inputs of a general workload. Packed: q [Tq, Hq, D], k and v [Tk, Hkv, D]
    plus int32 cu_seqlens_q / cu_seqlens_k; dense: [B, H, N, D] ("HND") or [B, N, H, D]
    ("NHD") tensors (every sequence then has the same lengths)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    Tq, Tk = sum(w.lens_q), sum(w.lens_k)
    q = torch.randn((Tq, w.Hq, w.D), generator=g, dtype=torch.float32)
    k = torch.randn((Tk, w.Hkv, w.D), generator=g, dtype=torch.float32)
    v = torch.randn((Tk, w.Hkv, w.D), generator=g, dtype=torch.float32)
    bias = torch.randn((w.B, w.Hkv, w.D), generator=g, dtype=torch.float32) * w.bias_sigma
    cu_q = torch.tensor([0] + list(itertools.accumulate(w.lens_q)), dtype=torch.int32)
    cu_k = torch.tensor([0] + list(itertools.accumulate(w.lens_k)), dtype=torch.int32)
    for b in range(w.B):
        k[cu_k[b]:cu_k[b + 1]] += bias[b]
    if w.q_bias_sigma > 0:
        qbias = torch.randn((w.B, w.Hq, w.D), generator=g, dtype=torch.float32) * w.q_bias_sigma
        for b in range(w.B):
            q[cu_q[b]:cu_q[b + 1]] += qbias[b]
    q, k, v = (q * w.q_scale).to(w.dtype), (k * w.k_scale).to(w.dtype), (v * w.v_scale).to(w.dtype)
    out = {"cu_seqlens_q": cu_q, "cu_seqlens_k": cu_k}
    if w.packed:
        out.update(q=q, k=k, v=v)
    else:
        if len(set(w.lens_q)) != 1 or len(set(w.lens_k)) != 1:
            raise ValueError("a dense workload needs equal lengths")
        Nq, Nk = w.lens_q[0], w.lens_k[0]
        qd = q.reshape(w.B, Nq, w.Hq, w.D)
        kd = k.reshape(w.B, Nk, w.Hkv, w.D)
        vd = v.reshape(w.B, Nk, w.Hkv, w.D)
        if w.layout == "HND":
            qd, kd, vd = (t.permute(0, 2, 1, 3).contiguous() for t in (qd, kd, vd))
        out.update(q=qd, k=kd, v=vd)
    if device is not None:
        out = {n: t.to(device) for n, t in out.items()}
    return out

