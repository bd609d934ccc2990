"""Test-side helpers: turn the CUDA library's tiled layouts into the oracle's canonical
ones (index functions as documented in include/sage_fp4.h), and run the oracle on a
subset of heads / rows of a workload."""
from __future__ import annotations

import numpy as np
import torch


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def qk_sf_index(BH: int, N: int, Np: int, D: int) -> np.ndarray:
    """Flat byte index into q_sf / k_sf for canonical [BH, N, D/16]."""
    bh = np.arange(BH)[:, None, None]
    n = np.arange(N)[None, :, None]
    c = np.arange(D // 16)[None, None, :]
    return (((bh * (Np // 128) + n // 128) * (D // 64) + (16 * c) // 64) * 512
            + (n % 32) * 16 + ((n % 128) // 32) * 4 + c % 4)


def vt_sf_index(BH: int, Nb: int, Np: int, D: int) -> np.ndarray:
    """Flat byte index into vt_sf for canonical [BH, D, Nb] (token blocks of 16)."""
    bh = np.arange(BH)[:, None, None]
    d = np.arange(D)[None, :, None]
    t = np.arange(Nb)[None, None, :]
    return (((bh * (Np // 128) + (16 * t) // 128) * 2 + ((16 * t) % 128) // 64) * 512
            + (d % 32) * 16 + (d // 32) * 4 + t % 4)


def canonical(qz: dict) -> dict:
    """GPU quantized tensors -> oracle canonical numpy layouts (padding stripped)."""
    B, H, N, D, Np = qz["B"], qz["H"], qz["N"], qz["D"], qz["Np"]
    BH = B * H
    N16 = (N + 15) // 16 * 16
    g = {k: qz[k].cpu().numpy() for k in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf")}
    out = {
        "q_codes": g["q_fp4"][: BH * Np * D // 2].reshape(BH, Np, D // 2)[:, :N],
        "k_codes": g["k_fp4"][: BH * Np * D // 2].reshape(BH, Np, D // 2)[:, :N],
        "vt_codes": g["vt_fp4"][: BH * D * Np // 2].reshape(BH, D, Np // 2)[:, :, : N16 // 2],
        "q_sf": g["q_sf"][qk_sf_index(BH, N, Np, D)],
        "k_sf": g["k_sf"][qk_sf_index(BH, N, Np, D)],
        "vt_sf": g["vt_sf"][vt_sf_index(BH, N16 // 16, Np, D)],
        "k_mean": qz["k_mean"].cpu().numpy()[: BH * D].reshape(BH, D),
        "BH": BH, "N": N, "D": D,
    }
    # padding must be zero
    pads = {
        "q_fp4": g["q_fp4"][: BH * Np * D // 2].reshape(BH, Np, D // 2)[:, N:],
        "k_fp4": g["k_fp4"][: BH * Np * D // 2].reshape(BH, Np, D // 2)[:, N:],
        "vt_fp4": g["vt_fp4"][: BH * D * Np // 2].reshape(BH, D, Np // 2)[:, :, (N + 1) // 2:],
    }
    out["pads_zero"] = all(not p.any() for p in pads.values())
    for k in ("q_codes", "k_codes", "vt_codes"):
        out[k] = np.ascontiguousarray(out[k])
    return out


def heads_view(t: torch.Tensor, heads) -> np.ndarray:
    """[B, H, N, D] tensor -> float32 numpy [len(heads), N, D] for flat head ids."""
    B, H, N, D = t.shape
    flat = t.reshape(B * H, N, D)
    return np.stack([f32(flat[h]) for h in heads])


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    base = [0, N - 1, min(N - 1, 127), min(N - 1, 128)]
    extra = rng.choice(N, size=min(N, count), replace=False)
    return np.unique(np.concatenate([base, extra]))
