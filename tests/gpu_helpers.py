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


def _vt_rows(vt: np.ndarray, BH: int, Np: int, D: int) -> np.ndarray:
    """Tile-major V^T [BH * Np/128, D, 64] -> [BH, D, Np/2]."""
    t = vt[: BH * Np * D // 2].reshape(BH, Np // 128, D, 64)
    return np.ascontiguousarray(t.transpose(0, 2, 1, 3).reshape(BH, D, Np // 2))


def canonical(qz: dict) -> dict:
    """GPU quantized tensors -> oracle canonical numpy layouts (padding stripped)."""
    B, H, N, D, Np = qz["B"], qz["H"], qz["N"], qz["D"], qz["Np"]
    BH = B * H
    N16 = (N + 15) // 16 * 16
    g = {k: qz[k].cpu().numpy() for k in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf")}
    vt = _vt_rows(g["vt_fp4"], BH, Np, D)
    out = {
        "q_codes": g["q_fp4"][: BH * Np * D // 2].reshape(BH, Np, D // 2)[:, :N],
        "k_codes": g["k_fp4"][: BH * Np * D // 2].reshape(BH, Np, D // 2)[:, :N],
        "vt_codes": vt[:, :, : N16 // 2],
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
        "vt_fp4": vt[:, :, (N + 1) // 2:],
    }
    out["pads_zero"] = all(not p.any() for p in pads.values())
    for k in ("q_codes", "k_codes", "vt_codes"):
        out[k] = np.ascontiguousarray(out[k])
    return out


def padded_offsets(lens) -> np.ndarray:
    """Exclusive prefix sums of the lengths rounded up to 128."""
    r = [(int(n) + 127) // 128 * 128 for n in lens]
    return np.concatenate([[0], np.cumsum(r)]).astype(np.int64)


def _sf_rows(sf: np.ndarray, rows: np.ndarray, D: int) -> np.ndarray:
    """Scale bytes of padded rows `rows` (all D/16 channel blocks) -> [len(rows), D/16]."""
    r = rows[:, None]
    c = np.arange(D // 16)[None, :]
    idx = ((r // 128) * (D // 64) + (16 * c) // 64) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    return sf[idx]


def decode_bias(buf: np.ndarray, row0: int, n: int) -> np.ndarray:
    """Sum of the three bf16 terms of keys 0..n-1 of the bias operand starting at padded
    row row0 (a multiple of 128) -> float64 [n]."""
    keys = np.arange(n)
    tile = row0 + (keys // 128) * 128
    k = keys % 128
    off = tile * 32 + (k // 8) * 256 + (k % 8) * 16
    words = np.stack([buf[off + 2 * i].astype(np.uint16) | (buf[off + 2 * i + 1].astype(np.uint16) << 8)
                      for i in range(3)])
    vals = (words.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return vals.sum(axis=0)


def canonical_problem(qz: dict, lens_q, lens_k, Hq: int, Hkv: int, D: int) -> list:
    """Per sequence, the GPU's quantized tensors of a general problem in the oracle's
    canonical layouts: q_codes [Hq, Lq, D/2], q_sf [Hq, Lq, D/16], k_codes / k_sf
    [Hkv, Lk, ...], vt_codes [Hkv, D, ceil16(Lk)/2], vt_sf [Hkv, D, ceil16(Lk)/16],
    k_mean [Hkv, D]; plus pads_zero (the padding rows and tokens hold zeros)."""
    g = {k: qz[k].cpu().numpy() for k in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf")}
    kmean = qz["k_mean"].cpu().numpy()
    qmean = qz["q_mean"].cpu().numpy() if "q_mean" in qz else None
    bias = qz["qk_bias"].cpu().numpy() if "qk_bias" in qz else None
    pq, pk = padded_offsets(lens_q), padded_offsets(lens_k)
    res = []
    for b, (Lq, Lk) in enumerate(zip(lens_q, lens_k)):
        Pq, Pk = (Lq + 127) // 128 * 128, (Lk + 127) // 128 * 128
        o = {"pads_zero": True}
        qc, qs, kc, ks = [], [], [], []
        for h in range(Hq):
            r0 = Hq * pq[b] + h * Pq
            rows = np.arange(r0, r0 + Pq)
            blk = g["q_fp4"][r0 * (D // 2):(r0 + Pq) * (D // 2)].reshape(Pq, D // 2)
            qc.append(blk[:Lq])
            qs.append(_sf_rows(g["q_sf"], rows[:Lq], D))
            o["pads_zero"] &= not blk[Lq:].any()
        vc, vs = [], []
        L16 = (Lk + 15) // 16 * 16
        for h in range(Hkv):
            r0 = Hkv * pk[b] + h * Pk
            rows = np.arange(r0, r0 + Pk)
            blk = g["k_fp4"][r0 * (D // 2):(r0 + Pk) * (D // 2)].reshape(Pk, D // 2)
            kc.append(blk[:Lk])
            ks.append(_sf_rows(g["k_sf"], rows[:Lk], D))
            o["pads_zero"] &= not blk[Lk:].any()
            t0 = r0 // 128
            vt = g["vt_fp4"][t0 * D * 64:(t0 + Pk // 128) * D * 64].reshape(Pk // 128, D, 64)
            vt = vt.transpose(1, 0, 2).reshape(D, Pk // 2)
            vc.append(vt[:, : L16 // 2])
            o["pads_zero"] &= not vt[:, (Lk + 1) // 2:].any()
            u = np.arange(L16 // 16)[None, :]
            d = np.arange(D)[:, None]
            t = t0 + (16 * u) // 128
            uu = u % 8
            vs.append(g["vt_sf"][(t * 2 + uu // 4) * 512 + (d % 32) * 16 + (d // 32) * 4 + uu % 4])
        o["q_codes"], o["q_sf"] = np.stack(qc), np.stack(qs)
        o["k_codes"], o["k_sf"] = np.stack(kc), np.stack(ks)
        o["vt_codes"], o["vt_sf"] = np.stack(vc), np.stack(vs)
        o["k_mean"] = kmean[b * Hkv * D:(b + 1) * Hkv * D].reshape(Hkv, D)
        if qmean is not None and qmean.size >= (b + 1) * Hq * D:
            o["q_mean"] = qmean[b * Hq * D:(b + 1) * Hq * D].reshape(Hq, D)
        if bias is not None and bias.size >= 32 * Hq * (pk[b] + Pk):
            # the Q-smoothing bias operand: 32 bytes per (query head, padded key row), three
            # bf16 terms in elements 0-2, key n of a tile at (n/8)*256 + (n%8)*16
            o["qk_bias"] = np.stack([decode_bias(bias, Hq * pk[b] + h * Pk, Lk) for h in range(Hq)])
        res.append(o)
    return res


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


def canonical8(qz: dict, lens_q, lens_k, Hq: int, Hkv: int, D: int) -> list:
    """Per sequence, the GPU's 8-bit quantized tensors in the oracle's layouts: q8 [Hq, Lq, D]
    int8, q_scale [Hq, ceil(Lq/128)], k8 / k_scale likewise with Hkv, vt8 [Hkv, D, Lk]
    (E4M3 bytes), v_scale [Hkv, D], k_mean [Hkv, D]; plus pads_zero."""
    g = {k: qz[k].cpu().numpy() for k in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf")}
    q_scale, k_scale, v_scale = (g[n].view(np.float32) for n in ("q_sf", "k_sf", "vt_sf"))
    kmean = qz["k_mean"].cpu().numpy()
    pq, pk = padded_offsets(lens_q), padded_offsets(lens_k)
    res = []
    for b, (Lq, Lk) in enumerate(zip(lens_q, lens_k)):
        Pq, Pk = (Lq + 127) // 128 * 128, (Lk + 127) // 128 * 128
        o = {"pads_zero": True}
        q8, qs = [], []
        for h in range(Hq):
            r0 = Hq * pq[b] + h * Pq
            blk = g["q_fp4"][r0 * D:(r0 + Pq) * D].reshape(Pq, D)
            q8.append(blk[:Lq].view(np.int8))
            qs.append(q_scale[r0 // 128:(r0 + Pq) // 128])
            o["pads_zero"] &= not blk[Lq:].any()
        k8, ks, vt, vs = [], [], [], []
        for h in range(Hkv):
            r0 = Hkv * pk[b] + h * Pk
            blk = g["k_fp4"][r0 * D:(r0 + Pk) * D].reshape(Pk, D)
            k8.append(blk[:Lk].view(np.int8))
            ks.append(k_scale[r0 // 128:(r0 + Pk) // 128])
            o["pads_zero"] &= not blk[Lk:].any()
            t0 = r0 // 128
            t = g["vt_fp4"][t0 * D * 128:(t0 + Pk // 128) * D * 128].reshape(Pk // 128, D, 128)
            t = t.transpose(1, 0, 2).reshape(D, Pk)
            vt.append(t[:, :Lk])
            o["pads_zero"] &= not t[:, Lk:].any()
            vs.append(v_scale[(b * Hkv + h) * D:(b * Hkv + h + 1) * D])
        o["q8"], o["q_scale"] = np.stack(q8), np.stack(qs)
        o["k8"], o["k_scale"] = np.stack(k8), np.stack(ks)
        o["vt8"], o["v_scale"] = np.stack(vt), np.stack(vs)
        o["k_mean"] = kmean[b * Hkv * D:(b + 1) * Hkv * D].reshape(Hkv, D)
        res.append(o)
    return res


def gpu_row_scores(sage, qz: dict, lens_q, lens_k, Hq: int, Hkv: int, D: int, b: int, h: int) -> np.ndarray:
    """The GPU tensor core's own FP32 products Q^ K^^T (no scale) of query head h of
    sequence b of a general problem, from the quantized buffers of sage.quantize:
    [Lq, Lk] float64. The (sequence, head) blocks of Q and of key/value head h / (Hq/Hkv)
    are copied into a dense one-head problem padded to a common length, and the
    library's scores kernel (the attention kernel's MMA form) runs on it."""
    pq, pk = padded_offsets(lens_q), padded_offsets(lens_k)
    Lq, Lk = int(lens_q[b]), int(lens_k[b])
    Pq, Pk = (Lq + 127) // 128 * 128, (Lk + 127) // 128 * 128
    Np = max(Pq, Pk)
    hk = h // (Hq // Hkv)
    rq, rk = Hq * int(pq[b]) + h * Pq, Hkv * int(pk[b]) + hk * Pk
    row_b, tile_b = D // 2, (D // 64) * 512
    dev = qz["q_fp4"].device
    dense = {n: torch.zeros(Np * row_b if n.endswith("fp4") else (Np // 128) * tile_b, dtype=torch.uint8,
                            device=dev) for n in ("q_fp4", "k_fp4", "q_sf", "k_sf")}
    dense["q_fp4"][: Pq * row_b] = qz["q_fp4"][rq * row_b:(rq + Pq) * row_b]
    dense["k_fp4"][: Pk * row_b] = qz["k_fp4"][rk * row_b:(rk + Pk) * row_b]
    dense["q_sf"][: (Pq // 128) * tile_b] = qz["q_sf"][(rq // 128) * tile_b:((rq + Pq) // 128) * tile_b]
    dense["k_sf"][: (Pk // 128) * tile_b] = qz["k_sf"][(rk // 128) * tile_b:((rk + Pk) // 128) * tile_b]
    dense.update({"B": 1, "H": 1, "N": Np, "D": D, "Np": Np})
    s = sage.qk_scores(dense, sm_scale=1.0)
    torch.cuda.synchronize()
    return s[0, :Lq, :Lk].double().cpu().numpy()
