"""CPU oracle for microscaling-FP4 attention (SageAttention3 forward).

TEST INFRASTRUCTURE ONLY. This package wraps ``sage_oracle.cpp``: a slow, plain,
binary64 reference with a bit-faithful emulation of the FP4/FP8 block quantizer.
Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
leg of ``bench.py`` may import it. The CUDA library never calls it and shares no
code with it; the two meet only in the tests, on inputs from the seeded generators.

Pins (what checks this oracle against something other than itself) live in
``tests/test_oracle_*.py``. Every function here is pinned except the absolute
accuracy of the emulated attention against exact attention, which the pages do not
fix ("parity unpinned" for that comparison; it is reported, not asserted).

Layouts (canonical, row-major; FP4 nibble 2i is the low half of byte i):
  q_codes, k_codes [BH, N, D/2] uint8; q_sf, k_sf [BH, N, D/16] uint8 (E4M3 bytes)
  vt_codes [BH, D, Np/2] uint8; vt_sf [BH, D, Np/16] uint8, Np = N rounded up to 16
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sage_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libsage_oracle.so")
_lib = None

TWO_LEVEL_TARGET = 448.0 * 6.0


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (-O2, OpenMP, no FP contraction, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["g++", "-std=c++17", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", _SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        c_long, c_int, c_double, vp = ctypes.c_long, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        sigs = {
            "so_e2m1_encode": [vp, c_long, vp],
            "so_e2m1_decode": [vp, c_long, vp],
            "so_e4m3_encode": [vp, c_long, vp],
            "so_e4m3_decode": [vp, c_long, vp],
            "so_quant_block16": [vp, c_long, vp, vp],
            "so_kmean": [vp, c_long, c_long, c_long, vp],
            "so_quantize_qkv": [vp, vp, vp, c_long, c_long, c_long, c_int, vp,
                                vp, vp, vp, vp, vp, vp, vp],
            "so_attn_emulated": [vp, vp, vp, vp, vp, vp, c_long, c_long, c_long, c_int,
                                 c_double, c_long, vp, c_long, vp],
            "so_attn_exact": [vp, vp, vp, c_long, c_long, c_long, c_int, c_double, vp, c_long, vp],
            "so_attn_online": [vp, vp, vp, c_long, c_long, c_long, c_int, c_double, c_long,
                               vp, c_long, vp],
        }
        for name, args in sigs.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = None
        lib.so_num_threads.restype = c_int
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def num_threads() -> int:
    return int(_L().so_num_threads())


# ------------------------------------------------------------------ formats --

def e2m1_encode(x) -> np.ndarray:
    x = _f32(x)
    out = np.empty(x.shape, np.uint8)
    _L().so_e2m1_encode(_p(x), x.size, _p(out))
    return out


def e2m1_decode(codes) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.empty(c.shape, np.float64)
    _L().so_e2m1_decode(_p(c), c.size, _p(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    x = _f32(x)
    out = np.empty(x.shape, np.uint8)
    _L().so_e4m3_encode(_p(x), x.size, _p(out))
    return out


def e4m3_decode(b) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint8))
    out = np.empty(b.shape, np.float64)
    _L().so_e4m3_decode(_p(b), b.size, _p(out))
    return out


def quant_block16(x):
    """x [..., 16] float32 -> (codes [..., 16] uint8 unpacked, scale bytes [...] uint8)."""
    x = _f32(x)
    assert x.shape[-1] == 16
    nb = x.size // 16
    codes = np.empty(x.shape, np.uint8)
    sb = np.empty(x.shape[:-1], np.uint8)
    _L().so_quant_block16(_p(x), nb, _p(codes), _p(sb))
    return codes, sb


def unpack_fp4(packed: np.ndarray) -> np.ndarray:
    """[..., n/2] uint8 -> [..., n] codes (low nibble first)."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


# ----------------------------------------------------------- quantization --

def kmean(k) -> np.ndarray:
    """k [BH, N, D] -> fp32 [BH, D], binary64 accumulation rounded once to binary32."""
    k = _f32(k)
    BH, N, D = k.shape
    out = np.empty((BH, D), np.float32)
    _L().so_kmean(_p(k), BH, N, D, _p(out))
    return out


def quantize_qkv(q, k, v, smooth_k: bool = True, kmean_in=None) -> dict:
    """q, k, v [BH, N, D] (float32 values of the bf16/fp16 inputs) -> canonical arrays."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BH, N, D = q.shape
    assert k.shape == q.shape == v.shape and D % 16 == 0
    Np = (N + 15) // 16 * 16
    r = {
        "q_codes": np.zeros((BH, N, D // 2), np.uint8), "q_sf": np.zeros((BH, N, D // 16), np.uint8),
        "k_codes": np.zeros((BH, N, D // 2), np.uint8), "k_sf": np.zeros((BH, N, D // 16), np.uint8),
        "vt_codes": np.zeros((BH, D, Np // 2), np.uint8), "vt_sf": np.zeros((BH, D, Np // 16), np.uint8),
        "k_mean": np.zeros((BH, D), np.float32), "BH": BH, "N": N, "D": D,
    }
    km = None
    if kmean_in is not None:
        km = _f32(kmean_in).reshape(BH, D)
    _L().so_quantize_qkv(_p(q), _p(k), _p(v), BH, N, D, int(bool(smooth_k)),
                         _p(km) if km is not None else None,
                         _p(r["q_codes"]), _p(r["q_sf"]), _p(r["k_codes"]), _p(r["k_sf"]),
                         _p(r["vt_codes"]), _p(r["vt_sf"]), _p(r["k_mean"]))
    return r


def _rows(BH: int, N: int, rows) -> np.ndarray:
    if rows is None:
        bh, i = np.meshgrid(np.arange(BH), np.arange(N), indexing="ij")
        return np.ascontiguousarray(np.stack([bh.ravel(), i.ravel()], 1).astype(np.int64))
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    assert (r[:, 0] >= 0).all() and (r[:, 0] < BH).all() and (r[:, 1] >= 0).all() and (r[:, 1] < N).all()
    return r


def attn_emulated(qz: dict, causal: bool, sm_scale: float, Bk: int = 128, rows=None) -> np.ndarray:
    """Emulated FP4 attention on quantized inputs -> [n_rows, D] binary64 (or [BH, N, D])."""
    BH, N, D = qz["BH"], qz["N"], qz["D"]
    r = _rows(BH, N, rows)
    out = np.empty((r.shape[0], D), np.float64)
    arrs = [np.ascontiguousarray(qz[n]) for n in ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf")]
    _L().so_attn_emulated(*[_p(a) for a in arrs], BH, N, D, int(bool(causal)), float(sm_scale),
                          int(Bk), _p(r), r.shape[0], _p(out))
    return out.reshape(BH, N, D) if rows is None else out


def attn_exact(q, k, v, causal: bool, sm_scale: float, rows=None) -> np.ndarray:
    """Two-pass softmax attention in binary64 -> [n_rows, D] (or [BH, N, D])."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BH, N, D = q.shape
    r = _rows(BH, N, rows)
    out = np.empty((r.shape[0], D), np.float64)
    _L().so_attn_exact(_p(q), _p(k), _p(v), BH, N, D, int(bool(causal)), float(sm_scale),
                       _p(r), r.shape[0], _p(out))
    return out.reshape(BH, N, D) if rows is None else out


def attn_online(q, k, v, causal: bool, sm_scale: float, Bk: int = 128, rows=None) -> np.ndarray:
    """Tiled online-softmax attention in binary64, no quantization."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BH, N, D = q.shape
    r = _rows(BH, N, rows)
    out = np.empty((r.shape[0], D), np.float64)
    _L().so_attn_online(_p(q), _p(k), _p(v), BH, N, D, int(bool(causal)), float(sm_scale),
                        int(Bk), _p(r), r.shape[0], _p(out))
    return out.reshape(BH, N, D) if rows is None else out


def attention(q, k, v, causal: bool, sm_scale: float, Bk: int = 128, rows=None,
              smooth_k: bool = True, kmean_in=None):
    """Full emulated pipeline: K mean, block quantization, emulated FP4 attention."""
    qz = quantize_qkv(q, k, v, smooth_k=smooth_k, kmean_in=kmean_in)
    return attn_emulated(qz, causal, sm_scale, Bk=Bk, rows=rows), qz


# ----------------------------------------------------------- error metrics --

def metrics(x: np.ndarray, ref: np.ndarray) -> dict:
    """Cosine similarity, relative L1 and RMSE (the accuracy metrics the SageAttention
    thread reports): cos = sum(xy)/sqrt(sum x^2 sum y^2), relL1 = sum|x-y|/sum|y|,
    rmse = sqrt(mean((x-y)^2)); plus max |x - y|."""
    x = np.asarray(x, np.float64).ravel()
    y = np.asarray(ref, np.float64).ravel()
    den = np.sqrt((x * x).sum() * (y * y).sum())
    return {
        "cos": float((x * y).sum() / den) if den > 0 else 1.0,
        "rel_l1": float(np.abs(x - y).sum() / max(np.abs(y).sum(), 1e-300)),
        "rmse": float(np.sqrt(np.mean((x - y) ** 2))),
        "max_abs": float(np.abs(x - y).max()) if x.size else 0.0,
    }
