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
  q_codes [B*Hq, Nq, D/2], k_codes [B*Hkv, Nk, D/2] uint8; q_sf, k_sf [..., D/16] uint8
  (E4M3 bytes); vt_codes [B*Hkv, D, Np/2] uint8; vt_sf [B*Hkv, D, Np/16] uint8, Np = Nk
  rounded up to 16. Query head h of batch b reads key/value head h / (Hq / Hkv).
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
            "so_group_amax": [vp, c_long, c_long, c_long, vp, vp],
            "so_second_level_scale": [vp, c_long, vp],
            "so_quantize_rows": [vp, c_long, c_long, c_long, vp, vp, vp, vp],
            "so_quantize_vt": [vp, c_long, c_long, c_long, vp, vp, vp],
            "so_attn_emulated": [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, c_long, c_long, c_long,
                                 c_long, c_long, c_long, c_int, c_double, c_long, vp, c_long, vp],
            "so_qk_bias": [vp, vp, vp, c_long, c_long, c_long, c_long, c_long, vp],
            "so_attn_from_scores": [vp, c_long, c_long, vp, vp, vp, vp, vp, c_long, c_long, vp],
            "so_quant_int8_rows": [vp, c_long, c_long, c_long, c_long, vp, vp, vp],
            "so_quant_e4m3_channels": [vp, c_long, c_long, c_long, vp, vp],
            "so_attn_emulated8": [vp, vp, vp, vp, vp, vp, c_long, c_long, c_long, c_long, c_long,
                                  c_long, c_long, c_int, c_double, c_long, vp, c_long, vp],
            "so_attn_exact": [vp, vp, vp, c_long, c_long, c_long, c_long, c_long, c_long, c_int,
                              c_double, vp, c_long, vp],
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


def group_amax(x, mean=None) -> np.ndarray:
    """x [G, N, D] -> float32 [G]: max |x - mean| (binary32 difference) per group."""
    x = _f32(x)
    G, N, D = x.shape
    m = None if mean is None else _f32(mean).reshape(G, D)
    out = np.empty(G, np.float32)
    _L().so_group_amax(_p(x), G, N, D, _p(m) if m is not None else None, _p(out))
    return out


def second_level_scale(amax) -> np.ndarray:
    """amax -> float32 second-level scales fp32(amax / 2688) (1 where that is 0)."""
    a = _f32(amax).ravel()
    out = np.empty(a.shape, np.float32)
    _L().so_second_level_scale(_p(a), a.size, _p(out))
    return out.reshape(np.shape(amax))


def quantize_rows(x, mean=None, gscale=None):
    """x [G, N, D] -> (codes [G, N, D/2], sf [G, N, D/16]) along D, after the optional
    smoothing mean [G, D] and second-level scale [G]."""
    x = _f32(x)
    G, N, D = x.shape
    m = None if mean is None else _f32(mean).reshape(G, D)
    g = None if gscale is None else _f32(gscale).reshape(G)
    codes = np.zeros((G, N, D // 2), np.uint8)
    sf = np.zeros((G, N, D // 16), np.uint8)
    _L().so_quantize_rows(_p(x), G, N, D, _p(m) if m is not None else None,
                          _p(g) if g is not None else None, _p(codes), _p(sf))
    return codes, sf


def quantize_vt(v, gscale=None):
    """v [G, N, D] -> (vt codes [G, D, Np/2], vt sf [G, D, Np/16]), Np = N rounded up to 16."""
    v = _f32(v)
    G, N, D = v.shape
    Np = (N + 15) // 16 * 16
    g = None if gscale is None else _f32(gscale).reshape(G)
    codes = np.zeros((G, D, Np // 2), np.uint8)
    sf = np.zeros((G, D, Np // 16), np.uint8)
    _L().so_quantize_vt(_p(v), G, N, D, _p(g) if g is not None else None, _p(codes), _p(sf))
    return codes, sf


GSCALE_MODES = ("none", "tensor", "head")


def qk_bias(mu_q, k, mu_k, heads) -> np.ndarray:
    """The Q-smoothing bias [B*Hq, Nk] (binary64): mu_q . fp32(k - mu_k) per key."""
    k = _f32(k)
    B, Hq, Hkv = heads
    BHkv, Nk, D = k.shape
    mq = _f32(mu_q).reshape(B * Hq, D)
    mk = None if mu_k is None else _f32(mu_k).reshape(BHkv, D)
    out = np.empty((B * Hq, Nk), np.float64)
    _L().so_qk_bias(_p(mq), _p(k), _p(mk) if mk is not None else None, B, Hq, Hkv, Nk, D, _p(out))
    return out


def quantize_qkv(q, k, v, smooth_k: bool = True, kmean_in=None, gscale: str = "none",
                 amax_in=None, heads=None, smooth_q: bool = False, qmean_in=None) -> dict:
    """Quantize one problem of equal-length sequences.

    q [B*Hq, Nq, D], k and v [B*Hkv, Nk, D] (float32 values of the bf16/fp16 inputs);
    heads = (B, Hq, Hkv), default (1, q.shape[0], k.shape[0]). K is smoothed by its
    per-head token mean (kmean_in [B*Hkv, D] supplies it instead). gscale: "none", or a
    second-level scale per tensor ("tensor") or per head ("head") from the amax of Q,
    of the smoothed K and of V; amax_in = {"q": [B*Hq], "k": [B*Hkv], "v": [B*Hkv]}
    supplies those maxima (already reduced for "tensor" mode). smooth_q: Q is quantized
    as q - mu_q (mu_q its per-head token mean, qmean_in [B*Hq, D] supplies it) and the
    emulation adds back qk_bias = mu_q . (k - mu_k) per key.
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    BHq, Nq, D = q.shape
    BHkv, Nk, Dk = k.shape
    assert v.shape == k.shape and Dk == D and D % 16 == 0
    B, Hq, Hkv = heads if heads is not None else (1, BHq, BHkv)
    assert B * Hq == BHq and B * Hkv == BHkv and Hq % Hkv == 0
    assert gscale in GSCALE_MODES
    km = np.zeros((BHkv, D), np.float32)
    if smooth_k:
        km = _f32(kmean_in).reshape(BHkv, D) if kmean_in is not None else kmean(k)
    qm = None
    if smooth_q:
        qm = _f32(qmean_in).reshape(BHq, D) if qmean_in is not None else kmean(q)
    r = {"B": B, "Hq": Hq, "Hkv": Hkv, "Nq": Nq, "Nk": Nk, "D": D, "k_mean": km, "q_mean": qm,
         "gq": None, "gk": None, "gv": None, "amax": None, "qk_bias": None}
    if smooth_q:
        r["qk_bias"] = qk_bias(qm, k, km if smooth_k else None, (B, Hq, Hkv))
    if gscale != "none":
        if amax_in is not None:
            am = {n: _f32(amax_in[n]).ravel() for n in ("q", "k", "v")}
        else:
            am = {"q": group_amax(q, qm), "k": group_amax(k, km if smooth_k else None), "v": group_amax(v)}
            if gscale == "tensor":
                am = {n: np.full(a.shape, a.max(initial=0.0), np.float32) for n, a in am.items()}
        r["amax"] = am
        r["gq"], r["gk"], r["gv"] = (second_level_scale(am[n]) for n in ("q", "k", "v"))
    r["q_codes"], r["q_sf"] = quantize_rows(q, qm, r["gq"])
    r["k_codes"], r["k_sf"] = quantize_rows(k, km if smooth_k else None, r["gk"])
    r["vt_codes"], r["vt_sf"] = quantize_vt(v, r["gv"])
    return r


def _rows(G: int, N: int, rows) -> np.ndarray:
    if rows is None:
        g, i = np.meshgrid(np.arange(G), np.arange(N), indexing="ij")
        return np.ascontiguousarray(np.stack([g.ravel(), i.ravel()], 1).astype(np.int64))
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    assert (r[:, 0] >= 0).all() and (r[:, 0] < G).all() and (r[:, 1] >= 0).all() and (r[:, 1] < N).all()
    return r


def attn_emulated(qz: dict, causal: bool, sm_scale: float, Bk: int = 128, rows=None) -> np.ndarray:
    """Emulated FP4 attention on quantized inputs -> [n_rows, D] binary64 (or
    [B*Hq, Nq, D] when rows is None). rows are (query head, query index) pairs."""
    B, Hq, Hkv, Nq, Nk, D = (qz[n] for n in ("B", "Hq", "Hkv", "Nq", "Nk", "D"))
    r = _rows(B * Hq, Nq, rows)
    out = np.empty((r.shape[0], D), np.float64)
    arrs = [np.ascontiguousarray(qz[n]) for n in ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf")]
    gs = [None if qz[n] is None else _f32(qz[n]) for n in ("gq", "gk", "gv")]
    bias = qz.get("qk_bias")
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    _L().so_attn_emulated(*[_p(a) for a in arrs], *[_p(g) if g is not None else None for g in gs],
                          _p(bias) if bias is not None else None,
                          B, Hq, Hkv, Nq, Nk, D, int(bool(causal)), float(sm_scale), int(Bk),
                          _p(r), r.shape[0], _p(out))
    return out.reshape(B * Hq, Nq, D) if rows is None else out


def attn_from_scores(S, kv, n_keys, qz: dict, Bk: int = 128) -> np.ndarray:
    """The emulated attention's softmax, two-level P~ quantization and P^ V~ accumulation
    applied to GIVEN scores: S [n_rows, Nk] (already multiplied by sm_scale, and by the Q
    and K second-level scales when there are any), row r reading the values of key/value
    head kv[r] of qz (the output of quantize_qkv) and seeing keys 0 .. n_keys[r] - 1.
    Returns [n_rows, D] binary64. Used to check a GPU row against the method applied to
    that GPU's own FP32 scores."""
    S = np.ascontiguousarray(np.asarray(S, np.float64))
    n_rows, Nk = S.shape
    assert Nk == qz["Nk"]
    kv = np.ascontiguousarray(np.asarray(kv, np.int64).reshape(n_rows))
    nk = np.ascontiguousarray(np.asarray(n_keys, np.int64).reshape(n_rows))
    D = qz["D"]
    out = np.empty((n_rows, D), np.float64)
    vt, vsf = np.ascontiguousarray(qz["vt_codes"]), np.ascontiguousarray(qz["vt_sf"])
    gv = None if qz["gv"] is None else _f32(qz["gv"])
    _L().so_attn_from_scores(_p(S), n_rows, Nk, _p(kv), _p(nk), _p(vt), _p(vsf),
                             _p(gv) if gv is not None else None, D, int(Bk), _p(out))
    return out


def attn_exact(q, k, v, causal: bool, sm_scale: float, rows=None, heads=None) -> np.ndarray:
    """Two-pass softmax attention in binary64 -> [n_rows, D] (or [B*Hq, Nq, D]).
    q [B*Hq, Nq, D]; k, v [B*Hkv, Nk, D]; heads = (B, Hq, Hkv) as in quantize_qkv."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BHq, Nq, D = q.shape
    BHkv, Nk, _ = k.shape
    B, Hq, Hkv = heads if heads is not None else (1, BHq, BHkv)
    r = _rows(BHq, Nq, rows)
    out = np.empty((r.shape[0], D), np.float64)
    _L().so_attn_exact(_p(q), _p(k), _p(v), B, Hq, Hkv, Nq, Nk, D, int(bool(causal)),
                       float(sm_scale), _p(r), r.shape[0], _p(out))
    return out.reshape(BHq, Nq, D) if rows is None else out


def attn_online(q, k, v, causal: bool, sm_scale: float, Bk: int = 128, rows=None) -> np.ndarray:
    """Tiled online-softmax attention in binary64, no quantization (Nq == Nk, one head map)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BH, N, D = q.shape
    r = _rows(BH, N, rows)
    out = np.empty((r.shape[0], D), np.float64)
    _L().so_attn_online(_p(q), _p(k), _p(v), BH, N, D, int(bool(causal)), float(sm_scale),
                        int(Bk), _p(r), r.shape[0], _p(out))
    return out.reshape(BH, N, D) if rows is None else out


def attention(q, k, v, causal: bool, sm_scale: float, Bk: int = 128, rows=None,
              smooth_k: bool = True, kmean_in=None, gscale: str = "none", heads=None,
              amax_in=None, smooth_q: bool = False, qmean_in=None):
    """Full emulated pipeline: K mean, block quantization, emulated FP4 attention."""
    qz = quantize_qkv(q, k, v, smooth_k=smooth_k, kmean_in=kmean_in, gscale=gscale,
                      amax_in=amax_in, heads=heads, smooth_q=smooth_q, qmean_in=qmean_in)
    return attn_emulated(qz, causal, sm_scale, Bk=Bk, rows=rows), qz


def varlen_amax(q, k, v, cu_q, cu_k, smooth_k: bool = True, kmeans=None, smooth_q: bool = False,
                qmeans=None) -> dict:
    """Per-tensor maxima of packed sequences (q [Tq, Hq, D], k, v [Tk, Hkv, D]) for the
    "tensor" second-level scale: max over every sequence and head, K (and Q with
    smooth_q) smoothed by the mean of its own sequence (kmeans[b] [Hkv, D] and qmeans[b]
    [Hq, D] supply those)."""
    a = {"q": 0.0, "k": 0.0, "v": 0.0}
    for b in range(len(cu_q) - 1):
        qs = _f32(q[cu_q[b]:cu_q[b + 1]]).transpose(1, 0, 2)
        ks = _f32(k[cu_k[b]:cu_k[b + 1]]).transpose(1, 0, 2)
        vs = _f32(v[cu_k[b]:cu_k[b + 1]]).transpose(1, 0, 2)
        km = None
        if smooth_k and ks.shape[1] > 0:
            km = kmeans[b] if kmeans is not None else kmean(ks)
        if qs.shape[1] > 0:
            qm = None
            if smooth_q:
                qm = qmeans[b] if qmeans is not None else kmean(qs)
            a["q"] = max(a["q"], float(group_amax(qs, qm).max()))
        if ks.shape[1] > 0:
            a["k"] = max(a["k"], float(group_amax(ks, km).max()))
            a["v"] = max(a["v"], float(group_amax(vs).max()))
    return {n: np.float32(x) for n, x in a.items()}


def attention_varlen(q, k, v, cu_q, cu_k, causal: bool, sm_scale: float, Bk: int = 128,
                     smooth_k: bool = True, gscale: str = "none", kmeans=None, rows=None,
                     smooth_q: bool = False, qmeans=None):
    """Packed variable-length sequences, each an independent problem.

    q [Tq, Hq, D], k and v [Tk, Hkv, D]; sequence b holds query tokens cu_q[b]..cu_q[b+1]
    and key tokens cu_k[b]..cu_k[b+1]. Second-level scales: "head" per (sequence, head),
    "tensor" over all sequences and heads. kmeans[b] [Hkv, D] supplies the K means.
    rows: (token, head) pairs (None = all). Returns (out [n_rows, D] or [Tq, Hq, D],
    list of per-sequence quantized dicts).
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    Tq, Hq, D = q.shape
    Hkv = k.shape[1]
    nseq = len(cu_q) - 1
    am = None
    if gscale == "tensor":
        t = varlen_amax(q, k, v, cu_q, cu_k, smooth_k, kmeans, smooth_q, qmeans)
    want = np.asarray(rows, np.int64).reshape(-1, 2) if rows is not None else None
    full = np.zeros((Tq, Hq, D), np.float64)
    qzs = []
    for b in range(nseq):
        Lq, Lk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        qs = q[cu_q[b]:cu_q[b + 1]].transpose(1, 0, 2)
        ks = k[cu_k[b]:cu_k[b + 1]].transpose(1, 0, 2)
        vs = v[cu_k[b]:cu_k[b + 1]].transpose(1, 0, 2)
        if Lk == 0 or Lq == 0:
            qzs.append(None)
            continue
        if gscale == "tensor":
            am = {"q": np.full(Hq, t["q"], np.float32), "k": np.full(Hkv, t["k"], np.float32),
                  "v": np.full(Hkv, t["v"], np.float32)}
        sel = None
        if want is not None:
            m = (want[:, 0] >= cu_q[b]) & (want[:, 0] < cu_q[b + 1])
            if not m.any():
                qzs.append(None)
                continue
            sel = np.stack([want[m, 1], want[m, 0] - cu_q[b]], 1)
        o, qz = attention(qs, ks, vs, causal, sm_scale, Bk=Bk, rows=sel, smooth_k=smooth_k,
                          kmean_in=None if kmeans is None else kmeans[b], gscale=gscale,
                          heads=(1, Hq, Hkv), amax_in=am, smooth_q=smooth_q,
                          qmean_in=None if qmeans is None else qmeans[b])
        qzs.append(qz)
        if sel is None:
            full[cu_q[b]:cu_q[b + 1]] = o.transpose(1, 0, 2)
        else:
            full[sel[:, 1] + cu_q[b], sel[:, 0]] = o
    if want is not None:
        return full[want[:, 0], want[:, 1]], qzs
    return full, qzs


def attn_exact_varlen(q, k, v, cu_q, cu_k, causal: bool, sm_scale: float) -> np.ndarray:
    """Exact attention of packed sequences -> [Tq, Hq, D] binary64."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    Tq, Hq, D = q.shape
    Hkv = k.shape[1]
    full = np.zeros((Tq, Hq, D), np.float64)
    for b in range(len(cu_q) - 1):
        if cu_q[b + 1] == cu_q[b] or cu_k[b + 1] == cu_k[b]:
            continue
        qs = q[cu_q[b]:cu_q[b + 1]].transpose(1, 0, 2)
        ks = k[cu_k[b]:cu_k[b + 1]].transpose(1, 0, 2)
        vs = v[cu_k[b]:cu_k[b + 1]].transpose(1, 0, 2)
        o = attn_exact(qs, ks, vs, causal, sm_scale, heads=(1, Hq, Hkv))
        full[cu_q[b]:cu_q[b + 1]] = o.transpose(1, 0, 2)
    return full


# ------------------------------------------------------------- 8-bit path --

INT8_BLOCK = 128


def quant_int8_rows(x, block: int = INT8_BLOCK, mean=None):
    """x [G, N, D] -> (int8 codes [G, N, D], scales [G, ceil(N/block)]): symmetric INT8 with
    one scale fp32(absmax / 127) per block of tokens, codes RNE-rounded and clamped to 127."""
    x = _f32(x)
    G, N, D = x.shape
    nb = (N + block - 1) // block
    m = None if mean is None else _f32(mean).reshape(G, D)
    codes = np.zeros((G, N, D), np.int8)
    sc = np.zeros((G, nb), np.float32)
    _L().so_quant_int8_rows(_p(x), G, N, D, block, _p(m) if m is not None else None, _p(codes), _p(sc))
    return codes, sc


def quant_e4m3_channels(v):
    """v [G, N, D] -> (E4M3 codes of V^T [G, D, N], scales [G, D] = fp32(absmax_d / 448))."""
    v = _f32(v)
    G, N, D = v.shape
    codes = np.zeros((G, D, N), np.uint8)
    sc = np.zeros((G, D), np.float32)
    _L().so_quant_e4m3_channels(_p(v), G, N, D, _p(codes), _p(sc))
    return codes, sc


def quantize8(q, k, v, smooth_k: bool = True, kmean_in=None, heads=None, block: int = INT8_BLOCK) -> dict:
    """The 8-bit path's quantization: INT8 Q and (smoothed) K per token block, E4M3 V^T
    per channel. Shapes as quantize_qkv."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BHq, Nq, D = q.shape
    BHkv, Nk, _ = k.shape
    B, Hq, Hkv = heads if heads is not None else (1, BHq, BHkv)
    km = np.zeros((BHkv, D), np.float32)
    if smooth_k:
        km = _f32(kmean_in).reshape(BHkv, D) if kmean_in is not None else kmean(k)
    r = {"B": B, "Hq": Hq, "Hkv": Hkv, "Nq": Nq, "Nk": Nk, "D": D, "block": block, "k_mean": km}
    r["q8"], r["q_scale"] = quant_int8_rows(q, block)
    r["k8"], r["k_scale"] = quant_int8_rows(k, block, km if smooth_k else None)
    r["vt8"], r["v_scale"] = quant_e4m3_channels(v)
    return r


def attn_emulated8(qz: dict, causal: bool, sm_scale: float, Bk: int = 128, rows=None) -> np.ndarray:
    """Emulated 8-bit attention on the output of quantize8 -> [n_rows, D] (or [B*Hq, Nq, D])."""
    B, Hq, Hkv, Nq, Nk, D = (qz[n] for n in ("B", "Hq", "Hkv", "Nq", "Nk", "D"))
    r = _rows(B * Hq, Nq, rows)
    out = np.empty((r.shape[0], D), np.float64)
    arrs = [np.ascontiguousarray(qz[n]) for n in ("q8", "q_scale", "k8", "k_scale", "vt8", "v_scale")]
    _L().so_attn_emulated8(*[_p(a) for a in arrs], B, Hq, Hkv, Nq, Nk, D, int(qz["block"]),
                           int(bool(causal)), float(sm_scale), int(Bk), _p(r), r.shape[0], _p(out))
    return out.reshape(B * Hq, Nq, D) if rows is None else out


def attention8(q, k, v, causal: bool, sm_scale: float, Bk: int = 128, rows=None, smooth_k: bool = True,
               kmean_in=None, heads=None):
    """Full emulated 8-bit pipeline."""
    qz = quantize8(q, k, v, smooth_k=smooth_k, kmean_in=kmean_in, heads=heads)
    return attn_emulated8(qz, causal, sm_scale, Bk=Bk, rows=rows), qz


# ----------------------------------------------------------- error metrics --

def metrics(x: np.ndarray, ref: np.ndarray) -> dict:
    """Cosine similarity, relative L1 and RMSE (the accuracy metrics the SageAttention
    thread reports, reply to reviewer tyTT W1): cos = sum(xy)/sqrt(sum x^2 sum y^2),
    relL1 = sum|x-y|/sum|y|, rmse = sqrt(mean((x-y)^2)); plus max |x - y| over every
    element. x and ref must have the same shape. cos is 1 when both are all zeros and 0
    when exactly one of them is (an all-zero output never passes as similar)."""
    x = np.asarray(x, np.float64)
    y = np.asarray(ref, np.float64)
    if x.shape != y.shape:
        raise ValueError(f"metrics: shapes differ {x.shape} vs {y.shape}")
    x, y = x.ravel(), y.ravel()
    nx, ny = (x * x).sum(), (y * y).sum()
    if nx > 0 and ny > 0:
        cos = float((x * y).sum() / np.sqrt(nx * ny))
    else:
        cos = 1.0 if nx == 0 and ny == 0 else 0.0
    sy = np.abs(y).sum()
    return {
        "cos": cos,
        "rel_l1": float(np.abs(x - y).sum() / sy) if sy > 0 else (0.0 if not np.abs(x).any() else float("inf")),
        "rmse": float(np.sqrt(np.mean((x - y) ** 2))) if x.size else 0.0,
        "max_abs": float(np.abs(x - y).max()) if x.size else 0.0,
    }
