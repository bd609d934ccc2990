"""Microscaling-FP4 attention forward (SageAttention3 method) for NVIDIA B200, sm_100a.

Thin Python binding over the C ABI in ``include/sage_fp4.h`` (``libsage_fp4.so``, built
in-tree by ``microscaling_fp4_quantized_b200.build``). Every step of the computation
runs in the library's CUDA kernels; this module only checks arguments, allocates
outputs/workspace with torch and passes pointers plus the current CUDA stream. There is
no CPU fallback: if the library cannot be loaded, every call raises.

    import microscaling_fp4_quantized_b200 as sage
    out = sage.attn(q, k, v, causal=False)          # q, k, v: [B, H, N, D] bf16/fp16 CUDA
    out = sage.sageattn(q, k, v, tensor_layout="NHD", is_causal=True)   # strided, GQA
    out = sage.sageattn_varlen(q, k, v, cu_q, cu_k, max_q, max_k)      # packed sequences
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

from . import workloads  # noqa: F401  (seeded synthetic inputs)

_HERE = os.path.dirname(os.path.abspath(__file__))
# SAGE_FP4_LIB may point at another build of the same library (A/B comparisons).
LIB_PATH = os.environ.get("SAGE_FP4_LIB") or os.path.join(_HERE, "libsage_fp4.so")

SAGE_OK, SAGE_ERR_INVALID_ARG, SAGE_ERR_UNSUPPORTED, SAGE_ERR_CUDA, SAGE_ERR_TIMEOUT, SAGE_ERR_BOUNDS = range(6)
SAGE_BF16, SAGE_F16 = 0, 1
GSCALE = {"none": 0, "tensor": 1, "head": 2}
PRECISION = {"fp4": 0, "8bit": 1}

EXPORTED = [
    "sage_status_string", "sage_fp4_quantized_sizes", "sage_fp4_quantize_scratch_bytes",
    "sage_fp4_quantize_qkv", "sage_fp4_attn_fwd_quantized", "sage_fp4_workspace_bytes",
    "sage_fp4_attn_fwd_ex", "sage_fp4_attn_fwd", "sage_fp4_qk_scores",
    "sage_fp4_get_device_error", "sage_fp4_set_wait_timeout_ns", "sage_fp4_attn_fwd_noalloc",
    "sage_fp4_last_cuda_error", "sage_fp4_set_debug_flags", "sage_fp4_problem_sizes",
    "sage_fp4_quantize", "sage_fp4_attn_quantized", "sage_fp4_attn", "sage_fp4_mma_rate",
    "sage_fp4_bounds_checked",
]


class SageError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        detail = ""
        if status == SAGE_ERR_CUDA:
            try:
                detail = " (" + lib().sage_fp4_last_cuda_error().decode() + ")"
            except Exception:
                pass
        super().__init__(f"{what}: {_status_name(status)}{detail}")


class _Sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf", "k_mean")]


class _Problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("D", ctypes.c_int),
                ("Nq", ctypes.c_int), ("Nk", ctypes.c_int),
                ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
                ("total_q", ctypes.c_int), ("total_k", ctypes.c_int),
                ("q_stride", ctypes.c_int64 * 3), ("k_stride", ctypes.c_int64 * 3),
                ("v_stride", ctypes.c_int64 * 3), ("o_stride", ctypes.c_int64 * 3),
                ("dtype", ctypes.c_int), ("causal", ctypes.c_int), ("sm_scale", ctypes.c_float),
                ("smooth_k", ctypes.c_int), ("gscale", ctypes.c_int), ("smooth_q", ctypes.c_int),
                ("precision", ctypes.c_int)]


_QZ_FIELDS = ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf", "k_mean", "amax", "seq", "q_mean",
              "qk_bias")


class _Quantized(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _QZ_FIELDS]


class _ProblemSizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in _QZ_FIELDS + ("scratch", "workspace")]


_lib = None


def lib():
    """The loaded CUDA library (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m microscaling_fp4_quantized_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i, u8p, vp, sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
        f = ctypes.c_float
        L.sage_status_string.argtypes = [i]
        L.sage_status_string.restype = ctypes.c_char_p
        L.sage_fp4_quantized_sizes.argtypes = [i, i, i, i, ctypes.POINTER(_Sizes)]
        L.sage_fp4_quantize_scratch_bytes.argtypes = [i, i, i, i]
        L.sage_fp4_quantize_scratch_bytes.restype = sz
        L.sage_fp4_quantize_qkv.argtypes = [vp, vp, vp, i, i, i, i, i, i, u8p, u8p, u8p, u8p, u8p,
                                            u8p, vp, vp, sz, vp]
        L.sage_fp4_attn_fwd_quantized.argtypes = [u8p, u8p, u8p, u8p, u8p, u8p, vp, i, i, i, i, i,
                                                  i, f, vp]
        L.sage_fp4_workspace_bytes.argtypes = [i, i, i, i]
        L.sage_fp4_workspace_bytes.restype = sz
        L.sage_fp4_attn_fwd_ex.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, vp, sz, vp]
        L.sage_fp4_attn_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, vp]
        L.sage_fp4_qk_scores.argtypes = [u8p, u8p, u8p, u8p, vp, i, i, i, i, f, vp]
        L.sage_fp4_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), vp]
        L.sage_fp4_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
        L.sage_fp4_set_debug_flags.argtypes = [ctypes.c_uint32]
        L.sage_fp4_last_cuda_error.argtypes = []
        L.sage_fp4_last_cuda_error.restype = ctypes.c_char_p
        L.sage_fp4_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
        pp = ctypes.POINTER(_Problem)
        L.sage_fp4_problem_sizes.argtypes = [pp, ctypes.POINTER(_ProblemSizes)]
        L.sage_fp4_quantize.argtypes = [pp, vp, vp, vp, ctypes.POINTER(_Quantized), vp, sz, vp]
        L.sage_fp4_attn_quantized.argtypes = [pp, ctypes.POINTER(_Quantized), vp, vp]
        L.sage_fp4_attn.argtypes = [pp, vp, vp, vp, vp, vp, sz, vp]
        L.sage_fp4_mma_rate.argtypes = [i, i, i, vp]
        L.sage_fp4_bounds_checked.argtypes = []
        for n in EXPORTED[1:]:
            if n not in ("sage_fp4_quantize_scratch_bytes", "sage_fp4_workspace_bytes",
                         "sage_fp4_last_cuda_error"):
                getattr(L, n).restype = i  # sage_status_t
        _lib = L
    return _lib


def _status_name(s: int) -> str:
    try:
        return lib().sage_status_string(int(s)).decode()
    except Exception:  # library not loadable: still report the number
        return f"status {s}"


def _check(status: int, what: str):
    if status != SAGE_OK:
        raise SageError(status, what)


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return SAGE_BF16
    if dt == torch.float16:
        return SAGE_F16
    raise TypeError(f"unsupported dtype {dt}; use bfloat16 or float16")


def _check_qkv(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dim() != 4:
            raise ValueError(f"{name} must be [B, H, N, D]")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must have the same dtype")
    return q.shape


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def sizes(B: int, H: int, N: int, D: int) -> dict:
    s = _Sizes()
    _check(lib().sage_fp4_quantized_sizes(B, H, N, D, ctypes.byref(s)), "sage_fp4_quantized_sizes")
    return {n: int(getattr(s, n)) for n, _ in _Sizes._fields_}


def padded_tokens(N: int) -> int:
    return (N + 127) // 128 * 128


def quantize_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, smooth_k: bool = True) -> dict:
    """K mean and FP4 quantization of Q, K (smoothed), V^T in the library's layouts."""
    B, H, N, D = _check_qkv(q, k, v)
    sz = sizes(B, H, N, D)
    dev = q.device
    out = {n: torch.empty(max(sz[n], 16), dtype=torch.uint8, device=dev) for n in
           ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf")}
    out["k_mean"] = torch.empty(max(sz["k_mean"] // 4, 4), dtype=torch.float32, device=dev)
    scratch_bytes = lib().sage_fp4_quantize_scratch_bytes(B, H, N, D)
    scratch = torch.empty(max(scratch_bytes, 16), dtype=torch.uint8, device=dev)
    _check(lib().sage_fp4_quantize_qkv(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), B, H, N, D, int(bool(smooth_k)),
        _ptr(out["q_fp4"]), _ptr(out["q_sf"]), _ptr(out["k_fp4"]), _ptr(out["k_sf"]),
        _ptr(out["vt_fp4"]), _ptr(out["vt_sf"]), _ptr(out["k_mean"]), _ptr(scratch),
        scratch_bytes, _stream(dev)), "sage_fp4_quantize_qkv")
    out.update(B=B, H=H, N=N, D=D, Np=padded_tokens(N), dtype=q.dtype)
    return out


def attn_quantized(qz: dict, causal: bool = False, sm_scale: Optional[float] = None,
                   out_dtype: Optional[torch.dtype] = None) -> torch.Tensor:
    """Fused FP4 attention on the output of :func:`quantize_qkv`."""
    B, H, N, D = qz["B"], qz["H"], qz["N"], qz["D"]
    odt = out_dtype or qz["dtype"]
    dev = qz["q_fp4"].device
    out = torch.empty((B, H, N, D), dtype=odt, device=dev)
    _check(lib().sage_fp4_attn_fwd_quantized(
        _ptr(qz["q_fp4"]), _ptr(qz["q_sf"]), _ptr(qz["k_fp4"]), _ptr(qz["k_sf"]), _ptr(qz["vt_fp4"]),
        _ptr(qz["vt_sf"]), _ptr(out), _dtype_code(odt), B, H, N, D, int(bool(causal)),
        float(sm_scale or 0.0), _stream(dev)), "sage_fp4_attn_fwd_quantized")
    return out


def workspace_bytes(B: int, H: int, N: int, D: int) -> int:
    return int(lib().sage_fp4_workspace_bytes(B, H, N, D))


def attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
         sm_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
         workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """FP4 attention forward: softmax(sm_scale Q K^T [causal]) V, [B, H, N, D] in and out."""
    B, H, N, D = _check_qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    ws_bytes = workspace_bytes(B, H, N, D)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=q.device)
    _check(lib().sage_fp4_attn_fwd_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q.dtype), B, H, N, D, int(bool(causal)),
        float(sm_scale or 0.0), _ptr(workspace), workspace.numel(), _stream(q.device)),
        "sage_fp4_attn_fwd_ex")
    return out


def attn_bf16_library_workspace(q, k, v, causal: bool = False, sm_scale: Optional[float] = None):
    """The bf16 entry point whose workspace comes from the stream-ordered allocator."""
    B, H, N, D = _check_qkv(q, k, v)
    out = torch.empty_like(q)
    _check(lib().sage_fp4_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, D,
                                   int(bool(causal)), float(sm_scale or 0.0), _stream(q.device)),
           "sage_fp4_attn_fwd")
    return out


def attn_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                 sm_scale: Optional[float] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The forward through the entry point that allocates no device memory (its scratch is
    a fixed 16 MiB device array inside the library; larger problems raise). For callers
    that cannot allocate; calls on different streams of one device must not overlap."""
    B, H, N, D = _check_qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sage_fp4_attn_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q.dtype), B, H, N, D, int(bool(causal)),
        float(sm_scale or 0.0), _stream(q.device)), "sage_fp4_attn_fwd_noalloc")
    return out


def qk_scores(qz: dict, sm_scale: Optional[float] = None) -> torch.Tensor:
    """S = sm_scale * Q^ K^^T for all (padded) query/key pairs: [B*H, Np, Np] float32."""
    BH, Np = qz["B"] * qz["H"], qz["Np"]
    s = torch.empty((BH, Np, Np), dtype=torch.float32, device=qz["q_fp4"].device)
    _check(lib().sage_fp4_qk_scores(
        _ptr(qz["q_fp4"]), _ptr(qz["q_sf"]), _ptr(qz["k_fp4"]), _ptr(qz["k_sf"]), _ptr(s),
        qz["B"], qz["H"], qz["N"], qz["D"], float(sm_scale or 0.0), _stream(s.device)),
        "sage_fp4_qk_scores")
    return s


DEV_ERR_TIMEOUT, DEV_ERR_SEQLENS, DEV_ERR_BOUNDS = 1, 2, 4


def device_error(device=None) -> int:
    """Read and clear the device error word (synchronizes the current stream): bit 0 a
    bounded wait ran out, bit 1 a packed problem's sequence table failed its check."""
    w = ctypes.c_uint32(0)
    st = lib().sage_fp4_get_device_error(ctypes.byref(w), _stream(device))
    if st not in (SAGE_OK, SAGE_ERR_TIMEOUT, SAGE_ERR_INVALID_ARG, SAGE_ERR_BOUNDS):
        raise SageError(st, "sage_fp4_get_device_error")
    return int(w.value)


def set_wait_timeout_ns(ns: int) -> None:
    _check(lib().sage_fp4_set_wait_timeout_ns(int(ns)), "sage_fp4_set_wait_timeout_ns")


def set_debug_flags(flags: int) -> None:
    """Test switch: bit 0 makes the attention kernel issue no loads, so its bounded waits
    run out and the device error word reports a timeout (0 restores normal operation)."""
    _check(lib().sage_fp4_set_debug_flags(int(flags)), "sage_fp4_set_debug_flags")


def mma_rate(n: int = 128, iters: int = 200000, ctas: Optional[int] = None, repeats: int = 5,
             device=None) -> dict:
    """Measured rate of the block-scaled FP4 tensor-core instruction (M128 x N x K64) with
    one CTA per SM: the best of `repeats` CUDA-event timings of sage_fp4_mma_rate after one
    warm-up launch. Returns {"tflops", "ms", "ops", "ctas", "n"}."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if ctas is None:
        ctas = torch.cuda.get_device_properties(dev).multi_processor_count
    s = _stream(dev)
    _check(lib().sage_fp4_mma_rate(n, max(1, iters // 10), ctas, s), "sage_fp4_mma_rate")
    best = None
    for _ in range(repeats):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        _check(lib().sage_fp4_mma_rate(n, iters, ctas, s), "sage_fp4_mma_rate")
        b.record()
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b)
        best = ms if best is None else min(best, ms)
    if device_error(dev) != 0:
        raise SageError(SAGE_ERR_TIMEOUT, "sage_fp4_mma_rate")
    ops = 2.0 * 128 * n * 64 * iters * ctas
    return {"tflops": ops / best / 1e9, "ms": best, "ops": ops, "ctas": ctas, "n": n}


def default_sm_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


class Plan:
    """Preallocated buffers for one problem shape: the forward as two C-ABI calls
    (quantize, then fused attention) with no allocation per call."""

    def __init__(self, B: int, H: int, N: int, D: int, dtype: torch.dtype = torch.bfloat16,
                 device="cuda"):
        self.B, self.H, self.N, self.D, self.dtype = B, H, N, D, dtype
        self.device = torch.device(device)
        sz = sizes(B, H, N, D)
        self.buf = {n: torch.empty(max(sz[n], 16), dtype=torch.uint8, device=self.device) for n in
                    ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf")}
        self.k_mean = torch.empty(max(sz["k_mean"] // 4, 4), dtype=torch.float32, device=self.device)
        self.scratch_bytes = int(lib().sage_fp4_quantize_scratch_bytes(B, H, N, D))
        self.scratch = torch.empty(max(self.scratch_bytes, 16), dtype=torch.uint8, device=self.device)

    def quantize(self, q, k, v, smooth_k: bool = True) -> None:
        b = self.buf
        _check(lib().sage_fp4_quantize_qkv(
            _ptr(q), _ptr(k), _ptr(v), _dtype_code(self.dtype), self.B, self.H, self.N, self.D,
            int(bool(smooth_k)), _ptr(b["q_fp4"]), _ptr(b["q_sf"]), _ptr(b["k_fp4"]), _ptr(b["k_sf"]),
            _ptr(b["vt_fp4"]), _ptr(b["vt_sf"]), _ptr(self.k_mean), _ptr(self.scratch),
            self.scratch_bytes, _stream(self.device)), "sage_fp4_quantize_qkv")

    def attention(self, out: torch.Tensor, causal: bool = False, sm_scale: Optional[float] = None) -> None:
        b = self.buf
        _check(lib().sage_fp4_attn_fwd_quantized(
            _ptr(b["q_fp4"]), _ptr(b["q_sf"]), _ptr(b["k_fp4"]), _ptr(b["k_sf"]), _ptr(b["vt_fp4"]),
            _ptr(b["vt_sf"]), _ptr(out), _dtype_code(out.dtype), self.B, self.H, self.N, self.D,
            int(bool(causal)), float(sm_scale or 0.0), _stream(self.device)),
            "sage_fp4_attn_fwd_quantized")


# ------------------------------------------------------------------ general problems --

def _strides3(t: torch.Tensor, dims) -> tuple:
    if t.stride(-1) != 1:
        raise ValueError("the channel (last) dimension must be contiguous")
    return tuple(int(t.stride(d)) for d in dims)


def make_problem(*, B: int, Hq: int, Hkv: int, D: int, Nq: int, Nk: int, dtype: torch.dtype,
                 q_stride, k_stride, v_stride, o_stride, causal: bool = False,
                 sm_scale: Optional[float] = None, smooth_k: bool = True, gscale: str = "none",
                 cu_seqlens_q: Optional[torch.Tensor] = None,
                 cu_seqlens_k: Optional[torch.Tensor] = None, total_q: int = 0,
                 total_k: int = 0, smooth_q: bool = False, precision: str = "fp4") -> _Problem:
    """The C problem descriptor (strides in elements of (sequence, head, token))."""
    if gscale not in GSCALE:
        raise ValueError(f"gscale must be one of {tuple(GSCALE)}")
    if precision not in PRECISION:
        raise ValueError(f"precision must be one of {tuple(PRECISION)}")
    pr = _Problem()
    pr.B, pr.Hq, pr.Hkv, pr.D, pr.Nq, pr.Nk = B, Hq, Hkv, D, Nq, Nk
    pr.cu_seqlens_q = cu_seqlens_q.data_ptr() if cu_seqlens_q is not None else None
    pr.cu_seqlens_k = cu_seqlens_k.data_ptr() if cu_seqlens_k is not None else None
    pr.total_q, pr.total_k = total_q, total_k
    for name, st in (("q_stride", q_stride), ("k_stride", k_stride), ("v_stride", v_stride),
                     ("o_stride", o_stride)):
        arr = getattr(pr, name)
        for i in range(3):
            arr[i] = int(st[i])
    pr.dtype = _dtype_code(dtype)
    pr.causal = int(bool(causal))
    pr.sm_scale = float(sm_scale or 0.0)
    pr.smooth_k = int(bool(smooth_k))
    pr.gscale = GSCALE[gscale]
    pr.smooth_q = int(bool(smooth_q))
    pr.precision = PRECISION[precision]
    return pr


def problem_sizes(pr: _Problem) -> dict:
    z = _ProblemSizes()
    _check(lib().sage_fp4_problem_sizes(ctypes.byref(pr), ctypes.byref(z)), "sage_fp4_problem_sizes")
    return {n: int(getattr(z, n)) for n, _ in _ProblemSizes._fields_}


def quantize(pr: _Problem, q, k, v) -> dict:
    """K statistics, second-level maxima and FP4 quantization of a general problem into
    freshly allocated buffers (returned as uint8 / float32 / int32 tensors)."""
    z = problem_sizes(pr)
    dev = q.device
    buf = {n: torch.empty(max(z[n], 16), dtype=torch.uint8, device=dev) for n in _QZ_FIELDS}
    scratch = torch.empty(max(z["scratch"], 16), dtype=torch.uint8, device=dev)
    qz = _Quantized(*[ctypes.c_void_p(buf[n].data_ptr()) for n in _QZ_FIELDS])
    _check(lib().sage_fp4_quantize(ctypes.byref(pr), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(qz),
                                   _ptr(scratch), z["scratch"], _stream(dev)), "sage_fp4_quantize")
    buf["k_mean"] = buf["k_mean"].view(torch.float32)
    buf["amax"] = buf["amax"].view(torch.float32)
    buf["seq"] = buf["seq"].view(torch.int32)
    buf["q_mean"] = buf["q_mean"].view(torch.float32)
    buf["problem"] = pr
    return buf


def attn_quantized_problem(qz: dict, out: torch.Tensor) -> torch.Tensor:
    """Fused attention on the output of :func:`quantize` (same problem), into `out`."""
    pr = qz["problem"]
    c = _Quantized(*[ctypes.c_void_p(qz[n].data_ptr()) for n in _QZ_FIELDS])
    _check(lib().sage_fp4_attn_quantized(ctypes.byref(pr), ctypes.byref(c), _ptr(out), _stream(out.device)),
           "sage_fp4_attn_quantized")
    return out


def _run(pr: _Problem, q, k, v, out, workspace):
    ws = problem_sizes(pr)["workspace"]
    if workspace is None or workspace.numel() < ws:
        workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=q.device)
    _check(lib().sage_fp4_attn(ctypes.byref(pr), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(workspace),
                               workspace.numel(), _stream(q.device)), "sage_fp4_attn")
    return out


def _same_kind(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must have the same dtype")
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")


def sageattn_problem(q, k, v, out, tensor_layout: str = "HND", is_causal: bool = False,
                     sm_scale: Optional[float] = None, smooth_k: bool = True,
                     gscale: str = "none", smooth_q: bool = False, precision: str = "fp4") -> _Problem:
    """The problem descriptor :func:`sageattn` passes to the library."""
    _same_kind(q, k, v)
    if tensor_layout == "HND":
        B, Hq, Nq, D = q.shape
        _, Hkv, Nk, _ = k.shape
        dims = (0, 1, 2)
    elif tensor_layout == "NHD":
        B, Nq, Hq, D = q.shape
        _, Nk, Hkv, _ = k.shape
        dims = (0, 2, 1)
    else:
        raise ValueError("tensor_layout must be 'HND' or 'NHD'")
    if k.shape[0] != B or k.shape[-1] != D:
        raise ValueError("q and k disagree on batch or head dimension")
    return make_problem(B=B, Hq=Hq, Hkv=Hkv, D=D, Nq=Nq, Nk=Nk, dtype=q.dtype,
                        q_stride=_strides3(q, dims), k_stride=_strides3(k, dims),
                        v_stride=_strides3(v, dims), o_stride=_strides3(out, dims), causal=is_causal,
                        sm_scale=sm_scale, smooth_k=smooth_k, gscale=gscale, smooth_q=smooth_q,
                        precision=precision)


def sageattn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, tensor_layout: str = "HND",
             is_causal: bool = False, sm_scale: Optional[float] = None, smooth_k: bool = True,
             gscale: str = "none", out: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None, smooth_q: bool = False,
             precision: str = "fp4") -> torch.Tensor:
    """FP4 attention on [B, H, N, D] ("HND") or [B, N, H, D] ("NHD") tensors with any
    strides (channels contiguous). k and v may have fewer heads than q (each shared by
    Hq / Hkv query heads) and a different length (the causal mask then aligns the last
    query with the last key). gscale adds a second-level FP32 scale per tensor ("tensor")
    or per (batch, head) ("head"); smooth_q subtracts each head's query mean before
    quantization and adds its product with the keys back to the scores. precision="8bit"
    runs the 8-bit path instead (INT8 Q/K per 128-token tile, E4M3 P~ and V)."""
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    pr = sageattn_problem(q, k, v, out, tensor_layout, is_causal, sm_scale, smooth_k, gscale, smooth_q,
                          precision)
    return _run(pr, q, k, v, out, workspace)


def sageattn_varlen_problem(q, k, v, out, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                            max_seqlen_k: int, is_causal: bool = False,
                            sm_scale: Optional[float] = None, smooth_k: bool = True,
                            gscale: str = "none", smooth_q: bool = False,
                            precision: str = "fp4") -> _Problem:
    """The problem descriptor :func:`sageattn_varlen` passes to the library."""
    _same_kind(q, k, v)
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("packed tensors are [total, H, D]")
    for t in (cu_seqlens_q, cu_seqlens_k):
        if t.dtype != torch.int32 or not t.is_cuda or t.dim() != 1 or not t.is_contiguous():
            raise ValueError("cu_seqlens must be contiguous int32 CUDA tensors")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold B + 1 offsets")
    total_q, Hq, D = q.shape
    total_k, Hkv, _ = k.shape
    dims = (0, 1, 0)
    return make_problem(B=cu_seqlens_q.numel() - 1, Hq=Hq, Hkv=Hkv, D=D, Nq=int(max_seqlen_q),
                      Nk=int(max_seqlen_k), dtype=q.dtype, q_stride=_strides3(q, dims),
                      k_stride=_strides3(k, dims), v_stride=_strides3(v, dims),
                      o_stride=_strides3(out, dims), causal=is_causal, sm_scale=sm_scale,
                      smooth_k=smooth_k, gscale=gscale, cu_seqlens_q=cu_seqlens_q,
                      cu_seqlens_k=cu_seqlens_k, total_q=total_q, total_k=total_k,
                      smooth_q=smooth_q, precision=precision)


def sageattn_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q: torch.Tensor,
                    cu_seqlens_k: torch.Tensor, max_seqlen_q: int, max_seqlen_k: int,
                    is_causal: bool = False, sm_scale: Optional[float] = None,
                    smooth_k: bool = True, gscale: str = "none",
                    out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, smooth_q: bool = False,
                    precision: str = "fp4") -> torch.Tensor:
    """FP4 attention on packed sequences: q [total_q, Hq, D], k and v [total_k, Hkv, D];
    sequence b holds tokens cu_seqlens_q[b] .. cu_seqlens_q[b+1] (int32 CUDA tensors of
    B+1 offsets; a bad table is reported by device_error(), never by a fault). Each
    sequence is its own problem: its own K mean, causal mask and ("head") scales."""
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    pr = sageattn_varlen_problem(q, k, v, out, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                                 max_seqlen_k, is_causal, sm_scale, smooth_k, gscale, smooth_q, precision)
    return _run(pr, q, k, v, out, workspace)


class ProblemPlan:
    """Preallocated quantized buffers, scratch and the C problem descriptor for one general
    problem (see :func:`sageattn_problem` / :func:`sageattn_varlen_problem`): the forward as
    two C-ABI calls, sage_fp4_quantize and sage_fp4_attn_quantized, with no allocation per
    call. The tensors passed to quantize() must have the shapes and strides the problem
    was built from."""

    def __init__(self, problem: _Problem, device="cuda"):
        self.problem = problem
        self.device = torch.device(device)
        z = problem_sizes(problem)
        self.sizes = z
        self.buf = {n: torch.empty(max(z[n], 16), dtype=torch.uint8, device=self.device) for n in _QZ_FIELDS}
        self.scratch = torch.empty(max(z["scratch"], 16), dtype=torch.uint8, device=self.device)
        self._qz = _Quantized(*[ctypes.c_void_p(self.buf[n].data_ptr()) for n in _QZ_FIELDS])

    def quantize(self, q, k, v) -> None:
        _check(lib().sage_fp4_quantize(ctypes.byref(self.problem), _ptr(q), _ptr(k), _ptr(v),
                                       ctypes.byref(self._qz), _ptr(self.scratch), self.sizes["scratch"],
                                       _stream(self.device)), "sage_fp4_quantize")

    def attention(self, out: torch.Tensor) -> None:
        _check(lib().sage_fp4_attn_quantized(ctypes.byref(self.problem), ctypes.byref(self._qz), _ptr(out),
                                             _stream(self.device)), "sage_fp4_attn_quantized")
