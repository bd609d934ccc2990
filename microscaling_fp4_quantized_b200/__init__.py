"""Microscaling-FP4 attention forward (SageAttention3 method) for NVIDIA B200, sm_100a.

Thin Python binding over the C ABI in ``include/sage_fp4.h`` (``libsage_fp4.so``, built
in-tree by ``microscaling_fp4_quantized_b200.build``). Every step of the computation
runs in the library's CUDA kernels; this module only checks arguments, allocates
outputs/workspace with torch and passes pointers plus the current CUDA stream. There is
no CPU fallback: if the library cannot be loaded, every call raises.

    import microscaling_fp4_quantized_b200 as sage
    out = sage.attn(q, k, v, causal=False)          # q, k, v: [B, H, N, D] bf16/fp16 CUDA
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

SAGE_OK, SAGE_ERR_INVALID_ARG, SAGE_ERR_UNSUPPORTED, SAGE_ERR_CUDA, SAGE_ERR_TIMEOUT = range(5)
SAGE_BF16, SAGE_F16 = 0, 1

EXPORTED = [
    "sage_status_string", "sage_fp4_quantized_sizes", "sage_fp4_quantize_scratch_bytes",
    "sage_fp4_quantize_qkv", "sage_fp4_attn_fwd_quantized", "sage_fp4_workspace_bytes",
    "sage_fp4_attn_fwd_ex", "sage_fp4_attn_fwd", "sage_fp4_qk_scores",
    "sage_fp4_get_device_error", "sage_fp4_set_wait_timeout_ns", "sage_fp4_attn_fwd_noalloc",
    "sage_fp4_last_cuda_error", "sage_fp4_set_debug_flags",
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


def device_error(device=None) -> int:
    """Read and clear the device error word (synchronizes the current stream)."""
    w = ctypes.c_uint32(0)
    st = lib().sage_fp4_get_device_error(ctypes.byref(w), _stream(device))
    if st not in (SAGE_OK, SAGE_ERR_TIMEOUT):
        raise SageError(st, "sage_fp4_get_device_error")
    return int(w.value)


def set_wait_timeout_ns(ns: int) -> None:
    _check(lib().sage_fp4_set_wait_timeout_ns(int(ns)), "sage_fp4_set_wait_timeout_ns")


def set_debug_flags(flags: int) -> None:
    """Test switch: bit 0 makes the attention kernel issue no loads, so its bounded waits
    run out and the device error word reports a timeout (0 restores normal operation)."""
    _check(lib().sage_fp4_set_debug_flags(int(flags)), "sage_fp4_set_debug_flags")


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
