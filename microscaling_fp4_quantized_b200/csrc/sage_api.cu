// C ABI of the FP4 attention library (declared in include/sage_fp4.h): argument checks,
// workspace carving, TMA descriptors and kernel launches. Host code only, apart from the
// device error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "sage_fp4.h"
#include "sage_internal.h"

namespace {

__device__ uint32_t g_sage_dev_error;

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<uint32_t> g_debug_flags{0};

constexpr int kMaxDevices = 64;
uint32_t* g_err_ptr[kMaxDevices] = {};
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

thread_local char g_last_error[256] = "";

sage_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SAGE_OK;
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return SAGE_ERR_CUDA;
}

// Address of the device error word on the current device.
sage_status_t error_word(uint32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sage_dev_error) != cudaSuccess) return SAGE_ERR_CUDA;
    g_err_ptr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_err_ptr[dev];
  return SAGE_OK;
}

sage_status_t encoder(EncodeTiledFn* fn) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || f == nullptr)
      return SAGE_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(f);
  }
  *fn = g_encode;
  return SAGE_OK;
}

// 2-D byte tensor [rows, inner] with a box of [box_rows, box_inner], swizzled.
sage_status_t make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                       uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn;
  if (sage_status_t s = encoder(&fn); s != SAGE_OK) return s;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SAGE_OK : SAGE_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Shape {
  int64_t BH, N, Np, D, nsplit;
  bool empty;
};

sage_status_t check_shape(int B, int H, int N, int D, Shape* s) {
  if (B < 0 || H < 0 || N < 0) return SAGE_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
  s->BH = static_cast<int64_t>(B) * H;
  s->N = N;
  s->Np = (static_cast<int64_t>(N) + 127) / 128 * 128;
  s->D = D;
  s->nsplit = (static_cast<int64_t>(N) + 511) / 512;
  s->empty = (s->BH == 0 || N == 0);
  if (s->empty) return SAGE_OK;
  // Grid y/z limits and 32-bit TMA coordinates / element counts.
  if (s->BH > 65535 || s->BH * s->Np >= (int64_t(1) << 31) || s->BH * s->Np * D >= (int64_t(1) << 33))
    return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

sage_fp4_sizes_t sizes_of(const Shape& s) {
  sage_fp4_sizes_t z;
  if (s.empty) {
    std::memset(&z, 0, sizeof(z));
    return z;
  }
  z.q_fp4 = z.k_fp4 = static_cast<size_t>(s.BH * s.Np * s.D / 2);
  z.q_sf = z.k_sf = static_cast<size_t>(s.BH * s.Np * s.D / 16);
  z.vt_fp4 = static_cast<size_t>(s.BH * s.D * s.Np / 2);
  z.vt_sf = static_cast<size_t>(s.BH * (s.Np / 128) * 1024);
  z.k_mean = static_cast<size_t>(s.BH * s.D * 4);
  return z;
}

size_t scratch_of(const Shape& s) {
  return s.empty ? 0 : static_cast<size_t>(s.BH * s.nsplit * s.D * 8);
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

struct Carved {
  uint8_t *q_fp4, *q_sf, *k_fp4, *k_sf, *vt_fp4, *vt_sf;
  float* k_mean;
  void* scratch;
  size_t total;
};

Carved carve(const Shape& s, void* base) {
  const sage_fp4_sizes_t z = sizes_of(s);
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  Carved c;
  auto take = [&](size_t n) { uint8_t* r = p ? p + off : nullptr; off += up256(n); return r; };
  c.q_fp4 = take(z.q_fp4);
  c.q_sf = take(z.q_sf);
  c.k_fp4 = take(z.k_fp4);
  c.k_sf = take(z.k_sf);
  c.vt_fp4 = take(z.vt_fp4);
  c.vt_sf = take(z.vt_sf);
  c.k_mean = reinterpret_cast<float*>(take(z.k_mean));
  c.scratch = take(scratch_of(s));
  c.total = off;
  return c;
}

sage_status_t run_quantize(const Shape& s, const void* q, const void* k, const void* v, int dtype,
                           int smooth_k, uint8_t* q_fp4, uint8_t* q_sf, uint8_t* k_fp4, uint8_t* k_sf,
                           uint8_t* vt_fp4, uint8_t* vt_sf, float* k_mean, void* scratch,
                           cudaStream_t stream) {
  sage::QuantParams p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.dtype = dtype;
  p.BH = static_cast<int>(s.BH);
  p.N = static_cast<int>(s.N);
  p.Np = static_cast<int>(s.Np);
  p.D = static_cast<int>(s.D);
  p.smooth_k = smooth_k ? 1 : 0;
  p.nsplit = static_cast<int>(s.nsplit);
  p.q_fp4 = q_fp4;
  p.q_sf = q_sf;
  p.k_fp4 = k_fp4;
  p.k_sf = k_sf;
  p.vt_fp4 = vt_fp4;
  p.vt_sf = vt_sf;
  p.k_mean = k_mean;
  p.partial = static_cast<double*>(scratch);
  return cuda_status(sage::launch_quantize(p, stream));
}

sage_status_t build_maps(const Shape& s, const uint8_t* q_fp4, const uint8_t* k_fp4,
                         const uint8_t* vt_fp4, sage::TensorMaps* m) {
  const uint64_t inner = static_cast<uint64_t>(s.D / 2);
  const CUtensorMapSwizzle swqk = s.D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  sage_status_t st;
  if ((st = make_map(&m->q, q_fp4, inner, s.BH * s.Np, static_cast<uint32_t>(inner), 128, swqk)) != SAGE_OK) return st;
  if ((st = make_map(&m->k, k_fp4, inner, s.BH * s.Np, static_cast<uint32_t>(inner), 128, swqk)) != SAGE_OK) return st;
  if (vt_fp4 != nullptr &&
      (st = make_map(&m->v, vt_fp4, s.Np / 2, s.BH * s.D, 64, static_cast<uint32_t>(s.D), CU_TENSOR_MAP_SWIZZLE_64B)) != SAGE_OK)
    return st;
  return SAGE_OK;
}

sage_status_t fill_attn_params(const Shape& s, float sm_scale, int causal, sage::AttnParams* p) {
  uint32_t* err = nullptr;
  if (sage_status_t st = error_word(&err); st != SAGE_OK) return st;
  const float scale = sm_scale > 0.0f ? sm_scale : 1.0f / std::sqrt(static_cast<float>(s.D));
  p->BH = static_cast<int>(s.BH);
  p->N = static_cast<int>(s.N);
  p->Np = static_cast<int>(s.Np);
  p->D = static_cast<int>(s.D);
  p->causal = causal ? 1 : 0;
  p->sm_scale = scale;
  p->sm_scale_log2 = scale * 1.4426950408889634f;
  p->err = err;
  p->timeout_ns = g_timeout_ns.load();
  p->debug_flags = g_debug_flags.load();
  return SAGE_OK;
}

sage_status_t run_attention(const Shape& s, const uint8_t* q_fp4, const uint8_t* q_sf,
                            const uint8_t* k_fp4, const uint8_t* k_sf, const uint8_t* vt_fp4,
                            const uint8_t* vt_sf, void* out, int out_dtype, int causal,
                            float sm_scale, cudaStream_t stream) {
  sage::TensorMaps m;
  if (sage_status_t st = build_maps(s, q_fp4, k_fp4, vt_fp4, &m); st != SAGE_OK) return st;
  sage::AttnParams p;
  if (sage_status_t st = fill_attn_params(s, sm_scale, causal, &p); st != SAGE_OK) return st;
  p.q_sf = q_sf;
  p.k_sf = k_sf;
  p.vt_sf = vt_sf;
  p.out = out;
  p.out_dtype = out_dtype;
  return cuda_status(sage::launch_attention(m, p, stream));
}

bool valid_dtype(sage_dtype_t d) { return d == SAGE_BF16 || d == SAGE_F16; }

}  // namespace

extern "C" {

const char* sage_status_string(sage_status_t status) {
  switch (status) {
    case SAGE_OK: return "SAGE_OK";
    case SAGE_ERR_INVALID_ARG: return "SAGE_ERR_INVALID_ARG";
    case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
    case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
    case SAGE_ERR_TIMEOUT: return "SAGE_ERR_TIMEOUT";
  }
  return "SAGE_ERR_UNKNOWN";
}

sage_status_t sage_fp4_quantized_sizes(int B, int H, int N, int D, sage_fp4_sizes_t* sizes) {
  if (sizes == nullptr) return SAGE_ERR_INVALID_ARG;
  Shape s;
  if (sage_status_t st = check_shape(B, H, N, D, &s); st != SAGE_OK) return st;
  *sizes = sizes_of(s);
  return SAGE_OK;
}

size_t sage_fp4_quantize_scratch_bytes(int B, int H, int N, int D) {
  Shape s;
  if (check_shape(B, H, N, D, &s) != SAGE_OK) return 0;
  return scratch_of(s);
}

size_t sage_fp4_workspace_bytes(int B, int H, int N, int D) {
  Shape s;
  if (check_shape(B, H, N, D, &s) != SAGE_OK || s.empty) return 0;
  return carve(s, nullptr).total;
}

sage_status_t sage_fp4_quantize_qkv(const void* q, const void* k, const void* v, sage_dtype_t dtype,
                                    int B, int H, int N, int D, int smooth_k, uint8_t* q_fp4,
                                    uint8_t* q_sf, uint8_t* k_fp4, uint8_t* k_sf, uint8_t* vt_fp4,
                                    uint8_t* vt_sf, float* k_mean, void* scratch,
                                    size_t scratch_bytes, void* stream) {
  Shape s;
  if (sage_status_t st = check_shape(B, H, N, D, &s); st != SAGE_OK) return st;
  if (!valid_dtype(dtype)) return SAGE_ERR_INVALID_ARG;
  if (s.empty) return SAGE_OK;
  const void* ptrs[] = {q, k, v, q_fp4, q_sf, k_fp4, k_sf, vt_fp4, vt_sf};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  if (smooth_k) {
    if (scratch == nullptr || !aligned16(scratch) || scratch_bytes < scratch_of(s)) return SAGE_ERR_INVALID_ARG;
    if (k_mean != nullptr && !aligned16(k_mean)) return SAGE_ERR_INVALID_ARG;
  }
  return run_quantize(s, q, k, v, dtype, smooth_k, q_fp4, q_sf, k_fp4, k_sf, vt_fp4, vt_sf, k_mean,
                      scratch, static_cast<cudaStream_t>(stream));
}

sage_status_t sage_fp4_attn_fwd_quantized(const uint8_t* q_fp4, const uint8_t* q_sf,
                                          const uint8_t* k_fp4, const uint8_t* k_sf,
                                          const uint8_t* vt_fp4, const uint8_t* vt_sf, void* out,
                                          sage_dtype_t out_dtype, int B, int H, int N, int D,
                                          int causal, float sm_scale, void* stream) {
  Shape s;
  if (sage_status_t st = check_shape(B, H, N, D, &s); st != SAGE_OK) return st;
  if (!valid_dtype(out_dtype)) return SAGE_ERR_INVALID_ARG;
  if (s.empty) return SAGE_OK;
  const void* ptrs[] = {q_fp4, q_sf, k_fp4, k_sf, vt_fp4, vt_sf, out};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  return run_attention(s, q_fp4, q_sf, k_fp4, k_sf, vt_fp4, vt_sf, out, out_dtype, causal, sm_scale,
                       static_cast<cudaStream_t>(stream));
}

sage_status_t sage_fp4_attn_fwd_ex(const void* q, const void* k, const void* v, void* out,
                                   sage_dtype_t dtype, int B, int H, int N, int D, int causal,
                                   float sm_scale, void* workspace, size_t ws_bytes, void* stream) {
  Shape s;
  if (sage_status_t st = check_shape(B, H, N, D, &s); st != SAGE_OK) return st;
  if (!valid_dtype(dtype)) return SAGE_ERR_INVALID_ARG;
  if (s.empty) return SAGE_OK;
  const void* ptrs[] = {q, k, v, out};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SAGE_ERR_INVALID_ARG;
  Carved c = carve(s, workspace);
  if (ws_bytes < c.total) return SAGE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  sage_status_t r = run_quantize(s, q, k, v, dtype, 1, c.q_fp4, c.q_sf, c.k_fp4, c.k_sf, c.vt_fp4,
                                 c.vt_sf, c.k_mean, c.scratch, st);
  if (r != SAGE_OK) return r;
  return run_attention(s, c.q_fp4, c.q_sf, c.k_fp4, c.k_sf, c.vt_fp4, c.vt_sf, out, dtype, causal,
                       sm_scale, st);
}

sage_status_t sage_fp4_attn_fwd(const void* q, const void* k, const void* v, void* out, int B,
                                int H, int N, int D, int causal, float sm_scale, void* stream) {
  Shape s;
  if (sage_status_t st = check_shape(B, H, N, D, &s); st != SAGE_OK) return st;
  if (s.empty) return SAGE_OK;
  const void* ptrs[] = {q, k, v, out};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = carve(s, nullptr).total;
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, bytes, st) != cudaSuccess) return SAGE_ERR_CUDA;
  sage_status_t r = sage_fp4_attn_fwd_ex(q, k, v, out, SAGE_BF16, B, H, N, D, causal, sm_scale, ws,
                                         bytes, stream);
  const cudaError_t e = cudaFreeAsync(ws, st);
  if (r == SAGE_OK && e != cudaSuccess) r = SAGE_ERR_CUDA;
  return r;
}

sage_status_t sage_fp4_qk_scores(const uint8_t* q_fp4, const uint8_t* q_sf, const uint8_t* k_fp4,
                                 const uint8_t* k_sf, float* s_out, int B, int H, int N, int D,
                                 float sm_scale, void* stream) {
  Shape s;
  if (sage_status_t st = check_shape(B, H, N, D, &s); st != SAGE_OK) return st;
  if (s.empty) return SAGE_OK;
  const void* ptrs[] = {q_fp4, q_sf, k_fp4, k_sf, s_out};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if (s.Np / 128 > 65535) return SAGE_ERR_UNSUPPORTED;
  sage::TensorMaps m;
  if (sage_status_t st = build_maps(s, q_fp4, k_fp4, nullptr, &m); st != SAGE_OK) return st;
  sage::AttnParams p;
  if (sage_status_t st = fill_attn_params(s, sm_scale, 0, &p); st != SAGE_OK) return st;
  p.q_sf = q_sf;
  p.k_sf = k_sf;
  p.vt_sf = nullptr;
  p.out = s_out;
  p.out_dtype = 0;
  return cuda_status(sage::launch_qk_scores(m, p, static_cast<cudaStream_t>(stream)));
}

sage_status_t sage_fp4_get_device_error(uint32_t* word, void* stream) {
  if (word == nullptr) return SAGE_ERR_INVALID_ARG;
  uint32_t* dev = nullptr;
  if (sage_status_t st = error_word(&dev); st != SAGE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  if (cudaMemcpyAsync(&host, dev, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess) return SAGE_ERR_CUDA;
  if (cudaMemsetAsync(dev, 0, sizeof(uint32_t), s) != cudaSuccess) return SAGE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SAGE_ERR_CUDA;
  *word = host;
  return host == 0 ? SAGE_OK : SAGE_ERR_TIMEOUT;
}

const char* sage_fp4_last_cuda_error(void) { return g_last_error; }

sage_status_t sage_fp4_set_debug_flags(uint32_t flags) {
  if (flags & ~1u) return SAGE_ERR_INVALID_ARG;
  g_debug_flags.store(flags);
  return SAGE_OK;
}

sage_status_t sage_fp4_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : ns);
  return SAGE_OK;
}

}  // extern "C"
