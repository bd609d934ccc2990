// C ABI of the FP4 attention library (declared in include/sage_fp4.h): argument checks,
// workspace carving, TMA descriptors and kernel launches. Host code only, apart from the
// device error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
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
bool valid_dtype(int d) { return d == SAGE_BF16 || d == SAGE_F16; }
int64_t round128(int64_t x) { return (x + 127) / 128 * 128; }
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// A checked problem with everything derived from it.
struct Prob {
  sage_fp4_problem_t u;  // the caller's description (sm_scale resolved)
  bool packed, empty, gs, sq, b8;
  int64_t rows_q, rows_k;  // padded token rows per head (packed: an upper bound)
  int tiles_q, tiles_k, nsplit;
};

sage_status_t check_problem(const sage_fp4_problem_t* in, Prob* p) {
  if (in == nullptr) return SAGE_ERR_INVALID_ARG;
  const sage_fp4_problem_t& u = *in;
  p->u = u;
  if (u.B < 0 || u.Hq < 0 || u.Hkv < 0 || u.Nq < 0 || u.Nk < 0) return SAGE_ERR_INVALID_ARG;
  if (u.D != 64 && u.D != 128) return SAGE_ERR_UNSUPPORTED;
  if (!valid_dtype(u.dtype)) return SAGE_ERR_INVALID_ARG;
  if (u.gscale != SAGE_GSCALE_NONE && u.gscale != SAGE_GSCALE_TENSOR && u.gscale != SAGE_GSCALE_HEAD)
    return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(u.sm_scale)) return SAGE_ERR_INVALID_ARG;
  p->u.sm_scale = u.sm_scale > 0.0f ? u.sm_scale : 1.0f / std::sqrt(static_cast<float>(u.D));
  p->packed = u.cu_seqlens_q != nullptr || u.cu_seqlens_k != nullptr;
  if (p->packed) {
    if (u.cu_seqlens_q == nullptr || u.cu_seqlens_k == nullptr) return SAGE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(u.cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(u.cu_seqlens_k) & 3u))
      return SAGE_ERR_INVALID_ARG;
    if (u.total_q < 0 || u.total_k < 0) return SAGE_ERR_INVALID_ARG;
    p->u.q_stride[0] = p->u.k_stride[0] = p->u.v_stride[0] = p->u.o_stride[0] = 0;
  }
  p->gs = u.gscale != SAGE_GSCALE_NONE;
  p->sq = u.smooth_q != 0;
  if (u.precision != SAGE_PRECISION_FP4 && u.precision != SAGE_PRECISION_8BIT) return SAGE_ERR_INVALID_ARG;
  p->b8 = u.precision == SAGE_PRECISION_8BIT;
  if (p->b8 && (p->gs || p->sq)) return SAGE_ERR_UNSUPPORTED;
  const int64_t* strides[4] = {p->u.q_stride, p->u.k_stride, p->u.v_stride, p->u.o_stride};
  for (const int64_t* s : strides)
    for (int i = 0; i < 3; ++i)
      if (s[i] < 0 || (s[i] % 8) != 0) return SAGE_ERR_INVALID_ARG;
  p->empty = u.B == 0 || u.Hq == 0 || u.Nq == 0 || (p->packed && u.total_q == 0);
  if (p->empty) return SAGE_OK;
  if (u.Hkv == 0 || u.Hq % u.Hkv != 0) return SAGE_ERR_INVALID_ARG;
  const int64_t B = u.B;
  if (p->packed) {
    p->rows_q = std::min<int64_t>(B * round128(u.Nq), (int64_t(u.total_q) + 127 * B) / 128 * 128);
    p->rows_k = std::min<int64_t>(B * round128(u.Nk), (int64_t(u.total_k) + 127 * B) / 128 * 128);
  } else {
    p->rows_q = B * round128(u.Nq);
    p->rows_k = B * round128(u.Nk);
  }
  p->rows_k = std::max<int64_t>(p->rows_k, 128);  // the K / V^T maps need one tile even with no keys
  p->tiles_q = static_cast<int>(round128(u.Nq) / 128);
  p->tiles_k = static_cast<int>(round128(u.Nk) / 128);
  p->nsplit = static_cast<int>((std::max<int64_t>(u.Nq, u.Nk) + 511) / 512);
  // Grid limits and 32-bit TMA coordinates / row indices.
  const int64_t lim = int64_t(1) << 31;
  if (u.B > 65535 || u.Hq > 65535) return SAGE_ERR_UNSUPPORTED;
  if (int64_t(u.Hq) * p->rows_q >= lim || int64_t(u.Hkv) * p->rows_k >= lim ||
      int64_t(u.Hkv) * p->rows_k / 128 * u.D >= lim || 3 * int64_t(std::max(p->tiles_q, p->tiles_k)) >= lim)
    return SAGE_ERR_UNSUPPORTED;
  if (p->packed && (int64_t(u.total_q) + 127 * B >= lim || int64_t(u.total_k) + 127 * B >= lim))
    return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

sage_fp4_problem_sizes_t sizes_of(const Prob& p) {
  sage_fp4_problem_sizes_t z;
  std::memset(&z, 0, sizeof(z));
  if (p.empty) return z;
  const int64_t D = p.u.D, B = p.u.B, Hq = p.u.Hq, Hkv = p.u.Hkv;
  if (p.b8) {
    const int64_t ns = p.nsplit;
    z.q_fp4 = static_cast<size_t>(Hq * p.rows_q * D);
    z.q_sf = static_cast<size_t>(Hq * p.rows_q / 128 * 4);
    z.k_fp4 = static_cast<size_t>(Hkv * p.rows_k * D);
    z.k_sf = static_cast<size_t>(Hkv * p.rows_k / 128 * 4);
    z.vt_fp4 = static_cast<size_t>(Hkv * p.rows_k * D);
    z.vt_sf = static_cast<size_t>(B * Hkv * D * 4);
    z.k_mean = static_cast<size_t>(B * Hkv * D * 4);
    z.amax = 0;
    z.seq = p.packed ? static_cast<size_t>((2 * (B + 1) + 4) * 4) : 0;
    z.scratch = up256(static_cast<size_t>(B * Hkv * ns * D * 8)) * 2 + 2 * up256(static_cast<size_t>(B * Hkv * ns * D * 4));
    z.workspace = up256(z.q_fp4) + up256(z.q_sf) + up256(z.k_fp4) + up256(z.k_sf) + up256(z.vt_fp4) +
                  up256(z.vt_sf) + up256(z.k_mean) + up256(z.seq) + z.scratch;
    return z;
  }
  z.q_fp4 = static_cast<size_t>(Hq * p.rows_q * D / 2);
  z.q_sf = static_cast<size_t>(Hq * p.rows_q * D / 16);
  z.k_fp4 = static_cast<size_t>(Hkv * p.rows_k * D / 2);
  z.k_sf = static_cast<size_t>(Hkv * p.rows_k * D / 16);
  z.vt_fp4 = static_cast<size_t>(Hkv * p.rows_k * D / 2);
  z.vt_sf = static_cast<size_t>(Hkv * p.rows_k / 128 * 1024);
  z.k_mean = static_cast<size_t>(B * Hkv * D * 4);
  z.amax = static_cast<size_t>(3 * B * Hq * 4);
  z.seq = p.packed ? static_cast<size_t>((2 * (B + 1) + 4) * 4) : 0;
  z.q_mean = p.sq ? static_cast<size_t>(B * Hq * D * 4) : 0;
  z.qk_bias = p.sq ? static_cast<size_t>(Hq * p.rows_k * 32) : 0;
  const int64_t ns = p.nsplit;
  size_t scratch = 0;
  if (p.u.smooth_k || p.gs || p.sq) scratch += up256(static_cast<size_t>(B * Hkv * ns * D * 8));
  if (p.gs)
    scratch += 2 * up256(static_cast<size_t>(B * Hkv * ns * D * 4)) + up256(static_cast<size_t>(B * Hq * ns * 4)) +
               up256(static_cast<size_t>(B * Hkv * ns * 4));
  if (p.sq) scratch += up256(static_cast<size_t>(B * Hq * ns * D * 8));
  if (p.sq && p.gs) scratch += 2 * up256(static_cast<size_t>(B * Hq * ns * D * 4));
  z.scratch = scratch;
  z.workspace = up256(z.q_fp4) + up256(z.q_sf) + up256(z.k_fp4) + up256(z.k_sf) + up256(z.vt_fp4) +
                up256(z.vt_sf) + up256(z.k_mean) + up256(z.amax) + up256(z.seq) + up256(z.q_mean) +
                up256(z.qk_bias) + z.scratch;
  return z;
}

// Elements of a caller tensor the problem can reach: the largest offset of a (sequence,
// head, token) row through the strides, plus the row's D channels (0 when empty).
uint64_t extent_el(const int64_t* st, int64_t B, int64_t H, int64_t tokens, bool packed, int64_t D) {
  if (B <= 0 || H <= 0 || tokens <= 0) return 0;
  const int64_t last = (packed ? 0 : (B - 1) * st[0]) + (H - 1) * st[1] + (tokens - 1) * st[2];
  return static_cast<uint64_t>(last + D);
}

// The extents every kernel of the problem may touch (see sage::Limits).
sage::Limits limits_of(const Prob& p) {
  sage::Limits l;
  std::memset(&l, 0, sizeof(l));
  if (p.empty) return l;
  const sage_fp4_problem_sizes_t z = sizes_of(p);
  const int64_t B = p.u.B, Hq = p.u.Hq, Hkv = p.u.Hkv, D = p.u.D, ns = p.nsplit;
  const int64_t tq = p.packed ? p.u.total_q : p.u.Nq, tk = p.packed ? p.u.total_k : p.u.Nk;
  l.q_el = extent_el(p.u.q_stride, B, Hq, tq, p.packed, D);
  l.k_el = extent_el(p.u.k_stride, B, Hkv, tk, p.packed, D);
  l.v_el = extent_el(p.u.v_stride, B, Hkv, tk, p.packed, D);
  l.o_el = extent_el(p.u.o_stride, B, Hq, tq, p.packed, D);
  l.q_fp4 = z.q_fp4;
  l.k_fp4 = z.k_fp4;
  l.vt_fp4 = z.vt_fp4;
  l.q_sf = z.q_sf;
  l.k_sf = z.k_sf;
  l.vt_sf = z.vt_sf;
  l.qk_bias = z.qk_bias;
  l.k_mean_el = z.k_mean / 4;
  l.q_mean_el = z.q_mean / 4;
  l.amax_el = z.amax / 4;
  l.stat_el = static_cast<uint64_t>(B * Hkv * ns * D);
  l.qstat_el = static_cast<uint64_t>(B * Hq * ns * D);
  l.qamax_el = static_cast<uint64_t>(B * Hq * ns);
  l.vamax_el = static_cast<uint64_t>(B * Hkv * ns);
  l.rows_q = static_cast<uint64_t>(Hq * p.rows_q);
  l.rows_k = static_cast<uint64_t>(Hkv * p.rows_k);
  l.rows_v = static_cast<uint64_t>(Hkv * p.rows_k / 128 * D);
  return l;
}

// Carve a workspace (256-byte aligned) into the quantized bundle followed by the scratch.
void carve(const Prob& p, void* base, sage_fp4_quantized_t* qz, void** scratch) {
  const sage_fp4_problem_sizes_t z = sizes_of(p);
  uint8_t* b = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t n) { uint8_t* r = b + off; off += up256(n); return r; };
  qz->q_fp4 = take(z.q_fp4);
  qz->q_sf = take(z.q_sf);
  qz->k_fp4 = take(z.k_fp4);
  qz->k_sf = take(z.k_sf);
  qz->vt_fp4 = take(z.vt_fp4);
  qz->vt_sf = take(z.vt_sf);
  qz->k_mean = reinterpret_cast<float*>(take(z.k_mean));
  qz->amax = z.amax ? reinterpret_cast<float*>(take(z.amax)) : nullptr;
  qz->seq = p.packed ? reinterpret_cast<int32_t*>(take(z.seq)) : nullptr;
  qz->q_mean = p.sq ? reinterpret_cast<float*>(take(z.q_mean)) : nullptr;
  qz->qk_bias = p.sq ? take(z.qk_bias) : nullptr;
  *scratch = z.scratch ? b + off : nullptr;
}

sage::SeqMap seq_map(const Prob& p, const sage_fp4_quantized_t& qz) {
  sage::SeqMap m;
  m.Nq = p.u.Nq;
  m.Nk = p.u.Nk;
  if (p.packed) {
    m.cu_q = p.u.cu_seqlens_q;
    m.cu_k = p.u.cu_seqlens_k;
    m.pad_q = qz.seq;
    m.pad_k = qz.seq + (p.u.B + 1);
    m.bad = reinterpret_cast<const uint32_t*>(qz.seq + 2 * (p.u.B + 1));
  } else {
    m.cu_q = m.cu_k = m.pad_q = m.pad_k = nullptr;
    m.bad = nullptr;
  }
  return m;
}

sage::Strides strides_of(const int64_t s[3]) { return sage::Strides{s[0], s[1], s[2]}; }

sage_status_t check_bundle(const Prob& p, const sage_fp4_quantized_t* qz, bool need_kmean) {
  if (qz == nullptr) return SAGE_ERR_INVALID_ARG;
  const void* ptrs[] = {qz->q_fp4, qz->q_sf, qz->k_fp4, qz->k_sf, qz->vt_fp4, qz->vt_sf};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  if (need_kmean && (qz->k_mean == nullptr || !aligned16(qz->k_mean))) return SAGE_ERR_INVALID_ARG;
  if (p.gs && (qz->amax == nullptr || !aligned16(qz->amax))) return SAGE_ERR_INVALID_ARG;
  if (p.b8 && need_kmean && (qz->k_mean == nullptr || !aligned16(qz->k_mean))) return SAGE_ERR_INVALID_ARG;
  if (p.packed && (qz->seq == nullptr || !aligned16(qz->seq))) return SAGE_ERR_INVALID_ARG;
  if (p.sq && (qz->qk_bias == nullptr || !aligned16(qz->qk_bias))) return SAGE_ERR_INVALID_ARG;
  if (p.sq && need_kmean && (qz->q_mean == nullptr || !aligned16(qz->q_mean))) return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

sage_status_t run_quantize(const Prob& p, const void* q, const void* k, const void* v,
                           const sage_fp4_quantized_t& qz, void* scratch, cudaStream_t stream) {
  uint32_t* err = nullptr;
  if (sage_status_t st = error_word(&err); st != SAGE_OK) return st;
  sage::QuantParams k_;
  std::memset(&k_, 0, sizeof(k_));
  k_.q = q;
  k_.k = k;
  k_.v = v;
  k_.sq = strides_of(p.u.q_stride);
  k_.sk = strides_of(p.u.k_stride);
  k_.sv = strides_of(p.u.v_stride);
  k_.dtype = p.u.dtype;
  k_.B = p.u.B;
  k_.Hq = p.u.Hq;
  k_.Hkv = p.u.Hkv;
  k_.D = p.u.D;
  k_.seq = seq_map(p, qz);
  k_.smooth_k = p.u.smooth_k ? 1 : 0;
  k_.smooth_q = p.sq ? 1 : 0;
  k_.bits8 = p.b8 ? 1 : 0;
  k_.q_mean = p.sq ? qz.q_mean : nullptr;
  k_.qk_bias = p.sq ? qz.qk_bias : nullptr;
  k_.gscale = p.u.gscale;
  k_.nsplit = p.nsplit;
  k_.amax_stride = p.u.B * p.u.Hq;
  k_.q_fp4 = qz.q_fp4;
  k_.q_sf = qz.q_sf;
  k_.k_fp4 = qz.k_fp4;
  k_.k_sf = qz.k_sf;
  k_.vt_fp4 = qz.vt_fp4;
  k_.vt_sf = qz.vt_sf;
  k_.k_mean = qz.k_mean;
  k_.amax = qz.amax;
  const int64_t B = p.u.B, Hq = p.u.Hq, Hkv = p.u.Hkv, ns = p.nsplit, D = p.u.D;
  uint8_t* s = static_cast<uint8_t*>(scratch);
  auto take = [&](size_t n) { uint8_t* r = s; s += up256(n); return r; };
  if (p.b8) {
    // 8-bit path: K sums, then V channel sums / maxima / minima (the sums are not used).
    k_.ksum = reinterpret_cast<double*>(take(static_cast<size_t>(B * Hkv * ns * D * 8)));
    k_.vsum = reinterpret_cast<double*>(take(static_cast<size_t>(B * Hkv * ns * D * 8)));
    k_.vmax = reinterpret_cast<float*>(take(static_cast<size_t>(B * Hkv * ns * D * 4)));
    k_.vmin = reinterpret_cast<float*>(take(static_cast<size_t>(B * Hkv * ns * D * 4)));
    k_.v_scale = reinterpret_cast<float*>(qz.vt_sf);
  } else if (p.u.smooth_k || p.gs || p.sq) {
    k_.ksum = reinterpret_cast<double*>(take(static_cast<size_t>(B * Hkv * ns * D * 8)));
  }
  if (p.gs) {
    k_.kmax = reinterpret_cast<float*>(take(static_cast<size_t>(B * Hkv * ns * D * 4)));
    k_.kmin = reinterpret_cast<float*>(take(static_cast<size_t>(B * Hkv * ns * D * 4)));
    k_.qamax = reinterpret_cast<float*>(take(static_cast<size_t>(B * Hq * ns * 4)));
    k_.vamax = reinterpret_cast<float*>(take(static_cast<size_t>(B * Hkv * ns * 4)));
  }
  if (p.sq) k_.qsum = reinterpret_cast<double*>(take(static_cast<size_t>(B * Hq * ns * D * 8)));
  if (p.sq && p.gs) {
    k_.qmax = reinterpret_cast<float*>(take(static_cast<size_t>(B * Hq * ns * D * 4)));
    k_.qmin = reinterpret_cast<float*>(take(static_cast<size_t>(B * Hq * ns * D * 4)));
  }
  if (p.packed) {
    k_.total_q = p.u.total_q;
    k_.total_k = p.u.total_k;
    k_.pad_q_out = qz.seq;
    k_.pad_k_out = qz.seq + (p.u.B + 1);
    k_.bad_out = reinterpret_cast<uint32_t*>(qz.seq + 2 * (p.u.B + 1));
  }
  k_.err = err;
  k_.lim = limits_of(p);
  if (p.b8) return cuda_status(sage::launch_quantize8(k_, sage::QuantLaunch{p.tiles_q, p.tiles_k}, stream));
  return cuda_status(sage::launch_quantize(k_, sage::QuantLaunch{p.tiles_q, p.tiles_k}, stream));
}

sage_status_t build_maps8(const Prob& p, const uint8_t* q8, const uint8_t* k8, const uint8_t* vt8,
                          sage::TensorMaps* m) {
  const uint64_t D = static_cast<uint64_t>(p.u.D);
  const CUtensorMapSwizzle swqk = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  sage_status_t st;
  if ((st = make_map(&m->q, q8, D, p.u.Hq * p.rows_q, static_cast<uint32_t>(D), 128, swqk)) != SAGE_OK) return st;
  if ((st = make_map(&m->k, k8, D, p.u.Hkv * p.rows_k, static_cast<uint32_t>(D), 128, swqk)) != SAGE_OK) return st;
  return make_map(&m->v, vt8, 128, p.u.Hkv * p.rows_k / 128 * D, 128, static_cast<uint32_t>(D),
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

sage_status_t build_maps(const Prob& p, const uint8_t* q_fp4, const uint8_t* k_fp4, const uint8_t* vt_fp4,
                         sage::TensorMaps* m) {
  const uint64_t inner = static_cast<uint64_t>(p.u.D / 2);
  const CUtensorMapSwizzle swqk = p.u.D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  sage_status_t st;
  if ((st = make_map(&m->q, q_fp4, inner, p.u.Hq * p.rows_q, static_cast<uint32_t>(inner), 128, swqk)) != SAGE_OK) return st;
  if ((st = make_map(&m->k, k_fp4, inner, p.u.Hkv * p.rows_k, static_cast<uint32_t>(inner), 128, swqk)) != SAGE_OK) return st;
  if (vt_fp4 != nullptr &&
      (st = make_map(&m->v, vt_fp4, 64, p.u.Hkv * p.rows_k / 128 * p.u.D, 64, static_cast<uint32_t>(p.u.D),
                     CU_TENSOR_MAP_SWIZZLE_64B)) != SAGE_OK)
    return st;
  return SAGE_OK;
}

sage_status_t base_params(int D, float sm_scale, int causal, sage::AttnParams* a) {
  std::memset(a, 0, sizeof(*a));
  uint32_t* err = nullptr;
  if (sage_status_t st = error_word(&err); st != SAGE_OK) return st;
  a->D = D;
  a->causal = causal ? 1 : 0;
  a->sm_scale = sm_scale;
  a->sm_scale_log2 = sm_scale * 1.4426950408889634f;
  a->err = err;
  a->timeout_ns = g_timeout_ns.load();
  a->debug_flags = g_debug_flags.load();
  return SAGE_OK;
}

sage_status_t run_attention(const Prob& p, const sage_fp4_quantized_t& qz, void* out, cudaStream_t stream) {
  sage::TensorMaps m;
  if (p.b8) {
    if (sage_status_t st = build_maps8(p, qz.q_fp4, qz.k_fp4, qz.vt_fp4, &m); st != SAGE_OK) return st;
  } else if (sage_status_t st = build_maps(p, qz.q_fp4, qz.k_fp4, qz.vt_fp4, &m); st != SAGE_OK) {
    return st;
  }
  sage::AttnParams a;
  if (sage_status_t st = base_params(p.u.D, p.u.sm_scale, p.u.causal, &a); st != SAGE_OK) return st;
  a.q_sf = qz.q_sf;
  a.k_sf = qz.k_sf;
  a.vt_sf = qz.vt_sf;
  a.out = out;
  a.so = strides_of(p.u.o_stride);
  a.out_dtype = p.u.dtype;
  a.B = p.u.B;
  a.Hq = p.u.Hq;
  a.Hkv = p.u.Hkv;
  a.group = p.u.Hq / p.u.Hkv;
  a.seq = seq_map(p, qz);
  a.lim = limits_of(p);
  if (a.debug_flags & sage::kDebugNoOutput) a.lim.o_el = 0;
  a.amax = p.gs ? qz.amax : nullptr;
  a.qk_bias = p.sq ? qz.qk_bias : nullptr;
  if (p.b8) {
    a.q_scale8 = reinterpret_cast<const float*>(qz.q_sf);
    a.k_scale8 = reinterpret_cast<const float*>(qz.k_sf);
    a.v_scale8 = reinterpret_cast<const float*>(qz.vt_sf);
    a.amax = nullptr;
    return cuda_status(sage::launch_attention8(m, a, p.tiles_q, stream));
  }
  a.gscale = p.u.gscale;
  a.amax_stride = p.u.B * p.u.Hq;
  return cuda_status(sage::launch_attention(m, a, p.tiles_q, stream));
}

// The dense [B, H, N, D] contiguous problem of the original entry points.
sage_fp4_problem_t dense_problem(int B, int H, int N, int D, int dtype, int causal, float sm_scale, int smooth_k) {
  sage_fp4_problem_t u;
  std::memset(&u, 0, sizeof(u));
  u.B = B;
  u.Hq = u.Hkv = H;
  u.D = D;
  u.Nq = u.Nk = N;
  const int64_t s[3] = {int64_t(H) * N * D, int64_t(N) * D, D};
  for (int i = 0; i < 3; ++i) u.q_stride[i] = u.k_stride[i] = u.v_stride[i] = u.o_stride[i] = s[i];
  u.dtype = static_cast<sage_dtype_t>(dtype);
  u.causal = causal;
  u.sm_scale = sm_scale;
  u.smooth_k = smooth_k;
  u.gscale = SAGE_GSCALE_NONE;
  return u;
}

}  // namespace

extern "C" {

const char* sage_status_string(sage_status_t status) {
  switch (status) {
    case SAGE_OK: return "SAGE_OK";
    case SAGE_ERR_INVALID_ARG: return "SAGE_ERR_INVALID_ARG";
    case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
    case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
    case SAGE_ERR_TIMEOUT: return "SAGE_ERR_TIMEOUT";
    case SAGE_ERR_BOUNDS: return "SAGE_ERR_BOUNDS";
  }
  return "SAGE_ERR_UNKNOWN";
}

// ------------------------------------------------------------ general problem ----

sage_status_t sage_fp4_problem_sizes(const sage_fp4_problem_t* problem, sage_fp4_problem_sizes_t* sizes) {
  if (sizes == nullptr) return SAGE_ERR_INVALID_ARG;
  Prob p;
  if (sage_status_t st = check_problem(problem, &p); st != SAGE_OK) return st;
  *sizes = sizes_of(p);
  return SAGE_OK;
}

sage_status_t sage_fp4_quantize(const sage_fp4_problem_t* problem, const void* q, const void* k,
                                const void* v, const sage_fp4_quantized_t* qz, void* scratch,
                                size_t scratch_bytes, void* stream) {
  Prob p;
  if (sage_status_t st = check_problem(problem, &p); st != SAGE_OK) return st;
  if (p.empty) return SAGE_OK;
  const void* ptrs[] = {q, k, v};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  if (sage_status_t st = check_bundle(p, qz, true); st != SAGE_OK) return st;
  const size_t need = sizes_of(p).scratch;
  if (need > 0 && (scratch == nullptr || !aligned16(scratch) || scratch_bytes < need)) return SAGE_ERR_INVALID_ARG;
  return run_quantize(p, q, k, v, *qz, scratch, static_cast<cudaStream_t>(stream));
}

sage_status_t sage_fp4_attn_quantized(const sage_fp4_problem_t* problem, const sage_fp4_quantized_t* qz,
                                      void* out, void* stream) {
  Prob p;
  if (sage_status_t st = check_problem(problem, &p); st != SAGE_OK) return st;
  if (p.empty) return SAGE_OK;
  if (out == nullptr || !aligned16(out)) return SAGE_ERR_INVALID_ARG;
  if (sage_status_t st = check_bundle(p, qz, false); st != SAGE_OK) return st;
  return run_attention(p, *qz, out, static_cast<cudaStream_t>(stream));
}

sage_status_t sage_fp4_attn(const sage_fp4_problem_t* problem, const void* q, const void* k, const void* v,
                            void* out, void* workspace, size_t ws_bytes, void* stream) {
  Prob p;
  if (sage_status_t st = check_problem(problem, &p); st != SAGE_OK) return st;
  if (p.empty) return SAGE_OK;
  const void* ptrs[] = {q, k, v, out};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < sizes_of(p).workspace) return SAGE_ERR_INVALID_ARG;
  sage_fp4_quantized_t qz;
  void* scratch = nullptr;
  carve(p, workspace, &qz, &scratch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (sage_status_t r = run_quantize(p, q, k, v, qz, scratch, st); r != SAGE_OK) return r;
  return run_attention(p, qz, out, st);
}

// ------------------------------------------------- dense [B, H, N, D] problems ----

sage_status_t sage_fp4_quantized_sizes(int B, int H, int N, int D, sage_fp4_sizes_t* sizes) {
  if (sizes == nullptr) return SAGE_ERR_INVALID_ARG;
  const sage_fp4_problem_t u = dense_problem(B, H, N, D, SAGE_BF16, 0, 0.0f, 1);
  Prob p;
  if (sage_status_t st = check_problem(&u, &p); st != SAGE_OK) return st;
  const sage_fp4_problem_sizes_t z = sizes_of(p);
  sizes->q_fp4 = z.q_fp4;
  sizes->q_sf = z.q_sf;
  sizes->k_fp4 = z.k_fp4;
  sizes->k_sf = z.k_sf;
  sizes->vt_fp4 = z.vt_fp4;
  sizes->vt_sf = z.vt_sf;
  sizes->k_mean = z.k_mean;
  return SAGE_OK;
}

size_t sage_fp4_quantize_scratch_bytes(int B, int H, int N, int D) {
  const sage_fp4_problem_t u = dense_problem(B, H, N, D, SAGE_BF16, 0, 0.0f, 1);
  Prob p;
  if (check_problem(&u, &p) != SAGE_OK || p.empty) return 0;
  // The binary64 partial sums, then room for the K mean when the caller passes none.
  return sizes_of(p).scratch + up256(sizes_of(p).k_mean);
}

size_t sage_fp4_workspace_bytes(int B, int H, int N, int D) {
  const sage_fp4_problem_t u = dense_problem(B, H, N, D, SAGE_BF16, 0, 0.0f, 1);
  Prob p;
  if (check_problem(&u, &p) != SAGE_OK || p.empty) return 0;
  return sizes_of(p).workspace;
}

sage_status_t sage_fp4_quantize_qkv(const void* q, const void* k, const void* v, sage_dtype_t dtype,
                                    int B, int H, int N, int D, int smooth_k, uint8_t* q_fp4,
                                    uint8_t* q_sf, uint8_t* k_fp4, uint8_t* k_sf, uint8_t* vt_fp4,
                                    uint8_t* vt_sf, float* k_mean, void* scratch,
                                    size_t scratch_bytes, void* stream) {
  if (!valid_dtype(dtype)) return SAGE_ERR_INVALID_ARG;
  const sage_fp4_problem_t u = dense_problem(B, H, N, D, dtype, 0, 0.0f, smooth_k ? 1 : 0);
  Prob p;
  if (sage_status_t st = check_problem(&u, &p); st != SAGE_OK) return st;
  if (p.empty) return SAGE_OK;
  const void* ptrs[] = {q, k, v};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  sage_fp4_quantized_t qz;
  std::memset(&qz, 0, sizeof(qz));
  qz.q_fp4 = q_fp4;
  qz.q_sf = q_sf;
  qz.k_fp4 = k_fp4;
  qz.k_sf = k_sf;
  qz.vt_fp4 = vt_fp4;
  qz.vt_sf = vt_sf;
  qz.k_mean = k_mean;
  if (sage_status_t st = check_bundle(p, &qz, false); st != SAGE_OK) return st;
  if (k_mean != nullptr && !aligned16(k_mean)) return SAGE_ERR_INVALID_ARG;
  const sage_fp4_problem_sizes_t z = sizes_of(p);
  const size_t need = smooth_k ? z.scratch + (k_mean ? 0 : up256(z.k_mean)) : 0;
  if (need > 0 && (scratch == nullptr || !aligned16(scratch) || scratch_bytes < need)) return SAGE_ERR_INVALID_ARG;
  if (smooth_k && k_mean == nullptr) qz.k_mean = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + z.scratch);
  return run_quantize(p, q, k, v, qz, smooth_k ? scratch : nullptr, static_cast<cudaStream_t>(stream));
}

sage_status_t sage_fp4_attn_fwd_quantized(const uint8_t* q_fp4, const uint8_t* q_sf,
                                          const uint8_t* k_fp4, const uint8_t* k_sf,
                                          const uint8_t* vt_fp4, const uint8_t* vt_sf, void* out,
                                          sage_dtype_t out_dtype, int B, int H, int N, int D,
                                          int causal, float sm_scale, void* stream) {
  const sage_fp4_problem_t u = dense_problem(B, H, N, D, out_dtype, causal, sm_scale, 1);
  sage_fp4_quantized_t qz;
  std::memset(&qz, 0, sizeof(qz));
  qz.q_fp4 = const_cast<uint8_t*>(q_fp4);
  qz.q_sf = const_cast<uint8_t*>(q_sf);
  qz.k_fp4 = const_cast<uint8_t*>(k_fp4);
  qz.k_sf = const_cast<uint8_t*>(k_sf);
  qz.vt_fp4 = const_cast<uint8_t*>(vt_fp4);
  qz.vt_sf = const_cast<uint8_t*>(vt_sf);
  return sage_fp4_attn_quantized(&u, &qz, out, stream);
}

sage_status_t sage_fp4_attn_fwd_ex(const void* q, const void* k, const void* v, void* out,
                                   sage_dtype_t dtype, int B, int H, int N, int D, int causal,
                                   float sm_scale, void* workspace, size_t ws_bytes, void* stream) {
  const sage_fp4_problem_t u = dense_problem(B, H, N, D, dtype, causal, sm_scale, 1);
  return sage_fp4_attn(&u, q, k, v, out, workspace, ws_bytes, stream);
}

sage_status_t sage_fp4_attn_fwd(const void* q, const void* k, const void* v, void* out, int B,
                                int H, int N, int D, int causal, float sm_scale, void* stream) {
  const sage_fp4_problem_t u = dense_problem(B, H, N, D, SAGE_BF16, causal, sm_scale, 1);
  Prob p;
  if (sage_status_t st = check_problem(&u, &p); st != SAGE_OK) return st;
  if (p.empty) return SAGE_OK;
  const void* ptrs[] = {q, k, v, out};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = sizes_of(p).workspace;
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, bytes, st) != cudaSuccess) return SAGE_ERR_CUDA;
  sage_status_t r = sage_fp4_attn(&u, q, k, v, out, ws, bytes, stream);
  const cudaError_t e = cudaFreeAsync(ws, st);
  if (r == SAGE_OK && e != cudaSuccess) r = SAGE_ERR_CUDA;
  return r;
}

sage_status_t sage_fp4_qk_scores(const uint8_t* q_fp4, const uint8_t* q_sf, const uint8_t* k_fp4,
                                 const uint8_t* k_sf, float* s_out, int B, int H, int N, int D,
                                 float sm_scale, void* stream) {
  const sage_fp4_problem_t u = dense_problem(B, H, N, D, SAGE_BF16, 0, sm_scale, 1);
  Prob p;
  if (sage_status_t st = check_problem(&u, &p); st != SAGE_OK) return st;
  if (p.empty) return SAGE_OK;
  const void* ptrs[] = {q_fp4, q_sf, k_fp4, k_sf, s_out};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SAGE_ERR_INVALID_ARG;
  if (p.tiles_q > 65535) return SAGE_ERR_UNSUPPORTED;
  sage::TensorMaps m;
  if (sage_status_t st = build_maps(p, q_fp4, k_fp4, nullptr, &m); st != SAGE_OK) return st;
  sage::AttnParams a;
  if (sage_status_t st = base_params(D, p.u.sm_scale, 0, &a); st != SAGE_OK) return st;
  a.q_sf = q_sf;
  a.k_sf = k_sf;
  a.out = s_out;
  a.BH = B * H;
  a.Np = static_cast<int>(round128(N));
  return cuda_status(sage::launch_qk_scores(m, a, static_cast<cudaStream_t>(stream)));
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
  if (host == 0) return SAGE_OK;
  if (host & sage::kDevErrTimeout) return SAGE_ERR_TIMEOUT;
  if (host & sage::kDevErrBounds) return SAGE_ERR_BOUNDS;
  return SAGE_ERR_INVALID_ARG;
}

const char* sage_fp4_last_cuda_error(void) { return g_last_error; }

sage_status_t sage_fp4_set_debug_flags(uint32_t flags) {
  if (flags & ~3u) return SAGE_ERR_INVALID_ARG;
#ifndef SAGE_CHECKS
  if (flags & sage::kDebugNoOutput) return SAGE_ERR_UNSUPPORTED;  // only the bounds-checked build has it
#endif
  g_debug_flags.store(flags);
  return SAGE_OK;
}

int sage_fp4_bounds_checked(void) {
#ifdef SAGE_CHECKS
  return 1;
#else
  return 0;
#endif
}

sage_status_t sage_fp4_mma_rate(int n, int iters, int ctas, void* stream) {
  if ((n != 64 && n != 128) || iters < 1 || ctas < 1 || ctas > 65535) return SAGE_ERR_INVALID_ARG;
  uint32_t* err = nullptr;
  if (sage_status_t st = error_word(&err); st != SAGE_OK) return st;
  return cuda_status(sage::launch_mma_rate(n, iters, ctas, err, g_timeout_ns.load(), static_cast<cudaStream_t>(stream)));
}

sage_status_t sage_fp4_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : ns);
  return SAGE_OK;
}

}  // extern "C"
