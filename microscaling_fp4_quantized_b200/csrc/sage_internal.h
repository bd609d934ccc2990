// Internal launch interfaces of the CUDA library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace sage {

enum : int { kDtypeBF16 = 0, kDtypeF16 = 1 };

// Bits of the device error word.
enum : uint32_t { kDevErrTimeout = 1u, kDevErrSeqlens = 2u, kDevErrBounds = 4u };

// Extents the kernels may touch, derived on the host from the problem: elements of the
// caller's q, k, v and out reachable through the strides, bytes of each quantized
// buffer, elements of the statistics buffers, and rows of the TMA maps. The bounds-checked
// build (compiled with SAGE_CHECKS) tests every computed global index against them before
// the access; a failed check sets kDevErrBounds in the device error word, raises the CTA's
// abort flag where the kernel has one, and skips the access. Without SAGE_CHECKS the
// checks compile to nothing and these fields are unused.
struct Limits {
  uint64_t q_el, k_el, v_el, o_el;
  uint64_t q_fp4, k_fp4, vt_fp4, q_sf, k_sf, vt_sf, qk_bias;
  uint64_t k_mean_el, q_mean_el, amax_el, stat_el, qstat_el, qamax_el, vamax_el;
  uint64_t rows_q, rows_k, rows_v;
};

#ifdef SAGE_CHECKS
// True when `cond` holds; otherwise records a bounds failure (and raises *abort_flag when
// it is not null) and returns false so that the caller skips the access.
__device__ __forceinline__ bool sage_in_bounds(bool cond, uint32_t* err, volatile uint32_t* abort_flag) {
  if (cond) return true;
  atomicOr(err, kDevErrBounds);
  if (abort_flag != nullptr) *abort_flag = 1u;
  return false;
}
#define SAGE_IN_BOUNDS(cond, err, abort_flag) ::sage::sage_in_bounds((cond), (err), (abort_flag))
#else
#define SAGE_IN_BOUNDS(cond, err, abort_flag) true
#endif

// Second-level scale modes (one FP32 factor per tensor or per (sequence, head)).
enum : int { kGscaleNone = 0, kGscaleTensor = 1, kGscaleHead = 2 };

// 448 * 6: E4M3 max times E2M1 max, the target of every two-level scaling.
constexpr float kTwoLevelTarget = 2688.0f;

// Element strides of (sequence, head, token); channels are contiguous.
struct Strides {
  int64_t b, h, n;
};

// Where each sequence lives. Dense problems (cu_q == nullptr): B sequences of Nq queries
// and Nk keys, sequence b starting at token 0 of batch b. Packed problems: sequence b
// holds tokens cu_q[b] .. cu_q[b+1] of the packed tensors; pad_q[b] is the number of
// padded (multiple-of-128) query tokens of the sequences before it, computed on the
// device; *bad != 0 when the sequence table failed validation (kernels then do nothing).
struct SeqMap {
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* pad_q;
  const int32_t* pad_k;
  const uint32_t* bad;
  int Nq, Nk;
};

struct SeqInfo {
  int len_q, len_k;    // tokens
  int tok_q, tok_k;    // first token in the (packed) input / output tensors
  int prow_q, prow_k;  // padded tokens of all earlier sequences
};

__device__ __forceinline__ int round128(int x) { return (x + 127) & ~127; }

__device__ __forceinline__ SeqInfo seq_info(const SeqMap& m, int b) {
  SeqInfo s;
  if (m.cu_q == nullptr) {
    s.len_q = m.Nq;
    s.len_k = m.Nk;
    s.tok_q = 0;
    s.tok_k = 0;
    s.prow_q = b * round128(m.Nq);
    s.prow_k = b * round128(m.Nk);
  } else {
    s.tok_q = m.cu_q[b];
    s.tok_k = m.cu_k[b];
    s.len_q = m.cu_q[b + 1] - s.tok_q;
    s.len_k = m.cu_k[b + 1] - s.tok_k;
    s.prow_q = m.pad_q[b];
    s.prow_k = m.pad_k[b];
  }
  return s;
}

__device__ __forceinline__ bool seq_table_bad(const SeqMap& m) {
  return m.bad != nullptr && *reinterpret_cast<const volatile uint32_t*>(m.bad) != 0u;
}

// Second-level scale from a group maximum: fp32(amax / 2688), or 1 when that is 0. The
// quotient is the double product amax * RN64(1/2688) rounded to binary32, which equals the
// IEEE binary32 division for every non-negative binary32 amax (checked exhaustively on the
// CPU: the exact quotient's binary fraction repeats with period 6, 2688 = 21 * 2^7, so it
// never lies within the double product's error of a binary32 rounding midpoint). It keeps
// the division's subroutine out of the attention kernel (measured 1053 -> 1082 TFLOP/s for
// its general instance on the long workload).
__device__ __forceinline__ float second_level_scale(float amax) {
  constexpr double kInvTarget = 1.0 / static_cast<double>(kTwoLevelTarget);
  const float g = __double2float_rn(static_cast<double>(amax) * kInvTarget);
  return g > 0.0f ? g : 1.0f;
}

// Quantized layouts: the padded-token row of (sequence b, head h, token n) of Q is
//   Hq * prow_q + h * round128(len_q) + n
// (K and V^T likewise with Hkv, prow_k, len_k); a 128-row tile t of those rows is
// the scale-factor tile t and the V^T tile t.
struct QuantParams {
  const void* q;
  const void* k;
  const void* v;
  Strides sq, sk, sv;
  int dtype;
  int B, Hq, Hkv, D;
  SeqMap seq;
  int smooth_k;
  int smooth_q;      // subtract the per-(sequence, head) query mean; emit the per-key bias
  int bits8;         // the 8-bit path: INT8 Q/K per 128-token tile, E4M3 V^T per channel
  int gscale;
  int nsplit;        // 512-token chunks of the longest sequence
  int amax_stride;   // B * Hq: distance between the Q, K and V maxima
  uint8_t* q_fp4;
  uint8_t* q_sf;
  uint8_t* k_fp4;
  uint8_t* k_sf;
  uint8_t* vt_fp4;
  uint8_t* vt_sf;
  float* k_mean;     // [B * Hkv, D]
  float* q_mean;     // [B * Hq, D]              (smooth_q)
  uint8_t* qk_bias;  // (smooth_q) per (query head, padded key row) 32 bytes: the bias
                     // mu_q . (k - mu_k) / (g_q g_k) as three bf16 terms, MMA operand layout
  float* amax;       // [3, B * Hq]; tensor mode uses element 0 of each
  double* ksum;      // [B * Hkv, nsplit, D]
  float* kmax;       // [B * Hkv, nsplit, D]  (second-level scale only)
  float* kmin;       // [B * Hkv, nsplit, D]
  double* qsum;      // [B * Hq, nsplit, D]   (smooth_q)
  float* qmax;       // [B * Hq, nsplit, D]   (smooth_q with a second-level scale)
  float* qmin;       // [B * Hq, nsplit, D]
  float* qamax;      // [B * Hq, nsplit]
  float* vamax;      // [B * Hkv, nsplit]
  // 8-bit path: q_fp4 / k_fp4 hold int8 codes [rows, D], q_sf / k_sf one float scale per
  // 128-row tile, vt_fp4 E4M3 codes [key tiles, D, 128], v_scale the channel scales.
  float* v_scale;    // [B * Hkv, D]
  double* vsum;      // [B * Hkv, nsplit, D]  (channel statistics of V, 8-bit path)
  float* vmax;       // [B * Hkv, nsplit, D]
  float* vmin;       // [B * Hkv, nsplit, D]
  // Packed problems: the plan kernel's inputs and outputs.
  int total_q, total_k;
  int32_t* pad_q_out;
  int32_t* pad_k_out;
  uint32_t* bad_out;
  uint32_t* err;
  Limits lim;
};

struct AttnParams {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* vt_sf;
  void* out;            // attention: element (b, h, n) at b*so.b + h*so.h + (tok_q + n)*so.n;
                        // scores: float [BH, Np, Np]
  Strides so;
  int out_dtype;
  int B, Hq, Hkv, group, D;
  SeqMap seq;
  const float* amax;    // second-level maxima, or nullptr
  const uint8_t* qk_bias; // Q-smoothing bias operand per (query head, padded key row), or nullptr
  const float* q_scale8;  // 8-bit path: scale per 128-row Q tile
  const float* k_scale8;  // 8-bit path: scale per 128-row K tile
  const float* v_scale8;  // 8-bit path: [B * Hkv, D] channel scales of V
  int gscale;
  int amax_stride;
  int BH, Np;           // dense S = Q^ K^^T (scores kernel only)
  int causal;
  float sm_scale;       // scale of the dot products
  float sm_scale_log2;  // sm_scale * log2(e)
  uint32_t* err;        // device error word
  uint64_t timeout_ns;  // bound on every wait
  uint32_t debug_flags; // kDebugNoLoads: the producer issues no copies (test of the error path)
  int tiles_q;          // query tiles of the longest sequence (work items: B * Hq * tiles_q)
  Limits lim;
};

// Test switches: kDebugNoLoads, the attention kernel's copy warps issue no loads (every
// bounded wait then runs out); kDebugNoOutput (bounds-checked build only), the output
// extent is taken as 0, so every output store fails its check and is skipped.
enum : uint32_t { kDebugNoLoads = 1u, kDebugNoOutput = 2u };

struct TensorMaps {
  CUtensorMap q, k, v;
};

struct QuantLaunch {
  int tiles_q, tiles_k;  // 128-token tiles of the longest query / key sequence
};

cudaError_t launch_quantize(const QuantParams& p, const QuantLaunch& l, cudaStream_t stream);
cudaError_t launch_quantize8(const QuantParams& p, const QuantLaunch& l, cudaStream_t stream);
cudaError_t launch_attention(const TensorMaps& maps, const AttnParams& p, int tiles_q, cudaStream_t stream);
cudaError_t launch_qk_scores(const TensorMaps& maps, const AttnParams& p, cudaStream_t stream);
cudaError_t launch_attention8(const TensorMaps& maps, const AttnParams& p, int tiles_q, cudaStream_t stream);
// Tensor-core rate probe (mma_rate.cu): `ctas` CTAs, each issuing `iters` block-scaled FP4
// products of M = 128, N = n, K = 64.
cudaError_t launch_mma_rate(int n, int iters, int ctas, uint32_t* err, uint64_t timeout_ns, cudaStream_t stream);

}  // namespace sage
