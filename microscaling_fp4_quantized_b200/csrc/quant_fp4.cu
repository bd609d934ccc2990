// Quantization kernels of the FP4 attention forward (sm_100a):
//   kmean_partial_kernel : binary64 column sums of K over 512-token chunks
//   quant_kernel         : Q, K - mean and V^T -> packed E2M1 codes + UE4M3 scale tiles
//
// The block rule follows the microscaling FP4 statement of SageAttention3 (arXiv
// 2505.11594, abstract): per 16 consecutive elements, s = E4M3(absmax / 6) and
// code = E2M1(x / s), both round-to-nearest-even with saturation; "smoothing K"
// (SageAttention OpenReview thread, reply to W1) subtracts the per-channel token mean
// of K first. Every arithmetic step is IEEE binary32 with RNE (true divisions, no
// reciprocal), so codes and scale bytes are reproducible bit for bit.
//
// Both kernels are HBM-bound: 16-byte coalesced loads, tiles of 128 tokens, scale
// factors and V^T codes staged in shared memory and written out as 16-byte chunks.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sage_internal.h"
#include "sm100_ptx.cuh"

namespace sage {

namespace {

__device__ __forceinline__ void unpack8(uint4 raw, int dtype, float (&x)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (dtype == kDtypeBF16) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      x[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xFFFFu)));
      x[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
    }
  }
}

__device__ __forceinline__ uint4 ld_nc_16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Codes of 8 values against a decoded scale s (s == 0 -> zero codes); element 0 lands
// in the low nibble of the low byte.
__device__ __forceinline__ uint32_t encode8(const float (&x)[8], float s) {
  if (s == 0.0f) return 0u;
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = __fdiv_rn(x[2 * i], s);
    const float b = __fdiv_rn(x[2 * i + 1], s);
    w |= f32x2_to_e2m1(a, b) << (8 * i);
  }
  return w;
}

constexpr int kThreads = 256;
constexpr int kMeanChunk = 512;  // tokens per K-mean partial

}  // namespace

// grid (nsplit, BH); partial[bh, split, d] = sum over tokens of the chunk, binary64.
template <int D>
__global__ void __launch_bounds__(kThreads) kmean_partial_kernel(QuantParams p) {
  constexpr int CPR = D / 8;          // 16-byte chunks per row
  constexpr int RG = kThreads / CPR;  // row groups
  __shared__ double red[RG][D];
  const int t = threadIdx.x, c = t % CPR, rg = t / CPR;
  const int bh = blockIdx.y;
  const int n0 = blockIdx.x * kMeanChunk;
  const int n1 = min(n0 + kMeanChunk, p.N);
  const char* base = static_cast<const char*>(p.k) + (static_cast<size_t>(bh) * p.N) * D * 2;
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
  for (int n = n0 + rg; n < n1; n += RG) {
    float x[8];
    unpack8(ld_nc_16(base + (static_cast<size_t>(n) * D + c * 8) * 2), p.dtype, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += static_cast<double>(x[e]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rg][c * 8 + e] = acc[e];
  __syncthreads();
  for (int d = t; d < D; d += kThreads) {
    double s = 0.0;
    for (int g = 0; g < RG; ++g) s += red[g][d];
    p.partial[(static_cast<size_t>(bh) * p.nsplit + blockIdx.x) * D + d] = s;
  }
}

// grid (Np/128, BH, 3): z = 0 quantizes Q rows, 1 quantizes K rows (smoothed), 2 V^T.
template <int D>
__global__ void __launch_bounds__(kThreads) quant_kernel(QuantParams p) {
  constexpr int CPR = D / 8;
  constexpr int kVRowBytes = (D + 8) * 2;  // padded V tile row (16-byte multiple)
  constexpr int kCodeRow = 80;             // padded V^T code staging row (64 used)
  constexpr int kSfBytesQK = (D / 64) * 512;
  __shared__ __align__(16) uint8_t smem[128 * kVRowBytes + D * kCodeRow + 1024 + D * 4];
  const int t = threadIdx.x;
  const int bh = blockIdx.y;
  const int tile = blockIdx.x;
  const int row0 = tile * 128;
  const int job = blockIdx.z;
  const int ntiles = p.Np / 128;

  if (job < 2) {
    uint8_t* sfbuf = smem;                                  // kSfBytesQK
    float* mu = reinterpret_cast<float*>(smem + 1024);      // D floats
    const bool smooth = (job == 1) && p.smooth_k;
    for (int d = t; d < D; d += kThreads) {
      float m = 0.0f;
      if (smooth) {
        double s = 0.0;
        for (int g = 0; g < p.nsplit; ++g) s += p.partial[(static_cast<size_t>(bh) * p.nsplit + g) * D + d];
        m = static_cast<float>(s / static_cast<double>(p.N));
        if (tile == 0 && p.k_mean != nullptr) p.k_mean[static_cast<size_t>(bh) * D + d] = m;
      }
      mu[d] = m;
    }
    for (int i = t; i < kSfBytesQK / 16; i += kThreads) reinterpret_cast<uint4*>(sfbuf)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    const char* src = static_cast<const char*>(job == 0 ? p.q : p.k) + static_cast<size_t>(bh) * p.N * D * 2;
    uint8_t* dst = (job == 0 ? p.q_fp4 : p.k_fp4) + static_cast<size_t>(bh) * p.Np * (D / 2);
#pragma unroll 2
    for (int g = t; g < 128 * CPR; g += kThreads) {
      const int rl = g / CPR, c = g % CPR;
      const int n = row0 + rl;
      float x[8];
      if (n < p.N) {
        unpack8(ld_nc_16(src + (static_cast<size_t>(n) * D + c * 8) * 2), p.dtype, x);
        if (smooth) {
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], mu[c * 8 + e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 0.0f;
      }
      float a = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(x[e]));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));  // partner holds the other 8 of the block
      const uint32_t sb = f32_to_e4m3(__fdiv_rn(a, 6.0f));
      const float s = e4m3_to_f32(sb);
      const uint32_t w = encode8(x, s);
      *reinterpret_cast<uint32_t*>(dst + static_cast<size_t>(n) * (D / 2) + c * 4) = w;
      if ((c & 1) == 0) {
        const int col = c * 8;
        sfbuf[(col / 64) * 512 + (rl % 32) * 16 + (rl / 32) * 4 + (col % 64) / 16] = static_cast<uint8_t>(sb);
      }
    }
    __syncthreads();
    uint8_t* sf_out = (job == 0 ? p.q_sf : p.k_sf) + (static_cast<size_t>(bh) * ntiles + tile) * kSfBytesQK;
    for (int i = t; i < kSfBytesQK / 16; i += kThreads)
      reinterpret_cast<uint4*>(sf_out)[i] = reinterpret_cast<const uint4*>(sfbuf)[i];
    return;
  }

  // ---- V^T: tokens become the contiguous (contraction) dimension ----
  uint8_t* vtile = smem;                                // 128 x kVRowBytes
  uint8_t* cbuf = smem + 128 * kVRowBytes;              // D x kCodeRow
  uint8_t* sfbuf = cbuf + D * kCodeRow;                 // 1024
  const char* src = static_cast<const char*>(p.v) + static_cast<size_t>(bh) * p.N * D * 2;
  for (int i = t; i < 1024 / 16; i += kThreads) reinterpret_cast<uint4*>(sfbuf)[i] = make_uint4(0, 0, 0, 0);
  for (int g = t; g < 128 * CPR; g += kThreads) {
    const int rl = g / CPR, c = g % CPR;
    const int n = row0 + rl;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (n < p.N) raw = ld_nc_16(src + (static_cast<size_t>(n) * D + c * 8) * 2);
    *reinterpret_cast<uint4*>(vtile + rl * kVRowBytes + c * 16) = raw;
  }
  __syncthreads();
  for (int item = t; item < D * 8; item += kThreads) {
    const int d = item % D, tb = item / D;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint16_t h = *reinterpret_cast<const uint16_t*>(vtile + (tb * 16 + i) * kVRowBytes + d * 2);
      x[i] = (p.dtype == kDtypeBF16) ? __uint_as_float(static_cast<uint32_t>(h) << 16)
                                     : __half2float(__ushort_as_half(h));
    }
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
    const uint32_t sb = f32_to_e4m3(__fdiv_rn(a, 6.0f));
    const float s = e4m3_to_f32(sb);
    float lo[8], hi[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lo[i] = x[i];
      hi[i] = x[8 + i];
    }
    const uint32_t w0 = encode8(lo, s), w1 = encode8(hi, s);
    *reinterpret_cast<uint2*>(cbuf + d * kCodeRow + tb * 8) = make_uint2(w0, w1);
    sfbuf[(tb / 4) * 512 + (d % 32) * 16 + (d / 32) * 4 + (tb % 4)] = static_cast<uint8_t>(sb);
  }
  __syncthreads();
  uint8_t* vt = p.vt_fp4 + static_cast<size_t>(bh) * D * (p.Np / 2) + tile * 64;
  for (int g = t; g < D * 4; g += kThreads) {
    const int d = g / 4, k = g % 4;
    *reinterpret_cast<uint4*>(vt + static_cast<size_t>(d) * (p.Np / 2) + k * 16) =
        *reinterpret_cast<const uint4*>(cbuf + d * kCodeRow + k * 16);
  }
  uint8_t* sf_out = p.vt_sf + (static_cast<size_t>(bh) * ntiles + tile) * 1024;
  for (int i = t; i < 1024 / 16; i += kThreads)
    reinterpret_cast<uint4*>(sf_out)[i] = reinterpret_cast<const uint4*>(sfbuf)[i];
}

cudaError_t launch_quantize(const QuantParams& p, cudaStream_t stream) {
  if (p.BH == 0 || p.N == 0) return cudaSuccess;
  const int ntiles = p.Np / 128;
  if (p.smooth_k) {
    dim3 g1(p.nsplit, p.BH);
    if (p.D == 64) kmean_partial_kernel<64><<<g1, kThreads, 0, stream>>>(p);
    else kmean_partial_kernel<128><<<g1, kThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  dim3 g2(ntiles, p.BH, 3);
  if (p.D == 64) quant_kernel<64><<<g2, kThreads, 0, stream>>>(p);
  else quant_kernel<128><<<g2, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace sage
