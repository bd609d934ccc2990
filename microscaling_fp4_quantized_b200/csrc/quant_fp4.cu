// Quantization kernels of the FP4 attention forward (sm_100a):
//   seq_plan_kernel  : packed sequences only -- checks the sequence table and prefix-sums
//                      the padded (multiple-of-128) lengths
//   stats_kernel     : per 512-token chunk: binary64 column sums of K; with a second-level
//                      scale also the column maxima / minima of K and the maxima of |Q|, |V|
//   finalize_kernel  : per (sequence, head): the K mean and the second-level maxima
//   quant_kernel     : Q, K - mean (one launch) and V^T (another) -> packed E2M1 codes +
//                      UE4M3 scale tiles
//
// The block rule follows the microscaling FP4 statement of SageAttention3 (arXiv
// 2505.11594, abstract): per 16 consecutive elements, s = E4M3(absmax / 6) and
// code = E2M1(x / s), both round-to-nearest-even with saturation; "smoothing K"
// (SageAttention OpenReview thread, reply to W1) subtracts the per-channel token mean
// of K first. The optional second-level scale (NVFP4's FP32 factor, named on the
// author page, "TetraJet-v2" abstract) divides a whole tensor, or one head of one
// sequence, by g = amax / 2688 before the block rule -- the same two-level shape the
// method gives P~. Every arithmetic step is IEEE binary32 with RNE, and every quotient is
// the IEEE binary32 quotient (an IEEE division, or one of the two forms below proven to
// equal it where they are used), so codes and scale bytes are reproducible bit for bit.
//
// All four kernels are HBM-bound (or tiny): 16-byte coalesced loads, tiles of 128
// tokens, scale factors and V^T codes staged in shared memory and written out as
// 16-byte chunks; V^T is stored tile-major (one contiguous D x 64-byte block per tile).
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

// x / d rounded to nearest even, from r = RN(1/d): the FMA-corrected quotient of
// Markstein ("IA-64 and Elementary Functions: Speed and Precision", 2000, ch. 8):
// q = RN(x r), e = x - q d (exact with an FMA), result RN(q + e r). It is not correctly
// rounded for every divisor, so it is used only where it was checked exhaustively on the
// CPU against IEEE binary32 division: d = any positive E4M3 value with |x/d| in
// [2^-4, 2^4) (E2M1 codes outside that range do not depend on the last bit of the
// quotient), and d = 6 for every positive binary32 x with a normal quotient (a subnormal
// a/6 gives scale byte 0 either way). The sign is copied from x so that -0 / d = -0.
__device__ __forceinline__ float div_fma(float x, float d, float r) {
  const float q = __fmul_rn(x, r);
  const float e = __fmaf_rn(-q, d, x);
  return copysignf(__fmaf_rn(e, r, q), x);
}

// x / d rounded to binary32 exactly as the IEEE division, from c ~ 1/d in double formed
// once per divisor (recip_d): the double product x * c is within ~2^-52 (relative) of
// x / d, while for binary32 x and d the quotient is either representable or at least
// 2^-49 (relative) away from every binary32 rounding midpoint (x - d * mid is a nonzero
// multiple of ulp(d) * ulp(mid) / 2, and a midpoint has 25 significant bits), so rounding
// the product gives the correctly rounded quotient -- subnormal quotients included.
// Checked on the CPU for random divisors with the same reciprocal sequence.
__device__ __forceinline__ float div_by(float x, double c) {
  return __double2float_rn(static_cast<double>(x) * c);
}

// 1/d in double to ~2^-53 relative for a positive finite binary32 d: the binary32
// reciprocal refined by two Newton steps (each squares the relative error) in double
// FMAs; d below 2^-64 is scaled by 2^64 first so that the binary32 reciprocal stays
// finite. No division, so no division subroutine in the kernel.
__device__ __forceinline__ double recip_d(float d) {
  const bool tiny = d < 5.421010862427522e-20f;  // 2^-64
  const float ds = tiny ? d * 18446744073709551616.0f : d;
  const double dd = static_cast<double>(ds);
  double y = static_cast<double>(__frcp_rn(ds));
  y = fma(y, fma(-dd, y, 1.0), y);
  y = fma(y, fma(-dd, y, 1.0), y);
  return tiny ? y * 18446744073709551616.0 : y;
}

// RN(1/6) in binary32.
constexpr float kRecip6 = 0.16666667163372039794921875f;

// E4M3 scale byte of a block with maximum magnitude a: E4M3(RN(a / 6)).
__device__ __forceinline__ uint32_t block_scale_byte(float a) {
  return f32_to_e4m3(div_fma(a, 6.0f, kRecip6));
}

// Codes of 8 values against a decoded scale s (s == 0 -> zero codes); element 0 lands
// in the low nibble of the low byte. Each code is E2M1(RN(x / s)).
__device__ __forceinline__ uint32_t encode8(const float (&x)[8], float s) {
  if (s == 0.0f) return 0u;
  const float r = __frcp_rn(s);
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = div_fma(x[2 * i], s, r);
    const float b = div_fma(x[2 * i + 1], s, r);
    w |= f32x2_to_e2m1(a, b) << (8 * i);
  }
  return w;
}

// Address of element (b, h, token) of a [.., D] input whose channels are contiguous.
__device__ __forceinline__ const char* row_ptr(const void* base, const Strides& s, int b, int h, int64_t tok) {
  return static_cast<const char*>(base) + (static_cast<int64_t>(b) * s.b + static_cast<int64_t>(h) * s.h + tok * s.n) * 2;
}

// 16 bytes (8 elements, channels 8c .. 8c + 7) of row (b, h, tok) of a caller tensor;
// the bounds-checked build refuses an offset outside the problem's extent (zeros).
__device__ __forceinline__ uint4 ld_row16(const void* base, const Strides& s, int b, int h, int64_t tok, int c,
                                          uint64_t lim_el, uint32_t* err) {
  const int64_t off = static_cast<int64_t>(b) * s.b + static_cast<int64_t>(h) * s.h + tok * s.n + 8 * c;
  (void)lim_el;
  (void)err;
  if (!SAGE_IN_BOUNDS(off >= 0 && static_cast<uint64_t>(off) + 8 <= lim_el, err, nullptr)) return make_uint4(0, 0, 0, 0);
  return ld_nc_16(static_cast<const char*>(base) + off * 2);
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x / 32, nw = blockDim.x / 32;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = 0.0f;
  for (int i = 0; i < nw; ++i) r = fmaxf(r, red[i]);
  return r;
}

__device__ __forceinline__ void amax_store(float* slot, int mode, float a) {
  if (mode == kGscaleTensor) atomicMax(reinterpret_cast<unsigned int*>(slot), __float_as_uint(a));
  else *slot = a;
}

constexpr int kThreads = 256;
constexpr int kChunk = 512;  // tokens per statistics chunk

}  // namespace

// One CTA. Checks cu_q / cu_k (start at 0, non-decreasing, end at the packed totals,
// no sequence longer than its stated maximum) and writes the exclusive prefix sums of
// the padded lengths; a failed check sets *bad and the device error bit instead.
__global__ void __launch_bounds__(1024) seq_plan_kernel(QuantParams p) {
  __shared__ long long wq[32], wk[32];
  __shared__ int s_bad;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  if (t == 0) s_bad = 0;
  __syncthreads();
  const int B = p.B;
  const int per = (B + 1023) / 1024;
  const int b0 = min(B, t * per), b1 = min(B, b0 + per);
  long long sq = 0, sk = 0;
  int bad = 0;
  for (int b = b0; b < b1; ++b) {
    const int lq = p.seq.cu_q[b + 1] - p.seq.cu_q[b];
    const int lk = p.seq.cu_k[b + 1] - p.seq.cu_k[b];
    if (lq < 0 || lk < 0 || lq > p.seq.Nq || lk > p.seq.Nk) bad = 1;
    sq += (max(lq, 0) + 127) / 128 * 128;
    sk += (max(lk, 0) + 127) / 128 * 128;
  }
  if (t == 0 && (p.seq.cu_q[0] != 0 || p.seq.cu_k[0] != 0 || p.seq.cu_q[B] != p.total_q ||
                 p.seq.cu_k[B] != p.total_k))
    bad = 1;
  if (bad) atomicOr(&s_bad, 1);
  // Block-wide inclusive scan of (sq, sk).
  long long iq = sq, ik = sk;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long a = __shfl_up_sync(0xffffffffu, iq, o), c = __shfl_up_sync(0xffffffffu, ik, o);
    if (lane >= o) {
      iq += a;
      ik += c;
    }
  }
  if (lane == 31) {
    wq[w] = iq;
    wk[w] = ik;
  }
  __syncthreads();
  long long oq = 0, ok = 0;
  for (int i = 0; i < w; ++i) {
    oq += wq[i];
    ok += wk[i];
  }
  long long eq = oq + iq - sq, ek = ok + ik - sk;  // exclusive prefix of this thread's range
  __syncthreads();
  if (s_bad) {
    if (t == 0) {
      *p.bad_out = 1u;
      atomicOr(p.err, kDevErrSeqlens);
    }
    return;
  }
  for (int b = b0; b < b1; ++b) {
    p.pad_q_out[b] = static_cast<int32_t>(eq);
    p.pad_k_out[b] = static_cast<int32_t>(ek);
    eq += (p.seq.cu_q[b + 1] - p.seq.cu_q[b] + 127) / 128 * 128;
    ek += (p.seq.cu_k[b + 1] - p.seq.cu_k[b] + 127) / 128 * 128;
  }
  if (b1 == B) {
    p.pad_q_out[B] = static_cast<int32_t>(eq);
    p.pad_k_out[B] = static_cast<int32_t>(ek);
  }
  if (t == 0) *p.bad_out = 0u;
}

// Channel statistics of one 512-token chunk of one (sequence, head) of a [.., D] input:
// binary64 sums into sum[.., D]; with extremes also float maxima / minima per channel.
template <int D>
__device__ __forceinline__ void chunk_channel_stats(const void* src, const Strides& st, int dtype, int b, int h,
                                                    int64_t tok0, int n0, int n1, bool extremes,
                                                    double* sum, float* cmax, float* cmin,
                                                    double (*red)[D], float (*redmx)[D], float (*redmn)[D],
                                                    uint64_t lim_el, uint32_t* err) {
  constexpr int CPR = D / 8;
  constexpr int RG = kThreads / CPR;
  const int t = threadIdx.x, c = t % CPR, rg = t / CPR;
  double acc[8];
  float mx[8], mn[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    acc[e] = 0.0;
    mx[e] = -INFINITY;
    mn[e] = INFINITY;
  }
#pragma unroll 8
  for (int n = n0 + rg; n < n1; n += RG) {
    float x[8];
    unpack8(ld_row16(src, st, b, h, tok0 + n, c, lim_el, err), dtype, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      acc[e] += static_cast<double>(x[e]);
      mx[e] = fmaxf(mx[e], x[e]);
      mn[e] = fminf(mn[e], x[e]);
    }
  }
  __syncthreads();  // the reduction buffers may still be read by a previous call
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    red[rg][c * 8 + e] = acc[e];
    redmx[rg][c * 8 + e] = mx[e];
    redmn[rg][c * 8 + e] = mn[e];
  }
  __syncthreads();
  for (int d = t; d < D; d += kThreads) {
    double sacc = 0.0;
    float a = -INFINITY, z = INFINITY;
    for (int g = 0; g < RG; ++g) {
      sacc += red[g][d];
      a = fmaxf(a, redmx[g][d]);
      z = fminf(z, redmn[g][d]);
    }
    sum[d] = sacc;
    if (extremes) {
      cmax[d] = a;
      cmin[d] = z;
    }
  }
}

// grid (nsplit, Hq, B): chunk `split` of sequence b, head h.
//   K (h < Hkv, K smoothing or a second-level scale): ksum[bh, split, d] = sum over the
//     chunk's tokens, binary64; with a second-level scale also kmax / kmin per channel.
//   Q (h < Hq, Q smoothing): the same statistics of Q into qsum / qmax / qmin.
//   Q without smoothing (h < Hq) and V (h < Hkv), second-level scale only: max |x| over
//   the chunk.
template <int D>
__global__ void __launch_bounds__(kThreads, 4) stats_kernel(QuantParams p) {
  constexpr int CPR = D / 8;          // 16-byte chunks per row
  constexpr int RG = kThreads / CPR;  // row groups
  __shared__ double red[RG][D];
  __shared__ float redmx[RG][D], redmn[RG][D];
  __shared__ float redw[kThreads / 32];
  if (seq_table_bad(p.seq)) return;
  const int t = threadIdx.x, c = t % CPR, rg = t / CPR;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const SeqInfo si = seq_info(p.seq, b);
  const bool gs = p.gscale != kGscaleNone;
  if (gs && p.gscale == kGscaleTensor && split == 0 && h == 0 && b == 0 && t < 3) p.amax[t * p.amax_stride] = 0.0f;
  const int n0 = split * kChunk;

  if (h < p.Hkv && (p.smooth_k || gs) && n0 < si.len_k) {
    const size_t base = (static_cast<size_t>(b * p.Hkv + h) * p.nsplit + split) * D;
    if (!SAGE_IN_BOUNDS(base + D <= p.lim.stat_el, p.err, nullptr)) return;
    chunk_channel_stats<D>(p.k, p.sk, p.dtype, b, h, si.tok_k, n0, min(n0 + kChunk, si.len_k), gs,
                           p.ksum + base, gs ? p.kmax + base : nullptr, gs ? p.kmin + base : nullptr,
                           red, redmx, redmn, p.lim.k_el, p.err);
  }
  if (h < p.Hkv && p.bits8 && n0 < si.len_k) {
    const size_t base = (static_cast<size_t>(b * p.Hkv + h) * p.nsplit + split) * D;
    if (!SAGE_IN_BOUNDS(base + D <= p.lim.stat_el, p.err, nullptr)) return;
    chunk_channel_stats<D>(p.v, p.sv, p.dtype, b, h, si.tok_k, n0, min(n0 + kChunk, si.len_k), true,
                           p.vsum + base, p.vmax + base, p.vmin + base, red, redmx, redmn, p.lim.v_el, p.err);
  }
  if (h < p.Hq && p.smooth_q && n0 < si.len_q) {
    const size_t base = (static_cast<size_t>(b * p.Hq + h) * p.nsplit + split) * D;
    if (!SAGE_IN_BOUNDS(base + D <= p.lim.qstat_el, p.err, nullptr)) return;
    chunk_channel_stats<D>(p.q, p.sq, p.dtype, b, h, si.tok_q, n0, min(n0 + kChunk, si.len_q), gs,
                           p.qsum + base, gs ? p.qmax + base : nullptr, gs ? p.qmin + base : nullptr,
                           red, redmx, redmn, p.lim.q_el, p.err);
  }
  if (!gs) return;
  for (int job = 0; job < 2; ++job) {  // 0: Q (unsmoothed), 1: V
    if (job == 0 && p.smooth_q) continue;
    const int H = job == 0 ? p.Hq : p.Hkv;
    const int len = job == 0 ? si.len_q : si.len_k;
    if (h >= H || n0 >= len) continue;
    const int n1 = min(n0 + kChunk, len);
    const void* src = job == 0 ? p.q : p.v;
    const Strides& st = job == 0 ? p.sq : p.sv;
    const int tok = job == 0 ? si.tok_q : si.tok_k;
    float a = 0.0f;
#pragma unroll 8
    for (int n = n0 + rg; n < n1; n += RG) {
      float x[8];
      unpack8(ld_row16(src, st, b, h, static_cast<int64_t>(tok) + n, c, job == 0 ? p.lim.q_el : p.lim.v_el, p.err), p.dtype, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(x[e]));
    }
    a = block_max(a, redw);
    const size_t ia = static_cast<size_t>(b * H + h) * p.nsplit + split;
    if (t == 0 && SAGE_IN_BOUNDS(ia < (job == 0 ? p.lim.qamax_el : p.lim.vamax_el), p.err, nullptr))
      (job == 0 ? p.qamax : p.vamax)[ia] = a;
  }
}

// grid (Hq, B), D threads: the K mean of (sequence b, key/value head h), the Q mean of
// query head h (Q smoothing), and the second-level maxima of Q (or Q - mean) for head h
// and of K - mean and V for head h.
template <int D>
__global__ void __launch_bounds__(D) finalize_kernel(QuantParams p) {
  __shared__ float redw[D / 32];
  if (seq_table_bad(p.seq)) return;
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const SeqInfo si = seq_info(p.seq, b);
  const bool gs = p.gscale != kGscaleNone;
  if (h < p.Hkv) {
    const int ns = (si.len_k + kChunk - 1) / kChunk;
    const size_t base = static_cast<size_t>(b * p.Hkv + h) * p.nsplit * D + d;
    float mu = 0.0f;
    if (p.smooth_k && si.len_k > 0) {
      double s = 0.0;
      for (int g = 0; g < ns; ++g) s += p.ksum[base + static_cast<size_t>(g) * D];
      mu = static_cast<float>(s / static_cast<double>(si.len_k));
    }
    if (SAGE_IN_BOUNDS(static_cast<size_t>(b * p.Hkv + h) * D + d < p.lim.k_mean_el, p.err, nullptr))
      p.k_mean[static_cast<size_t>(b * p.Hkv + h) * D + d] = mu;
    if (p.bits8) {
      // E4M3 scale of V's channel d: fp32(max |v| / 448) over the sequence's tokens.
      float mx = -INFINITY, mn = INFINITY;
      for (int g = 0; g < ns; ++g) {
        mx = fmaxf(mx, p.vmax[base + static_cast<size_t>(g) * D]);
        mn = fminf(mn, p.vmin[base + static_cast<size_t>(g) * D]);
      }
      const float a = si.len_k > 0 ? fmaxf(fabsf(mx), fabsf(mn)) : 0.0f;
      p.v_scale[static_cast<size_t>(b * p.Hkv + h) * D + d] = __fdiv_rn(a, 448.0f);
    }
    if (gs) {
      float mx = -INFINITY, mn = INFINITY, av = 0.0f;
      for (int g = 0; g < ns; ++g) {
        mx = fmaxf(mx, p.kmax[base + static_cast<size_t>(g) * D]);
        mn = fminf(mn, p.kmin[base + static_cast<size_t>(g) * D]);
      }
      // Rounding is monotone, so max |fp32(k - mu)| over the tokens is reached at the
      // channel's largest or smallest k.
      float ak = si.len_k > 0 ? fmaxf(fabsf(__fsub_rn(mx, mu)), fabsf(__fsub_rn(mn, mu))) : 0.0f;
      ak = block_max(ak, redw);
      for (int g = d; g < ns; g += D) av = fmaxf(av, p.vamax[static_cast<size_t>(b * p.Hkv + h) * p.nsplit + g]);
      av = block_max(av, redw);
      if (d == 0) {
        const int i = p.gscale == kGscaleHead ? b * p.Hkv + h : 0;
        amax_store(p.amax + p.amax_stride + i, p.gscale, ak);
        amax_store(p.amax + 2 * p.amax_stride + i, p.gscale, av);
      }
    }
  }
  if (h < p.Hq && (gs || p.smooth_q)) {
    const int ns = (si.len_q + kChunk - 1) / kChunk;
    float aq = 0.0f;
    if (p.smooth_q) {
      // The query mean, and (second-level scale) the maximum of |fp32(q - mu_q)|.
      const size_t base = static_cast<size_t>(b * p.Hq + h) * p.nsplit * D + d;
      float mu = 0.0f;
      if (si.len_q > 0) {
        double s = 0.0;
        for (int g = 0; g < ns; ++g) s += p.qsum[base + static_cast<size_t>(g) * D];
        mu = static_cast<float>(s / static_cast<double>(si.len_q));
      }
      if (SAGE_IN_BOUNDS(static_cast<size_t>(b * p.Hq + h) * D + d < p.lim.q_mean_el, p.err, nullptr))
        p.q_mean[static_cast<size_t>(b * p.Hq + h) * D + d] = mu;
      if (gs && si.len_q > 0) {
        float mx = -INFINITY, mn = INFINITY;
        for (int g = 0; g < ns; ++g) {
          mx = fmaxf(mx, p.qmax[base + static_cast<size_t>(g) * D]);
          mn = fminf(mn, p.qmin[base + static_cast<size_t>(g) * D]);
        }
        aq = fmaxf(fabsf(__fsub_rn(mx, mu)), fabsf(__fsub_rn(mn, mu)));
      }
    } else {
      for (int g = d; g < ns; g += D) aq = fmaxf(aq, p.qamax[static_cast<size_t>(b * p.Hq + h) * p.nsplit + g]);
    }
    if (gs) {
      aq = block_max(aq, redw);
      if (d == 0) amax_store(p.amax + (p.gscale == kGscaleHead ? b * p.Hq + h : 0), p.gscale, aq);
    }
  }
}

// Two launches: VJOB = false, grid (2 * tiles, Hq, B), x = 2 * tile + job, job 0 quantizes
// Q rows and 1 K rows (smoothed); VJOB = true, grid (key tiles, Hkv, B), V^T. Only the V
// transpose needs a large shared-memory tile, so the Q/K launch keeps many CTAs per SM.
// CTAs past a sequence's tiles or heads return at once.
// At most 64 registers (4 CTAs per SM): the extra resident warps hide more load latency
// than the few spilled values cost (measured 0.35 -> 0.31 ms for the long workload's
// quantization with the statistics loop unrolled 8-deep; identical output bytes).
template <int D, bool VJOB, bool GS>
__global__ void __launch_bounds__(kThreads, 4) quant_kernel(QuantParams p) {
  constexpr int CPR = D / 8;
  constexpr int kVRowBytes = (D + 8) * 2;  // padded V tile row (16-byte multiple)
  constexpr int kCodeRow = 80;             // padded V^T code staging row (64 used)
  constexpr int kSfBytesQK = (D / 64) * 512;
  __shared__ __align__(16) uint8_t smem[VJOB ? 128 * kVRowBytes + D * kCodeRow + 1024 : 1024 + D * 4];
  if (seq_table_bad(p.seq)) return;
  const int t = threadIdx.x;
  const int job = VJOB ? 2 : static_cast<int>(blockIdx.x % 2);
  const int tile = VJOB ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x / 2);
  const int h = blockIdx.y, b = blockIdx.z;
  const int H = job == 0 ? p.Hq : p.Hkv;
  if (h >= H) return;
  const SeqInfo si = seq_info(p.seq, b);
  const int len = job == 0 ? si.len_q : si.len_k;
  const int ntile = (len + 127) >> 7;
  if (tile >= ntile) return;
  const int prow = job == 0 ? si.prow_q : si.prow_k;
  const int64_t tok0 = static_cast<int64_t>(job == 0 ? si.tok_q : si.tok_k) + tile * 128;
  const int64_t row0 = static_cast<int64_t>(H) * prow + static_cast<int64_t>(h) * ntile * 128 + tile * 128;
  const int64_t T = row0 >> 7;  // scale-factor / V^T tile index
  const int rows = min(128, len - tile * 128);
  constexpr bool gs = GS;  // second-level scale (its own instance, so the plain one carries none of its code)
  float g = 1.0f;
  if (gs) g = second_level_scale(p.amax[job * p.amax_stride + (p.gscale == kGscaleHead ? b * H + h : 0)]);
  const double cg = gs ? recip_d(g) : 1.0;  // x / g = div_by(x, cg)

  if constexpr (!VJOB) {
    uint8_t* sfbuf = smem;                                  // kSfBytesQK
    float* mu = reinterpret_cast<float*>(smem + 1024);      // D floats
    const bool smooth = (job == 1) ? p.smooth_k != 0 : p.smooth_q != 0;
    const float* mean_src = (job == 1 ? p.k_mean : p.q_mean) + static_cast<size_t>(b * H + h) * D;
    for (int d = t; d < D; d += kThreads) mu[d] = smooth ? mean_src[d] : 0.0f;
    for (int i = t; i < kSfBytesQK / 16; i += kThreads) reinterpret_cast<uint4*>(sfbuf)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    const void* src = job == 0 ? p.q : p.k;
    const Strides& st = job == 0 ? p.sq : p.sk;
    uint8_t* dst = (job == 0 ? p.q_fp4 : p.k_fp4) + row0 * (D / 2);
    // Every thread owns one 8-channel chunk c of rows rl0, rl0 + kRowStep, ...: all of its
    // 16-byte loads are issued before any of them is used.
    constexpr int kRowStep = kThreads / CPR, kIter = 128 / kRowStep;
    const int c = t % CPR, rl0 = t / CPR;
    float m8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m8[e] = mu[c * 8 + e];
    uint4 raw[kIter];
#pragma unroll
    for (int it = 0; it < kIter; ++it) {
      const int rl = rl0 + it * kRowStep;
      raw[it] = rl < rows ? ld_row16(src, st, b, h, tok0 + rl, c, job == 0 ? p.lim.q_el : p.lim.k_el, p.err)
                          : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int it = 0; it < kIter; ++it) {
      const int rl = rl0 + it * kRowStep;
      float x[8];
      unpack8(raw[it], p.dtype, x);
      if (rl < rows && smooth) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], m8[e]);
      }
      if (job == 1 && p.smooth_q) {
        // Q smoothing bias of this key for every query head of the group:
        // mu_q . (k - mu_k), over the CPR lanes that hold the row (zero for padding).
        const int G = p.Hq / p.Hkv;
        for (int gi = 0; gi < G; ++gi) {
          const int hq = h * G + gi;
          const float4* mq = reinterpret_cast<const float4*>(p.q_mean + static_cast<size_t>(b * p.Hq + hq) * D + c * 8);
          const float4 m0 = mq[0], m1 = mq[1];
          float acc = x[0] * m0.x;
          acc = fmaf(x[1], m0.y, acc);
          acc = fmaf(x[2], m0.z, acc);
          acc = fmaf(x[3], m0.w, acc);
          acc = fmaf(x[4], m1.x, acc);
          acc = fmaf(x[5], m1.y, acc);
          acc = fmaf(x[6], m1.z, acc);
          acc = fmaf(x[7], m1.w, acc);
#pragma unroll
          for (int o = CPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (c == 0) {
            if (gs) {
              const float gq = second_level_scale(p.amax[p.gscale == kGscaleHead ? b * p.Hq + hq : 0]);
              acc = __fdiv_rn(acc, gq * g);
            }
            // Three bf16 terms (their sum is acc to about 2^-24 relative) in the operand
            // layout the attention kernel's bias MMA reads: 8-key groups of 256 bytes, two
            // 128-byte halves of 8 keys x 16 bytes.
            const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
            const float r1 = acc - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
            const uint32_t w0 = static_cast<uint32_t>(__bfloat16_as_ushort(hi)) |
                                (static_cast<uint32_t>(__bfloat16_as_ushort(mid)) << 16);
            const uint32_t w1 = static_cast<uint32_t>(__bfloat16_as_ushort(lo));
            uint8_t* tb = p.qk_bias + (static_cast<int64_t>(p.Hq) * prow + static_cast<int64_t>(hq) * ntile * 128 +
                                       tile * 128) * 32;
            uint8_t* row = tb + (rl >> 3) * 256 + (rl & 7) * 16;
            if (SAGE_IN_BOUNDS(static_cast<uint64_t>(row + 144 - p.qk_bias) <= p.lim.qk_bias, p.err, nullptr)) {
              *reinterpret_cast<uint4*>(row) = make_uint4(w0, w1, 0u, 0u);
              *reinterpret_cast<uint4*>(row + 128) = make_uint4(0u, 0u, 0u, 0u);
            }
          }
        }
      }
      if (rl < rows && gs) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = div_by(x[e], cg);
      }
      float a = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(x[e]));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));  // partner holds the other 8 of the block
      const uint32_t sb = block_scale_byte(a);
      const float s = e4m3_to_f32(sb);
      const uint32_t w = encode8(x, s);
      if (SAGE_IN_BOUNDS(static_cast<uint64_t>(row0 + rl) * (D / 2) + c * 4 + 4 <= (job == 0 ? p.lim.q_fp4 : p.lim.k_fp4),
                         p.err, nullptr))
        *reinterpret_cast<uint32_t*>(dst + static_cast<size_t>(rl) * (D / 2) + c * 4) = w;
      if ((c & 1) == 0) {
        const int col = c * 8;
        sfbuf[(col / 64) * 512 + (rl % 32) * 16 + (rl / 32) * 4 + (col % 64) / 16] = static_cast<uint8_t>(sb);
      }
    }
    __syncthreads();
    uint8_t* sf_out = (job == 0 ? p.q_sf : p.k_sf) + T * kSfBytesQK;
    if (SAGE_IN_BOUNDS(static_cast<uint64_t>(T + 1) * kSfBytesQK <= (job == 0 ? p.lim.q_sf : p.lim.k_sf), p.err, nullptr))
      for (int i = t; i < kSfBytesQK / 16; i += kThreads)
        reinterpret_cast<uint4*>(sf_out)[i] = reinterpret_cast<const uint4*>(sfbuf)[i];
  } else {
    // ---- V^T: tokens become the contiguous (contraction) dimension ----
    uint8_t* vtile = smem;                                // 128 x kVRowBytes
    uint8_t* cbuf = smem + 128 * kVRowBytes;              // D x kCodeRow
    uint8_t* sfbuf = cbuf + D * kCodeRow;                 // 1024
    for (int i = t; i < 1024 / 16; i += kThreads) reinterpret_cast<uint4*>(sfbuf)[i] = make_uint4(0, 0, 0, 0);
    {
      constexpr int kRowStep = kThreads / CPR, kIter = 128 / kRowStep;
      const int c = t % CPR, rl0 = t / CPR;
      uint4 raw[kIter];
  #pragma unroll
      for (int it = 0; it < kIter; ++it) {
        const int rl = rl0 + it * kRowStep;
        raw[it] = rl < rows ? ld_row16(p.v, p.sv, b, h, tok0 + rl, c, p.lim.v_el, p.err) : make_uint4(0, 0, 0, 0);
      }
  #pragma unroll
      for (int it = 0; it < kIter; ++it)
        *reinterpret_cast<uint4*>(vtile + (rl0 + it * kRowStep) * kVRowBytes + c * 16) = raw[it];
    }
    __syncthreads();
    for (int item = t; item < D * 8; item += kThreads) {
      const int d = item % D, tb = item / D;
      float x[16];
  #pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint16_t hv = *reinterpret_cast<const uint16_t*>(vtile + (tb * 16 + i) * kVRowBytes + d * 2);
        x[i] = (p.dtype == kDtypeBF16) ? __uint_as_float(static_cast<uint32_t>(hv) << 16)
                                       : __half2float(__ushort_as_half(hv));
        if (gs) x[i] = div_by(x[i], cg);
      }
      float a = 0.0f;
  #pragma unroll
      for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
      const uint32_t sb = block_scale_byte(a);
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
    uint8_t* vt = p.vt_fp4 + T * (D * 64);
    if (SAGE_IN_BOUNDS(static_cast<uint64_t>(T + 1) * (D * 64) <= p.lim.vt_fp4, p.err, nullptr))
      for (int gi = t; gi < D * 4; gi += kThreads) {
        const int d = gi / 4, k = gi % 4;
        *reinterpret_cast<uint4*>(vt + d * 64 + k * 16) = *reinterpret_cast<const uint4*>(cbuf + d * kCodeRow + k * 16);
      }
    uint8_t* sf_out = p.vt_sf + T * 1024;
    if (SAGE_IN_BOUNDS(static_cast<uint64_t>(T + 1) * 1024 <= p.lim.vt_sf, p.err, nullptr))
      for (int i = t; i < 1024 / 16; i += kThreads)
        reinterpret_cast<uint4*>(sf_out)[i] = reinterpret_cast<const uint4*>(sfbuf)[i];
  }
}

// ------------------------------------------------------------- 8-bit path ----
// Two launches, split like quant_kernel. VJOB = false, grid (2 * tiles, Hq, B),
// x = 2 * tile + job: jobs 0 and 1 turn a 128-row tile of Q or K - mean into symmetric
// INT8 with one scale s = fp32(absmax / 127) for the tile and codes
// clamp(RNE(fp32(x / s)), -127, 127). VJOB = true, grid (key tiles, Hkv, B): a 128-token
// tile of V becomes E4M3 codes fp32(v / s_d) with the channel scales of the finalize
// pass, transposed (tokens contiguous) and stored tile-major [key tiles, D, 128].
// Bounded to 4 CTAs per SM like quant_kernel (0.48 -> 0.46 ms for the long workload's
// 8-bit quantization, identical output bytes).
template <int D, bool VJOB>
__global__ void __launch_bounds__(kThreads, 4) quant8_kernel(QuantParams p) {
  constexpr int CPR = D / 8;
  constexpr int kVRowBytes = (D + 8) * 2;  // padded V tile row (16-byte multiple)
  constexpr int kCodeRow = 144;            // padded V^T code staging row (128 used)
  __shared__ __align__(16) uint8_t smem[VJOB ? 128 * kVRowBytes + D * 4 : D * 4];
  __shared__ float redw[kThreads / 32];
  static_assert(D * kCodeRow <= 128 * kVRowBytes, "V^T codes reuse the V tile's staging");
  if (seq_table_bad(p.seq)) return;
  const int t = threadIdx.x;
  const int job = VJOB ? 2 : static_cast<int>(blockIdx.x % 2);
  const int tile = VJOB ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x / 2);
  const int h = blockIdx.y, b = blockIdx.z;
  const int H = job == 0 ? p.Hq : p.Hkv;
  if (h >= H) return;
  const SeqInfo si = seq_info(p.seq, b);
  const int len = job == 0 ? si.len_q : si.len_k;
  const int ntile = (len + 127) >> 7;
  if (tile >= ntile) return;
  const int prow = job == 0 ? si.prow_q : si.prow_k;
  const int64_t tok0 = static_cast<int64_t>(job == 0 ? si.tok_q : si.tok_k) + tile * 128;
  const int64_t row0 = static_cast<int64_t>(H) * prow + static_cast<int64_t>(h) * ntile * 128 + tile * 128;
  const int64_t T = row0 >> 7;
  const int rows = min(128, len - tile * 128);
  constexpr int kRowStep = kThreads / CPR, kIter = 128 / kRowStep;
  const int c = t % CPR, rl0 = t / CPR;

  if constexpr (!VJOB) {
    float* mu = reinterpret_cast<float*>(smem);
    const bool smooth = job == 1 && p.smooth_k;
    for (int d = t; d < D; d += kThreads)
      mu[d] = smooth ? p.k_mean[static_cast<size_t>(b * p.Hkv + h) * D + d] : 0.0f;
    __syncthreads();
    float m8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m8[e] = mu[c * 8 + e];
    const void* src = job == 0 ? p.q : p.k;
    const Strides& st = job == 0 ? p.sq : p.sk;
    uint4 raw[kIter];
#pragma unroll
    for (int it = 0; it < kIter; ++it) {
      const int rl = rl0 + it * kRowStep;
      raw[it] = rl < rows ? ld_row16(src, st, b, h, tok0 + rl, c, job == 0 ? p.lim.q_el : p.lim.k_el, p.err)
                          : make_uint4(0, 0, 0, 0);
    }
    auto values = [&](int it, float (&x)[8]) {
      unpack8(raw[it], p.dtype, x);
      if (smooth && rl0 + it * kRowStep < rows) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], m8[e]);
      }
    };
    float a = 0.0f;
#pragma unroll
    for (int it = 0; it < kIter; ++it) {
      float x[8];
      values(it, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(x[e]));
    }
    a = block_max(a, redw);
    const float s = __fdiv_rn(a, 127.0f);
    const double cs = s > 0.0f ? recip_d(s) : 0.0;  // x / s = div_by(x, cs)
    if (t == 0 && SAGE_IN_BOUNDS(static_cast<uint64_t>(T + 1) * 4 <= (job == 0 ? p.lim.q_sf : p.lim.k_sf), p.err, nullptr))
      reinterpret_cast<float*>(job == 0 ? p.q_sf : p.k_sf)[T] = s;
    uint8_t* dst = (job == 0 ? p.q_fp4 : p.k_fp4) + row0 * D;
#pragma unroll
    for (int it = 0; it < kIter; ++it) {
      float x[8];
      values(it, x);
      uint32_t w[2] = {0u, 0u};
      if (s > 0.0f) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float r = fminf(127.0f, fmaxf(-127.0f, rintf(div_by(x[e], cs))));
          w[e >> 2] |= (static_cast<uint32_t>(static_cast<int>(r)) & 0xFFu) << (8 * (e & 3));
        }
      }
      if (SAGE_IN_BOUNDS(static_cast<uint64_t>(row0 + rl0 + it * kRowStep) * D + c * 8 + 8 <=
                             (job == 0 ? p.lim.q_fp4 : p.lim.k_fp4), p.err, nullptr))
        *reinterpret_cast<uint2*>(dst + static_cast<size_t>(rl0 + it * kRowStep) * D + c * 8) = make_uint2(w[0], w[1]);
    }
  } else {
  // ---- V^T: E4M3 with one scale per channel ----
  uint8_t* vtile = smem;                                         // 128 x kVRowBytes
  float* sv = reinterpret_cast<float*>(smem + 128 * kVRowBytes); // D channel scales
  for (int d = t; d < D; d += kThreads) sv[d] = p.v_scale[static_cast<size_t>(b * p.Hkv + h) * D + d];
  {
    uint4 raw[kIter];
#pragma unroll
    for (int it = 0; it < kIter; ++it) {
      const int rl = rl0 + it * kRowStep;
      raw[it] = rl < rows ? ld_row16(p.v, p.sv, b, h, tok0 + rl, c, p.lim.v_el, p.err) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int it = 0; it < kIter; ++it)
      *reinterpret_cast<uint4*>(vtile + (rl0 + it * kRowStep) * kVRowBytes + c * 16) = raw[it];
  }
  __syncthreads();
  constexpr int kItems = D * 8 / kThreads;  // (channel, 16-token block) pairs per thread
  uint4 codes[kItems];
#pragma unroll
  for (int k = 0; k < kItems; ++k) {
    const int item = t + k * kThreads;
    const int d = item % D, tb = item / D;
    const float s = sv[d];
    const double cs = s > 0.0f ? recip_d(s) : 0.0;  // x / s = div_by(x, cs)
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (s > 0.0f) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint16_t hv = *reinterpret_cast<const uint16_t*>(vtile + (tb * 16 + i) * kVRowBytes + d * 2);
        const float x = (p.dtype == kDtypeBF16) ? __uint_as_float(static_cast<uint32_t>(hv) << 16)
                                                : __half2float(__ushort_as_half(hv));
        w[i >> 2] |= f32_to_e4m3(div_by(x, cs)) << (8 * (i & 3));
      }
    }
    codes[k] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __syncthreads();  // the tile is read; its storage now stages the codes
  uint8_t* cbuf = smem;
#pragma unroll
  for (int k = 0; k < kItems; ++k) {
    const int item = t + k * kThreads;
    *reinterpret_cast<uint4*>(cbuf + (item % D) * kCodeRow + (item / D) * 16) = codes[k];
  }
  __syncthreads();
  uint8_t* vt = p.vt_fp4 + T * (D * 128);
  for (int gi = t; gi < D * 8; gi += kThreads) {
    const int d = gi / 8, k = gi % 8;
    if (SAGE_IN_BOUNDS(static_cast<uint64_t>(T) * (D * 128) + d * 128 + k * 16 + 16 <= p.lim.vt_fp4, p.err, nullptr))
      *reinterpret_cast<uint4*>(vt + d * 128 + k * 16) = *reinterpret_cast<const uint4*>(cbuf + d * kCodeRow + k * 16);
  }
  }
}

cudaError_t launch_quantize8(const QuantParams& p, const QuantLaunch& l, cudaStream_t stream) {
  if (p.B == 0 || p.Hq == 0) return cudaSuccess;
  if (p.seq.cu_q != nullptr) {
    seq_plan_kernel<<<1, 1024, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.nsplit > 0) {
    dim3 g1(p.nsplit, p.Hq, p.B);
    if (p.D == 64) stats_kernel<64><<<g1, kThreads, 0, stream>>>(p);
    else stats_kernel<128><<<g1, kThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    dim3 g2(p.Hq, p.B);
    if (p.D == 64) finalize_kernel<64><<<g2, 64, 0, stream>>>(p);
    else finalize_kernel<128><<<g2, 128, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int tiles = l.tiles_q > l.tiles_k ? l.tiles_q : l.tiles_k;
  if (tiles == 0) return cudaSuccess;
  dim3 g3(2 * tiles, p.Hq, p.B);
  if (p.D == 64) quant8_kernel<64, false><<<g3, kThreads, 0, stream>>>(p);
  else quant8_kernel<128, false><<<g3, kThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || l.tiles_k == 0) return e;
  dim3 g4(l.tiles_k, p.Hkv, p.B);
  if (p.D == 64) quant8_kernel<64, true><<<g4, kThreads, 0, stream>>>(p);
  else quant8_kernel<128, true><<<g4, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantParams& p, const QuantLaunch& l, cudaStream_t stream) {
  if (p.B == 0 || p.Hq == 0) return cudaSuccess;
  if (p.seq.cu_q != nullptr) {
    seq_plan_kernel<<<1, 1024, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const bool gs = p.gscale != kGscaleNone;
  if ((p.smooth_k || p.smooth_q || gs) && p.nsplit > 0) {
    dim3 g1(p.nsplit, p.Hq, p.B);
    if (p.D == 64) stats_kernel<64><<<g1, kThreads, 0, stream>>>(p);
    else stats_kernel<128><<<g1, kThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // The finalize pass writes the K mean (zeros without smoothing) and the maxima.
  if (p.k_mean != nullptr || gs || p.smooth_q) {
    dim3 g2(p.Hq, p.B);
    if (p.D == 64) finalize_kernel<64><<<g2, 64, 0, stream>>>(p);
    else finalize_kernel<128><<<g2, 128, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int tiles = l.tiles_q > l.tiles_k ? l.tiles_q : l.tiles_k;
  if (tiles == 0) return cudaSuccess;
  dim3 g3(2 * tiles, p.Hq, p.B);
  if (gs) {
    if (p.D == 64) quant_kernel<64, false, true><<<g3, kThreads, 0, stream>>>(p);
    else quant_kernel<128, false, true><<<g3, kThreads, 0, stream>>>(p);
  } else {
    if (p.D == 64) quant_kernel<64, false, false><<<g3, kThreads, 0, stream>>>(p);
    else quant_kernel<128, false, false><<<g3, kThreads, 0, stream>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || l.tiles_k == 0) return e;
  dim3 g4(l.tiles_k, p.Hkv, p.B);
  if (gs) {
    if (p.D == 64) quant_kernel<64, true, true><<<g4, kThreads, 0, stream>>>(p);
    else quant_kernel<128, true, true><<<g4, kThreads, 0, stream>>>(p);
  } else {
    if (p.D == 64) quant_kernel<64, true, false><<<g4, kThreads, 0, stream>>>(p);
    else quant_kernel<128, true, false><<<g4, kThreads, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace sage
