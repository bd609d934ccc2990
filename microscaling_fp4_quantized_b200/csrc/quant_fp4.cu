// Quantization kernels of the FP4 attention forward (sm_100a):
//   seq_plan_kernel   : packed sequences only -- checks the sequence table and prefix-sums
//                       the padded (multiple-of-128) lengths
//   quant_pass_kernel : one launch over jobs of up to four kinds -- K tiles, Q tiles, V^T
//                       tiles and statistics chunks; run twice, before and after finalize
//     statistics job  : per 512-token chunk: binary64 column sums of K; with a second-level
//                       scale also the column maxima / minima of K and the maxima of |Q|, |V|
//     Q / K tile job  : Q or K - mean, one 128-row tile -> packed E2M1 codes + UE4M3 scale tile
//     V^T tile job    : one 128-token tile of V, transposed -> packed codes + scale tile
//   finalize_kernel   : per (sequence, head): the K mean and the second-level maxima
//   stats_kernel      : the statistics jobs alone (the 8-bit path)
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
// The passes are HBM-bound: coalesced 16- or 32-byte loads, tiles of 128 tokens, scale
// factors staged in shared memory and written out as 16-byte chunks; V^T is stored
// tile-major (one contiguous D x 64-byte block per tile).
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
template <int D, bool EXTREMES>
__device__ __forceinline__ void chunk_channel_stats(const void* src, const Strides& st, int dtype, int b, int h,
                                                    int64_t tok0, int n0, int n1,
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
      if (EXTREMES) {
        mx[e] = fmaxf(mx[e], x[e]);
        mn[e] = fminf(mn[e], x[e]);
      }
    }
  }
  __syncthreads();  // the reduction buffers may still be read by a previous call
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    red[rg][c * 8 + e] = acc[e];
    if (EXTREMES) {
      redmx[rg][c * 8 + e] = mx[e];
      redmn[rg][c * 8 + e] = mn[e];
    }
  }
  __syncthreads();
  for (int d = t; d < D; d += kThreads) {
    double sacc = 0.0;
    float a = -INFINITY, z = INFINITY;
    for (int g = 0; g < RG; ++g) {
      sacc += red[g][d];
      if (EXTREMES) {
        a = fmaxf(a, redmx[g][d]);
        z = fminf(z, redmn[g][d]);
      }
    }
    sum[d] = sacc;
    if (EXTREMES) {
      cmax[d] = a;
      cmin[d] = z;
    }
  }
}

// Shared memory of one quantization job; the jobs of a pass share one buffer.
template <int D>
struct QuantSmem {
  static constexpr int kCPR = D / 8;                 // 16-byte chunks per row
  static constexpr int kRG = kThreads / kCPR;        // row groups of the statistics job
  static constexpr int kVRowBytes = (D + 8) * 2;     // padded V tile row (16-byte multiple)
  static constexpr int kStats = kRG * D * 8 + 2 * kRG * D * 4 + (kThreads / 32) * 4;
  static constexpr int kVt = 128 * kVRowBytes + 1024;
  static constexpr int kRows = (D / 64) * 512;  // the Q / K tile's scale tile
};

// Statistics job (split, h, b): chunk `split` of sequence b, head h.
//   K (h < Hkv, K smoothing or a second-level scale): ksum[bh, split, d] = sum over the
//     chunk's tokens, binary64; with a second-level scale also kmax / kmin per channel.
//   V (h < Hkv, 8-bit path): the same statistics of V into vsum / vmax / vmin.
//   Q (h < Hq, Q smoothing): the same statistics of Q into qsum / qmax / qmin.
//   Q without smoothing (h < Hq) and V (h < Hkv), second-level scale only: max |x| over
//   the chunk.
template <int D>
__device__ __forceinline__ void stats_job(const QuantParams& p, int split, int h, int b, uint8_t* smem) {
  using S = QuantSmem<D>;
  constexpr int CPR = S::kCPR, RG = S::kRG;
  auto red = reinterpret_cast<double (*)[D]>(smem);
  auto redmx = reinterpret_cast<float (*)[D]>(smem + RG * D * 8);
  auto redmn = reinterpret_cast<float (*)[D]>(smem + RG * D * 12);
  float* redw = reinterpret_cast<float*>(smem + RG * D * 16);
  const int t = threadIdx.x, c = t % CPR, rg = t / CPR;
  const SeqInfo si = seq_info(p.seq, b);
  const bool gs = p.gscale != kGscaleNone;
  if (gs && p.gscale == kGscaleTensor && split == 0 && h == 0 && b == 0 && t < 3) p.amax[t * p.amax_stride] = 0.0f;
  const int n0 = split * kChunk;

  if (h < p.Hkv && (p.smooth_k || gs) && n0 < si.len_k) {
    const size_t base = (static_cast<size_t>(b * p.Hkv + h) * p.nsplit + split) * D;
    if (!SAGE_IN_BOUNDS(base + D <= p.lim.stat_el, p.err, nullptr)) return;
    if (gs)
      chunk_channel_stats<D, true>(p.k, p.sk, p.dtype, b, h, si.tok_k, n0, min(n0 + kChunk, si.len_k), p.ksum + base,
                                   p.kmax + base, p.kmin + base, red, redmx, redmn, p.lim.k_el, p.err);
    else
      chunk_channel_stats<D, false>(p.k, p.sk, p.dtype, b, h, si.tok_k, n0, min(n0 + kChunk, si.len_k), p.ksum + base,
                                    nullptr, nullptr, red, redmx, redmn, p.lim.k_el, p.err);
  }
  if (h < p.Hkv && p.bits8 && n0 < si.len_k) {
    const size_t base = (static_cast<size_t>(b * p.Hkv + h) * p.nsplit + split) * D;
    if (!SAGE_IN_BOUNDS(base + D <= p.lim.stat_el, p.err, nullptr)) return;
    chunk_channel_stats<D, true>(p.v, p.sv, p.dtype, b, h, si.tok_k, n0, min(n0 + kChunk, si.len_k), p.vsum + base,
                                 p.vmax + base, p.vmin + base, red, redmx, redmn, p.lim.v_el, p.err);
  }
  if (h < p.Hq && p.smooth_q && n0 < si.len_q) {
    const size_t base = (static_cast<size_t>(b * p.Hq + h) * p.nsplit + split) * D;
    if (!SAGE_IN_BOUNDS(base + D <= p.lim.qstat_el, p.err, nullptr)) return;
    if (gs)
      chunk_channel_stats<D, true>(p.q, p.sq, p.dtype, b, h, si.tok_q, n0, min(n0 + kChunk, si.len_q), p.qsum + base,
                                   p.qmax + base, p.qmin + base, red, redmx, redmn, p.lim.q_el, p.err);
    else
      chunk_channel_stats<D, false>(p.q, p.sq, p.dtype, b, h, si.tok_q, n0, min(n0 + kChunk, si.len_q), p.qsum + base,
                                    nullptr, nullptr, red, redmx, redmn, p.lim.q_el, p.err);
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

// grid (nsplit, Hq, B): the statistics jobs alone (the 8-bit path's first launch).
template <int D>
__global__ void __launch_bounds__(kThreads, 4) stats_kernel(QuantParams p) {
  __shared__ __align__(16) uint8_t smem[QuantSmem<D>::kStats];
  if (seq_table_bad(p.seq)) return;
  stats_job<D>(p, blockIdx.x, blockIdx.y, blockIdx.z, smem);
}

// Programmatic dependent launch: wait for the previous kernel of the stream (a no-op when
// the launch did not overlap it), and let the next one start launching.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// grid (Hq, B), 4 D threads: the K mean of (sequence b, key/value head h), the Q mean of
// query head h (Q smoothing), and the second-level maxima of Q (or Q - mean) for head h
// and of K - mean and V for head h. A channel's mean is its ns chunk sums added in chunk
// order, a quarter of the chunks per thread, then the four quarters in order.
template <int D>
__global__ void __launch_bounds__(4 * D) finalize_kernel(QuantParams p) {
  __shared__ float redw[4 * D / 32];
  __shared__ double part[4][D];
  grid_dependency_wait();
  grid_dependents_launch();  // pass B launches while this small grid runs
  if (seq_table_bad(p.seq)) return;
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x, d = t % D, qp = t / D;
  const bool lead = qp == 0;  // the thread that writes channel d
  const SeqInfo si = seq_info(p.seq, b);
  const bool gs = p.gscale != kGscaleNone;
  auto chunk_mean = [&](const double* src, int ns, int len) -> float {
    const int g0 = ns * qp / 4, g1 = ns * (qp + 1) / 4;
    double s = 0.0;
    for (int g = g0; g < g1; ++g) s += src[static_cast<size_t>(g) * D];
    part[qp][d] = s;
    __syncthreads();
    const double tot = ((part[0][d] + part[1][d]) + part[2][d]) + part[3][d];
    __syncthreads();
    return static_cast<float>(tot / static_cast<double>(len));
  };
  if (h < p.Hkv) {
    const int ns = (si.len_k + kChunk - 1) / kChunk;
    const size_t base = static_cast<size_t>(b * p.Hkv + h) * p.nsplit * D + d;
    float mu = 0.0f;
    if (p.smooth_k && si.len_k > 0) mu = chunk_mean(p.ksum + base, ns, si.len_k);
    if (lead && SAGE_IN_BOUNDS(static_cast<size_t>(b * p.Hkv + h) * D + d < p.lim.k_mean_el, p.err, nullptr))
      p.k_mean[static_cast<size_t>(b * p.Hkv + h) * D + d] = mu;
    if (p.bits8 && lead) {
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
      float ak = 0.0f, av = 0.0f;
      if (lead && si.len_k > 0) {
        float mx = -INFINITY, mn = INFINITY;
        for (int g = 0; g < ns; ++g) {
          mx = fmaxf(mx, p.kmax[base + static_cast<size_t>(g) * D]);
          mn = fminf(mn, p.kmin[base + static_cast<size_t>(g) * D]);
        }
        // Rounding is monotone, so max |fp32(k - mu)| over the tokens is reached at the
        // channel's largest or smallest k.
        ak = fmaxf(fabsf(__fsub_rn(mx, mu)), fabsf(__fsub_rn(mn, mu)));
      }
      ak = block_max(ak, redw);
      for (int g = t; g < ns; g += blockDim.x) av = fmaxf(av, p.vamax[static_cast<size_t>(b * p.Hkv + h) * p.nsplit + g]);
      av = block_max(av, redw);
      if (t == 0) {
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
      if (si.len_q > 0) mu = chunk_mean(p.qsum + base, ns, si.len_q);
      if (lead && SAGE_IN_BOUNDS(static_cast<size_t>(b * p.Hq + h) * D + d < p.lim.q_mean_el, p.err, nullptr))
        p.q_mean[static_cast<size_t>(b * p.Hq + h) * D + d] = mu;
      if (gs && si.len_q > 0 && lead) {
        float mx = -INFINITY, mn = INFINITY;
        for (int g = 0; g < ns; ++g) {
          mx = fmaxf(mx, p.qmax[base + static_cast<size_t>(g) * D]);
          mn = fminf(mn, p.qmin[base + static_cast<size_t>(g) * D]);
        }
        aq = fmaxf(fabsf(__fsub_rn(mx, mu)), fabsf(__fsub_rn(mn, mu)));
      }
    } else {
      for (int g = t; g < ns; g += blockDim.x) aq = fmaxf(aq, p.qamax[static_cast<size_t>(b * p.Hq + h) * p.nsplit + g]);
    }
    if (gs) {
      aq = block_max(aq, redw);
      if (t == 0) amax_store(p.amax + (p.gscale == kGscaleHead ? b * p.Hq + h : 0), p.gscale, aq);
    }
  }
}

// 32 bytes at p: one 256-bit load when p is 32-byte aligned (vec32), else two 128-bit ones.
__device__ __forceinline__ void ld_nc_32(const char* p, bool vec32, uint32_t (&r)[8]) {
  if (vec32) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "l"(p));
  } else {
    const uint4 a = ld_nc_16(p), b = ld_nc_16(p + 16);
    r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
    r[4] = b.x; r[5] = b.y; r[6] = b.z; r[7] = b.w;
  }
}

// 16 bf16 / fp16 values from 8 words, as floats in order.
__device__ __forceinline__ void unpack16(const uint32_t (&w)[8], int dtype, float (&x)[16]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (dtype == kDtypeBF16) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      x[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xFFFFu)));
      x[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
    }
  }
}

__device__ __forceinline__ float absmax16(const float (&x)[16]) {
  float a = max3(fabsf(x[0]), fabsf(x[1]), fabsf(x[2]));
#pragma unroll
  for (int i = 3; i < 15; i += 2) a = max3(a, fabsf(x[i]), fabsf(x[i + 1]));
  return fmaxf(a, fabsf(x[15]));
}

// Codes of 8 values (x[O .. O + 7]) against a decoded scale s (s == 0 -> zero codes);
// element O lands in the low nibble of the low byte. Each code is E2M1(RN(x / s)) with
// RN(x / s) formed as div_fma does, two lanes per instruction and with the reciprocal
// negated: q' = RN(x * -r) = -RN(x r); e = RN(x + q' s) = x - RN(x r) s, div_fma's exact
// remainder; RN(e * -r + q') = -RN(e r + RN(x r)). Rounding to nearest is symmetric, so
// every lane holds exactly -div_fma(x, s, r) -- and, for x = +-0 or a product that
// underflows, the zero of the sign opposite to x's, i.e. minus div_fma's copysign result.
// E2M1 rounding is symmetric too, so the codes come out with every sign bit inverted,
// which one XOR puts back. (Checked on the CPU for every E4M3 divisor and every finite
// quotient tried, +-0 and underflowing products included: tests/div_identity.c.)
template <int O, int N>
__device__ __forceinline__ uint32_t encode8_neg(const float (&x)[N], float s) {
  if (s == 0.0f) return 0u;
  const float nr = -__frcp_rn(s);
  const float2 nr2 = make_float2(nr, nr), s2 = make_float2(s, s);
  float y[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 xv = make_float2(x[O + 2 * i], x[O + 2 * i + 1]);
    const float2 nq = mul2(xv, nr2);
    const float2 e = fma2(nq, s2, xv);
    const float2 r = fma2(e, nr2, nq);
    y[2 * i] = r.x;
    y[2 * i + 1] = r.y;
  }
  return f32x8_to_e2m1(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]) ^ 0x88888888u;
}

// Q or K - mean (job 0 / 1), one 128-row tile: packed E2M1 codes [row][D/2] and the
// UE4M3 scale tile of the block-scaled MMA. Thread t owns the 16-element block t % (D/16)
// of rows t / (D/16) + (256 / (D/16)) i, and loads each as one 32-byte piece; all of its
// loads are issued before any is used.
template <int D, bool GS>
__device__ __forceinline__ void rows_job(const QuantParams& p, int job, int tile, int h, int b, bool vec32,
                                         uint8_t* smem) {
  constexpr int BPR = D / 16;               // 16-element blocks per row
  constexpr int kRowStep = kThreads / BPR;  // rows per sweep of the CTA
  constexpr int kIter = 128 / kRowStep;
  constexpr int kSfBytesQK = (D / 64) * 512;
  const int H = job == 0 ? p.Hq : p.Hkv;
  if (h >= H) return;
  const SeqInfo si = seq_info(p.seq, b);
  const int len = job == 0 ? si.len_q : si.len_k;
  const int ntile = (len + 127) >> 7;
  if (tile >= ntile) return;
  const int t = threadIdx.x;
  const int prow = job == 0 ? si.prow_q : si.prow_k;
  const int64_t tok0 = static_cast<int64_t>(job == 0 ? si.tok_q : si.tok_k) + tile * 128;
  const int64_t row0 = static_cast<int64_t>(H) * prow + static_cast<int64_t>(h) * ntile * 128 + tile * 128;
  const int64_t T = row0 >> 7;  // scale-factor tile index
  const int rows = min(128, len - tile * 128);
  float g = 1.0f;
  if (GS) g = second_level_scale(p.amax[job * p.amax_stride + (p.gscale == kGscaleHead ? b * H + h : 0)]);
  const double cg = GS ? recip_d(g) : 1.0;  // x / g = div_by(x, cg)

  uint8_t* sfbuf = smem;  // kSfBytesQK: every byte is written below
  const bool smooth = (job == 1) ? p.smooth_k != 0 : p.smooth_q != 0;
  const void* src = job == 0 ? p.q : p.k;
  const Strides& st = job == 0 ? p.sq : p.sk;
  const uint64_t lim_el = job == 0 ? p.lim.q_el : p.lim.k_el;
  (void)lim_el;  // read by the bounds-checked build only
  uint8_t* dst = (job == 0 ? p.q_fp4 : p.k_fp4) + row0 * (D / 2);
  const int c = t % BPR, rl0 = t / BPR;
  const int64_t off0 = static_cast<int64_t>(b) * st.b + static_cast<int64_t>(h) * st.h + (tok0 + rl0) * st.n + 16 * c;
  const int64_t step = static_cast<int64_t>(kRowStep) * st.n;
  uint32_t raw[kIter][8];
#pragma unroll
  for (int it = 0; it < kIter; ++it) {
    const int64_t off = off0 + it * step;
    const bool ok = rl0 + it * kRowStep < rows &&
                    SAGE_IN_BOUNDS(off >= 0 && static_cast<uint64_t>(off) + 16 <= lim_el, p.err, nullptr);
    if (ok) {
      ld_nc_32(static_cast<const char*>(src) + off * 2, vec32, raw[it]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) raw[it][i] = 0u;
    }
  }
  float2 nm[8];  // -mean of the block's channels, two per pair
  if (smooth) {
    const float4* mean = reinterpret_cast<const float4*>((job == 1 ? p.k_mean : p.q_mean) +
                                                         static_cast<size_t>(b * H + h) * D + 16 * c);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 m = mean[i];
      nm[2 * i] = make_float2(-m.x, -m.y);
      nm[2 * i + 1] = make_float2(-m.z, -m.w);
    }
  }
#pragma unroll
  for (int it = 0; it < kIter; ++it) {
    const int rl = rl0 + it * kRowStep;
    float x[16];
    unpack16(raw[it], p.dtype, x);
    if (rl < rows && smooth) {
      // x - mean as x + (-mean): the same binary32 sum, signed zeros included.
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 r = add2(make_float2(x[2 * i], x[2 * i + 1]), nm[i]);
        x[2 * i] = r.x;
        x[2 * i + 1] = r.y;
      }
    }
    if (job == 1 && p.smooth_q) {
      // Q smoothing bias of this key for every query head of the group:
      // mu_q . (k - mu_k), over the D/16 lanes that hold the row (zero for padding).
      const int Gq = p.Hq / p.Hkv;
      for (int gi = 0; gi < Gq; ++gi) {
        const int hq = h * Gq + gi;
        const float4* mq = reinterpret_cast<const float4*>(p.q_mean + static_cast<size_t>(b * p.Hq + hq) * D + c * 16);
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 m = mq[j];
          acc = fmaf(x[4 * j], m.x, acc);
          acc = fmaf(x[4 * j + 1], m.y, acc);
          acc = fmaf(x[4 * j + 2], m.z, acc);
          acc = fmaf(x[4 * j + 3], m.w, acc);
        }
#pragma unroll
        for (int o = BPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (c == 0) {
          if (GS) {
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
          const uint32_t b0 = static_cast<uint32_t>(__bfloat16_as_ushort(hi)) |
                              (static_cast<uint32_t>(__bfloat16_as_ushort(mid)) << 16);
          const uint32_t b1 = static_cast<uint32_t>(__bfloat16_as_ushort(lo));
          uint8_t* tb = p.qk_bias + (static_cast<int64_t>(p.Hq) * prow + static_cast<int64_t>(hq) * ntile * 128 +
                                     tile * 128) * 32;
          uint8_t* row = tb + (rl >> 3) * 256 + (rl & 7) * 16;
          if (SAGE_IN_BOUNDS(static_cast<uint64_t>(row + 144 - p.qk_bias) <= p.lim.qk_bias, p.err, nullptr)) {
            *reinterpret_cast<uint4*>(row) = make_uint4(b0, b1, 0u, 0u);
            *reinterpret_cast<uint4*>(row + 128) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
    }
    if (GS && rl < rows) {
#pragma unroll
      for (int e = 0; e < 16; ++e) x[e] = div_by(x[e], cg);
    }
    const uint32_t sb = block_scale_byte(absmax16(x));
    const float s = e4m3_to_f32(sb);
    const uint32_t c0 = encode8_neg<0>(x, s), c1 = encode8_neg<8>(x, s);
    if (SAGE_IN_BOUNDS(static_cast<uint64_t>(row0 + rl) * (D / 2) + c * 8 + 8 <= (job == 0 ? p.lim.q_fp4 : p.lim.k_fp4),
                       p.err, nullptr))
      *reinterpret_cast<uint2*>(dst + static_cast<size_t>(rl) * (D / 2) + c * 8) = make_uint2(c0, c1);
    const int col = c * 16;
    sfbuf[(col / 64) * 512 + (rl % 32) * 16 + (rl / 32) * 4 + (col % 64) / 16] = static_cast<uint8_t>(sb);
  }
  __syncthreads();
  uint8_t* sf_out = (job == 0 ? p.q_sf : p.k_sf) + T * kSfBytesQK;
  if (SAGE_IN_BOUNDS(static_cast<uint64_t>(T + 1) * kSfBytesQK <= (job == 0 ? p.lim.q_sf : p.lim.k_sf), p.err, nullptr))
    for (int i = t; i < kSfBytesQK / 16; i += kThreads)
      reinterpret_cast<uint4*>(sf_out)[i] = reinterpret_cast<const uint4*>(sfbuf)[i];
}

// V^T, one 128-token tile: tokens become the contiguous (contraction) dimension. The tile
// is staged in shared memory; thread t then owns the channel pair (2 (t % (D/2)),
// 2 (t % (D/2)) + 1) over tokens [G (t / (D/2)), G (t / (D/2)) + G), G = D / 4, reading one
// 32-bit word per token, and stores each channel's G/2 code bytes straight to the
// tile-major V^T block (one contiguous D x 64-byte block per tile).
template <int D, bool GS>
__device__ __forceinline__ void vt_job(const QuantParams& p, int tile, int h, int b, uint8_t* smem) {
  using S = QuantSmem<D>;
  constexpr int CPR = S::kCPR, kVRowBytes = S::kVRowBytes;
  constexpr int NP = D / 2;                 // channel pairs
  constexpr int G = 128 / (kThreads / NP);  // tokens per thread: 32 (D = 128) or 16 (D = 64)
  constexpr int NB = G / 16;                // 16-token blocks per thread
  if (h >= p.Hkv) return;
  const SeqInfo si = seq_info(p.seq, b);
  const int ntile = (si.len_k + 127) >> 7;
  if (tile >= ntile) return;
  const int t = threadIdx.x;
  const int64_t tok0 = static_cast<int64_t>(si.tok_k) + tile * 128;
  const int64_t row0 = static_cast<int64_t>(p.Hkv) * si.prow_k + static_cast<int64_t>(h) * ntile * 128 + tile * 128;
  const int64_t T = row0 >> 7;
  const int rows = min(128, si.len_k - tile * 128);
  float g = 1.0f;
  if (GS) g = second_level_scale(p.amax[2 * p.amax_stride + (p.gscale == kGscaleHead ? b * p.Hkv + h : 0)]);
  const double cg = GS ? recip_d(g) : 1.0;

  uint8_t* vtile = smem;                     // 128 x kVRowBytes
  uint8_t* sfbuf = smem + 128 * kVRowBytes;  // 1024
  if constexpr (D == 64)  // half of each 16-byte scale group is unused at D = 64
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
  const int pr = t % NP, grp = t / NP;
  const int d0 = 2 * pr;
  uint32_t code[2][NB * 2];  // per channel: NB blocks x 2 words
#pragma unroll
  for (int kb = 0; kb < NB; ++kb) {
    const int tb = grp * NB + kb;  // 16-token block within the tile
    float x0[16], x1[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(vtile + (tb * 16 + i) * kVRowBytes + pr * 4);
      if (p.dtype == kDtypeBF16) {
        x0[i] = __uint_as_float(w << 16);
        x1[i] = __uint_as_float(w & 0xFFFF0000u);
      } else {
        x0[i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
        x1[i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
      }
      if (GS) {
        x0[i] = div_by(x0[i], cg);
        x1[i] = div_by(x1[i], cg);
      }
    }
    const uint32_t sb0 = block_scale_byte(absmax16(x0)), sb1 = block_scale_byte(absmax16(x1));
    const float s0 = e4m3_to_f32(sb0), s1 = e4m3_to_f32(sb1);
    code[0][2 * kb] = encode8_neg<0>(x0, s0);
    code[0][2 * kb + 1] = encode8_neg<8>(x0, s0);
    code[1][2 * kb] = encode8_neg<0>(x1, s1);
    code[1][2 * kb + 1] = encode8_neg<8>(x1, s1);
    sfbuf[(tb / 4) * 512 + (d0 % 32) * 16 + (d0 / 32) * 4 + (tb % 4)] = static_cast<uint8_t>(sb0);
    sfbuf[(tb / 4) * 512 + ((d0 + 1) % 32) * 16 + ((d0 + 1) / 32) * 4 + (tb % 4)] = static_cast<uint8_t>(sb1);
  }
  uint8_t* vt = p.vt_fp4 + T * (D * 64);
  if (SAGE_IN_BOUNDS(static_cast<uint64_t>(T + 1) * (D * 64) <= p.lim.vt_fp4, p.err, nullptr)) {
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      uint8_t* dst = vt + (d0 + ch) * 64 + grp * (G / 2);
      if constexpr (NB == 2)
        *reinterpret_cast<uint4*>(dst) = make_uint4(code[ch][0], code[ch][1], code[ch][2], code[ch][3]);
      else
        *reinterpret_cast<uint2*>(dst) = make_uint2(code[ch][0], code[ch][1]);
    }
  }
  __syncthreads();
  uint8_t* sf_out = p.vt_sf + T * 1024;
  if (SAGE_IN_BOUNDS(static_cast<uint64_t>(T + 1) * 1024 <= p.lim.vt_sf, p.err, nullptr))
    for (int i = t; i < 1024 / 16; i += kThreads)
      reinterpret_cast<uint4*>(sf_out)[i] = reinterpret_cast<const uint4*>(sfbuf)[i];
}

// Job kinds of a pass (bits of the kernel's KINDS mask, which compiles only those).
enum : int { kKindRowsK = 1, kKindRowsQ = 2, kKindVt = 4, kKindStats = 8 };

// One launch of the FP4 quantizer: a 1-D grid over the jobs of up to four kinds, in this
// order: K tiles (last (sequence, head, tile) first), Q tiles, V^T tiles, statistics
// chunks. The first pass runs what does not need the finalize step's results (the
// statistics, and Q and V^T when no mean or maximum scales them); the second runs the
// rest. Taking K backwards in the second pass starts it on the keys that the first pass's
// statistics read last, which may still be in L2.
struct QuantPass {
  int n_k, n_q, n_v, n_stats;  // jobs of each kind
  int tiles_q, tiles_k;        // 128-token tiles per (sequence, head)
  int vec32;                   // Q and K rows can be read as aligned 32-byte pieces
};

template <int D, int KINDS>
struct PassSmem {
  using S = QuantSmem<D>;
  static constexpr int a = (KINDS & kKindStats) ? S::kStats : 0;
  static constexpr int b = (KINDS & kKindVt) ? S::kVt : 0;
  static constexpr int c = (KINDS & (kKindRowsK | kKindRowsQ)) ? S::kRows : 0;
  static constexpr int kBytes = a > b ? (a > c ? a : c) : (b > c ? b : c);
};

// CTAs per SM: four for the mixed passes (more resident warps hide the statistics' and the
// V^T jobs' latency), three for the K-only pass (room for its loads in registers: measured
// 57 against 65 us for the long workload's keys).
template <int KINDS>
constexpr int pass_min_blocks() { return KINDS == kKindRowsK ? 3 : 4; }

template <int D, bool GS, int KINDS>
__global__ void __launch_bounds__(kThreads, pass_min_blocks<KINDS>()) quant_pass_kernel(QuantParams p, QuantPass q) {
  __shared__ __align__(16) uint8_t smem[PassSmem<D, KINDS>::kBytes];
  grid_dependency_wait();  // the passes never let their successor start early: the next
                           // kernel's CTAs would hold SM slots the pass still uses
  if (seq_table_bad(p.seq)) return;
  if constexpr (KINDS == (kKindRowsQ | kKindVt | kKindStats)) {
    // Pass A of a problem without Q smoothing or a second-level scale, head-major: per
    // (sequence, query head) its statistics chunks, its Q tiles, then its V^T tiles (none
    // past the key/value heads), so the statistics jobs (binary64 sums) are spread over
    // the pass instead of forming its tail.
    const int U = p.nsplit + q.tiles_q + q.tiles_k;
    const int grp = blockIdx.x / U, r = blockIdx.x % U;
    const int h = grp % p.Hq, b = grp / p.Hq;
    if (r < p.nsplit) stats_job<D>(p, r, h, b, smem);
    else if (r < p.nsplit + q.tiles_q) rows_job<D, GS>(p, 0, r - p.nsplit, h, b, q.vec32 != 0, smem);
    else vt_job<D, GS>(p, r - p.nsplit - q.tiles_q, h, b, smem);
    return;
  }
  int i = blockIdx.x;
  if constexpr ((KINDS & kKindRowsK) != 0) {
    if (i < q.n_k) {
      i = q.n_k - 1 - i;
      rows_job<D, GS>(p, 1, i % q.tiles_k, (i / q.tiles_k) % p.Hkv, i / (q.tiles_k * p.Hkv), q.vec32 != 0, smem);
      return;
    }
  }
  i -= q.n_k;
  if constexpr ((KINDS & kKindRowsQ) != 0) {
    if (i < q.n_q) {
      rows_job<D, GS>(p, 0, i % q.tiles_q, (i / q.tiles_q) % p.Hq, i / (q.tiles_q * p.Hq), q.vec32 != 0, smem);
      return;
    }
  }
  i -= q.n_q;
  if constexpr ((KINDS & kKindVt) != 0) {
    if (i < q.n_v) {
      vt_job<D, GS>(p, i % q.tiles_k, (i / q.tiles_k) % p.Hkv, i / (q.tiles_k * p.Hkv), smem);
      return;
    }
  }
  i -= q.n_v;
  if constexpr ((KINDS & kKindStats) != 0) {
    if (i < q.n_stats) stats_job<D>(p, i % p.nsplit, (i / p.nsplit) % p.Hq, i / (p.nsplit * p.Hq), smem);
  }
}

// ------------------------------------------------------------- 8-bit path ----
// Two launches: VJOB = false, grid (2 * tiles, Hq, B),
// x = 2 * tile + job: jobs 0 and 1 turn a 128-row tile of Q or K - mean into symmetric
// INT8 with one scale s = fp32(absmax / 127) for the tile and codes
// clamp(RNE(fp32(x / s)), -127, 127). VJOB = true, grid (key tiles, Hkv, B): a 128-token
// tile of V becomes E4M3 codes fp32(v / s_d) with the channel scales of the finalize
// pass, transposed (tokens contiguous) and stored tile-major [key tiles, D, 128].
// Only the V^T launch needs the large shared-memory tile. Bounded to 4 CTAs per SM
// (0.48 -> 0.46 ms for the long workload's 8-bit quantization, identical output bytes).
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

// Host-side test of the 32-byte read of a row block: base and every stride (bytes) are
// multiples of 32.
static bool rows_vec32(const void* base, const Strides& st) {
  const uint64_t a = reinterpret_cast<uint64_t>(base);
  return a % 32 == 0 && (st.b * 2) % 32 == 0 && (st.h * 2) % 32 == 0 && (st.n * 2) % 32 == 0;
}

// A launch that may start while the previous kernel of the stream drains (programmatic
// dependent launch); the kernel waits for that kernel's results before it reads anything.
template <typename... Args>
static cudaError_t launch_ex(void (*kernel)(Args...), dim3 grid, dim3 block, bool dependent, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int D, bool GS, int KINDS>
static cudaError_t launch_kinds(const QuantParams& p, const QuantPass& q, unsigned n, bool dependent,
                                cudaStream_t stream) {
  return launch_ex(quant_pass_kernel<D, GS, KINDS>, dim3(n), dim3(kThreads), dependent, stream, p, q);
}

static cudaError_t launch_finalize(const QuantParams& p, bool dependent, cudaStream_t stream) {
  if (p.D == 64) return launch_ex(finalize_kernel<64>, dim3(p.Hq, p.B), dim3(4 * 64), dependent, stream, p);
  return launch_ex(finalize_kernel<128>, dim3(p.Hq, p.B), dim3(4 * 128), dependent, stream, p);
}

// The instance compiled for the job kinds present: the common passes get their own
// (pass A of a plain problem: Q, V^T, statistics; pass B: K alone), anything else the
// instance with all four.
template <int D, bool GS>
static cudaError_t launch_pass_d(const QuantParams& p, const QuantPass& q, bool dependent, cudaStream_t stream) {
  const long long n = static_cast<long long>(q.n_k) + q.n_q + q.n_v + q.n_stats;
  if (n == 0) return cudaSuccess;
  if (n > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  const int kinds = (q.n_k ? kKindRowsK : 0) | (q.n_q ? kKindRowsQ : 0) | (q.n_v ? kKindVt : 0) |
                    (q.n_stats ? kKindStats : 0);
  if (kinds == kKindRowsK) return launch_kinds<D, GS, kKindRowsK>(p, q, static_cast<unsigned>(n), dependent, stream);
  if (kinds == (kKindRowsQ | kKindVt | kKindStats)) {
    const long long hm = static_cast<long long>(p.B) * p.Hq * (p.nsplit + q.tiles_q + q.tiles_k);  // head-major grid
    if (hm > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    return launch_kinds<D, GS, kKindRowsQ | kKindVt | kKindStats>(p, q, static_cast<unsigned>(hm), dependent, stream);
  }
  return launch_kinds<D, GS, kKindRowsK | kKindRowsQ | kKindVt | kKindStats>(p, q, static_cast<unsigned>(n), dependent,
                                                                              stream);
}

static cudaError_t launch_pass(const QuantParams& p, const QuantPass& q, bool gs, bool dependent, cudaStream_t stream) {
  if (p.D == 64)
    return gs ? launch_pass_d<64, true>(p, q, dependent, stream) : launch_pass_d<64, false>(p, q, dependent, stream);
  return gs ? launch_pass_d<128, true>(p, q, dependent, stream) : launch_pass_d<128, false>(p, q, dependent, stream);
}

// Pass A: the statistics, plus Q and V^T when neither a mean nor a second-level scale
// of theirs is needed; finalize; pass B: K and whatever pass A left.
cudaError_t launch_quantize(const QuantParams& p, const QuantLaunch& l, cudaStream_t stream) {
  if (p.B == 0 || p.Hq == 0) return cudaSuccess;
  if (p.seq.cu_q != nullptr) {
    seq_plan_kernel<<<1, 1024, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const bool gs = p.gscale != kGscaleNone;
  const bool stats = (p.smooth_k || p.smooth_q || gs) && p.nsplit > 0;
  const bool q_early = !p.smooth_q && !gs, v_early = !gs;
  QuantPass a{}, b{};
  a.tiles_q = b.tiles_q = l.tiles_q;
  a.tiles_k = b.tiles_k = l.tiles_k;
  a.vec32 = b.vec32 = rows_vec32(p.q, p.sq) && rows_vec32(p.k, p.sk) ? 1 : 0;
  const int nq = l.tiles_q * p.Hq * p.B, nkv = l.tiles_k * p.Hkv * p.B;
  a.n_stats = stats ? p.nsplit * p.Hq * p.B : 0;
  (q_early ? a : b).n_q = nq;
  (v_early ? a : b).n_v = nkv;
  b.n_k = nkv;
  cudaError_t e = launch_pass(p, a, gs, false, stream);
  if (e != cudaSuccess) return e;
  const bool after_a = a.n_k + a.n_q + a.n_v + a.n_stats > 0;  // a kernel of this call precedes
  // The finalize pass writes the K mean (zeros without smoothing) and the maxima.
  bool fin = false;
  if (p.k_mean != nullptr || gs || p.smooth_q) {
    e = launch_finalize(p, after_a, stream);
    if (e != cudaSuccess) return e;
    fin = true;
  }
  return launch_pass(p, b, gs, fin || after_a, stream);
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
    cudaError_t e = launch_finalize(p, false, stream);
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

}  // namespace sage
