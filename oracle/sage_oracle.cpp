// CPU oracle for microscaling-FP4 attention (SageAttention3 forward).
//
// TEST INFRASTRUCTURE ONLY. This file is the slow, plain reference that the CUDA
// path is checked against. Only the test suite, the smoke check and the benchmark's
// CPU-baseline leg may load it. It shares no code, header or table with the CUDA
// library and must never be called from the product path.
//
// Sources followed (page titles, with the section of each page):
//  * "SageAttention3: Microscaling FP4 Attention for Inference and An Exploration of
//    8-Bit Training" (arXiv 2505.11594), abstract: FP4 microscaling attention on
//    Blackwell FP4 tensor cores.
//  * "SageAttention: Accurate 8-Bit Attention for Plug-and-play Inference
//    Acceleration" (OpenReview thread), reply to Q3: the online-softmax recurrence
//    m_0 = -inf, d_0 = 0, m_i = max(m_{i-1}, a_i), d_i = d_{i-1} e^{m_{i-1}-m_i} +
//    e^{a_i-m_i}, and FlashAttention tiling (S tile rows = query tokens of a Q tile,
//    columns = key tokens of a K tile); reply to Q2: diag(l)^-1 is applied only after
//    the last key tile; reply to W1: smoothing K.
//  * The formats (E2M1 elements, one unsigned E4M3 scale per 16 elements, K smoothed
//    by its per-head channel mean over tokens, two-level scaling of P~ with a per-row
//    factor then per-16 FP8 scales, FP32-or-better accumulation) are the method's
//    statement of the microscaling FP4 path; the pages name NVFP4 ("TetraJet-v2"
//    abstract on the author page) without printing the encodings, so the encodings
//    below are the plain OCP definitions of E2M1 and E4M3.
//
// Every step that the CUDA path must reproduce bit for bit (the 16-element block
// quantizer and the K mean) is done in IEEE binary32 with round-to-nearest-even;
// everything else (dot products, softmax, accumulation) is done in binary64.
// Build with -ffp-contract=off and without -ffast-math.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---------------------------------------------------------------- formats ----

// E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no inf/NaN.
// Exponent field 0 is subnormal: magnitude = mantissa * 0.5.
double e2m1_magnitude(int c) {
  const int e = (c >> 1) & 3;
  const int m = c & 1;
  if (e == 0) return 0.5 * m;
  return std::ldexp(1.0 + 0.5 * m, e - 1);
}

double e2m1_value(uint8_t code) {
  const double v = e2m1_magnitude(code & 7);
  return (code & 8) ? -v : v;
}

// Round to nearest representable E2M1 magnitude; a tie goes to the code whose
// mantissa bit is 0; magnitudes above the largest finite value (6) saturate to it.
// The sign is kept, so a negative input that rounds to zero gives code 0x8.
uint8_t e2m1_encode(float x) {
  const double a = std::fabs(static_cast<double>(x));
  int best = 7;
  if (!(a >= 6.0)) {
    double bestd = std::numeric_limits<double>::infinity();
    for (int c = 0; c < 8; ++c) {
      const double d = std::fabs(a - e2m1_magnitude(c));
      if (d < bestd || (d == bestd && (c & 1) == 0)) {
        bestd = d;
        best = c;
      }
    }
  }
  return static_cast<uint8_t>(best | (std::signbit(x) ? 8 : 0));
}

// E4M3 (the "FN" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits;
// exponent field 0 is subnormal (m * 2^-9); 0x7F / 0xFF are NaN; largest finite 448.
double e4m3_value(uint8_t b) {
  const int e = (b >> 3) & 15;
  const int m = b & 7;
  double v;
  if (e == 15 && m == 7) {
    v = std::numeric_limits<double>::quiet_NaN();
  } else if (e == 0) {
    v = std::ldexp(static_cast<double>(m), -9);
  } else {
    v = std::ldexp(1.0 + m / 8.0, e - 7);
  }
  return (b & 0x80) ? -v : v;
}

// Round to nearest finite E4M3 value, ties to an even mantissa, saturating at 448.
uint8_t e4m3_encode(float x) {
  const double a = std::fabs(static_cast<double>(x));
  int best = 0x7E;
  if (!(a >= 448.0)) {
    double bestd = std::numeric_limits<double>::infinity();
    for (int c = 0; c <= 0x7E; ++c) {
      const double d = std::fabs(a - e4m3_value(static_cast<uint8_t>(c)));
      if (d < bestd || (d == bestd && (c & 1) == 0)) {
        bestd = d;
        best = c;
      }
    }
  }
  return static_cast<uint8_t>(best | (std::signbit(x) ? 0x80 : 0));
}

// One microscaling block of 16 values x[i * stride]:
//   a = max |x_i| (binary32); s_f = a / 6 (binary32 division);
//   scale byte = E4M3(s_f); s = its value;
//   s == 0 -> all codes 0; else code_i = E2M1(x_i / s) with x_i / s a binary32 division.
void quant_block16(const float* x, long stride, int count, uint8_t codes[16], uint8_t* sbyte) {
  float a = 0.0f;
  for (int i = 0; i < count; ++i) a = std::max(a, std::fabs(x[i * stride]));
  const float sf = a / 6.0f;
  const uint8_t sb = e4m3_encode(sf);
  const float s = static_cast<float>(e4m3_value(sb));
  for (int i = 0; i < 16; ++i) {
    if (i >= count || s == 0.0f) {
      codes[i] = 0;
    } else {
      const float q = x[i * stride] / s;
      codes[i] = e2m1_encode(q);
    }
  }
  *sbyte = sb;
}

inline void put_nibble(uint8_t* row, long idx, uint8_t code) {
  uint8_t& byte = row[idx >> 1];
  if (idx & 1) byte = static_cast<uint8_t>((byte & 0x0F) | (code << 4));
  else         byte = static_cast<uint8_t>((byte & 0xF0) | (code & 0x0F));
}

inline uint8_t get_nibble(const uint8_t* row, long idx) {
  const uint8_t byte = row[idx >> 1];
  return (idx & 1) ? (byte >> 4) : (byte & 0x0F);
}

constexpr double kTwoLevelTarget = 448.0 * 6.0;  // E4M3 max * E2M1 max

}  // namespace

extern "C" {

// ------------------------------------------------------------- element ops ----

void so_e2m1_encode(const float* x, long n, uint8_t* codes) {
  for (long i = 0; i < n; ++i) codes[i] = e2m1_encode(x[i]);
}

void so_e2m1_decode(const uint8_t* codes, long n, double* out) {
  for (long i = 0; i < n; ++i) out[i] = e2m1_value(codes[i]);
}

void so_e4m3_encode(const float* x, long n, uint8_t* bytes) {
  for (long i = 0; i < n; ++i) bytes[i] = e4m3_encode(x[i]);
}

void so_e4m3_decode(const uint8_t* bytes, long n, double* out) {
  for (long i = 0; i < n; ++i) out[i] = e4m3_value(bytes[i]);
}

// nblocks contiguous blocks of 16 floats -> 16 unpacked codes and one scale byte each.
void so_quant_block16(const float* x, long nblocks, uint8_t* codes, uint8_t* sbytes) {
  for (long b = 0; b < nblocks; ++b) quant_block16(x + 16 * b, 1, 16, codes + 16 * b, sbytes + b);
}

// --------------------------------------------------------------- K mean ----
// mean[bh, d] = fp32( (sum_n k[bh, n, d], accumulated in binary64) / N ).
void so_kmean(const float* k, long BH, long N, long D, float* mean) {
#pragma omp parallel for schedule(static)
  for (long bh = 0; bh < BH; ++bh) {
    for (long d = 0; d < D; ++d) {
      double acc = 0.0;
      for (long n = 0; n < N; ++n) acc += static_cast<double>(k[(bh * N + n) * D + d]);
      mean[bh * D + d] = static_cast<float>(acc / static_cast<double>(N));
    }
  }
}

// ------------------------------------------------------------ quantize QKV ----
// Canonical layouts (all row-major, nibble 2i in the low half of byte i):
//   q_codes, k_codes : [BH, N, D/2]     q_sf, k_sf : [BH, N, D/16]
//   vt_codes         : [BH, D, Np/2]    vt_sf      : [BH, D, Np/16]
// where Np = N rounded up to a multiple of 16 (tokens past N count as zeros).
// K is smoothed as k' = fp32(k - mean) when smooth_k != 0; kmean_in (nullable)
// supplies the mean instead of computing it; kmean_out (nullable) receives it.
void so_quantize_qkv(const float* q, const float* k, const float* v, long BH, long N, long D,
                     int smooth_k, const float* kmean_in, uint8_t* q_codes, uint8_t* q_sf,
                     uint8_t* k_codes, uint8_t* k_sf, uint8_t* vt_codes, uint8_t* vt_sf,
                     float* kmean_out) {
  const long Np = (N + 15) / 16 * 16;
  std::vector<float> mean(static_cast<size_t>(BH * D), 0.0f);
  if (smooth_k) {
    if (kmean_in) std::memcpy(mean.data(), kmean_in, sizeof(float) * BH * D);
    else so_kmean(k, BH, N, D, mean.data());
  }
  if (kmean_out) std::memcpy(kmean_out, mean.data(), sizeof(float) * BH * D);

  const long nb_d = D / 16;
#pragma omp parallel for schedule(static)
  for (long row = 0; row < BH * N; ++row) {
    const long bh = row / N;
    float kk[16];
    uint8_t codes[16];
    for (long blk = 0; blk < nb_d; ++blk) {
      const float* qx = q + row * D + blk * 16;
      quant_block16(qx, 1, 16, codes, &q_sf[row * nb_d + blk]);
      for (int i = 0; i < 16; ++i) put_nibble(q_codes + row * (D / 2), blk * 16 + i, codes[i]);

      const float* kx = k + row * D + blk * 16;
      for (int i = 0; i < 16; ++i) kk[i] = kx[i] - mean[bh * D + blk * 16 + i];
      quant_block16(kk, 1, 16, codes, &k_sf[row * nb_d + blk]);
      for (int i = 0; i < 16; ++i) put_nibble(k_codes + row * (D / 2), blk * 16 + i, codes[i]);
    }
  }

  const long nb_n = Np / 16;
#pragma omp parallel for schedule(static)
  for (long bhd = 0; bhd < BH * D; ++bhd) {
    const long bh = bhd / D, d = bhd % D;
    uint8_t codes[16];
    for (long blk = 0; blk < nb_n; ++blk) {
      const long n0 = blk * 16;
      const int count = static_cast<int>(std::min<long>(16, N - n0));
      const float* vx = v + (bh * N + n0) * D + d;
      quant_block16(vx, D, count, codes, &vt_sf[bhd * nb_n + blk]);
      for (int i = 0; i < 16; ++i) put_nibble(vt_codes + bhd * (Np / 2), n0 + i, codes[i]);
    }
  }
}

// ------------------------------------------------------ emulated attention ----
// For each requested row (bh, i): dequantize Q^, K^, V^T exactly in binary64 and walk
// key tiles of width Bk (the GPU kernel's key-tile width) with the online softmax:
//   S_j   = sm_scale * sum_d q~_id k~_jd                      (binary64)
//   m'    = max(m, max_j S_j)   (masked keys excluded)
//   P~_j  = exp(S_j - m')                                      (masked keys -> 0)
//   l     = l * exp(m - m') + sum_j P~_j                       (unquantized P~)
//   r     = max_j P~_j ;  s1 = r / (448 * 6)                   (per-row factor)
//   P2_j  = fp32(P~_j / s1), quantized by the 16-block rule over the tile's keys
//   O     = O * exp(m - m') + s1 * sum_j p^_j v~_j             (binary64)
// and finally O / l. Causal masking keeps keys j <= i.
// rows: n_rows pairs (bh, i); out: [n_rows, D] binary64.
void so_attn_emulated(const uint8_t* q_codes, const uint8_t* q_sf, const uint8_t* k_codes,
                      const uint8_t* k_sf, const uint8_t* vt_codes, const uint8_t* vt_sf, long BH,
                      long N, long D, int causal, double sm_scale, long Bk, const long* rows,
                      long n_rows, double* out) {
  const long Np = (N + 15) / 16 * 16;
  const long nb_d = D / 16, nb_n = Np / 16;
  // Group rows by head so that K~ and V~ are dequantized once per head.
  std::vector<long> order(static_cast<size_t>(n_rows));
  for (long r = 0; r < n_rows; ++r) order[r] = r;
  std::stable_sort(order.begin(), order.end(),
                   [&](long a, long b) { return rows[2 * a] < rows[2 * b]; });

  std::vector<double> kd, vd;  // [N, D] each
  long r0 = 0;
  while (r0 < n_rows) {
    const long bh = rows[2 * order[r0]];
    long r1 = r0;
    while (r1 < n_rows && rows[2 * order[r1]] == bh) ++r1;

    kd.assign(static_cast<size_t>(N * D), 0.0);
    vd.assign(static_cast<size_t>(N * D), 0.0);
#pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n) {
      const uint8_t* kr = k_codes + (bh * N + n) * (D / 2);
      for (long d = 0; d < D; ++d) {
        const double s = e4m3_value(k_sf[(bh * N + n) * nb_d + d / 16]);
        kd[n * D + d] = e2m1_value(get_nibble(kr, d)) * s;
        const uint8_t* vr = vt_codes + (bh * D + d) * (Np / 2);
        const double sv = e4m3_value(vt_sf[(bh * D + d) * nb_n + n / 16]);
        vd[n * D + d] = e2m1_value(get_nibble(vr, n)) * sv;
      }
    }

#pragma omp parallel for schedule(dynamic, 1)
    for (long rr = r0; rr < r1; ++rr) {
      const long ridx = order[rr];
      const long i = rows[2 * ridx + 1];
      std::vector<double> qd(static_cast<size_t>(D)), O(static_cast<size_t>(D), 0.0);
      std::vector<double> S(static_cast<size_t>(Bk)), P(static_cast<size_t>(Bk));
      std::vector<float> P2(static_cast<size_t>(Bk + 16));
      std::vector<double> phat(static_cast<size_t>(Bk + 16));
      const uint8_t* qr = q_codes + (bh * N + i) * (D / 2);
      for (long d = 0; d < D; ++d)
        qd[d] = e2m1_value(get_nibble(qr, d)) * e4m3_value(q_sf[(bh * N + i) * nb_d + d / 16]);

      double m = -std::numeric_limits<double>::infinity(), l = 0.0;
      const long last_key = causal ? std::min(i, N - 1) : N - 1;
      for (long j0 = 0; j0 <= last_key; j0 += Bk) {
        const long j1 = std::min(j0 + Bk, last_key + 1);  // exclusive; keys past it are masked
        double tmax = -std::numeric_limits<double>::infinity();
        for (long j = j0; j < j1; ++j) {
          double acc = 0.0;
          for (long d = 0; d < D; ++d) acc += qd[d] * kd[j * D + d];
          S[j - j0] = sm_scale * acc;
          tmax = std::max(tmax, S[j - j0]);
        }
        const double m_new = std::max(m, tmax);
        const double alpha = std::exp(m - m_new);  // exp(-inf) = 0 on the first tile
        double rowsum = 0.0, r = 0.0;
        for (long j = j0; j < j1; ++j) {
          P[j - j0] = std::exp(S[j - j0] - m_new);
          rowsum += P[j - j0];
          r = std::max(r, P[j - j0]);
        }
        l = l * alpha + rowsum;
        const double s1 = r / kTwoLevelTarget;
        // P2 over the whole tile width (masked or absent keys are 0), blocks of 16.
        const long width = std::min(Bk, ((j1 - j0) + 15) / 16 * 16);
        for (long t = 0; t < width; ++t)
          P2[t] = (j0 + t < j1) ? static_cast<float>(P[t] / s1) : 0.0f;
        for (long b0 = 0; b0 < width; b0 += 16) {
          uint8_t codes[16], sb;
          quant_block16(&P2[b0], 1, 16, codes, &sb);
          const double s = e4m3_value(sb);
          for (int t = 0; t < 16; ++t) phat[b0 + t] = e2m1_value(codes[t]) * s;
        }
        for (long d = 0; d < D; ++d) {
          double acc = 0.0;
          for (long j = j0; j < j1; ++j) acc += phat[j - j0] * vd[j * D + d];
          O[d] = O[d] * alpha + s1 * acc;
        }
        m = m_new;
      }
      for (long d = 0; d < D; ++d) out[ridx * D + d] = O[d] / l;
    }
    r0 = r1;
  }
}

// --------------------------------------------------- unquantized attention ----
// Plain two-pass softmax attention in binary64 on the fp32 inputs (the definition):
//   O_i = sum_j exp(S_ij - max_j S_ij) v_j / sum_j exp(S_ij - max_j S_ij).
void so_attn_exact(const float* q, const float* k, const float* v, long BH, long N, long D,
                   int causal, double sm_scale, const long* rows, long n_rows, double* out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (long r = 0; r < n_rows; ++r) {
    const long bh = rows[2 * r], i = rows[2 * r + 1];
    const long nk = causal ? std::min(i + 1, N) : N;
    std::vector<double> S(static_cast<size_t>(nk));
    double mx = -std::numeric_limits<double>::infinity();
    for (long j = 0; j < nk; ++j) {
      double acc = 0.0;
      for (long d = 0; d < D; ++d)
        acc += static_cast<double>(q[(bh * N + i) * D + d]) * static_cast<double>(k[(bh * N + j) * D + d]);
      S[j] = sm_scale * acc;
      mx = std::max(mx, S[j]);
    }
    double l = 0.0;
    for (long j = 0; j < nk; ++j) {
      S[j] = std::exp(S[j] - mx);
      l += S[j];
    }
    for (long d = 0; d < D; ++d) {
      double acc = 0.0;
      for (long j = 0; j < nk; ++j) acc += S[j] * static_cast<double>(v[(bh * N + j) * D + d]);
      out[r * D + d] = acc / l;
    }
  }
}

// Online-softmax attention without quantization, key tiles of width Bk, binary64:
// the recurrence of the reply to Q3, with O scaled by diag(l)^-1 after the last tile.
void so_attn_online(const float* q, const float* k, const float* v, long BH, long N, long D,
                    int causal, double sm_scale, long Bk, const long* rows, long n_rows,
                    double* out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (long r = 0; r < n_rows; ++r) {
    const long bh = rows[2 * r], i = rows[2 * r + 1];
    const long last_key = causal ? std::min(i, N - 1) : N - 1;
    std::vector<double> O(static_cast<size_t>(D), 0.0), S(static_cast<size_t>(Bk));
    double m = -std::numeric_limits<double>::infinity(), l = 0.0;
    for (long j0 = 0; j0 <= last_key; j0 += Bk) {
      const long j1 = std::min(j0 + Bk, last_key + 1);
      double tmax = -std::numeric_limits<double>::infinity();
      for (long j = j0; j < j1; ++j) {
        double acc = 0.0;
        for (long d = 0; d < D; ++d)
          acc += static_cast<double>(q[(bh * N + i) * D + d]) * static_cast<double>(k[(bh * N + j) * D + d]);
        S[j - j0] = sm_scale * acc;
        tmax = std::max(tmax, S[j - j0]);
      }
      const double m_new = std::max(m, tmax);
      const double alpha = std::exp(m - m_new);
      double rowsum = 0.0;
      for (long j = j0; j < j1; ++j) {
        S[j - j0] = std::exp(S[j - j0] - m_new);
        rowsum += S[j - j0];
      }
      l = l * alpha + rowsum;
      for (long d = 0; d < D; ++d) {
        double acc = 0.0;
        for (long j = j0; j < j1; ++j) acc += S[j - j0] * static_cast<double>(v[(bh * N + j) * D + d]);
        O[d] = O[d] * alpha + acc;
      }
      m = m_new;
    }
    for (long d = 0; d < D; ++d) out[r * D + d] = O[d] / l;
  }
}

int so_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
