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

// ------------------------------------------------------ second-level scale ----
// NVFP4's per-tensor FP32 scale, named (not printed) on the author page ("TetraJet-v2"
// abstract, "double-block quantization" for NVFP4), read here the way the method scales
// P~ before its 16-element blocks: a coarse factor maps the largest magnitude of the
// group onto 448 * 6 (E4M3 max times E2M1 max), the values are divided by it, and the
// ordinary block rule runs on the quotient.
//   amax[g] = max |x'| over group g, x' = fp32(x - mean) when a mean is given, else x.
void so_group_amax(const float* x, long G, long N, long D, const float* mean, float* amax) {
#pragma omp parallel for schedule(static)
  for (long g = 0; g < G; ++g) {
    float a = 0.0f;
    for (long n = 0; n < N; ++n)
      for (long d = 0; d < D; ++d) {
        float v = x[(g * N + n) * D + d];
        if (mean) v = v - mean[g * D + d];
        a = std::max(a, std::fabs(v));
      }
    amax[g] = a;
  }
}

// gscale[i] = fp32(amax[i] / 2688) (binary32 division), or 1 when that is 0.
void so_second_level_scale(const float* amax, long n, float* gscale) {
  for (long i = 0; i < n; ++i) {
    const float g = amax[i] / static_cast<float>(kTwoLevelTarget);
    gscale[i] = g > 0.0f ? g : 1.0f;
  }
}

// ------------------------------------------------------------ quantize rows ----
// x [G, N, D] quantized along D (the Q and K direction):
//   x' = fp32(x - mean[g, d])   when mean != NULL (smoothing K),
//   x'' = fp32(x' / gscale[g])  when gscale != NULL (second-level scale),
// then the 16-element block rule on x''. Canonical outputs (nibble 2i in the low half
// of byte i): codes [G, N, D/2], sf [G, N, D/16].
void so_quantize_rows(const float* x, long G, long N, long D, const float* mean,
                      const float* gscale, uint8_t* codes, uint8_t* sf) {
  const long nb_d = D / 16;
#pragma omp parallel for schedule(static)
  for (long row = 0; row < G * N; ++row) {
    const long g = row / N;
    float blk[16];
    uint8_t c[16];
    for (long b = 0; b < nb_d; ++b) {
      for (int i = 0; i < 16; ++i) {
        float v = x[row * D + b * 16 + i];
        if (mean) v = v - mean[g * D + b * 16 + i];
        if (gscale) v = v / gscale[g];
        blk[i] = v;
      }
      quant_block16(blk, 1, 16, c, &sf[row * nb_d + b]);
      for (int i = 0; i < 16; ++i) put_nibble(codes + row * (D / 2), b * 16 + i, c[i]);
    }
  }
}

// v [G, N, D] quantized along tokens (the P~V contraction direction) and stored
// transposed: vt_codes [G, D, Np/2], vt_sf [G, D, Np/16], Np = N rounded up to 16
// (tokens past N count as zeros). gscale as for so_quantize_rows.
void so_quantize_vt(const float* v, long G, long N, long D, const float* gscale,
                    uint8_t* vt_codes, uint8_t* vt_sf) {
  const long Np = (N + 15) / 16 * 16;
  const long nb_n = Np / 16;
#pragma omp parallel for schedule(static)
  for (long gd = 0; gd < G * D; ++gd) {
    const long g = gd / D, d = gd % D;
    float blk[16];
    uint8_t c[16];
    for (long b = 0; b < nb_n; ++b) {
      const long n0 = b * 16;
      for (int i = 0; i < 16; ++i) {
        float x = (n0 + i < N) ? v[(g * N + n0 + i) * D + d] : 0.0f;
        if (gscale) x = x / gscale[g];
        blk[i] = x;
      }
      quant_block16(blk, 1, 16, c, &vt_sf[gd * nb_n + b]);
      for (int i = 0; i < 16; ++i) put_nibble(vt_codes + gd * (Np / 2), n0 + i, c[i]);
    }
  }
}

// ------------------------------------------------------------ Q smoothing ----
// Smoothing Q (named in the SageAttention2 abstract on the author page, the counterpart
// of smoothing K): each query row is quantized as q' = fp32(q - mu_q), mu_q the channel
// mean of the (sequence, query head) -- computed by so_kmean on Q -- and the part that
// was taken out returns as a per-key bias of the scores,
//   bias[bhq, j] = sum_d mu_q[bhq, d] * k'[kv(bhq), j, d]      (binary64),
// with k' = fp32(k - mu_k) the smoothed, unquantized keys (k itself when mu_k is NULL),
// so that q . k' = q' . k' + bias exactly. kv(bhq) follows the grouped-head map of
// so_attn_emulated. mu_q [B*Hq, D]; k [B*Hkv, Nk, D]; mu_k [B*Hkv, D]; bias [B*Hq, Nk].
void so_qk_bias(const float* mu_q, const float* k, const float* mu_k, long B, long Hq, long Hkv,
                long Nk, long D, double* bias) {
  const long group = Hq / Hkv;
#pragma omp parallel for schedule(static)
  for (long bhq = 0; bhq < B * Hq; ++bhq) {
    const long kv = (bhq / Hq) * Hkv + (bhq % Hq) / group;
    for (long j = 0; j < Nk; ++j) {
      double acc = 0.0;
      for (long d = 0; d < D; ++d) {
        float kk = k[(kv * Nk + j) * D + d];
        if (mu_k) kk = kk - mu_k[kv * D + d];
        acc += static_cast<double>(mu_q[bhq * D + d]) * static_cast<double>(kk);
      }
      bias[bhq * Nk + j] = acc;
    }
  }
}

}  // extern "C"

namespace {

// The key-tile walk of one query row (steps of so_attn_emulated below): S[0..n_keys) are
// the row's scaled scores (binary64), keys at or past n_keys are masked; vd [>= n_keys, D]
// the dequantized values. Writes O / l (0 for a row that sees no key) to out[0..D).
void walk_key_tiles(const double* S, long n_keys, const double* vd, long D, long Bk, double* out) {
  std::vector<double> O(static_cast<size_t>(D), 0.0), P(static_cast<size_t>(Bk));
  std::vector<float> P2(static_cast<size_t>(Bk + 16));
  std::vector<double> phat(static_cast<size_t>(Bk + 16));
  double m = -std::numeric_limits<double>::infinity(), l = 0.0;
  for (long j0 = 0; j0 < n_keys; j0 += Bk) {
    const long j1 = std::min(j0 + Bk, n_keys);  // exclusive; keys past it are masked
    double tmax = -std::numeric_limits<double>::infinity();
    for (long j = j0; j < j1; ++j) tmax = std::max(tmax, S[j]);
    const double m_new = std::max(m, tmax);
    const double alpha = std::exp(m - m_new);  // exp(-inf) = 0 on the first tile
    double rowsum = 0.0, r = 0.0;
    for (long j = j0; j < j1; ++j) {
      P[j - j0] = std::exp(S[j] - m_new);
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
  for (long d = 0; d < D; ++d) out[d] = l > 0.0 ? O[d] / l : 0.0;
}

// Dequantized V~ [Nk, D] of key/value head kv (binary64, exact): e2m1(code) * s * g_v.
void dequant_v(const uint8_t* vt_codes, const uint8_t* vt_sf, long kv, long Nk, long D, double g_v,
               std::vector<double>& vd) {
  const long Nkp = (Nk + 15) / 16 * 16, nb_n = Nkp / 16;
  vd.assign(static_cast<size_t>(Nk * D), 0.0);
#pragma omp parallel for schedule(static)
  for (long n = 0; n < Nk; ++n)
    for (long d = 0; d < D; ++d) {
      const uint8_t* vr = vt_codes + (kv * D + d) * (Nkp / 2);
      const double sv = e4m3_value(vt_sf[(kv * D + d) * nb_n + n / 16]);
      vd[n * D + d] = e2m1_value(get_nibble(vr, n)) * sv * g_v;
    }
}

}  // namespace

extern "C" {

// ------------------------------------------------------ emulated attention ----
// One or more sequences of equal lengths: B batches, Hq query heads, Hkv key/value heads
// (query head h reads key/value head h / (Hq / Hkv)), Nq queries and Nk keys each.
// Arrays: q codes/sf [B*Hq, Nq, ...]; k codes/sf [B*Hkv, Nk, ...]; vt [B*Hkv, D, ...];
// gq [B*Hq], gk, gv [B*Hkv] second-level scales (NULL = 1); qk_bias [B*Hq, Nk] the Q
// smoothing bias of so_qk_bias (NULL = none), added to the dot product before sm_scale.
// For each requested row (bhq, i): dequantize exactly in binary64 (code * scale * g)
// and walk key tiles of width Bk (the GPU kernel's key-tile width) from key 0:
//   S_j   = sm_scale * (sum_d q~_id k~_jd + qk_bias_j)         (binary64)
//   m'    = max(m, max_j S_j)   (masked keys excluded)
//   P~_j  = exp(S_j - m')                                      (masked keys -> 0)
//   l     = l * exp(m - m') + sum_j P~_j                       (unquantized P~)
//   r     = max_j P~_j ;  s1 = r / (448 * 6)                   (per-row factor)
//   P2_j  = fp32(P~_j / s1), quantized by the 16-block rule over the tile's keys
//   O     = O * exp(m - m') + s1 * sum_j p^_j v~_j             (binary64)
// and finally O / l. Causal masking keeps keys j <= i + (Nk - Nq) (the last query sees
// the last key; with Nq == Nk this is j <= i). A row that sees no key gives 0.
// rows: n_rows pairs (bhq, i); out: [n_rows, D] binary64.
void so_attn_emulated(const uint8_t* q_codes, const uint8_t* q_sf, const uint8_t* k_codes,
                      const uint8_t* k_sf, const uint8_t* vt_codes, const uint8_t* vt_sf,
                      const float* gq, const float* gk, const float* gv, const double* qk_bias,
                      long B, long Hq, long Hkv, long Nq, long Nk, long D, int causal,
                      double sm_scale, long Bk, const long* rows, long n_rows, double* out) {
  (void)B;
  const long group = Hq / Hkv;
  const long nb_d = D / 16;
  // Group rows by key/value head so that K~ and V~ are dequantized once per head.
  auto kv_of = [&](long bhq) { return (bhq / Hq) * Hkv + (bhq % Hq) / group; };
  std::vector<long> order(static_cast<size_t>(n_rows));
  for (long r = 0; r < n_rows; ++r) order[r] = r;
  std::stable_sort(order.begin(), order.end(),
                   [&](long a, long b) { return kv_of(rows[2 * a]) < kv_of(rows[2 * b]); });

  std::vector<double> kd, vd;  // [Nk, D] each
  long r0 = 0;
  while (r0 < n_rows) {
    const long kv = kv_of(rows[2 * order[r0]]);
    long r1 = r0;
    while (r1 < n_rows && kv_of(rows[2 * order[r1]]) == kv) ++r1;
    const double g_k = gk ? gk[kv] : 1.0, g_v = gv ? gv[kv] : 1.0;

    kd.assign(static_cast<size_t>(Nk * D), 0.0);
#pragma omp parallel for schedule(static)
    for (long n = 0; n < Nk; ++n) {
      const uint8_t* kr = k_codes + (kv * Nk + n) * (D / 2);
      for (long d = 0; d < D; ++d) {
        const double s = e4m3_value(k_sf[(kv * Nk + n) * nb_d + d / 16]);
        kd[n * D + d] = e2m1_value(get_nibble(kr, d)) * s * g_k;
      }
    }
    dequant_v(vt_codes, vt_sf, kv, Nk, D, g_v, vd);

#pragma omp parallel for schedule(dynamic, 1)
    for (long rr = r0; rr < r1; ++rr) {
      const long ridx = order[rr];
      const long bhq = rows[2 * ridx], i = rows[2 * ridx + 1];
      const double g_q = gq ? gq[bhq] : 1.0;
      std::vector<double> qd(static_cast<size_t>(D));
      const uint8_t* qr = q_codes + (bhq * Nq + i) * (D / 2);
      for (long d = 0; d < D; ++d)
        qd[d] = e2m1_value(get_nibble(qr, d)) * e4m3_value(q_sf[(bhq * Nq + i) * nb_d + d / 16]) * g_q;
      // Keys j <= last_key are visible; the rest of the row is masked.
      const long last_key = causal ? std::min(i + (Nk - Nq), Nk - 1) : Nk - 1;
      const long n_keys = std::max(last_key + 1, 0L);
      std::vector<double> S(static_cast<size_t>(std::max(n_keys, 1L)));
      for (long j = 0; j < n_keys; ++j) {
        double acc = 0.0;
        for (long d = 0; d < D; ++d) acc += qd[d] * kd[j * D + d];
        if (qk_bias) acc += qk_bias[bhq * Nk + j];
        S[j] = sm_scale * acc;
      }
      walk_key_tiles(S.data(), n_keys, vd.data(), D, Bk, out + ridx * D);
    }
    r0 = r1;
  }
}

// Steps 5-6 of so_attn_emulated on GIVEN scores: S [n_rows, Nk] binary64 are the
// already-scaled scores of each row (for instance a GPU's FP32 products, widened); row r
// reads values of key/value head kv[r] and sees keys 0 .. n_keys[r] - 1. The online
// softmax, the two-level P~ quantization and the P^ V~ accumulation are exactly those of
// so_attn_emulated; only the scores come from outside. out: [n_rows, D].
void so_attn_from_scores(const double* S, long n_rows, long Nk, const long* kv, const long* n_keys,
                         const uint8_t* vt_codes, const uint8_t* vt_sf, const float* gv, long D,
                         long Bk, double* out) {
  std::vector<double> vd;
  for (long r = 0; r < n_rows; ++r) {
    dequant_v(vt_codes, vt_sf, kv[r], Nk, D, gv ? gv[kv[r]] : 1.0, vd);
    walk_key_tiles(S + r * Nk, std::min(n_keys[r], Nk), vd.data(), D, Bk, out + r * D);
  }
}

// ------------------------------------------------------------ 8-bit path ----
// The 8-bit forward of the method's training exploration ("An Exploration of 8-Bit
// Training" in the SageAttention3 title; "trainable INT8 attention" in the SageBwd
// abstract; INT8 for QK^T per the SageAttention review thread, reply to W1). Formats:
//   Q, K (K smoothed first): symmetric INT8 with one binary32 scale per block of
//     `block` consecutive tokens of a head: s = fp32(absmax / 127) (0 -> codes 0),
//     code = clamp(RNE(fp32(x / s)), -127, 127);
//   V: E4M3 with one binary32 scale per channel over all tokens of a head:
//     s_d = fp32(absmax_d / 448), code = E4M3(fp32(v / s_d)) (0 scale -> code 0);
//   P~: per query row and key tile s1 = rowmax(P~) / 448, code = E4M3(fp32(P~ / s1)).

// x [G, N, D] -> codes [G, N, D] int8, scales [G, ceil(N / block)]; mean [G, D] or NULL.
void so_quant_int8_rows(const float* x, long G, long N, long D, long block, const float* mean,
                        int8_t* codes, float* scales) {
  const long nb = (N + block - 1) / block;
#pragma omp parallel for schedule(static)
  for (long gb = 0; gb < G * nb; ++gb) {
    const long g = gb / nb, b = gb % nb;
    const long n0 = b * block, n1 = std::min(N, n0 + block);
    auto val = [&](long n, long d) {
      float v = x[(g * N + n) * D + d];
      if (mean) v = v - mean[g * D + d];
      return v;
    };
    float a = 0.0f;
    for (long n = n0; n < n1; ++n)
      for (long d = 0; d < D; ++d) a = std::max(a, std::fabs(val(n, d)));
    const float s = a / 127.0f;
    scales[g * nb + b] = s;
    for (long n = n0; n < n1; ++n)
      for (long d = 0; d < D; ++d) {
        float c = 0.0f;
        if (s > 0.0f) c = std::nearbyint(val(n, d) / s);  // default rounding: to nearest even
        c = std::min(127.0f, std::max(-127.0f, c));
        codes[(g * N + n) * D + d] = static_cast<int8_t>(c);
      }
  }
}

// v [G, N, D] -> vt codes [G, D, N] (E4M3 bytes), scales [G, D].
void so_quant_e4m3_channels(const float* v, long G, long N, long D, uint8_t* vt_codes, float* scales) {
#pragma omp parallel for schedule(static)
  for (long gd = 0; gd < G * D; ++gd) {
    const long g = gd / D, d = gd % D;
    float a = 0.0f;
    for (long n = 0; n < N; ++n) a = std::max(a, std::fabs(v[(g * N + n) * D + d]));
    const float s = a / 448.0f;
    scales[gd] = s;
    for (long n = 0; n < N; ++n)
      vt_codes[gd * N + n] = s > 0.0f ? e4m3_encode(v[(g * N + n) * D + d] / s) : 0;
  }
}

// Emulated 8-bit attention: dequantize exactly in binary64 (q~ = code * s_q[block], and
// likewise k~; v~ = e4m3(code) * s_v[d]) and walk key tiles of Bk as so_attn_emulated,
// with P~ quantized as s1 = rowmax / 448 and p^ = e4m3(fp32(P~ / s1)) * s1.
// q codes [B*Hq, Nq, D], q scales [B*Hq, ceil(Nq/block)]; k likewise with Hkv, Nk;
// vt codes [B*Hkv, D, Nk], v scales [B*Hkv, D]. rows (bhq, i); out [n_rows, D].
void so_attn_emulated8(const int8_t* q_codes, const float* q_scales, const int8_t* k_codes,
                       const float* k_scales, const uint8_t* vt_codes, const float* v_scales,
                       long B, long Hq, long Hkv, long Nq, long Nk, long D, long block, int causal,
                       double sm_scale, long Bk, const long* rows, long n_rows, double* out) {
  (void)B;
  const long group = Hq / Hkv;
  const long nbq = (Nq + block - 1) / block, nbk = (Nk + block - 1) / block;
#pragma omp parallel for schedule(dynamic, 1)
  for (long r = 0; r < n_rows; ++r) {
    const long bhq = rows[2 * r], i = rows[2 * r + 1];
    const long kv = (bhq / Hq) * Hkv + (bhq % Hq) / group;
    std::vector<double> qd(static_cast<size_t>(D)), O(static_cast<size_t>(D), 0.0);
    std::vector<double> S(static_cast<size_t>(Bk)), P(static_cast<size_t>(Bk));
    const double sq = q_scales[bhq * nbq + i / block];
    for (long d = 0; d < D; ++d) qd[d] = q_codes[(bhq * Nq + i) * D + d] * sq;
    double m = -std::numeric_limits<double>::infinity(), l = 0.0;
    const long last_key = causal ? std::min(i + (Nk - Nq), Nk - 1) : Nk - 1;
    for (long j0 = 0; j0 <= last_key; j0 += Bk) {
      const long j1 = std::min(j0 + Bk, last_key + 1);
      double tmax = -std::numeric_limits<double>::infinity();
      for (long j = j0; j < j1; ++j) {
        const double sk = k_scales[kv * nbk + j / block];
        double acc = 0.0;
        for (long d = 0; d < D; ++d) acc += qd[d] * (k_codes[(kv * Nk + j) * D + d] * sk);
        S[j - j0] = sm_scale * acc;
        tmax = std::max(tmax, S[j - j0]);
      }
      const double m_new = std::max(m, tmax);
      const double alpha = std::exp(m - m_new);
      double rowsum = 0.0, rmax = 0.0;
      for (long j = j0; j < j1; ++j) {
        P[j - j0] = std::exp(S[j - j0] - m_new);
        rowsum += P[j - j0];
        rmax = std::max(rmax, P[j - j0]);
      }
      l = l * alpha + rowsum;
      const double s1 = rmax / 448.0;
      for (long j = j0; j < j1; ++j) {
        const float p2 = static_cast<float>(P[j - j0] / s1);
        P[j - j0] = e4m3_value(e4m3_encode(p2));
      }
      for (long d = 0; d < D; ++d) {
        const double sv = v_scales[kv * D + d];
        double acc = 0.0;
        for (long j = j0; j < j1; ++j) acc += P[j - j0] * (e4m3_value(vt_codes[(kv * D + d) * Nk + j]) * sv);
        O[d] = O[d] * alpha + s1 * acc;
      }
      m = m_new;
    }
    for (long d = 0; d < D; ++d) out[r * D + d] = l > 0.0 ? O[d] / l : 0.0;
  }
}

// --------------------------------------------------- unquantized attention ----
// Plain two-pass softmax attention in binary64 on the fp32 inputs (the definition):
//   O_i = sum_j exp(S_ij - max_j S_ij) v_j / sum_j exp(S_ij - max_j S_ij),
// with the head map and causal rule of so_attn_emulated (keys j <= i + Nk - Nq; a row
// with no visible key gives 0). q [B*Hq, Nq, D]; k, v [B*Hkv, Nk, D].
void so_attn_exact(const float* q, const float* k, const float* v, long B, long Hq, long Hkv,
                   long Nq, long Nk, long D, int causal, double sm_scale, const long* rows,
                   long n_rows, double* out) {
  (void)B;
  const long group = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
  for (long r = 0; r < n_rows; ++r) {
    const long bhq = rows[2 * r], i = rows[2 * r + 1];
    const long kv = (bhq / Hq) * Hkv + (bhq % Hq) / group;
    const long nk = causal ? std::max(0L, std::min(i + 1 + (Nk - Nq), Nk)) : Nk;
    std::vector<double> S(static_cast<size_t>(nk));
    double mx = -std::numeric_limits<double>::infinity();
    for (long j = 0; j < nk; ++j) {
      double acc = 0.0;
      for (long d = 0; d < D; ++d)
        acc += static_cast<double>(q[(bhq * Nq + i) * D + d]) * static_cast<double>(k[(kv * Nk + j) * D + d]);
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
      for (long j = 0; j < nk; ++j) acc += S[j] * static_cast<double>(v[(kv * Nk + j) * D + d]);
      out[r * D + d] = nk > 0 ? acc / l : 0.0;
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
