// Fused 8-bit attention forward for B200 (sm_100a): the 8-bit path of the method's
// training exploration (SageAttention3 title, "An Exploration of 8-Bit Training"; INT8
// for QK^T per the SageAttention review thread, reply to W1; "trainable INT8 attention"
// in the SageBwd abstract).
//
//   S  = (s_q s_k) * Q8 K8^T      tcgen05 kind::i8, INT32 accumulate in TMEM; one scale
//                                 per 128-row tile of Q and of K (sm_scale folded in)
//   P~ = exp(S - m), online softmax (m/d recurrence, lazy reference maximum)
//   P8 = E4M3(P~ / s1), s1 = rowmax(P~) / 448 per row and key tile
//   O  = O * alpha + s1 * P8 V8^T  tcgen05 kind::f8f6f4 (E4M3 x E4M3 -> FP32)
//   out = diag(s_v) O / l         s_v the channel scales of V
//
// Warp roles: warp 0 copies Q once and K / V^T tiles into a 3-stage ring (TMA, 128-byte
// swizzle), warp 1 allocates TMEM and issues the MMAs (S double-buffered), warps 2-9 are
// two softmax warpgroups splitting each row's keys (they exchange the row maxima every
// tile and each folds half of O). Every wait is bounded. This is the FP4 kernel's earlier
// design: the FP4 kernel's alternating-warpgroup design measured slower for these 8-bit
// products, which take twice the tensor time and twice the SMEM bytes of FP4. 8-bit
// operands carry no block scales, so there are no scale-factor copies and no per-16
// scale computation.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "attn_common.cuh"
#include "sage_internal.h"
#include "sm100_ptx.cuh"

namespace sage {

namespace {

using attn::Ctl;
using attn::store_out8;
using attn::tmem_wait_regs;
using attn::wait_bar;

constexpr int kStages8 = 3;
constexpr int kSoftmaxWarps8 = 8;
constexpr uint32_t kTmemCols8 = 512;
constexpr int kThreads8 = 320;
constexpr uint32_t kCol8S0 = 0;     // S buffers: 128 columns each (INT32), at 0 and 128
constexpr uint32_t kCol8PV = 256;   // PV accumulator: D columns (FP32)

constexpr int align1k8(int x) { return (x + 1023) & ~1023; }

template <int D>
struct Layout8 {
  static constexpr int kQBytes = 128 * D;   // int8 rows of D bytes
  static constexpr int kKBytes = 128 * D;
  static constexpr int kVBytes = D * 128;   // E4M3 V^T: D rows of 128 keys
  static constexpr int kPBytes = 128 * 128; // E4M3 P: 128 rows of 128 keys
  static constexpr int off_q = 0;
  static constexpr int st_k = 0;
  static constexpr int st_v = align1k8(kKBytes);
  static constexpr int kStageBytes = align1k8(st_v + kVBytes);
  static constexpr int off_stage = align1k8(off_q + kQBytes);
  static constexpr int off_p = off_stage + kStages8 * kStageBytes;
  static constexpr int off_xch = off_p + 2 * kPBytes;          // [2 tiles][2 halves][128] floats
  static constexpr int off_lsum = off_xch + 2 * 2 * 128 * 4;   // [2 halves][128] floats
  static constexpr int off_bar = off_lsum + 2 * 128 * 4;
  static constexpr int off_misc = off_bar + 32 * 8;            // tmem base, abort flags
  static constexpr int kBytes = off_misc + 16;
};

enum : int {
  E_QFULL = 0,
  E_KFULL = 1,                       // + stage
  E_VFULL = E_KFULL + kStages8,      // + stage
  E_KVEMPTY = E_VFULL + kStages8,    // + stage
  E_SFULL = E_KVEMPTY + kStages8,    // + buffer
  E_SEMPTY = E_SFULL + 2,
  E_PFULL = E_SEMPTY + 2,
  E_PEMPTY = E_PFULL + 2,
  E_PVFULL = E_PEMPTY + 2,
  E_PVEMPTY = E_PVFULL + 1,
  E_XCH = E_PVEMPTY + 1,             // + tile parity
  E_LSUM = E_XCH + 2,
  E_DRAIN = E_LSUM + 1,
  E_COUNT = E_DRAIN + 1
};
static_assert(E_COUNT <= 32, "barrier area");

// K-major operand rows of `row_bytes` bytes, swizzle = row width (128 or 64 bytes),
// 8-row groups row_bytes * 8 apart; one MMA consumes 32 bytes of each row.
__device__ __forceinline__ uint64_t rows_desc(uint32_t saddr, int row_bytes) {
  return make_sdesc(saddr, 16, 8 * row_bytes, row_bytes == 128 ? kLayoutSw128 : kLayoutSw64);
}

// Instruction descriptors (dense, K-major A and B, M = 128):
//   kind::i8     D S32 (2), A and B signed 8-bit (1)
//   kind::f8f6f4 D F32 (1), A and B E4M3 (0)
__host__ __device__ constexpr uint32_t idesc_i8(uint32_t n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_e4m3(uint32_t n) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t"
      "}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_mma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t"
      "}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// INT32 -> float, exact for |x| < 2^22 (|S| <= 127 * 127 * 128 here): place x in the
// mantissa of 1.5 * 2^23 and subtract that.
__device__ __forceinline__ float s32_to_f32(uint32_t raw) {
  return __uint_as_float(raw + 0x4B400000u) - 12582912.0f;
}

}  // namespace

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads8, 1)
    attn8_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using L = Layout8<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::off_bar;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + L::off_misc);
  float* xch = reinterpret_cast<float*>(smem + L::off_xch);
  float* lsum = reinterpret_cast<float*>(smem + L::off_lsum);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (seq_table_bad(p.seq)) return;
  const int bseq = blockIdx.z, hq = blockIdx.y;
  const SeqInfo si = seq_info(p.seq, bseq);
  const int nqt = (si.len_q + 127) >> 7;
  if (static_cast<int>(blockIdx.x) >= nqt) return;  // uniform: before any barrier or allocation
  const int qt = CAUSAL ? (nqt - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
  const int hk = hq / p.group;
  const int nkt = (si.len_k + 127) >> 7;
  const int coff = si.len_k - si.len_q;  // causal: query i sees keys j <= i + coff
  int nt = nkt;
  if (CAUSAL) {
    const int last = qt * 128 + 127 + coff;
    nt = last < 0 ? 0 : min(nkt, last / 128 + 1);
  }
  const int qrow0 = p.Hq * si.prow_q + hq * nqt * 128 + qt * 128;
  const int ktile0 = (p.Hkv * si.prow_k + hk * nkt * 128) >> 7;
  Ctl ctl{misc + 1, p.err, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(bar(E_QFULL), 1);
    for (int s = 0; s < kStages8; ++s) {
      mbar_init(bar(E_KFULL + s), 1);
      mbar_init(bar(E_VFULL + s), 1);
      mbar_init(bar(E_KVEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(E_SFULL + b), 1);
      mbar_init(bar(E_SEMPTY + b), kSoftmaxWarps8);
      mbar_init(bar(E_PFULL + b), kSoftmaxWarps8);
      mbar_init(bar(E_PEMPTY + b), 1);
      mbar_init(bar(E_XCH + b), kSoftmaxWarps8);
    }
    mbar_init(bar(E_PVFULL), 1);
    mbar_init(bar(E_PVEMPTY), kSoftmaxWarps8);
    mbar_init(bar(E_LSUM), kSoftmaxWarps8);
    mbar_init(bar(E_DRAIN), 1);
    misc[1] = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::off_misc, kTmemCols8);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ producer ----
    if (lane == 0 && !(p.debug_flags & kDebugNoLoads)) {
      const bool q_in = SAGE_IN_BOUNDS(static_cast<uint64_t>(qrow0) + 128 <= p.lim.rows_q, p.err, ctl.abort);
      if (q_in) {
        mbar_arrive_expect_tx(bar(E_QFULL), L::kQBytes);
        tma_load_2d(sbase + L::off_q, &tm_q, 0, qrow0, bar(E_QFULL));
      }
      int issued = 0;
      for (int j = 0; q_in && j < nt; ++j) {
        const int st = j % kStages8;
        if (!wait_bar(bar(E_KVEMPTY + st), ((j / kStages8) & 1) ^ 1, ctl)) break;
        if (!SAGE_IN_BOUNDS(static_cast<uint64_t>(ktile0 + j + 1) * 128 <= p.lim.rows_k &&
                                static_cast<uint64_t>(ktile0 + j + 1) * D <= p.lim.rows_v,
                            p.err, ctl.abort)) break;
        const uint32_t sst = sbase + L::off_stage + st * L::kStageBytes;
        mbar_arrive_expect_tx(bar(E_KFULL + st), L::kKBytes);
        tma_load_2d(sst + L::st_k, &tm_k, 0, (ktile0 + j) * 128, bar(E_KFULL + st));
        mbar_arrive_expect_tx(bar(E_VFULL + st), L::kVBytes);
        tma_load_2d(sst + L::st_v, &tm_v, 0, (ktile0 + j) * D, bar(E_VFULL + st));
        issued = j + 1;
      }
      if (*ctl.abort) {
        // Let every copy this thread started land before the CTA releases its memory.
        Ctl drain{misc + 2, p.err, p.timeout_ns};
        misc[2] = 0u;
        if (q_in) wait_bar(bar(E_QFULL), 0, drain);
        for (int j = (issued > kStages8 ? issued - kStages8 : 0); j < issued; ++j) {
          wait_bar(bar(E_KFULL + j % kStages8), (j / kStages8) & 1, drain);
          wait_bar(bar(E_VFULL + j % kStages8), (j / kStages8) & 1, drain);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer ----
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_i8(128);
      constexpr uint32_t id_pv = idesc_e4m3(D);
      bool ok = wait_bar(bar(E_QFULL), 0, ctl);
      for (int j = 0; ok && j <= nt; ++j) {
        if (j < nt) {
          const int st = j % kStages8, sb = j & 1;
          const uint32_t sst = sbase + L::off_stage + st * L::kStageBytes;
          if (!wait_bar(bar(E_KFULL + st), (j / kStages8) & 1, ctl)) { ok = false; break; }
          if (!wait_bar(bar(E_SEMPTY + sb), ((j >> 1) & 1) ^ 1, ctl)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c)
            tc_mma_i8(tmem + kCol8S0 + 128 * sb, rows_desc(sbase + L::off_q + 32 * c, D),
                      rows_desc(sst + L::st_k + 32 * c, D), id_s, c > 0 ? 1u : 0u);
          tc_commit(bar(E_SFULL + sb));
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj % kStages8, pb = jj & 1;
          const uint32_t sst = sbase + L::off_stage + st * L::kStageBytes;
          if (!wait_bar(bar(E_VFULL + st), (jj / kStages8) & 1, ctl)) { ok = false; break; }
          if (!wait_bar(bar(E_PFULL + pb), (jj >> 1) & 1, ctl)) { ok = false; break; }
          if (!wait_bar(bar(E_PVEMPTY), (jj & 1) ^ 1, ctl)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tc_mma_e4m3(tmem + kCol8PV, rows_desc(sbase + L::off_p + pb * L::kPBytes + 32 * c, 128),
                        rows_desc(sst + L::st_v + 32 * c, 128), id_pv, c > 0 ? 1u : 0u);
          tc_commit(bar(E_PVFULL));
          tc_commit(bar(E_PEMPTY + pb));
          tc_commit(bar(E_KVEMPTY + st));
        }
      }
      // Drain: every MMA issued above has completed before TMEM is released.
      tc_commit(bar(E_DRAIN));
      Ctl drain{misc + 3, p.err, p.timeout_ns};
      misc[3] = 0u;
      wait_bar(bar(E_DRAIN), 0, drain);
    }
  } else {
    // ------------------------------------------- softmax + correction (2 x 4 warps) ----
    constexpr int DH = D / 2;
    const int h = (warp - 2) >> 2;  // which half of the keys / output channels
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int qrow = qt * 128 + r;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    // exp2 scale of the integer scores: sm_scale * log2(e) * s_q * s_k(tile)
    const float xs_q = p.sm_scale_log2 * p.q_scale8[qrow0 >> 7];
    float o[DH];
#pragma unroll
    for (int d = 0; d < DH; ++d) o[d] = 0.0f;
    float m_run = -INFINITY, l_half = 0.0f, alpha_prev = 1.0f, s1_prev = 0.0f;
    bool ok = true;
    float sk_next = nt > 0 ? p.k_scale8[ktile0] : 0.0f;

    // O = O * alpha + s1 * PV for this thread's DH output channels (PV of tile jj).
    auto correct = [&](int jj, float alpha, float s1) -> bool {
      if (!__all_sync(0xffffffffu, wait_bar(bar(E_PVFULL), jj & 1, ctl))) return false;
      tc_fence_after();
      const bool unit = __all_sync(0xffffffffu, alpha == 1.0f);
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + kCol8PV + DH * h + 32 * c, v);
        tmem_wait_regs(v);
        const float2 s12 = make_float2(s1, s1), a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float2 acc = make_float2(o[32 * c + i], o[32 * c + i + 1]);
          if (!unit) acc = mul2(acc, a2);
          acc = fma2(make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])), s12, acc);
          o[32 * c + i] = acc.x;
          o[32 * c + i + 1] = acc.y;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(E_PVEMPTY));
      return true;
    };

    for (int j = 0; j < nt; ++j) {
      const int sb = j & 1, pb = j & 1;
      // A zero tile scale (all-zero Q or K - mean tile) makes every integer score 0; any
      // positive scale then gives the same values and keeps masked keys at -inf.
      const float xs_raw = xs_q * sk_next;
      const float xs = xs_raw > 0.0f ? xs_raw : 1.0f;
      if (j + 1 < nt) sk_next = p.k_scale8[ktile0 + j + 1];
      if (!__all_sync(0xffffffffu, wait_bar(bar(E_SFULL + sb), (j >> 1) & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(tmem + lane_base + kCol8S0 + 128 * sb + 64 * h, sr[0]);
      tmem_ld32(tmem + lane_base + kCol8S0 + 128 * sb + 64 * h + 32, sr[1]);
      tmem_wait_regs(sr[0]);
      tmem_wait_regs(sr[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(E_SEMPTY + sb));

      float s[64];
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 * c + i] = s32_to_f32(sr[c][i]);
      const int kbase = j * 128 + 64 * h;
      if ((j * 128 + 128 > si.len_k) || (CAUSAL && j * 128 + 127 > qt * 128 + coff)) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int key = kbase + c;
          if (key >= si.len_k || (CAUSAL && key > qrow + coff)) s[c] = -INFINITY;
        }
      }
      float hm = max3(s[0], s[1], s[2]);
#pragma unroll
      for (int i = 3; i < 63; i += 2) hm = max3(hm, s[i], s[i + 1]);
      hm = fmaxf(hm, s[63]);
      float* xb = xch + (j & 1) * 256;
      xb[h * 128 + r] = hm;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(E_XCH + (j & 1)));
      if (!__all_sync(0xffffffffu, wait_bar(bar(E_XCH + (j & 1)), (j >> 1) & 1, ctl))) { ok = false; break; }
      const float tm = fmaxf(hm, xb[(1 - h) * 128 + r]);
      const bool empty = tm == -INFINITY;  // the row sees no key of this tile

      const float tmx = tm * xs;
      // Lazy reference maximum, as in the FP4 kernel: it moves only when the tile maximum
      // exceeds it by more than 8 (log2 units); P8 is relative to the tile maximum.
      const bool move = tmx > m_run + 8.0f;
      const float m_new = move ? tmx : m_run;
      const float alpha = move ? ex2_approx(m_run - m_new) : 1.0f;
      const float rfac = empty ? 0.0f : ex2_approx(tmx - m_new);  // rowmax of P~ in this tile
      const float s1 = rfac * (1.0f / 448.0f);
      // P2 = P~ / s1 = exp2(S*xs - tmx) * 448, the E4M3 input (<= 448).
      const float nb = (empty ? 0.0f : -tmx) + 8.807354922057604f;  // log2(448)
      // P8 buffer pb must be free (PV of tile j-2 finished). Row r, keys 64h..64h+63:
      // 16-byte chunks 4h..4h+3 of a 128-byte row, 128-byte swizzle (chunk ^ row % 8);
      // each chunk is stored as soon as its 16 codes exist.
      if (!__all_sync(0xffffffffu, wait_bar(bar(E_PEMPTY + pb), ((j >> 1) & 1) ^ 1, ctl))) { ok = false; break; }
      uint8_t* prow = smem + L::off_p + pb * L::kPBytes + r * 128;
      const float2 xs2 = make_float2(xs, xs), nb2 = make_float2(nb, nb);
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i0 = 16 * c + 4 * k;
          const float2 a0 = fma2(make_float2(s[i0], s[i0 + 1]), xs2, nb2);
          const float2 a1 = fma2(make_float2(s[i0 + 2], s[i0 + 3]), xs2, nb2);
          const float2 e0 = make_float2(ex2_approx(a0.x), ex2_approx(a0.y));
          const float2 e1 = make_float2(ex2_approx(a1.x), ex2_approx(a1.y));
          acc = add2(acc, add2(e0, e1));
          pw[k] = f32x2_to_e4m3x2(e0.x, e0.y) | (f32x2_to_e4m3x2(e1.x, e1.y) << 16);
        }
        const int cs = (4 * h + c) ^ (r & 7);
        *reinterpret_cast<uint4*>(prow + cs * 16) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      }
      l_half = l_half * alpha + (acc.x + acc.y) * s1;
      m_run = m_new;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(E_PFULL + pb));

      if (j >= 1 && !correct(j - 1, alpha_prev, s1_prev)) { ok = false; break; }
      alpha_prev = alpha;
      s1_prev = s1;
    }
    if (ok && nt > 0) ok = correct(nt - 1, alpha_prev, s1_prev);
    if (ok) {
      lsum[h * 128 + r] = l_half;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(E_LSUM));
      ok = __all_sync(0xffffffffu, wait_bar(bar(E_LSUM), 0, ctl));
    }
    if (ok && qrow < si.len_q) {
      const float l = l_half + lsum[(1 - h) * 128 + r];
      const float il = l > 0.0f ? 1.0f / l : 0.0f;
      const float* sv = p.v_scale8 + static_cast<size_t>(bseq * p.Hkv + hk) * D + DH * h;
      const size_t base = static_cast<size_t>(static_cast<int64_t>(bseq) * p.so.b + static_cast<int64_t>(hq) * p.so.h +
                                              (static_cast<int64_t>(si.tok_q) + qrow) * p.so.n) + DH * h;
#pragma unroll
      for (int d = 0; d < DH; d += 8) {
        const float4 s0 = *reinterpret_cast<const float4*>(sv + d);
        const float4 s4 = *reinterpret_cast<const float4*>(sv + d + 4);
        const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s4.x, s4.y, s4.z, s4.w};
        float v8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v8[i] = o[d + i] * il * sc[i];
        if (SAGE_IN_BOUNDS(base + d + 8 <= p.lim.o_el, p.err, nullptr)) store_out8(p.out, base + d, v8, p.out_dtype);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols8);
  }
}

template <int D, bool CAUSAL>
static cudaError_t launch_attn8_t(const TensorMaps& m, const AttnParams& p, int tiles_q, cudaStream_t stream) {
  const int smem = Layout8<D>::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn8_fwd_kernel<D, CAUSAL>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles_q, p.Hq, p.B);
  attn8_fwd_kernel<D, CAUSAL><<<grid, kThreads8, smem, stream>>>(m.q, m.k, m.v, p);
  return cudaGetLastError();
}

cudaError_t launch_attention8(const TensorMaps& m, const AttnParams& p, int tiles_q, cudaStream_t stream) {
  if (p.B == 0 || p.Hq == 0 || tiles_q == 0) return cudaSuccess;
  if (p.D == 64) return p.causal ? launch_attn8_t<64, true>(m, p, tiles_q, stream) : launch_attn8_t<64, false>(m, p, tiles_q, stream);
  return p.causal ? launch_attn8_t<128, true>(m, p, tiles_q, stream) : launch_attn8_t<128, false>(m, p, tiles_q, stream);
}

}  // namespace sage
