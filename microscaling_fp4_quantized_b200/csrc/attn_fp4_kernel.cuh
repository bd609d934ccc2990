// Fused microscaling-FP4 attention forward for B200 (sm_100a): the kernel template,
// included by the two translation units that instantiate it (non-causal instances in
// attn_fp4_fwd.cu, causal ones in attn_fp4_causal.cu).
//
// Method: SageAttention3 (arXiv 2505.11594, abstract) -- FP4 Q, K, P~, V on the
// Blackwell FP4 tensor cores -- with FlashAttention tiling and the online softmax
// m/d recurrence as the SageAttention OpenReview thread states it (reply to Q3),
// diag(l)^-1 after the last key tile (reply to Q2), and the two-level P~ quantization
// (per-row factor s1 = rowmax(P~)/(448*6) per key tile, then 16-element E4M3 scales).
//
// One CTA per (128-query tile, query head, sequence); key tiles of 128. Sequences may be
// packed with different lengths, query heads may share key/value heads (head h reads
// key/value head h / (Hq / Hkv)), and the causal mask keeps key j <= i + (len_k - len_q)
// for query i (the last query sees the last key). Warp roles:
//   warp 0      TMA producer of Q^ + scales (once) and of the K^ tiles + scales, into a
//               4-stage ring whose slots return as soon as their S product is done.
//   warp 2      TMA producer of the V^T tiles + scales, into a 4-stage ring whose
//               slots return when their PV product is done (cp.async.bulk.tensor and
//               cp.async.bulk).
//   warp 1      allocates 512 tensor-memory columns; one thread issues the tcgen05
//               block-scaled MMAs S = Q^ K^^T (kind::mxf4nvf4, M128 N128 K64 steps)
//               into S buffer j % 2.
//   warp 3      one thread issues PV = P^ V^T (N = D) into the PV accumulator. Two
//               issuing threads, because one thread waiting on five barriers and
//               issuing ~15 tcgen05 operations per key tile on a busy sub-partition
//               took as long as the softmax of the tile.
//   warps 4-7   correction warpgroup. Thread r owns output row r in FP32 registers and
//               folds every tile's PV row in: O = O * alpha + s1 * 2^(e - m_O) * PV,
//               where e is the reference maximum the tile's softmax used and m_O its
//               own reference.
//   warps 8-15  two softmax warpgroups; warpgroup w takes key tiles j = w, w + 2, ...
//               Thread r owns query row r of its tiles: it reads the 128 scores from
//               TMEM (twice: block maxima first, then the exponentials), computes the
//               tile maximum, P~, the per-16 E4M3 scales, the P^ codes (written in the
//               swizzled layout the MMA reads) and the row sum relative to its own lazy
//               reference maximum, and hands (reference, s1) to the correction. The
//               two warpgroups never wait for each other, so one warpgroup's exp2 phase
//               overlaps the other's TMEM loads, scales and barrier hand-offs.
// Three instances per (D, causal): the general one (packed sequences, len_q != len_k,
// second-level scales: per-sequence lengths, a mask offset, an empty-row guard and a
// score scale read from the device), the general one with the Q-smoothing bias MMA, and
// a lean one for square dense problems with one-level scales, whose loop keeps the score
// scale and the lengths as kernel parameters (long non-causal workload: 1163 TFLOP/s
// lean, 1051 general with a per-tensor second-level scale).
// Every mbarrier wait is bounded (globaltimer); a wait that runs out raises the CTA's
// abort flag and the device error word, and all roles drain and return.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "attn_common.cuh"
#include "sage_internal.h"
#include "sm100_ptx.cuh"

namespace sage {

namespace {

using attn::Ctl;
using attn::kSuspendNs;
using attn::store_out8;
using attn::tmem_wait_regs;
using attn::wait_bar;

constexpr int kKStages = 4;
constexpr int kVStages = 4;
constexpr int kCorrWarps = 4;      // warps 4-7
constexpr uint32_t kTmemCols = 512;
constexpr int kAttnThreads = 512;  // 2 producers, 2 MMA issuers, 4 correction, 8 softmax warps
// Per-thread registers after setmaxnreg: each SM sub-partition holds one warp of every
// warpgroup, so 64 + 192 + 2 * 128 = 512 = 4 x the launch budget of 128. (72 / 184
// spills less but measured 2.5 % slower on long non-causal rows.)
constexpr uint32_t kRegsLow = 64;
constexpr uint32_t kRegsCorr = 192;

constexpr int align1k(int x) { return (x + 1023) & ~1023; }

// Tensor-memory column map of the attention kernel.
constexpr uint32_t kColS0 = 0;      // S buffers: 128 columns each, at 0 and 128
constexpr uint32_t kColPV = 256;    // PV accumulator: D columns
constexpr uint32_t kColSfQ = 384;   // 4 columns per 64-wide K chunk of D
constexpr uint32_t kColSfK = 392;   // + 8 * K stage
constexpr uint32_t kColSfV = 424;   // + 8 * V stage
constexpr uint32_t kColSfP = 456;   // + 8 * P buffer (ends at 472)
// The TMEM regions must not overlap (S buffers, PV, then the scale-factor columns).
static_assert(kColPV >= kColS0 + 2 * 128 && kColSfQ >= kColPV + 128, "TMEM: S / PV regions");
static_assert(kColSfK >= kColSfQ + 8 && kColSfV >= kColSfK + 8 * kKStages &&
                  kColSfP >= kColSfV + 8 * kVStages && kColSfP + 16 <= kTmemCols,
              "TMEM: scale-factor columns");

template <int D, bool QB = false>
struct Layout {
  // QB: the Q-smoothing instance, which adds the score bias with one bf16 MMA per key tile.
  static constexpr int kBiasBytes = QB ? 4096 : 0;   // per stage: 128 keys x 16 bf16, core-matrix layout
  static constexpr int kOnesBytes = QB ? 4096 : 0;   // 128 rows x 16 bf16: ones in columns 0-2
  static constexpr int kQBytes = 128 * D / 2;
  static constexpr int kSfQKBytes = (D / 64) * 512;
  static constexpr int kKBytes = 128 * D / 2;
  static constexpr int kVBytes = D * 64;
  static constexpr int kSfVBytes = 1024;
  static constexpr int kPBytes = 128 * 64;
  static constexpr int kSfPBytes = 1024;
  static constexpr int off_q = 0;
  static constexpr int off_sfq = align1k(off_q + kQBytes);
  // K ring slot: K^ tile, its scales, (Q smoothing) the bias operand; V ring slot: V^T
  // tile and its scales.
  static constexpr int st_k = 0;
  static constexpr int st_sfk = align1k(kKBytes);
  static constexpr int st_bias = align1k(st_sfk + kSfQKBytes);
  static constexpr int kKStageBytes = align1k(st_bias + kBiasBytes);
  static constexpr int st_v = 0;
  static constexpr int st_sfv = align1k(kVBytes);
  static constexpr int kVStageBytes = align1k(st_sfv + kSfVBytes);
  static constexpr int off_stage = align1k(off_sfq + kSfQKBytes);  // K ring
  static constexpr int off_vstage = off_stage + kKStages * kKStageBytes;
  static constexpr int off_p = off_vstage + kVStages * kVStageBytes;
  static constexpr int off_sfp = off_p + 2 * kPBytes;
  static constexpr int off_info = off_sfp + 2 * kSfPBytes;  // [2 warpgroups][128] (reference, s1)
  static constexpr int off_lsum = off_info + 2 * 128 * 8;    // [2 warpgroups][128] (l, reference)
  static constexpr int off_ones = align1k(off_lsum + 2 * 128 * 8);
  static constexpr int off_bar = off_ones + kOnesBytes;
  static constexpr int kNumBars = 40;
  static constexpr int off_misc = off_bar + kNumBars * 8;    // tmem base, abort flag, drain flags
  static constexpr int kBytes = off_misc + 32;
};

// Barrier indices.
enum : int {
  B_QFULL = 0,
  B_KFULL = 1,                     // + K stage
  B_KEMPTY = B_KFULL + kKStages,   // + K stage
  B_VFULL = B_KEMPTY + kKStages,   // + V stage
  B_VEMPTY = B_VFULL + kVStages,   // + V stage
  B_SFULL = B_VEMPTY + kVStages,   // + buffer
  B_SEMPTY = B_SFULL + 2,
  B_PFULL = B_SEMPTY + 2,
  B_PEMPTY = B_PFULL + 2,
  B_PVFULL = B_PEMPTY + 2,
  B_PVEMPTY = B_PVFULL + 1,
  B_IFULL = B_PVEMPTY + 1,        // + softmax warpgroup: per-row factors of its latest tile
  B_IEMPTY = B_IFULL + 2,
  B_LSUM = B_IEMPTY + 2,          // final row sums of both softmax warpgroups
  B_DRAIN = B_LSUM + 1,           // S issuer's last products done
  B_DRAIN2 = B_DRAIN + 1,         // PV issuer's last products done
  B_COUNT = B_DRAIN2 + 1
};
static_assert(B_COUNT <= 40, "barrier area");

__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  // 32 rows x 16 bytes, 8-row core matrices 128 bytes apart, no swizzle.
  return make_sdesc(saddr, 0, 128, kLayoutNone);
}

template <int D>
__device__ __forceinline__ uint64_t qk_desc(uint32_t saddr) {
  // Rows of D/2 bytes (K-major), 8-row groups D*4 bytes apart, swizzle = row width.
  return make_sdesc(saddr, 16, 8 * (D / 2), D == 128 ? kLayoutSw64 : kLayoutSw32);
}

__device__ __forceinline__ uint64_t row64_desc(uint32_t saddr) {
  return make_sdesc(saddr, 16, 512, kLayoutSw64);
}

}  // namespace

// MODE 0: square dense, one-level scales; 1: general; 2: general with the Q-smoothing
// score bias.
template <int D, bool CAUSAL, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fp4_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  constexpr bool GENERAL = MODE >= 1;
  constexpr bool QBIAS = MODE == 2;
  // Wait policy (see wait_bar): the copy and MMA-issuing threads always let themselves be
  // suspended; the softmax and correction warps do too, except in the causal instances.
  constexpr uint32_t kIdleNs = kSuspendNs;
  constexpr uint32_t kWaitNs = CAUSAL ? 0u : kSuspendNs;
  constexpr uint32_t kCheck = CAUSAL ? 31u : 0u;
  using L = Layout<D, QBIAS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::off_bar;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + L::off_misc);
  float2* info = reinterpret_cast<float2*>(smem + L::off_info);
  float2* lsum = reinterpret_cast<float2*>(smem + L::off_lsum);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (seq_table_bad(p.seq)) return;
  const int bseq = blockIdx.z, hq = blockIdx.y;
  SeqInfo si;
  if (GENERAL) {
    si = seq_info(p.seq, bseq);
  } else {
    si.len_q = p.seq.Nq;
    si.len_k = p.seq.Nk;
    si.tok_q = si.tok_k = 0;
    si.prow_q = bseq * round128(p.seq.Nq);
    si.prow_k = bseq * round128(p.seq.Nk);
  }
  const int nqt = (si.len_q + 127) >> 7;
  if (static_cast<int>(blockIdx.x) >= nqt) return;  // uniform: before any barrier or allocation
  const int qt = CAUSAL ? (nqt - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
  const int hk = hq / p.group;
  const int nkt = (si.len_k + 127) >> 7;
  const int coff = GENERAL ? si.len_k - si.len_q : 0;  // causal: query i sees keys j <= i + coff
  int nt = nkt;                          // key tiles to visit
  if (CAUSAL) {
    const int last = qt * 128 + 127 + coff;
    nt = last < 0 ? 0 : min(nkt, last / 128 + 1);
  }
  // Padded rows (TMA coordinates) of this Q tile and of key tile 0; 128-row tiles of
  // those rows index the scale-factor tiles and the V^T tiles.
  const int qrow0 = p.Hq * si.prow_q + hq * nqt * 128 + qt * 128;
  const int ktile0 = (p.Hkv * si.prow_k + hk * nkt * 128) >> 7;
  // Q-smoothing bias of (query head, key tile 0): 32 bytes (16 bf16) per padded key row.
  const size_t bias_row0 = static_cast<size_t>(p.Hq) * si.prow_k + static_cast<size_t>(hq) * nkt * 128;
  Ctl ctl{misc + 1, p.err, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_SFULL + b), 1);
      mbar_init(bar(B_SEMPTY + b), 4);
      mbar_init(bar(B_PFULL + b), 4);
      mbar_init(bar(B_PEMPTY + b), 1);
      mbar_init(bar(B_IFULL + b), 4);
      mbar_init(bar(B_IEMPTY + b), kCorrWarps);
    }
    mbar_init(bar(B_PVFULL), 1);
    mbar_init(bar(B_PVEMPTY), kCorrWarps);
    mbar_init(bar(B_LSUM), 8);
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_DRAIN2), 1);
    misc[1] = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::off_misc, kTmemCols);
    tmem_relinquish();
  }
  if (QBIAS && threadIdx.x < 128) {
    // A operand of the bias MMA: every row (1, 1, 1, 0, ...) in bf16, so that
    // S += A B^T adds the three bf16 terms of each key's bias to every query row.
    // Core-matrix layout (no swizzle): row r, 16-byte half c at (r/8)*256 + c*128 + (r%8)*16.
    const int r = threadIdx.x;
    uint8_t* row = smem + L::off_ones + (r >> 3) * 256 + (r & 7) * 16;
    *reinterpret_cast<uint4*>(row) = make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u);
    *reinterpret_cast<uint4*>(row + 128) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ producer ----
    regs_decrease<kRegsLow>();
    if (lane == 0 && !(p.debug_flags & kDebugNoLoads)) {
      const uint32_t sq = sbase + L::off_q;
      mbar_arrive_expect_tx(bar(B_QFULL), L::kQBytes + L::kSfQKBytes);
      tma_load_2d(sq, &tm_q, 0, qrow0, bar(B_QFULL));
      bulk_load(sbase + L::off_sfq, p.q_sf + static_cast<size_t>(qrow0 >> 7) * L::kSfQKBytes,
                L::kSfQKBytes, bar(B_QFULL));
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int st = j % kKStages;
        if (!wait_bar(bar(B_KEMPTY + st), ((j / kKStages) & 1) ^ 1, ctl, kIdleNs, kCheck)) break;
        const uint32_t sst = sbase + L::off_stage + st * L::kKStageBytes;
        mbar_arrive_expect_tx(bar(B_KFULL + st), L::kKBytes + L::kSfQKBytes + L::kBiasBytes);
        tma_load_2d(sst + L::st_k, &tm_k, 0, (ktile0 + j) * 128, bar(B_KFULL + st));
        bulk_load(sst + L::st_sfk, p.k_sf + static_cast<size_t>(ktile0 + j) * L::kSfQKBytes,
                  L::kSfQKBytes, bar(B_KFULL + st));
        if (QBIAS)
          bulk_load(sst + L::st_bias, p.qk_bias + (bias_row0 + static_cast<size_t>(j) * 128) * 32, L::kBiasBytes,
                    bar(B_KFULL + st));
        issued = j + 1;
      }
      if (*ctl.abort) {
        // Let every copy this thread started land before the CTA releases its memory.
        Ctl drain{misc + 2, p.err, p.timeout_ns};
        misc[2] = 0u;
        wait_bar(bar(B_QFULL), 0, drain, kIdleNs, kCheck);
        for (int j = (issued > kKStages ? issued - kKStages : 0); j < issued; ++j)
          wait_bar(bar(B_KFULL + j % kKStages), (j / kKStages) & 1, drain, kIdleNs, kCheck);
      }
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------- V producer ----
    regs_decrease<kRegsLow>();
    if (lane == 0 && !(p.debug_flags & kDebugNoLoads)) {
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int st = j % kVStages;
        if (!wait_bar(bar(B_VEMPTY + st), ((j / kVStages) & 1) ^ 1, ctl, kIdleNs, kCheck)) break;
        const uint32_t sst = sbase + L::off_vstage + st * L::kVStageBytes;
        mbar_arrive_expect_tx(bar(B_VFULL + st), L::kVBytes + L::kSfVBytes);
        tma_load_2d(sst + L::st_v, &tm_v, 0, (ktile0 + j) * D, bar(B_VFULL + st));
        bulk_load(sst + L::st_sfv, p.vt_sf + static_cast<size_t>(ktile0 + j) * L::kSfVBytes,
                  L::kSfVBytes, bar(B_VFULL + st));
        issued = j + 1;
      }
      if (*ctl.abort) {
        Ctl drain{misc + 4, p.err, p.timeout_ns};
        misc[4] = 0u;
        for (int j = (issued > kVStages ? issued - kVStages : 0); j < issued; ++j)
          wait_bar(bar(B_VFULL + j % kVStages), (j / kVStages) & 1, drain, kIdleNs, kCheck);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- S = Q^ K^^T issuer ----
    regs_decrease<kRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_fp4(128);
      constexpr int kc_qk = D / 64;
      bool ok = wait_bar(bar(B_QFULL), 0, ctl, kIdleNs, kCheck);
      if (ok) {
        tc_fence_after();
        for (int c = 0; c < kc_qk; ++c)
          tc_cp_sf(tmem + kColSfQ + 4 * c, sf_desc(sbase + L::off_sfq + 512 * c));
      }
      for (int j = 0; ok && j < nt; ++j) {
        const int st = j % kKStages, sb = j & 1;
        const uint32_t sst = sbase + L::off_stage + st * L::kKStageBytes;
        if (!wait_bar(bar(B_KFULL + st), (j / kKStages) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
        if (!wait_bar(bar(B_SEMPTY + sb), ((j >> 1) & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < kc_qk; ++c)
          tc_cp_sf(tmem + kColSfK + 8 * st + 4 * c, sf_desc(sst + L::st_sfk + 512 * c));
        for (int c = 0; c < kc_qk; ++c)
          tc_mma_fp4(tmem + kColS0 + 128 * sb, qk_desc<D>(sbase + L::off_q + 32 * c),
                     qk_desc<D>(sst + L::st_k + 32 * c), idesc_s, tmem + kColSfQ + 4 * c,
                     tmem + kColSfK + 8 * st + 4 * c, c > 0 ? 1u : 0u);
        if (QBIAS)  // S += ones * bias^T: the Q-smoothing bias of each key, on the tensor core
          tc_mma_bf16(tmem + kColS0 + 128 * sb, make_sdesc(sbase + L::off_ones, 128, 256, kLayoutNone),
                      make_sdesc(sst + L::st_bias, 128, 256, kLayoutNone), make_idesc_bf16(128), 1u);
        tc_commit(bar(B_SFULL + sb));
        tc_commit(bar(B_KEMPTY + st));
      }
      // Drain: every MMA / copy issued above has completed before TMEM is released.
      tc_commit(bar(B_DRAIN));
      Ctl drain{misc + 3, p.err, p.timeout_ns};
      misc[3] = 0u;
      wait_bar(bar(B_DRAIN), 0, drain, kIdleNs, kCheck);
    }
  } else if (warp == 3) {
    // ---------------------------------------------------------- PV = P^ V^T issuer ----
    // A second issuing thread: its products use other TMEM columns than the S products
    // and its own barriers, so neither chain waits behind the other's dependencies.
    regs_decrease<kRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_pv = make_idesc_fp4(D);
      bool ok = true;
      for (int j = 0; ok && j < nt; ++j) {
        const int st = j % kVStages, pb = j & 1;
        const uint32_t sst = sbase + L::off_vstage + st * L::kVStageBytes;
        if (!wait_bar(bar(B_VFULL + st), (j / kVStages) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
        if (!wait_bar(bar(B_PFULL + pb), (j >> 1) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
        if (!wait_bar(bar(B_PVEMPTY), (j & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < 2; ++c) {
          tc_cp_sf(tmem + kColSfP + 8 * pb + 4 * c, sf_desc(sbase + L::off_sfp + pb * L::kSfPBytes + 512 * c));
          tc_cp_sf(tmem + kColSfV + 8 * st + 4 * c, sf_desc(sst + L::st_sfv + 512 * c));
        }
        for (int c = 0; c < 2; ++c)
          tc_mma_fp4(tmem + kColPV, row64_desc(sbase + L::off_p + pb * L::kPBytes + 32 * c),
                     row64_desc(sst + L::st_v + 32 * c), idesc_pv, tmem + kColSfP + 8 * pb + 4 * c,
                     tmem + kColSfV + 8 * st + 4 * c, c > 0 ? 1u : 0u);
        tc_commit(bar(B_PVFULL));
        tc_commit(bar(B_PEMPTY + pb));
        tc_commit(bar(B_VEMPTY + st));
      }
      tc_commit(bar(B_DRAIN2));
      Ctl drain{misc + 5, p.err, p.timeout_ns};
      misc[5] = 0u;
      wait_bar(bar(B_DRAIN2), 0, drain, kIdleNs, kCheck);
    }
  } else if (warp < 4 + kCorrWarps) {
    // ----------------------------------------------------- correction (4 warps) ----
    regs_increase<kRegsCorr>();
    constexpr int DH = D;
    constexpr int cg = 0;
    const int quad = warp & 3;       // TMEM lane quarter = rows 32*quad ..
    const int r = quad * 32 + lane;
    const int qrow = qt * 128 + r;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    float gv = 1.0f;
    if (GENERAL && p.amax != nullptr)
      gv = second_level_scale(p.amax[2 * p.amax_stride + (p.gscale == kGscaleHead ? bseq * p.Hkv + hk : 0)]);
    float o[DH];
#pragma unroll
    for (int d = 0; d < DH; ++d) o[d] = 0.0f;
    // O is kept relative to 2^m_o; m_o moves (and O is rescaled) only when a tile's
    // reference exceeds it by more than 8, so the factor 2^(e - m_o) stays <= 2^8.
    float m_o = -INFINITY;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int w = j & 1;
      if (!__all_sync(0xffffffffu, wait_bar(bar(B_IFULL + w), (j >> 1) & 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
      const float2 f = info[w * 128 + r];  // (reference e, s1) of tile j for this row
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_IEMPTY + w));
      float alpha = 1.0f, c = 0.0f;
      if (f.y > 0.0f) {  // s1 = 0: the row saw no key of this tile
        if (f.x > m_o + 8.0f) {
          alpha = ex2_approx(m_o - f.x);  // 0 on the first contribution (m_o = -inf)
          m_o = f.x;
        }
        c = f.y * ex2_approx(f.x - m_o);
      }
      if (!__all_sync(0xffffffffu, wait_bar(bar(B_PVFULL), j & 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
      tc_fence_after();
      const bool unit = __all_sync(0xffffffffu, alpha == 1.0f);
      const float2 c2 = make_float2(c, c), a2 = make_float2(alpha, alpha);
#pragma unroll
      for (int cc = 0; cc < DH / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + kColPV + DH * cg + 32 * cc, v);
        tmem_wait_regs(v);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float2 acc = make_float2(o[32 * cc + i], o[32 * cc + i + 1]);
          if (!unit) acc = mul2(acc, a2);
          acc = fma2(make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])), c2, acc);
          o[32 * cc + i] = acc.x;
          o[32 * cc + i + 1] = acc.y;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PVEMPTY));
    }
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(bar(B_LSUM), 0, ctl, kWaitNs, kCheck));
    if (ok && qrow < si.len_q) {
      // l = sum over the two softmax warpgroups of l_w * 2^(m_w - m_o); a row that saw
      // no key (l = 0) is written as 0.
      float l = 0.0f;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const float2 e = lsum[w * 128 + r];
        if (e.x > 0.0f) l += e.x * ex2_approx(e.y - m_o);
      }
      const float il = l > 0.0f ? gv / l : 0.0f;
      const size_t base = static_cast<size_t>(static_cast<int64_t>(bseq) * p.so.b + static_cast<int64_t>(hq) * p.so.h +
                                              (static_cast<int64_t>(si.tok_q) + qrow) * p.so.n) + DH * cg;
#pragma unroll
      for (int d = 0; d < DH; d += 8) {
        float v8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v8[i] = o[d + i] * il;
        store_out8(p.out, base + d, v8, p.out_dtype);
      }
    }
  } else {
    // ----------------------------------------------------- softmax (2 x 4 warps) ----
    const int sw = (warp - 4 - kCorrWarps) >> 2;  // key tiles j = sw, sw + 2, ...
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int qrow = qt * 128 + r;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    float xs = p.sm_scale_log2;
    if (GENERAL && p.amax != nullptr) {
      // Second-level scales of Q and K fold into the score scale.
      const bool head = p.gscale == kGscaleHead;
      const float gq = second_level_scale(p.amax[head ? bseq * p.Hq + hq : 0]);
      const float gk = second_level_scale(p.amax[p.amax_stride + (head ? bseq * p.Hkv + hk : 0)]);
      xs = xs * gq * gk;
    }
    const float2 xs2 = make_float2(xs, xs);
    float m_w = -INFINITY, l_w = 0.0f;
    bool ok = true;
    uint8_t* prow = smem + L::off_p + sw * L::kPBytes + r * 64;
    uint8_t* sfrow = smem + L::off_sfp + sw * L::kSfPBytes + (r % 32) * 16 + (r / 32) * 4;
    const uint32_t scol = tmem + lane_base + kColS0 + 128 * sw;

    for (int j = sw; j < nt; j += 2) {
      const int use = j >> 1;  // use count of S / P buffer sw
      if (!__all_sync(0xffffffffu, wait_bar(bar(B_SFULL + sw), use & 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
      tc_fence_after();
      const int kbase = j * 128;
      const bool need_mask = GENERAL ? ((j * 128 + 128 > si.len_k) || (CAUSAL && j * 128 + 127 > qt * 128 + coff))
                                     : (CAUSAL ? (j == nt - 1) : (j * 128 + 128 > p.seq.Nk));
      // Scores of keys k0 .. k0 + 31 as floats, masked keys -> -inf.
      auto load_mask = [&](uint32_t (&v)[32], int k0) {
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int key = kbase + k0 + i;
            if (GENERAL ? (key >= si.len_k || (CAUSAL && key > qrow + coff))
                        : (key >= p.seq.Nk || (CAUSAL && key > qrow)))
              v[i] = __float_as_uint(-INFINITY);
          }
        }
      };
      auto block_max16 = [&](const uint32_t (&v)[32], int i0) {
        float m0 = max3(__uint_as_float(v[i0]), __uint_as_float(v[i0 + 1]), __uint_as_float(v[i0 + 2]));
#pragma unroll
        for (int i = 3; i < 15; i += 2) m0 = max3(m0, __uint_as_float(v[i0 + i]), __uint_as_float(v[i0 + i + 1]));
        return fmaxf(m0, __uint_as_float(v[i0 + 15]));
      };
      // Pass 1: block maxima of the raw scores (sm_scale > 0, so they order like P~).
      uint32_t sa[32], sb[32];
      float bm[8];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        tmem_ld32(scol + 64 * hh, sa);
        tmem_ld32(scol + 64 * hh + 32, sb);
        tmem_wait_regs(sa);
        tmem_wait_regs(sb);
        load_mask(sa, 64 * hh);
        load_mask(sb, 64 * hh + 32);
        bm[4 * hh] = block_max16(sa, 0);
        bm[4 * hh + 1] = block_max16(sa, 16);
        bm[4 * hh + 2] = block_max16(sb, 0);
        bm[4 * hh + 3] = block_max16(sb, 16);
      }
      const float tm = fmaxf(fmaxf(max3(bm[0], bm[1], bm[2]), max3(bm[3], bm[4], bm[5])), fmaxf(bm[6], bm[7]));
      // A row can see no key of this tile (causal with len_q > len_k, or a mask offset
      // that is not a multiple of 128): it then adds nothing, and its P^ codes are 0.
      const bool empty = GENERAL && tm == -INFINITY;
      const float tmx = tm * xs;
      // Lazy reference maximum: it moves only when the tile maximum exceeds it by more
      // than 8 (log2 units). It cancels in O / l, and P~ is quantized relative to the
      // tile maximum, so it only decides how often l and O are rescaled.
      const bool move = tmx > m_w + 8.0f;  // always true on the first tile (m_w = -inf)
      const float m_new = move ? tmx : m_w;
      const float alpha = move ? ex2_approx(m_w - m_new) : 1.0f;
      const float rfac = empty ? 0.0f : ex2_approx(tmx - m_new);  // rowmax of P~ in this tile (<= 2^8)
      const float tref = empty ? 0.0f : tmx;
      // Per-16 scales of P2 = P~ / s1 = exp2(S*xs - tmx) * 2688 (E4M3 of blockmax / 6).
      uint32_t sfw[2] = {0u, 0u};
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const float amax = ex2_approx(fmaf(bm[b], xs, -tref)) * 2688.0f;
        sfw[b >> 2] |= f32_to_e4m3(amax * (1.0f / 6.0f)) << (8 * (b & 3));
      }
      // P^ buffer sw must be free (PV of tile j - 2 finished).
      if (!__all_sync(0xffffffffu, wait_bar(bar(B_PEMPTY + sw), (use & 1) ^ 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
      float rsum = 0.0f;
      // Codes of keys 32c .. 32c + 31. The division by the decoded block scale is folded
      // into the exp2 argument: v = exp2(S*xs - nb) = P2 / s. A block whose scale rounds
      // to zero keeps the plain exp2 (for the row sum) and gets zero codes.
      auto emit = [&](const uint32_t (&v)[32], int c) {
        uint32_t pw[4];
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const int b = 2 * c + bb;
          const uint32_t sbyte = (sfw[b >> 2] >> (8 * (b & 3))) & 0xFFu;
          float nb = -tref, mult = 1.0f;
          if (sbyte != 0u) {
            const float sdec = e4m3_to_f32(sbyte);
            nb = -(tref + lg2_approx(sdec) - 11.392317422778761f);  // log2(2688)
            mult = sdec * (1.0f / 2688.0f);
          }
          const float2 nb2 = make_float2(nb, nb);
          float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            float e[8];
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
              const int k0 = 16 * bb + 8 * w + 2 * q2;
              const float2 arg = fma2(make_float2(__uint_as_float(v[k0]), __uint_as_float(v[k0 + 1])), xs2, nb2);
              const float2 ee = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
              acc = add2(acc, ee);
              e[2 * q2] = ee.x;
              e[2 * q2 + 1] = ee.y;
            }
            const uint32_t word = f32x8_to_e2m1(e[0], e[1], e[2], e[3], e[4], e[5], e[6], e[7]);
            pw[2 * bb + w] = sbyte != 0u ? word : 0u;
          }
          rsum += (acc.x + acc.y) * mult;
        }
        *reinterpret_cast<uint4*>(prow + ((c ^ ((r >> 1) & 3)) * 16)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      };
      // Pass 2: keys 64-127 are still in registers; keys 0-63 are read again, after
      // which the S buffer goes back to the MMA warp.
      emit(sa, 2);
      emit(sb, 3);
      tmem_ld32(scol, sa);
      tmem_ld32(scol + 32, sb);
      tmem_wait_regs(sa);
      tmem_wait_regs(sb);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_SEMPTY + sw));
      load_mask(sa, 0);
      load_mask(sb, 32);
      emit(sa, 0);
      emit(sb, 1);
      *reinterpret_cast<uint32_t*>(sfrow) = sfw[0];
      *reinterpret_cast<uint32_t*>(sfrow + 512) = sfw[1];
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PFULL + sw));

      // (reference, s1) of this tile for the correction warpgroups.
      if (!__all_sync(0xffffffffu, wait_bar(bar(B_IEMPTY + sw), (use & 1) ^ 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
      info[sw * 128 + r] = make_float2(m_new, rfac * (1.0f / 2688.0f));
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_IFULL + sw));
      l_w = l_w * alpha + rsum * rfac;
      m_w = m_new;
    }
    if (ok) {
      lsum[sw * 128 + r] = make_float2(l_w, m_w);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_LSUM));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool QB>
static int attn_smem_bytes() {
  const int need = Layout<D, QB>::kBytes + 1024;
  // At least 116 KiB so that two CTAs never share an SM (each holds all 512 TMEM columns).
  return need > 116 * 1024 ? need : 116 * 1024;
}

template <int D, bool CAUSAL, int MODE>
static cudaError_t launch_attn_t(const TensorMaps& m, const AttnParams& p, int tiles_q, cudaStream_t stream) {
  const int smem = attn_smem_bytes<D, MODE == 2>();
  cudaError_t e = cudaFuncSetAttribute(attn_fp4_fwd_kernel<D, CAUSAL, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles_q, p.Hq, p.B);
  attn_fp4_fwd_kernel<D, CAUSAL, MODE><<<grid, kAttnThreads, smem, stream>>>(m.q, m.k, m.v, p);
  return cudaGetLastError();
}

// Causal instances (attn_fp4_causal.cu); mode as in launch_attention.
cudaError_t launch_attention_causal(const TensorMaps& m, const AttnParams& p, int tiles_q, int mode,
                                    cudaStream_t stream);

}  // namespace sage
