// FP4 attention forward for short sequences (sm_100a): the persistent form of the kernel
// in attn_fp4_kernel.cuh. One CTA per SM walks the list of (sequence, query head, query
// tile) work items c, c + gridDim.x, ...; every role derives the same list, the next
// item's copies and products start while the current item's last tiles and epilogue
// finish, and barrier phases follow a CTA-wide count of key tiles and of items (Q is
// double-buffered). This hides the ~5 us start-up and drain a CTA pays per query tile,
// which dominates when a query tile has few key tiles: measured 803 against 727 TFLOP/s
// on B64 H32 N1024 D128, while on long rows it was slower (938 against 1163), so the
// library uses it only for square dense non-causal D = 128 problems of at most
// kShortTiles query tiles. Roles, layouts, arithmetic and waits are those of attn_fp4_kernel.cuh.

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
constexpr uint32_t kRegsSoft = 128;

constexpr int align1k(int x) { return (x + 1023) & ~1023; }

// Tensor-memory column map of the attention kernel.
constexpr uint32_t kColS0 = 0;      // S buffers: 128 columns each, at 0 and 128
constexpr uint32_t kColPV = 256;    // PV accumulator: D columns
constexpr uint32_t kColSfQ = 384;   // + 8 * Q slot; 4 columns per 64-wide K chunk of D
constexpr uint32_t kColSfK = 400;   // + 8 * K stage
constexpr uint32_t kColSfV = 432;   // + 8 * V stage
constexpr uint32_t kColSfP = 464;   // + 8 * P buffer (ends at 480)
// The TMEM regions must not overlap (S buffers, PV, then the scale-factor columns).
static_assert(kColPV >= kColS0 + 2 * 128 && kColSfQ >= kColPV + 128, "TMEM: S / PV regions");
static_assert(kColSfK >= kColSfQ + 16 && kColSfV >= kColSfK + 8 * kKStages &&
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
  // Two Q slots (the next work item's Q^ loads while the current one's S products run),
  // each the Q^ tile and its scales.
  static constexpr int off_q = 0;
  static constexpr int off_sfq = align1k(off_q + kQBytes);
  static constexpr int kQSlotBytes = align1k(off_sfq + kSfQKBytes);
  // K ring slot: K^ tile, its scales, (Q smoothing) the bias operand; V ring slot: V^T
  // tile and its scales.
  static constexpr int st_k = 0;
  static constexpr int st_sfk = align1k(kKBytes);
  static constexpr int st_bias = align1k(st_sfk + kSfQKBytes);
  static constexpr int kKStageBytes = align1k(st_bias + kBiasBytes);
  static constexpr int st_v = 0;
  static constexpr int st_sfv = align1k(kVBytes);
  static constexpr int kVStageBytes = align1k(st_sfv + kSfVBytes);
  static constexpr int off_stage = 2 * kQSlotBytes;  // K ring
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
  B_QFULL = 0,                     // + Q slot
  B_QEMPTY = B_QFULL + 2,          // + Q slot
  B_KFULL = B_QEMPTY + 2,          // + K stage
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
  B_LFULL = B_IEMPTY + 2,         // a work item's row sums from both softmax warpgroups
  B_LEMPTY = B_LFULL + 1,
  B_DRAIN = B_LEMPTY + 1,         // S issuer's last products done
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

// One work item: query tile qt of query head hq of sequence bseq.
struct WorkItem {
  SeqInfo si;
  int bseq, hq, hk, qt, nt, coff;
  int qrow0;         // padded Q row of the tile (TMA coordinate; /128 = its scale tile)
  int ktile0;        // 128-row tile index of key tile 0 of the key/value head
  size_t bias_row0;  // Q-smoothing bias row of (query head, key tile 0)
  bool valid;        // the sequence has this query tile
};

}  // namespace

// MODE 0: square dense, one-level scales; 1: general; 2: general with the Q-smoothing
// score bias. Persistent: CTA c takes work items c, c + gridDim.x, ... of the list
// (sequence, query head, query tile) -- every role walks the same list, so the roles need
// no scheduler between them -- and the next item's copies and products start while the
// current item's last tiles and epilogue finish. Causal items go longest first within a
// head. Barrier phases follow a CTA-wide count of key tiles (gt) and of items.
template <int D, bool CAUSAL, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fp4_persistent_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
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
  const int per_head = p.tiles_q;  // query tiles of the longest sequence
  const int n_items = p.B * p.Hq * per_head;
  if (static_cast<int>(blockIdx.x) >= n_items) return;  // uniform: before any barrier or allocation

  auto decode = [&](int w, WorkItem& it) {
    it.bseq = w / (p.Hq * per_head);
    const int rem = w - it.bseq * p.Hq * per_head;
    it.hq = rem / per_head;
    const int x = rem - it.hq * per_head;
    if (GENERAL) {
      it.si = seq_info(p.seq, it.bseq);
    } else {
      it.si.len_q = p.seq.Nq;
      it.si.len_k = p.seq.Nk;
      it.si.tok_q = it.si.tok_k = 0;
      it.si.prow_q = it.bseq * round128(p.seq.Nq);
      it.si.prow_k = it.bseq * round128(p.seq.Nk);
    }
    const int nqt = (it.si.len_q + 127) >> 7;
    it.valid = x < nqt;
    it.qt = CAUSAL ? (nqt - 1 - x) : x;
    it.hk = it.hq / p.group;
    const int nkt = (it.si.len_k + 127) >> 7;
    it.coff = GENERAL ? it.si.len_k - it.si.len_q : 0;  // causal: query i sees keys j <= i + coff
    it.nt = nkt;                                          // key tiles to visit
    if (CAUSAL) {
      const int last = it.qt * 128 + 127 + it.coff;
      it.nt = last < 0 ? 0 : min(nkt, last / 128 + 1);
    }
    it.qrow0 = p.Hq * it.si.prow_q + it.hq * nqt * 128 + it.qt * 128;
    it.ktile0 = (p.Hkv * it.si.prow_k + it.hk * nkt * 128) >> 7;
    it.bias_row0 = static_cast<size_t>(p.Hq) * it.si.prow_k + static_cast<size_t>(it.hq) * nkt * 128;
  };
  Ctl ctl{misc + 1, p.err, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_QFULL + s), 1);
      mbar_init(bar(B_QEMPTY + s), 1);
    }
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
    mbar_init(bar(B_LFULL), 8);
    mbar_init(bar(B_LEMPTY), kCorrWarps);
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
    // ------------------------------------------------- Q and K producer ----
    regs_decrease<kRegsLow>();
    if (lane == 0 && !(p.debug_flags & kDebugNoLoads)) {
      int gt = 0, qi = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
        WorkItem it;
        decode(w, it);
        if (!it.valid || it.nt == 0) continue;
        const int qs = qi & 1;
        if (!wait_bar(bar(B_QEMPTY + qs), ((qi >> 1) & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
        const uint32_t sq = sbase + L::off_q + qs * L::kQSlotBytes;
        mbar_arrive_expect_tx(bar(B_QFULL + qs), L::kQBytes + L::kSfQKBytes);
        tma_load_2d(sq, &tm_q, 0, it.qrow0, bar(B_QFULL + qs));
        bulk_load(sq + L::off_sfq, p.q_sf + static_cast<size_t>(it.qrow0 >> 7) * L::kSfQKBytes, L::kSfQKBytes,
                  bar(B_QFULL + qs));
        ++qi;
        for (int j = 0; j < it.nt; ++j, ++gt) {
          const int st = gt % kKStages;
          if (!wait_bar(bar(B_KEMPTY + st), ((gt / kKStages) & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          const uint32_t sst = sbase + L::off_stage + st * L::kKStageBytes;
          mbar_arrive_expect_tx(bar(B_KFULL + st), L::kKBytes + L::kSfQKBytes + L::kBiasBytes);
          tma_load_2d(sst + L::st_k, &tm_k, 0, (it.ktile0 + j) * 128, bar(B_KFULL + st));
          bulk_load(sst + L::st_sfk, p.k_sf + static_cast<size_t>(it.ktile0 + j) * L::kSfQKBytes,
                    L::kSfQKBytes, bar(B_KFULL + st));
          if (QBIAS)
            bulk_load(sst + L::st_bias, p.qk_bias + (it.bias_row0 + static_cast<size_t>(j) * 128) * 32,
                      L::kBiasBytes, bar(B_KFULL + st));
        }
      }
      if (*ctl.abort) {
        // Let every copy this thread started land before the CTA releases its memory.
        Ctl drain{misc + 2, p.err, p.timeout_ns};
        misc[2] = 0u;
        for (int k = (qi > 2 ? qi - 2 : 0); k < qi; ++k)
          wait_bar(bar(B_QFULL + (k & 1)), (k >> 1) & 1, drain, kIdleNs, kCheck);
        for (int g = (gt > kKStages ? gt - kKStages : 0); g < gt; ++g)
          wait_bar(bar(B_KFULL + g % kKStages), (g / kKStages) & 1, drain, kIdleNs, kCheck);
      }
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------- V producer ----
    regs_decrease<kRegsLow>();
    if (lane == 0 && !(p.debug_flags & kDebugNoLoads)) {
      int gt = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
        WorkItem it;
        decode(w, it);
        if (!it.valid) continue;
        for (int j = 0; j < it.nt; ++j, ++gt) {
          const int st = gt % kVStages;
          if (!wait_bar(bar(B_VEMPTY + st), ((gt / kVStages) & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          const uint32_t sst = sbase + L::off_vstage + st * L::kVStageBytes;
          mbar_arrive_expect_tx(bar(B_VFULL + st), L::kVBytes + L::kSfVBytes);
          tma_load_2d(sst + L::st_v, &tm_v, 0, (it.ktile0 + j) * D, bar(B_VFULL + st));
          bulk_load(sst + L::st_sfv, p.vt_sf + static_cast<size_t>(it.ktile0 + j) * L::kSfVBytes,
                    L::kSfVBytes, bar(B_VFULL + st));
        }
      }
      if (*ctl.abort) {
        Ctl drain{misc + 4, p.err, p.timeout_ns};
        misc[4] = 0u;
        for (int g = (gt > kVStages ? gt - kVStages : 0); g < gt; ++g)
          wait_bar(bar(B_VFULL + g % kVStages), (g / kVStages) & 1, drain, kIdleNs, kCheck);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- S = Q^ K^^T issuer ----
    regs_decrease<kRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_fp4(128);
      constexpr int kc_qk = D / 64;
      int gt = 0, qi = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
        WorkItem it;
        decode(w, it);
        if (!it.valid || it.nt == 0) continue;
        const int qs = qi & 1;
        const uint32_t sq = sbase + L::off_q + qs * L::kQSlotBytes;
        if (!wait_bar(bar(B_QFULL + qs), (qi >> 1) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < kc_qk; ++c)
          tc_cp_sf(tmem + kColSfQ + 8 * qs + 4 * c, sf_desc(sq + L::off_sfq + 512 * c));
        for (int j = 0; j < it.nt; ++j, ++gt) {
          const int st = gt % kKStages, sb = gt & 1;
          const uint32_t sst = sbase + L::off_stage + st * L::kKStageBytes;
          if (!wait_bar(bar(B_KFULL + st), (gt / kKStages) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          if (!wait_bar(bar(B_SEMPTY + sb), ((gt >> 1) & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          tc_fence_after();
          for (int c = 0; c < kc_qk; ++c)
            tc_cp_sf(tmem + kColSfK + 8 * st + 4 * c, sf_desc(sst + L::st_sfk + 512 * c));
          for (int c = 0; c < kc_qk; ++c)
            tc_mma_fp4(tmem + kColS0 + 128 * sb, qk_desc<D>(sq + 32 * c), qk_desc<D>(sst + L::st_k + 32 * c), idesc_s,
                       tmem + kColSfQ + 8 * qs + 4 * c, tmem + kColSfK + 8 * st + 4 * c, c > 0 ? 1u : 0u);
          if (QBIAS)  // S += ones * bias^T: the Q-smoothing bias of each key, on the tensor core
            tc_mma_bf16(tmem + kColS0 + 128 * sb, make_sdesc(sbase + L::off_ones, 128, 256, kLayoutNone),
                        make_sdesc(sst + L::st_bias, 128, 256, kLayoutNone), make_idesc_bf16(128), 1u);
          tc_commit(bar(B_SFULL + sb));
          tc_commit(bar(B_KEMPTY + st));
        }
        if (!ok) break;
        tc_commit(bar(B_QEMPTY + qs));  // the Q slot returns once this item's S products are done
        ++qi;
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
      int gt = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
        WorkItem it;
        decode(w, it);
        if (!it.valid) continue;
        for (int j = 0; j < it.nt; ++j, ++gt) {
          const int st = gt % kVStages, pb = gt & 1;
          const uint32_t sst = sbase + L::off_vstage + st * L::kVStageBytes;
          if (!wait_bar(bar(B_VFULL + st), (gt / kVStages) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          if (!wait_bar(bar(B_PFULL + pb), (gt >> 1) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          if (!wait_bar(bar(B_PVEMPTY), (gt & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
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
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int gt = 0, itc = 0;
    bool ok = true;
    for (int wi = blockIdx.x; ok && wi < n_items; wi += gridDim.x) {
    WorkItem it;
    decode(wi, it);
    if (!it.valid) continue;
    const int qrow = it.qt * 128 + r;
    float gv = 1.0f;
    if (GENERAL && p.amax != nullptr)
      gv = second_level_scale(p.amax[2 * p.amax_stride + (p.gscale == kGscaleHead ? it.bseq * p.Hkv + it.hk : 0)]);
    float o[DH];
#pragma unroll
    for (int d = 0; d < DH; ++d) o[d] = 0.0f;
    // O is kept relative to 2^m_o; m_o moves (and O is rescaled) only when a tile's
    // reference exceeds it by more than 8, so the factor 2^(e - m_o) stays <= 2^8.
    float m_o = -INFINITY;
    for (int j = 0; j < it.nt; ++j, ++gt) {
      const int w = gt & 1;
      if (!__all_sync(0xffffffffu, wait_bar(bar(B_IFULL + w), (gt >> 1) & 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
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
      if (!__all_sync(0xffffffffu, wait_bar(bar(B_PVFULL), gt & 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
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
    if (!ok) break;
    // The item's row sums: l = sum over the two softmax warpgroups of l_w * 2^(m_w - m_o);
    // a row that saw no key (l = 0) is written as 0.
    if (!__all_sync(0xffffffffu, wait_bar(bar(B_LFULL), itc & 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
    float l = 0.0f;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const float2 e = lsum[w * 128 + r];
      if (e.x > 0.0f) l += e.x * ex2_approx(e.y - m_o);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(B_LEMPTY));
    ++itc;
    if (qrow < it.si.len_q) {
      const float il = l > 0.0f ? gv / l : 0.0f;
      const size_t base = static_cast<size_t>(static_cast<int64_t>(it.bseq) * p.so.b + static_cast<int64_t>(it.hq) * p.so.h +
                                              (static_cast<int64_t>(it.si.tok_q) + qrow) * p.so.n) + DH * cg;
#pragma unroll
      for (int d = 0; d < DH; d += 8) {
        float v8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v8[i] = o[d + i] * il;
        store_out8(p.out, base + d, v8, p.out_dtype);
      }
    }
    }  // work items
  } else {
    // ----------------------------------------------------- softmax (2 x 4 warps) ----
    if constexpr (kRegsSoft > 128) regs_increase<kRegsSoft>();
    const int sw = (warp - 4 - kCorrWarps) >> 2;  // key tiles j = sw, sw + 2, ...
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    uint8_t* prow = smem + L::off_p + sw * L::kPBytes + r * 64;
    uint8_t* sfrow = smem + L::off_sfp + sw * L::kSfPBytes + (r % 32) * 16 + (r / 32) * 4;
    const uint32_t scol = tmem + lane_base + kColS0 + 128 * sw;
    int gt = 0, itc = 0;
    bool ok = true;
    for (int wi = blockIdx.x; ok && wi < n_items; wi += gridDim.x) {
    WorkItem it;
    decode(wi, it);
    if (!it.valid) continue;
    const SeqInfo& si = it.si;
    const int qt = it.qt, nt = it.nt, coff = it.coff;
    const int qrow = qt * 128 + r;
    float xs = p.sm_scale_log2;
    if (GENERAL && p.amax != nullptr) {
      // Second-level scales of Q and K fold into the score scale.
      const bool head = p.gscale == kGscaleHead;
      const float gq = second_level_scale(p.amax[head ? it.bseq * p.Hq + it.hq : 0]);
      const float gk = second_level_scale(p.amax[p.amax_stride + (head ? it.bseq * p.Hkv + it.hk : 0)]);
      xs = xs * gq * gk;
    }
    const float2 xs2 = make_float2(xs, xs);
    float m_w = -INFINITY, l_w = 0.0f;
    const int gt0 = gt;  // CTA-wide index of the item's key tile 0
    gt += nt;
    // This warpgroup takes the item's key tiles whose CTA-wide index has its parity.
    for (int j = (sw - gt0) & 1; j < nt; j += 2) {
      const int use = (gt0 + j) >> 1;  // use count of S / P buffer sw
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
    if (!ok) break;
    // The item's row sum and reference for the correction warpgroup.
    if (!__all_sync(0xffffffffu, wait_bar(bar(B_LEMPTY), (itc & 1) ^ 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
    lsum[sw * 128 + r] = make_float2(l_w, m_w);
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(B_LFULL));
    ++itc;
    }  // work items
  }


  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool QB>
static int persistent_smem_bytes() {
  const int need = Layout<D, QB>::kBytes + 1024;
  // At least 116 KiB so that two CTAs never share an SM (each holds all 512 TMEM columns).
  return need > 116 * 1024 ? need : 116 * 1024;
}

template <int D, bool CAUSAL, int MODE>
static cudaError_t launch_persistent_t(const TensorMaps& m, const AttnParams& p, int tiles_q, cudaStream_t stream) {
  const int smem = persistent_smem_bytes<D, MODE == 2>();
  cudaError_t e = cudaFuncSetAttribute(attn_fp4_persistent_kernel<D, CAUSAL, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // Persistent grid: one CTA per SM (the CTA holds all 512 TMEM columns), at most one
  // per work item.
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  AttnParams q = p;
  q.tiles_q = tiles_q;
  const long long items = static_cast<long long>(p.B) * p.Hq * tiles_q;
  const int grid = static_cast<int>(items < sms ? items : sms);
  attn_fp4_persistent_kernel<D, CAUSAL, MODE><<<grid, kAttnThreads, smem, stream>>>(m.q, m.k, m.v, q);
  return cudaGetLastError();
}

cudaError_t launch_attention_short(const TensorMaps& m, const AttnParams& p, int tiles_q, cudaStream_t stream) {
  return p.D == 64 ? launch_persistent_t<64, false, 0>(m, p, tiles_q, stream)
                   : launch_persistent_t<128, false, 0>(m, p, tiles_q, stream);
}

}  // namespace sage
