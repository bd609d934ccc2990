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
// Work items are (sequence, query head, 128-query tile); key tiles are 128 wide. The grid
// is at most one CTA per SM, and each CTA walks its share of the item list (next_item:
// plain order for non-causal problems, heaviest first and alternating rounds for causal
// ones); every role derives the same list, and barrier phases follow CTA-wide counts of
// key tiles and items, so the next item's copies and products start while the current
// item finishes. Sequences may
// be packed with different lengths, query heads may share key/value heads (head h reads
// key/value head h / (Hq / Hkv)), and the causal mask keeps key j <= i + (len_k - len_q).
//
// Warp roles (16 warps; warp w runs on SM sub-partition w % 4):
//   warp 0      TMA producer of Q^ + scales (two slots) and of the K^ tiles + scales into
//               a 4-stage ring whose slots return as soon as their S product is done.
//   warp 2      TMA producer of the V^T tiles + scales into a 4-stage ring whose slots
//               return when their PV product is done.
//   warp 1      allocates the 512 tensor-memory columns; one thread issues the
//               block-scaled MMAs S = Q^ K^^T (tcgen05 kind::mxf4nvf4, M128 N128 K64)
//               into the S buffer, one key tile g (g = CTA-wide key-tile count) after
//               another as soon as the softmax has read the previous one out.
//   warp 3      one thread issues PV = P^ V^T (N = D) into PV accumulator g % 2. Two
//               issuing threads, so that neither chain of products waits behind the
//               other's dependencies.
//   warps 4-7   correction warpgroup. Thread r owns output row r in FP32 registers and
//               folds every tile's PV row in: O = O * alpha + s1 * 2^(e - m_O) * PV,
//               where e is the reference maximum the tile's softmax used and m_O its own
//               reference.
//   warps 8-15  two softmax warpgroups; warpgroup w takes key tiles g = w (mod 2).
//               Thread r owns query row r of its tiles and holds all 128 scores of it in
//               registers: one read from TMEM, after which the S buffer goes straight
//               back to the MMA warp (the next S product, for the other warpgroup, runs
//               while this one works on its tile). It computes the tile maximum, P~, the per-16 E4M3
//               scales, the P^ codes (written in the swizzled layout the MMA reads) and
//               the row sum relative to its own lazy reference maximum, and hands
//               (reference, s1) to the correction. The two warpgroups never wait for each
//               other: one warpgroup's exp2 phase overlaps the other's TMEM loads, scales
//               and barrier hand-offs.
// Three instances per (D, causal): the general one (packed sequences, len_q != len_k,
// second-level scales: per-sequence lengths, a mask offset, an empty-row guard and a
// score scale read from the device), the general one with the Q-smoothing bias MMA, and
// a lean one for square dense problems with one-level scales, whose loop keeps the score
// scale and the lengths as kernel parameters.
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
using attn::tmem_wait_regs16;
using attn::wait_bar;

constexpr int kKStages = 4;
constexpr int kVStages = 4;
constexpr int kQSlots = 2;
constexpr int kBufs = 2;           // softmax warpgroups = P^ buffers = PV accumulators
constexpr int kCorrWarps = 4;      // warps 4-7
constexpr int kSoftWarps = 4 * kBufs;
constexpr uint32_t kTmemCols = 512;
constexpr int kAttnThreads = 32 * (8 + kSoftWarps);  // 2 producers, 2 issuers, 4 correction, 8 softmax
// Per-thread registers after setmaxnreg. Every SM sub-partition holds one warp of each of
// the four warpgroups; launched at 128, the budget per lane is 4 * 128 = 512 = 32 (copy /
// MMA warpgroup) + 160 (correction: O[128] plus a 16-column PV chunk) + 2 * 160 (softmax:
// the 128 scores of its row plus working registers).
constexpr uint32_t kRegsLow = 32;
constexpr uint32_t kRegsCorr = 160;
constexpr uint32_t kRegsSoft = 160;
static_assert(kRegsLow + kRegsCorr + 2 * kRegsSoft <= 4 * 128, "register split above the launch budget");

constexpr int align1k(int x) { return (x + 1023) & ~1023; }

// Tensor-memory column map: one 128-column S buffer (a softmax warpgroup reads its
// scores out at once and frees it, so the next S product overlaps that warpgroup's
// exponentials), two PV accumulators (the correction folds PV(g) in while PV(g + 1) runs),
// then the scale factors (4 columns per 64-wide K chunk).
constexpr uint32_t kColS = 0;       // 128 columns
constexpr uint32_t kColPV = 128;    // + 128 * accumulator (D columns each)
constexpr uint32_t kColSfQ = 384;   // + 8 * Q slot
constexpr uint32_t kColSfK = 400;   // + 8 * K stage
constexpr uint32_t kColSfV = 432;   // + 8 * V stage
constexpr uint32_t kColSfP = 464;   // + 8 * P buffer (ends at 480)
static_assert(kColPV >= kColS + 128 && kColSfQ >= kColPV + 128 * kBufs, "TMEM: S / PV regions");
static_assert(kColSfK >= kColSfQ + 8 * kQSlots && kColSfV >= kColSfK + 8 * kKStages &&
                  kColSfP >= kColSfV + 8 * kVStages && kColSfP + 8 * kBufs <= kTmemCols,
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
  // Q slot: the Q^ tile and its scales (slot 0 at off_q; off_sfq relative to a slot).
  static constexpr int off_q = 0;
  static constexpr int off_sfq = align1k(kQBytes);
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
  static constexpr int off_stage = kQSlots * kQSlotBytes;  // K ring
  static constexpr int off_vstage = off_stage + kKStages * kKStageBytes;
  static constexpr int off_p = off_vstage + kVStages * kVStageBytes;
  static constexpr int off_sfp = off_p + kBufs * kPBytes;
  static constexpr int off_info = off_sfp + kBufs * kSfPBytes;  // [softmax warpgroup][128] (reference, s1)
  static constexpr int off_lsum = off_info + kBufs * 128 * 8;    // [softmax warpgroup][128] (l, reference)
  static constexpr int off_ones = align1k(off_lsum + kBufs * 128 * 8);
  static constexpr int off_bar = off_ones + kOnesBytes;
  static constexpr int kNumBars = 40;
  static constexpr int off_misc = off_bar + kNumBars * 8;    // tmem base, abort flag, drain flags
  static constexpr int kBytes = off_misc + 32;
  static_assert(kBytes + 1024 <= 227 * 1024, "shared memory above the per-CTA limit");
};

// Barrier indices.
enum : int {
  B_QFULL = 0,                     // + Q slot
  B_QEMPTY = B_QFULL + kQSlots,    // + Q slot
  B_KFULL = B_QEMPTY + kQSlots,    // + K stage
  B_KEMPTY = B_KFULL + kKStages,   // + K stage
  B_VFULL = B_KEMPTY + kKStages,   // + V stage
  B_VEMPTY = B_VFULL + kVStages,   // + V stage
  B_SFULL = B_VEMPTY + kVStages,   // + softmax warpgroup: the S product of its key tile done
                                   //   (one barrier per consumer, so that a parity wait never
                                   //   sees the other warpgroup's phase)
  B_SEMPTY = B_SFULL + kBufs,      // scores read out of the S buffer
  B_PFULL = B_SEMPTY + 1,          // + P buffer: P^ tile and its scales written
  B_PEMPTY = B_PFULL + kBufs,      // + P buffer: its PV product done
  B_PVFULL = B_PEMPTY + kBufs,     // + accumulator: PV product done
  B_PVEMPTY = B_PVFULL + kBufs,    // + accumulator: PV folded into O
  B_IFULL = B_PVEMPTY + kBufs,     // + softmax warpgroup: (reference, s1) of its latest tile
  B_IEMPTY = B_IFULL + kBufs,
  B_LFULL = B_IEMPTY + kBufs,      // an item's row sums from both softmax warpgroups
  B_LEMPTY = B_LFULL + 1,
  B_DRAIN = B_LEMPTY + 1,          // S issuer's last products done
  B_DRAIN2 = B_DRAIN + 1,          // PV issuer's last products done
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

// The walk over the work items: round k hands items kG .. kG + G - 1 to the G CTAs.
// Causal items shrink along the list (heaviest first, see decode_item), so odd rounds go
// in reverse CTA order and every CTA ends with about the same work (measured on the causal
// LLM workload: 1033 against 924 TFLOP/s in plain order). Non-causal items are all alike
// and keep the plain order, which measured faster for them. next_item gets round k + 1 and
// the item of round k; the walk ends at an item >= the item count.
template <bool CAUSAL>
__device__ __forceinline__ int next_item(int k1, int w) {
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  if (!CAUSAL) return w + G;
  return k1 * G + ((k1 & 1) ? G - 1 - c : c);
}

// Item w of the list. Non-causal: query-tile index fastest (consecutive items share their
// key/value head, which keeps its K^ / V^T tiles in L2). Causal: heaviest first over all
// (sequence, head) pairs.
template <bool GENERAL, bool CAUSAL>
__device__ __forceinline__ void decode_item(const AttnParams& p, int w, WorkItem& it) {
  const int per_head = p.tiles_q;
  int bh, x;
  if (CAUSAL) {
    // Causal: the list runs heaviest first over all (sequence, head) pairs -- every pair's
    // last query tile, then every pair's second last, ...
    const int BH = p.B * p.Hq;
    x = w / BH;
    bh = w - x * BH;
  } else {
    bh = w / per_head;
    x = w - bh * per_head;
  }
  it.bseq = bh / p.Hq;
  it.hq = bh - it.bseq * p.Hq;
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
  // Wait policy (see wait_bar): every role polls, and checks the abort flag and the clock
  // on every 32nd probe (measured faster than suspending waits for this kernel: 1158
  // against 1100 TFLOP/s on the long non-causal workload, 822 against 781 causal).
  constexpr uint32_t kIdleNs = 0u;
  constexpr uint32_t kWaitNs = 0u;
  constexpr uint32_t kCheck = 31u;
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
  const int n_items = p.B * p.Hq * p.tiles_q;
  if (static_cast<int>(blockIdx.x) >= n_items) return;  // uniform: before any barrier or allocation
  if (static_cast<int>(gridDim.x) >= n_items) {
    // One item per CTA: a CTA past its sequence's query tiles exits before any set-up.
    WorkItem it;
    decode_item<GENERAL, CAUSAL>(p, blockIdx.x, it);
    if (!it.valid) return;
  }
  Ctl ctl{misc + 1, p.err, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQSlots; ++s) {
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
    mbar_init(bar(B_SEMPTY), 4);
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(bar(B_SFULL + b), 1);
      mbar_init(bar(B_PVFULL + b), 1);
      mbar_init(bar(B_PVEMPTY + b), kCorrWarps);
      mbar_init(bar(B_PFULL + b), 4);
      mbar_init(bar(B_PEMPTY + b), 1);
      mbar_init(bar(B_IFULL + b), 4);
      mbar_init(bar(B_IEMPTY + b), kCorrWarps);
    }
    mbar_init(bar(B_LFULL), kSoftWarps);
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
      for (int k = 0, w = blockIdx.x; ok && w < n_items; ++k, w = next_item<CAUSAL>(k, w)) {
        WorkItem it;
        decode_item<GENERAL, CAUSAL>(p, w, it);
        if (!it.valid || it.nt == 0) continue;
        const int qs = qi % kQSlots;
        if (!wait_bar(bar(B_QEMPTY + qs), ((qi / kQSlots) & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
        if (!SAGE_IN_BOUNDS(static_cast<uint64_t>(it.qrow0) + 128 <= p.lim.rows_q &&
                                static_cast<uint64_t>((it.qrow0 >> 7) + 1) * L::kSfQKBytes <= p.lim.q_sf,
                            p.err, ctl.abort)) { ok = false; break; }
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
          if (!SAGE_IN_BOUNDS(static_cast<uint64_t>(it.ktile0 + j + 1) * 128 <= p.lim.rows_k &&
                                  static_cast<uint64_t>(it.ktile0 + j + 1) * L::kSfQKBytes <= p.lim.k_sf &&
                                  (!QBIAS || (it.bias_row0 + static_cast<size_t>(j + 1) * 128) * 32 <= p.lim.qk_bias),
                              p.err, ctl.abort)) { ok = false; break; }
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
        for (int k = (qi > kQSlots ? qi - kQSlots : 0); k < qi; ++k)
          wait_bar(bar(B_QFULL + k % kQSlots), (k / kQSlots) & 1, drain, kIdleNs, kCheck);
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
      for (int k = 0, w = blockIdx.x; ok && w < n_items; ++k, w = next_item<CAUSAL>(k, w)) {
        WorkItem it;
        decode_item<GENERAL, CAUSAL>(p, w, it);
        if (!it.valid) continue;
        for (int j = 0; j < it.nt; ++j, ++gt) {
          const int st = gt % kVStages;
          if (!wait_bar(bar(B_VEMPTY + st), ((gt / kVStages) & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          const uint32_t sst = sbase + L::off_vstage + st * L::kVStageBytes;
          if (!SAGE_IN_BOUNDS(static_cast<uint64_t>(it.ktile0 + j + 1) * D <= p.lim.rows_v &&
                                  static_cast<uint64_t>(it.ktile0 + j + 1) * L::kSfVBytes <= p.lim.vt_sf,
                              p.err, ctl.abort)) { ok = false; break; }
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
      for (int k = 0, w = blockIdx.x; ok && w < n_items; ++k, w = next_item<CAUSAL>(k, w)) {
        WorkItem it;
        decode_item<GENERAL, CAUSAL>(p, w, it);
        if (!it.valid || it.nt == 0) continue;
        const int qs = qi % kQSlots;
        const uint32_t sq = sbase + L::off_q + qs * L::kQSlotBytes;
        if (!wait_bar(bar(B_QFULL + qs), (qi / kQSlots) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < kc_qk; ++c)
          tc_cp_sf(tmem + kColSfQ + 8 * qs + 4 * c, sf_desc(sq + L::off_sfq + 512 * c));
        for (int j = 0; j < it.nt; ++j, ++gt) {
          const int st = gt % kKStages;
          const uint32_t sst = sbase + L::off_stage + st * L::kKStageBytes;
          const uint32_t dst = tmem + kColS;
          if (!wait_bar(bar(B_KFULL + st), (gt / kKStages) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          tc_fence_after();
          for (int c = 0; c < kc_qk; ++c)
            tc_cp_sf(tmem + kColSfK + 8 * st + 4 * c, sf_desc(sst + L::st_sfk + 512 * c));
          if (!wait_bar(bar(B_SEMPTY), (gt & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          tc_fence_after();
          for (int c = 0; c < kc_qk; ++c)
            tc_mma_fp4(dst, qk_desc<D>(sq + 32 * c), qk_desc<D>(sst + L::st_k + 32 * c), idesc_s,
                       tmem + kColSfQ + 8 * qs + 4 * c, tmem + kColSfK + 8 * st + 4 * c, c > 0 ? 1u : 0u);
          if (QBIAS)  // S += ones * bias^T: the Q-smoothing bias of each key, on the tensor core
            tc_mma_bf16(dst, make_sdesc(sbase + L::off_ones, 128, 256, kLayoutNone),
                        make_sdesc(sst + L::st_bias, 128, 256, kLayoutNone), make_idesc_bf16(128), 1u);
          tc_commit(bar(B_SFULL + gt % kBufs));
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
      for (int k = 0, w = blockIdx.x; ok && w < n_items; ++k, w = next_item<CAUSAL>(k, w)) {
        WorkItem it;
        decode_item<GENERAL, CAUSAL>(p, w, it);
        if (!it.valid) continue;
        for (int j = 0; j < it.nt; ++j, ++gt) {
          const int st = gt % kVStages, b = gt % kBufs;
          const uint32_t sst = sbase + L::off_vstage + st * L::kVStageBytes;
          // The scale factors go to their own TMEM columns as soon as they are in shared
          // memory (the products that used those columns before are done: the V slot and
          // the P^ buffer were released by them); only the MMAs wait for the accumulator.
          if (!wait_bar(bar(B_VFULL + st), (gt / kVStages) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          tc_fence_after();
          for (int c = 0; c < 2; ++c) tc_cp_sf(tmem + kColSfV + 8 * st + 4 * c, sf_desc(sst + L::st_sfv + 512 * c));
          if (!wait_bar(bar(B_PFULL + b), (gt / kBufs) & 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          tc_fence_after();
          for (int c = 0; c < 2; ++c)
            tc_cp_sf(tmem + kColSfP + 8 * b + 4 * c, sf_desc(sbase + L::off_sfp + b * L::kSfPBytes + 512 * c));
          if (!wait_bar(bar(B_PVEMPTY + b), ((gt / kBufs) & 1) ^ 1, ctl, kIdleNs, kCheck)) { ok = false; break; }
          tc_fence_after();
          for (int c = 0; c < 2; ++c)
            tc_mma_fp4(tmem + kColPV + 128 * b, row64_desc(sbase + L::off_p + b * L::kPBytes + 32 * c),
                       row64_desc(sst + L::st_v + 32 * c), idesc_pv, tmem + kColSfP + 8 * b + 4 * c,
                       tmem + kColSfV + 8 * st + 4 * c, c > 0 ? 1u : 0u);
          tc_commit(bar(B_PVFULL + b));
          tc_commit(bar(B_PEMPTY + b));
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
    const int quad = warp & 3;       // TMEM lane quarter = rows 32*quad ..
    const int r = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int gt = 0, itc = 0;
    bool ok = true;
    for (int k = 0, wi = blockIdx.x; ok && wi < n_items; ++k, wi = next_item<CAUSAL>(k, wi)) {
      WorkItem it;
      decode_item<GENERAL, CAUSAL>(p, wi, it);
      if (!it.valid) continue;
      const int qrow = it.qt * 128 + r;
      float o[D];
#pragma unroll
      for (int d = 0; d < D; ++d) o[d] = 0.0f;
      // O is kept relative to 2^m_o; m_o moves (and O is rescaled) only when a tile's
      // reference exceeds it by more than 8, so the factor 2^(e - m_o) stays <= 2^8.
      float m_o = -INFINITY;
      for (int j = 0; j < it.nt; ++j, ++gt) {
        const int b = gt % kBufs, ph = (gt / kBufs) & 1;
        if (!__all_sync(0xffffffffu, wait_bar(bar(B_IFULL + b), ph, ctl, kWaitNs, kCheck))) { ok = false; break; }
        const float2 f = info[b * 128 + r];  // (reference e, s1) of tile j for this row
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_IEMPTY + b));
        float alpha = 1.0f, c = 0.0f;
        if (f.y > 0.0f) {  // s1 = 0: the row saw no key of this tile
          if (f.x > m_o + 8.0f) {
            alpha = ex2_approx(m_o - f.x);  // 0 on the first contribution (m_o = -inf)
            m_o = f.x;
          }
          c = f.y * ex2_approx(f.x - m_o);
        }
        if (!__all_sync(0xffffffffu, wait_bar(bar(B_PVFULL + b), ph, ctl, kWaitNs, kCheck))) { ok = false; break; }
        tc_fence_after();
        const bool unit = __all_sync(0xffffffffu, alpha == 1.0f);
        const float2 c2 = make_float2(c, c), a2 = make_float2(alpha, alpha);
        // 16-column chunks, the next chunk's load in flight while this one is folded in.
        uint32_t v[2][16];
        const uint32_t pvcol = tmem + lane_base + kColPV + 128 * b;
        tmem_ld16(pvcol, v[0]);
#pragma unroll
        for (int cc = 0; cc < D / 16; ++cc) {
          tmem_wait_regs16(v[cc & 1]);
          if (cc + 1 < D / 16) tmem_ld16(pvcol + 16 * (cc + 1), v[(cc + 1) & 1]);
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            float2 acc = make_float2(o[16 * cc + i], o[16 * cc + i + 1]);
            if (!unit) acc = mul2(acc, a2);
            acc = fma2(make_float2(__uint_as_float(v[cc & 1][i]), __uint_as_float(v[cc & 1][i + 1])), c2, acc);
            o[16 * cc + i] = acc.x;
            o[16 * cc + i + 1] = acc.y;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PVEMPTY + b));
      }
      if (!ok) break;
      // The item's row sums: l = sum over the softmax warpgroups of l_w * 2^(m_w - m_o);
      // a row that saw no key (l = 0) is written as 0.
      if (!__all_sync(0xffffffffu, wait_bar(bar(B_LFULL), itc & 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
      float l = 0.0f;
#pragma unroll
      for (int w = 0; w < kBufs; ++w) {
        const float2 e = lsum[w * 128 + r];
        if (e.x > 0.0f) l += e.x * ex2_approx(e.y - m_o);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_LEMPTY));
      ++itc;
      if (qrow < it.si.len_q) {
        float gv = 1.0f;
        if (GENERAL && p.amax != nullptr)
          gv = second_level_scale(p.amax[2 * p.amax_stride + (p.gscale == kGscaleHead ? it.bseq * p.Hkv + it.hk : 0)]);
        const float il = l > 0.0f ? gv / l : 0.0f;
        const size_t base = static_cast<size_t>(static_cast<int64_t>(it.bseq) * p.so.b +
                                                static_cast<int64_t>(it.hq) * p.so.h +
                                                (static_cast<int64_t>(it.si.tok_q) + qrow) * p.so.n);
#pragma unroll
        for (int d = 0; d < D; d += 8) {
          float v8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) v8[i] = o[d + i] * il;
          if (SAGE_IN_BOUNDS(base + d + 8 <= p.lim.o_el, p.err, nullptr)) store_out8(p.out, base + d, v8, p.out_dtype);
        }
      }
    }  // work items
  } else {
    // ----------------------------------------------------- softmax (2 x 4 warps) ----
    regs_increase<kRegsSoft>();
    const int sw = (warp - 4 - kCorrWarps) >> 2;  // key tiles g = sw (mod 2)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t scol = tmem + lane_base + kColS;
    uint8_t* prow = smem + L::off_p + sw * L::kPBytes + r * 64;
    uint8_t* sfrow = smem + L::off_sfp + sw * L::kSfPBytes + (r % 32) * 16 + (r / 32) * 4;
    int gt = 0, itc = 0;
    bool ok = true;
    for (int k = 0, wi = blockIdx.x; ok && wi < n_items; ++k, wi = next_item<CAUSAL>(k, wi)) {
      WorkItem it;
      decode_item<GENERAL, CAUSAL>(p, wi, it);
      if (!it.valid) continue;
      const int qt = it.qt, nt = it.nt, coff = it.coff;
      const int len_k = it.si.len_k;
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
      // This warpgroup takes the item's key tiles whose CTA-wide index is sw mod 2.
      for (int j = (sw - gt0 % kBufs + kBufs) % kBufs; j < nt; j += kBufs) {
        const int use = (gt0 + j) / kBufs;  // this warpgroup's tile count (S-full / P^ buffer phases)
        if (!__all_sync(0xffffffffu, wait_bar(bar(B_SFULL + sw), use & 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
        tc_fence_after();
        const int kbase = j * 128;
        const bool need_mask = GENERAL ? ((kbase + 128 > len_k) || (CAUSAL && kbase + 127 > qt * 128 + coff))
                                       : (CAUSAL ? (j == nt - 1) : (kbase + 128 > p.seq.Nk));
        // The row's 128 scores, read once; masked keys -> -inf.
        uint32_t sv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(scol + 32 * c, sv[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_wait_regs(sv[c]);
        // Every score is in registers: the S buffer goes back to the MMA warp.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_SEMPTY));
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int key = kbase + 32 * c + i;
              if (GENERAL ? (key >= len_k || (CAUSAL && key > qrow + coff))
                          : (key >= p.seq.Nk || (CAUSAL && key > qrow)))
                sv[c][i] = __float_as_uint(-INFINITY);
            }
        }
        // Block maxima of the raw scores (sm_scale > 0, so they order like P~).
        float bm[8];
#pragma unroll
        for (int bb = 0; bb < 8; ++bb) {
          const uint32_t* v = &sv[bb >> 1][16 * (bb & 1)];
          float m0 = max3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
          for (int i = 3; i < 15; i += 2) m0 = max3(m0, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
          bm[bb] = fmaxf(m0, __uint_as_float(v[15]));
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
        // Per-16 scales of P2 = P~ / s1 = exp2(S*xs - tmx) * 2688: the E4M3 byte of
        // blockmax / 6 = exp2(bm*xs - tmx + log2(448)), two blocks per conversion.
        uint32_t sfw[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t w4[2];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int b0 = 4 * h + 2 * q;
            const float a0 = ex2_approx(fmaf(bm[b0], xs, 8.807354922057604f - tref));  // log2(448)
            const float a1 = ex2_approx(fmaf(bm[b0 + 1], xs, 8.807354922057604f - tref));
            w4[q] = f32x2_to_e4m3x2(a0, a1);
          }
          sfw[h] = w4[0] | (w4[1] << 16);
        }
        // P^ buffer sw must be free (PV of tile g - 2 finished).
        if (!__all_sync(0xffffffffu, wait_bar(bar(B_PEMPTY + sw), (use & 1) ^ 1, ctl, kWaitNs, kCheck))) { ok = false; break; }
        float rsum = 0.0f;
        // Codes of keys 32c .. 32c + 31. The division by the decoded block scale is folded
        // into the exp2 argument: v = exp2(S*xs - nb) = P2 / s. A block whose scale rounds
        // to zero keeps the plain exp2 (for the row sum); its v = P2 / 2688 stays below
        // 2^-18, so its codes are 0 as the method's are.
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t* v = sv[c];
          uint32_t pw[4];
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            const int blk = 2 * c + bb;
            const uint32_t sbyte = (sfw[blk >> 2] >> (8 * (blk & 3))) & 0xFFu;
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
              pw[2 * bb + w] = f32x8_to_e2m1(e[0], e[1], e[2], e[3], e[4], e[5], e[6], e[7]);
            }
            rsum += (acc.x + acc.y) * mult;
          }
          *reinterpret_cast<uint4*>(prow + ((c ^ ((r >> 1) & 3)) * 16)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        }
        *reinterpret_cast<uint32_t*>(sfrow) = sfw[0];
        *reinterpret_cast<uint32_t*>(sfrow + 512) = sfw[1];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PFULL + sw));
        // (reference, s1) of this tile for the correction warpgroup.
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
static int attn_smem_bytes() {
  const int need = Layout<D, QB>::kBytes + 1024;
  // At least 116 KiB so that two CTAs never share an SM (each holds all 512 TMEM columns).
  return need > 116 * 1024 ? need : 116 * 1024;
}

// Grid: the smaller of the item count and `max_ctas`, every CTA walking its share.
template <int D, bool CAUSAL, int MODE>
static cudaError_t launch_attn_t(const TensorMaps& m, const AttnParams& p, int tiles_q, int max_ctas,
                                 cudaStream_t stream) {
  const int smem = attn_smem_bytes<D, MODE == 2>();
  cudaError_t e = cudaFuncSetAttribute(attn_fp4_fwd_kernel<D, CAUSAL, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  AttnParams q = p;
  q.tiles_q = tiles_q;
  const long long items = static_cast<long long>(p.B) * p.Hq * tiles_q;
  const int grid = static_cast<int>(max_ctas > 0 && items > max_ctas ? max_ctas : items);
  attn_fp4_fwd_kernel<D, CAUSAL, MODE><<<grid, kAttnThreads, smem, stream>>>(m.q, m.k, m.v, q);
  return cudaGetLastError();
}

// Causal instances (attn_fp4_causal.cu); mode as in launch_attention.
cudaError_t launch_attention_causal(const TensorMaps& m, const AttnParams& p, int tiles_q, int mode, int max_ctas,
                                    cudaStream_t stream);

}  // namespace sage
