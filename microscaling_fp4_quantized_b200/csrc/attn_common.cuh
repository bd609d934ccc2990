// Helpers shared by the attention kernels (sm_100a): the bounded mbarrier wait with its
// abort / timeout protocol, the TMEM load wait, and the 16-byte output store.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sage_internal.h"
#include "sm100_ptx.cuh"

namespace sage {
namespace attn {

struct Ctl {
  volatile uint32_t* abort;
  uint32_t* err;
  uint64_t timeout_ns;
};

// Suspend bound of one try_wait for threads that let themselves be suspended while they
// wait.
constexpr uint32_t kSuspendNs = 500;

__device__ __forceinline__ bool try_wait_for(uint32_t bar, uint32_t parity, uint32_t sleep_ns) {
  return sleep_ns != 0u ? mbar_try_wait_sleep(bar, parity, sleep_ns) : mbar_try_wait(bar, parity);
}

// Bounded wait: true when the phase with `parity` has completed, false on abort/timeout.
// sleep_ns != 0 lets the thread stay suspended in each probe for up to that long; the
// abort flag and the clock are read after every probe whose index & check_mask is 0.
// Measured on the FP4 attention kernel: every role waits fastest with plain probes and a
// check every 32nd (1158 against 1100 TFLOP/s with 500 ns suspended probes on long
// non-causal rows, 822 against 781 on causal ones); suspending only the copy and MMA
// warps lost on causal rows.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& c, uint32_t sleep_ns = 0u,
                                         uint32_t check_mask = 0u) {
  if (try_wait_for(bar, parity, sleep_ns)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (try_wait_for(bar, parity, sleep_ns)) return true;
    if ((it & check_mask) != 0u) continue;
    if (*c.abort) return false;
    if (globaltimer_ns() - t0 > c.timeout_ns) {
      *c.abort = 1u;
      atomicOr(c.err, kDevErrTimeout);
      return false;
    }
  }
}

// 32 columns from TMEM, with the wait::ld tied to the registers it produces.
__device__ __forceinline__ void tmem_wait_regs(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// 16 columns from TMEM, with the wait::ld tied to the registers it produces.
__device__ __forceinline__ void tmem_wait_regs16(uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15])
      :
      : "memory");
}

__device__ __forceinline__ void store_out8(void* out, size_t idx, const float* v, int dtype) {
  uint4 w;
  uint32_t* ww = reinterpret_cast<uint32_t*>(&w);
  if (dtype == kDtypeBF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      ww[i] = *reinterpret_cast<uint32_t*>(&h);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
      ww[i] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
  *reinterpret_cast<uint4*>(static_cast<char*>(out) + idx * 2) = w;
}

}  // namespace attn
}  // namespace sage
