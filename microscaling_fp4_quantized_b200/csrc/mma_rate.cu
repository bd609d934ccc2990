// Throughput probe of the block-scaled FP4 tensor-core instruction that the attention
// kernel issues for both of its contractions ("FP4 Tensor Cores in Blackwell GPUs",
// SageAttention3 abstract): tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16
// with M = 128, N = 64 or 128 and K = 64 per instruction, E2M1 operands and UE4M3 scales.
//
// One CTA per SM (the dynamic shared memory keeps a second one off the SM). Thread 0
// issues `iters` products back to back from operands resident in shared memory into two
// TMEM accumulators used alternately, commits once, and waits (bounded) for completion.
// The host times the launch with CUDA events; ops = 2 * 128 * N * 64 * iters * CTAs.
// The operand bytes are a fixed hash (no zero data path); every scale is 1.0.
#include <cuda_runtime.h>

#include <cstdint>

#include "attn_common.cuh"
#include "sage_internal.h"
#include "sm100_ptx.cuh"

namespace sage {

namespace {

constexpr int kRateThreads = 128;
constexpr uint32_t kRateCols = 512;
constexpr int kRateSmem = 120 * 1024;  // > half of an SM's shared memory: one CTA per SM

__global__ void __launch_bounds__(kRateThreads, 1)
    mma_rate_kernel(int n, int iters, uint32_t* err, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // A: 128 rows x 32 bytes; B: n rows x 32 bytes; scale blocks of 512 bytes each.
  constexpr int off_a = 0, off_b = 4096, off_sfa = 12288, off_sfb = 13312, off_bar = 14336, off_misc = 14400;
  const uint32_t sbase = smem_u32(smem);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + off_misc);
  for (int i = threadIdx.x; i < off_sfa / 4; i += kRateThreads) {
    uint32_t h = static_cast<uint32_t>(i) * 2654435761u;
    h ^= h >> 15;
    reinterpret_cast<uint32_t*>(smem)[i] = h * 2246822519u;
  }
  for (int i = threadIdx.x; i < 2048 / 4; i += kRateThreads)
    reinterpret_cast<uint32_t*>(smem + off_sfa)[i] = 0x38383838u;  // UE4M3 1.0
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(sbase + off_bar, 1);
    misc[1] = 0u;
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(sbase + off_misc, kRateCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  if (threadIdx.x == 0) {
    const uint32_t idesc = make_idesc_fp4(static_cast<uint32_t>(n));
    const uint64_t adesc = make_sdesc(sbase + off_a, 16, 256, kLayoutSw32);
    const uint64_t bdesc = make_sdesc(sbase + off_b, 16, 256, kLayoutSw32);
    const uint32_t sfa = tmem + 256, sfb = tmem + 264;
    tc_cp_sf(sfa, make_sdesc(sbase + off_sfa, 0, 128, kLayoutNone));
    tc_cp_sf(sfb, make_sdesc(sbase + off_sfb, 0, 128, kLayoutNone));
    for (int i = 0; i < iters; ++i)
      tc_mma_fp4(tmem + 128u * static_cast<uint32_t>(i & 1), adesc, bdesc, idesc, sfa, sfb, i >= 2 ? 1u : 0u);
    tc_commit(sbase + off_bar);
    attn::Ctl ctl{misc + 1, err, timeout_ns};
    attn::wait_bar(sbase + off_bar, 0, ctl, attn::kSuspendNs);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, kRateCols);
  }
}

}  // namespace

cudaError_t launch_mma_rate(int n, int iters, int ctas, uint32_t* err, uint64_t timeout_ns, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRateSmem);
  if (e != cudaSuccess) return e;
  mma_rate_kernel<<<ctas, kRateThreads, kRateSmem, stream>>>(n, iters, err, timeout_ns);
  return cudaGetLastError();
}

}  // namespace sage
