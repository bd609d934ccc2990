// FP4 attention forward (sm_100a): the non-causal instances of the kernel template in
// attn_fp4_kernel.cuh, the launch dispatch, and the S = Q^ K^^T check kernel. The causal
// instances live in their own translation unit (attn_fp4_causal.cu), which keeps the two
// sets of instances compiling in parallel.
#include "attn_fp4_kernel.cuh"

namespace sage {

namespace {

template <int D>
cudaError_t launch_attn_full_d(const TensorMaps& m, const AttnParams& p, int tiles_q, int mode, int max_ctas,
                               cudaStream_t stream) {
  if (mode == 2) return launch_attn_t<D, false, 2>(m, p, tiles_q, max_ctas, stream);
  if (mode == 1) return launch_attn_t<D, false, 1>(m, p, tiles_q, max_ctas, stream);
  return launch_attn_t<D, false, 0>(m, p, tiles_q, max_ctas, stream);
}

}  // namespace

cudaError_t launch_attention(const TensorMaps& m, const AttnParams& p, int tiles_q, cudaStream_t stream) {
  if (p.B == 0 || p.Hq == 0 || tiles_q == 0) return cudaSuccess;
  // The general instance serves packed sequences, Nq != Nk and second-level scales, the
  // third one adds the Q-smoothing bias; a square dense problem with one-level scales
  // gets the leaner loop (constant score scale, no mask offset, no empty-row guard).
  const bool general = p.seq.cu_q != nullptr || p.seq.Nq != p.seq.Nk || p.amax != nullptr;
  const int mode = p.qk_bias != nullptr ? 2 : (general ? 1 : 0);
  // One CTA per SM walks the work items: the next item's loads and products start while
  // the current one drains, so no item pays a CTA's start-up (measured against one CTA
  // per item: +10 % on B1 H16 N4096 D128, +4.5-6 % on causal rows, equal on N = 32768).
  int max_ctas = 0;
  {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&max_ctas, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  if (p.causal) return launch_attention_causal(m, p, tiles_q, mode, max_ctas, stream);
  return p.D == 64 ? launch_attn_full_d<64>(m, p, tiles_q, mode, max_ctas, stream)
                   : launch_attn_full_d<128>(m, p, tiles_q, mode, max_ctas, stream);
}

// S = sm_scale * Q^ K^^T for one (query tile, key tile, head): the QK^T stage alone.
template <int D>
__global__ void __launch_bounds__(192, 1)
    qk_scores_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const AttnParams p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  // Reuse the attention layout: Q tile at off_q, K tile in stage 0.
  const uint32_t bar_full = sbase + L::off_bar, bar_mma = bar_full + 8;
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + L::off_misc);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nqt = p.Np / 128;
  const int qt = blockIdx.x, kt = blockIdx.y, bh = blockIdx.z;
  Ctl ctl{misc + 1, p.err, p.timeout_ns};
  constexpr uint32_t kCols = 256;
  if (threadIdx.x == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_mma, 1);
    misc[1] = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::off_misc, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const uint32_t sk = sbase + L::off_stage;
  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_full, L::kQBytes + L::kKBytes + 2 * L::kSfQKBytes);
      tma_load_2d(sbase + L::off_q, &tm_q, 0, bh * p.Np + qt * 128, bar_full);
      tma_load_2d(sk + L::st_k, &tm_k, 0, bh * p.Np + kt * 128, bar_full);
      bulk_load(sbase + L::off_sfq, p.q_sf + (static_cast<size_t>(bh) * nqt + qt) * L::kSfQKBytes, L::kSfQKBytes, bar_full);
      bulk_load(sk + L::st_sfk, p.k_sf + (static_cast<size_t>(bh) * nqt + kt) * L::kSfQKBytes, L::kSfQKBytes, bar_full);
      Ctl drain{misc + 2, p.err, p.timeout_ns};
      misc[2] = 0u;
      wait_bar(bar_full, 0, drain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (wait_bar(bar_full, 0, ctl)) {
        tc_fence_after();
        constexpr int kc = D / 64;
        for (int c = 0; c < kc; ++c) {
          tc_cp_sf(tmem + 128 + 4 * c, sf_desc(sbase + L::off_sfq + 512 * c));
          tc_cp_sf(tmem + 144 + 4 * c, sf_desc(sk + L::st_sfk + 512 * c));
        }
        for (int c = 0; c < kc; ++c)
          tc_mma_fp4(tmem, qk_desc<D>(sbase + L::off_q + 32 * c), qk_desc<D>(sk + L::st_k + 32 * c),
                     make_idesc_fp4(128), tmem + 128 + 4 * c, tmem + 144 + 4 * c, c > 0 ? 1u : 0u);
      }
      tc_commit(bar_mma);
    }
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const bool ready = wait_bar(bar_mma, 0, ctl) && !*ctl.abort;
    if (__all_sync(0xffffffffu, ready)) {
      tc_fence_after();
      float* out = static_cast<float*>(p.out) + (static_cast<size_t>(bh) * p.Np + qt * 128 + r) * p.Np + kt * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + 32 * c, v);
        tmem_wait_regs(v);
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(out + 32 * c + i) =
              make_float4(__uint_as_float(v[i]) * p.sm_scale, __uint_as_float(v[i + 1]) * p.sm_scale,
                          __uint_as_float(v[i + 2]) * p.sm_scale, __uint_as_float(v[i + 3]) * p.sm_scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

template <int D>
static cudaError_t launch_scores_t(const TensorMaps& m, const AttnParams& p, cudaStream_t stream) {
  const int smem = Layout<D>::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(qk_scores_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.Np / 128, p.Np / 128, p.BH);
  qk_scores_kernel<D><<<grid, 192, smem, stream>>>(m.q, m.k, p);
  return cudaGetLastError();
}

cudaError_t launch_qk_scores(const TensorMaps& m, const AttnParams& p, cudaStream_t stream) {
  if (p.BH == 0 || p.Np == 0) return cudaSuccess;
  return p.D == 64 ? launch_scores_t<64>(m, p, stream) : launch_scores_t<128>(m, p, stream);
}

}  // namespace sage
