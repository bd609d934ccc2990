// FP4 attention forward (sm_100a): the causal instances of the kernel template in
// attn_fp4_kernel.cuh (a translation unit of their own; see attn_fp4_fwd.cu).
#include "attn_fp4_kernel.cuh"

namespace sage {

namespace {

template <int D>
cudaError_t launch_attn_causal_d(const TensorMaps& m, const AttnParams& p, int tiles_q, int mode, int max_ctas,
                                 cudaStream_t stream) {
  if (mode == 2) return launch_attn_t<D, true, 2>(m, p, tiles_q, max_ctas, stream);
  if (mode == 1) return launch_attn_t<D, true, 1>(m, p, tiles_q, max_ctas, stream);
  return launch_attn_t<D, true, 0>(m, p, tiles_q, max_ctas, stream);
}

}  // namespace

cudaError_t launch_attention_causal(const TensorMaps& m, const AttnParams& p, int tiles_q, int mode, int max_ctas,
                                    cudaStream_t stream) {
  return p.D == 64 ? launch_attn_causal_d<64>(m, p, tiles_q, mode, max_ctas, stream)
                   : launch_attn_causal_d<128>(m, p, tiles_q, mode, max_ctas, stream);
}

}  // namespace sage
