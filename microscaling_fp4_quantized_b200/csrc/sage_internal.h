// Internal launch interfaces of the CUDA library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace sage {

enum : int { kDtypeBF16 = 0, kDtypeF16 = 1 };

// Bits of the device error word.
enum : uint32_t { kDevErrTimeout = 1u };

struct QuantParams {
  const void* q;
  const void* k;
  const void* v;
  int dtype;
  int BH, N, Np, D;
  int smooth_k;
  int nsplit;  // number of 512-token chunks of the K mean
  uint8_t* q_fp4;
  uint8_t* q_sf;
  uint8_t* k_fp4;
  uint8_t* k_sf;
  uint8_t* vt_fp4;
  uint8_t* vt_sf;
  float* k_mean;
  double* partial;  // [BH, nsplit, D]
};

struct AttnParams {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* vt_sf;
  void* out;            // [BH, N, D] (attention) or float [BH, Np, Np] (scores)
  int out_dtype;
  int BH, N, Np, D;
  int causal;
  float sm_scale;       // scale of the dot products
  float sm_scale_log2;  // sm_scale * log2(e)
  uint32_t* err;        // device error word
  uint64_t timeout_ns;  // bound on every wait
  uint32_t debug_flags; // kDebugNoLoads: the producer issues no copies (test of the error path)
};

enum : uint32_t { kDebugNoLoads = 1u };

struct TensorMaps {
  CUtensorMap q, k, v;
};

cudaError_t launch_quantize(const QuantParams& p, cudaStream_t stream);
cudaError_t launch_attention(const TensorMaps& maps, const AttnParams& p, cudaStream_t stream);
cudaError_t launch_qk_scores(const TensorMaps& maps, const AttnParams& p, cudaStream_t stream);

}  // namespace sage
