/*
 * sage_fp4.h -- C ABI of the B200 (sm_100a) microscaling-FP4 attention forward.
 *
 * The operation (SageAttention3, "Microscaling FP4 Attention for Inference ...",
 * arXiv 2505.11594, abstract: plug-and-play FP4 attention on Blackwell FP4 tensor cores):
 *
 *   O = softmax(sm_scale * Q K^T [+ causal mask]) V        per (batch, head)
 *
 * computed as:
 *   1. K smoothing: K' = K - mean_over_tokens(K) per (b, h, channel)  (SageAttention
 *      OpenReview thread, reply to W1, "smoothing K"; softmax is invariant to it).
 *   2. Q, K', V quantized to FP4 E2M1 with one unsigned E4M3 scale per 16 consecutive
 *      elements (Q and K' along the head dimension, V along tokens).
 *   3. S = Q^ K^^T as a block-scaled FP4 tensor-core contraction (FP32 accumulate),
 *      FlashAttention tiling with the online softmax m/d recurrence (same thread, reply
 *      to Q3), diag(l)^-1 applied after the last key tile (reply to Q2).
 *   4. P~ quantized with two-level scaling: a per-row factor s1 = rowmax(P~)/(448*6)
 *      per key tile, then the same 16-element E4M3/E2M1 rule; P^ V^ as a second
 *      block-scaled FP4 contraction, accumulated in FP32.
 *   5. Optional (sage_fp4_problem_t.gscale): a second-level FP32 scale per tensor or per
 *      (sequence, head) for Q, K' and V, NVFP4's per-tensor factor (named on the author
 *      page, "TetraJet-v2" abstract: double-block quantization for NVFP4), applied the
 *      way step 4 scales P~: g = amax / (448*6), the 16-element rule runs on x / g, and
 *      g is folded back into the scores (Q, K) and the output (V).
 *   6. Optional (sage_fp4_problem_t.smooth_q): smoothing Q (SageAttention2 abstract on the
 *      author page), read as the counterpart of step 1: Q' = Q - mean_over_tokens(Q) is
 *      quantized, and the removed part returns as a per-key score bias mu_q . K' computed
 *      from the unquantized smoothed keys (one FP32 add per score).
 *
 * Conventions for every entry point
 *   - Tensors are device pointers unless stated; the caller owns all memory. The
 *     library keeps no per-call state and never frees caller memory.
 *   - Dense entry points: Q, K, V, O are [B, H, N, D] contiguous, element type bf16 or
 *     fp16 (sage_dtype_t). sage_fp4_problem_t describes the general case: any token /
 *     head / batch strides, packed variable-length sequences, key/value heads shared by
 *     groups of query heads, and query and key lengths that differ.
 *   - D must be 64 or 128; B, H, N >= 0 (any zero gives an empty problem: SAGE_OK,
 *     nothing launched); N need not be a multiple of anything.
 *   - Causal masking keeps key j for query i when j <= i + (len_k - len_q): the last
 *     query sees the last key (with len_q == len_k, j <= i). A query that sees no key
 *     (or a sequence with no keys) gets an output row of zeros.
 *   - All pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call is
 *     asynchronous on it; argument errors are returned before anything is launched.
 *   - sm_scale <= 0 selects 1/sqrt(D).
 *   - No C++ exception crosses this boundary.
 *   - Every wait inside the kernels is bounded (default 2 s). A wait that runs out sets
 *     a device error word, the kernel drains its own copies, frees its tensor memory
 *     and returns; sage_fp4_get_device_error() reports it (SAGE_ERR_TIMEOUT).
 *
 * Quantized layouts. Every sequence is padded to a multiple of 128 tokens (padding
 * tokens quantize as zeros). For the dense [B, H, N, D] entry points let Np = N rounded
 * up to 128; the padded row of (batch b, head h, token n) is then (b*H + h)*Np + n.
 * In general (sage_fp4_problem_t) the padded row of query (sequence b, head h, token n)
 * is  Hq * P_b + h * round128(len_q(b)) + n,  where P_b is the sum of round128(len_q)
 * over the sequences before b (b * round128(Nq) for dense problems); keys use Hkv,
 * len_k and their own P_b. A "tile" is 128 consecutive padded rows: tile t = row / 128.
 *   q_fp4, k_fp4 : [rows, D/2] bytes. Byte j of a row holds elements 2j (low nibble)
 *                  and 2j+1 (high nibble). E2M1 code = sign<<3 | magnitude.
 *   vt_fp4       : [key tiles, D, 64] bytes: V transposed per key tile; byte j of row d
 *                  of tile t holds tokens 128t + 2j (low nibble) and 128t + 2j + 1.
 *   q_sf, k_sf   : [tiles, D/64, 512] bytes, the tensor-core scale-factor tiling. The
 *                  scale of (row r, channels 16c..16c+15) is at
 *                    ((r/128) * (D/64) + (16c)/64) * 512 + (r%32)*16 + ((r%128)/32)*4 + c%4
 *   vt_sf        : [key tiles, 2, 512] bytes. The scale of (channel d, tokens
 *                  16u..16u+15 of tile t, u < 8) is at
 *                    (t * 2 + u/4) * 512 + (d%32)*16 + (d/32)*4 + u%4
 *                  (for D = 64 the bytes with d/32 >= 2 are 0).
 *   k_mean       : [B*Hkv, D] float32: fp32(sum_n K[b, h, n, d] in binary64 / len_k).
 *   amax         : [3, B*Hq] float32, second-level maxima of Q, K - mean and V (element
 *                  b*Hq + h for Q and b*Hkv + h for K and V; element 0 of each in the
 *                  per-tensor mode); the scale is fp32(amax / 2688), or 1 if that is 0.
 */
#ifndef SAGE_FP4_H
#define SAGE_FP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, short workspace,
                               (from sage_fp4_get_device_error) a bad sequence table */
  SAGE_ERR_UNSUPPORTED = 2, /* D not in {64, 128}, or a size beyond the 32-bit indexing limits */
  SAGE_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed */
  SAGE_ERR_TIMEOUT = 4,     /* a bounded wait inside a kernel ran out (see above) */
  SAGE_ERR_BOUNDS = 5       /* bounds-checked build only: a kernel refused an out-of-range
                               index (an internal error; the access was skipped) */
} sage_status_t;

typedef enum { SAGE_BF16 = 0, SAGE_F16 = 1 } sage_dtype_t;

/* Human-readable name of a status code (static storage). */
const char* sage_status_string(sage_status_t status);

/* ---------------------------------------------------------------- general problem ---- */

typedef enum {
  SAGE_GSCALE_NONE = 0,   /* one level: the 16-element E4M3 scales alone (the method as stated) */
  SAGE_GSCALE_TENSOR = 1, /* plus one FP32 scale per tensor (Q, K - mean, V): NVFP4's shape */
  SAGE_GSCALE_HEAD = 2    /* plus one FP32 scale per (sequence, head) of each tensor */
} sage_gscale_t;

typedef enum {
  SAGE_PRECISION_FP4 = 0,  /* microscaling FP4 Q, K, P~, V (the method; steps 1-6) */
  SAGE_PRECISION_8BIT = 1  /* the 8-bit path of the method's training exploration: INT8 Q, K
                              (after K smoothing) with one scale per 128-token tile, E4M3 V
                              with one scale per channel, E4M3 P~ with s1 = rowmax / 448 per
                              row and key tile; no second-level scale, no Q smoothing */
} sage_precision_t;

/*
 * One attention problem. Element (sequence b, head h, token n, channel d) of Q is at
 *   q + (b*q_stride[0] + h*q_stride[1] + (t0 + n)*q_stride[2] + d) elements,
 * t0 = 0 for dense problems and cu_seqlens_q[b] for packed ones (whose batch stride is
 * ignored); K, V and O likewise (K and V with cu_seqlens_k). Channels are contiguous;
 * every stride must be a non-negative multiple of 8 elements (16 bytes). The library
 * cannot check that the strides stay inside the caller's allocations.
 */
typedef struct {
  int B;                        /* sequences */
  int Hq, Hkv;                  /* query heads; key/value heads (Hq % Hkv == 0) */
  int D;                        /* head dimension: 64 or 128 */
  int Nq, Nk;                   /* dense: tokens per sequence; packed: the longest sequence */
  const int32_t* cu_seqlens_q;  /* packed: device [B+1] token offsets into q and out, else NULL */
  const int32_t* cu_seqlens_k;  /* packed: device [B+1] token offsets into k and v, else NULL */
  int total_q, total_k;         /* packed: tokens in the packed tensors (= cu_seqlens[B]) */
  int64_t q_stride[3];          /* elements between consecutive (sequence, head, token) */
  int64_t k_stride[3];
  int64_t v_stride[3];
  int64_t o_stride[3];
  sage_dtype_t dtype;           /* of q, k, v and out */
  int causal;
  float sm_scale;               /* <= 0: 1/sqrt(D) */
  int smooth_k;                 /* subtract the per-(sequence, head) channel mean of K */
  sage_gscale_t gscale;
  int smooth_q;                 /* subtract the per-(sequence, head) channel mean of Q before
                                   quantizing it, and add mu_q . (k - mu_k) back to the scores */
  sage_precision_t precision;   /* SAGE_PRECISION_FP4 (0) or SAGE_PRECISION_8BIT */
} sage_fp4_problem_t;

/* The quantized tensors of a problem (layouts above); device pointers, 16-byte aligned.
 * With SAGE_PRECISION_8BIT the same fields hold: q_fp4 / k_fp4 int8 codes [rows, D] (one
 * byte per element), q_sf / k_sf one float32 scale per 128-row tile, vt_fp4 E4M3 codes
 * [key tiles, D, 128] (V transposed per tile, one byte per token), vt_sf float32 channel
 * scales [B*Hkv, D]; amax, q_mean and qk_bias are unused. */
typedef struct {
  uint8_t *q_fp4, *q_sf, *k_fp4, *k_sf, *vt_fp4, *vt_sf;
  float* k_mean;                /* required by sage_fp4_quantize */
  float* amax;                  /* required when gscale != SAGE_GSCALE_NONE */
  int32_t* seq;                 /* packed problems: the padded offsets of every sequence,
                                   [2, B+1] int32 plus a validity word; else unused */
  float* q_mean;                /* smooth_q: [B*Hq, D] query means */
  uint8_t* qk_bias;             /* smooth_q: 32 bytes per query head and padded key row (the
                                   key rows' layout with Hq heads): b = mu_q . (k - mu_k)
                                   divided by the Q and K second-level scales (1 without), as
                                   bf16 terms hi, mid, lo (hi = bf16(b), mid = bf16(b - hi),
                                   lo = bf16(b - hi - mid)) in elements 0-2 of 16, zeros
                                   after; the 128 keys of a tile form a 4 KiB tensor-core
                                   operand: key n, 8-element half c at byte
                                   (n/8)*256 + c*128 + (n%8)*16 of the tile */
} sage_fp4_quantized_t;

/* Byte sizes for a problem (all 0 for an empty problem). For packed problems the
 * quantized sizes are upper bounds computed from B, Nq, Nk, total_q and total_k. */
typedef struct {
  size_t q_fp4, q_sf, k_fp4, k_sf, vt_fp4, vt_sf, k_mean, amax, seq, q_mean, qk_bias;
  size_t scratch;    /* scratch of sage_fp4_quantize */
  size_t workspace;  /* workspace of sage_fp4_attn: the above, each 256-byte aligned */
} sage_fp4_problem_sizes_t;

sage_status_t sage_fp4_problem_sizes(const sage_fp4_problem_t* problem, sage_fp4_problem_sizes_t* sizes);

/*
 * Steps 1-2 (and 5) for a general problem: K mean, second-level maxima, quantization of
 * Q, K - mean and V^T into the buffers of `qz`. Packed problems first check the sequence
 * table on the device (cu_seqlens start at 0, do not decrease, end at total_q / total_k,
 * no sequence longer than Nq / Nk); a table that fails sets the device error word
 * (sage_fp4_get_device_error returns SAGE_ERR_INVALID_ARG) and every later kernel of
 * the call leaves its outputs untouched. scratch: at least sizes.scratch bytes.
 */
sage_status_t sage_fp4_quantize(const sage_fp4_problem_t* problem, const void* q, const void* k,
                                const void* v, const sage_fp4_quantized_t* qz, void* scratch,
                                size_t scratch_bytes, void* stream);

/* Steps 3-4 on the output of sage_fp4_quantize for the same problem (k_mean unused). */
sage_status_t sage_fp4_attn_quantized(const sage_fp4_problem_t* problem, const sage_fp4_quantized_t* qz,
                                      void* out, void* stream);

/*
 * The whole forward of a general problem with a caller-owned workspace of at least
 * sizes.workspace bytes (256-byte aligned). Four kernel launches: quantization pass A
 * (the statistics, plus Q and V^T when they need no mean or second-level scale), the K
 * mean and maxima, quantization pass B (K and the rest), attention; packed problems add
 * the sequence-table kernel.
 */
sage_status_t sage_fp4_attn(const sage_fp4_problem_t* problem, const void* q, const void* k,
                            const void* v, void* out, void* workspace, size_t ws_bytes, void* stream);

/* -------------------------------------------------- dense [B, H, N, D] problems ---- */

/* Byte sizes of the quantized tensors for a problem (0 for an empty problem). */
typedef struct {
  size_t q_fp4, q_sf, k_fp4, k_sf, vt_fp4, vt_sf, k_mean;
} sage_fp4_sizes_t;
sage_status_t sage_fp4_quantized_sizes(int B, int H, int N, int D, sage_fp4_sizes_t* sizes);

/* Scratch bytes sage_fp4_quantize_qkv needs (binary64 partial sums for the K mean, and
 * room for the mean itself when k_mean is NULL). */
size_t sage_fp4_quantize_scratch_bytes(int B, int H, int N, int D);

/*
 * Steps 1-2 alone: K mean, then quantize Q, K - mean (smooth_k != 0) or K (smooth_k == 0),
 * and V^T into the layouts above. Outputs are written in full (padding included).
 * scratch: device memory of at least sage_fp4_quantize_scratch_bytes(); contents are
 * overwritten. k_mean may be NULL when smooth_k == 0.
 */
sage_status_t sage_fp4_quantize_qkv(const void* q, const void* k, const void* v, sage_dtype_t dtype,
                                    int B, int H, int N, int D, int smooth_k, uint8_t* q_fp4,
                                    uint8_t* q_sf, uint8_t* k_fp4, uint8_t* k_sf, uint8_t* vt_fp4,
                                    uint8_t* vt_sf, float* k_mean, void* scratch,
                                    size_t scratch_bytes, void* stream);

/*
 * Steps 3-4 on already-quantized inputs (layouts above): the fused tensor-core attention
 * kernel. out: [B, H, N, D] of out_dtype. Uses no scratch memory.
 */
sage_status_t sage_fp4_attn_fwd_quantized(const uint8_t* q_fp4, const uint8_t* q_sf,
                                          const uint8_t* k_fp4, const uint8_t* k_sf,
                                          const uint8_t* vt_fp4, const uint8_t* vt_sf, void* out,
                                          sage_dtype_t out_dtype, int B, int H, int N, int D,
                                          int causal, float sm_scale, void* stream);

/* Workspace bytes sage_fp4_attn_fwd_ex needs: the quantized tensors plus scratch. */
size_t sage_fp4_workspace_bytes(int B, int H, int N, int D);

/*
 * The whole forward (steps 1-4) with a caller-owned workspace of at least
 * sage_fp4_workspace_bytes() bytes (256-byte aligned). Four kernel launches (quantization
 * pass A, K mean, quantization pass B, attention).
 */
sage_status_t sage_fp4_attn_fwd_ex(const void* q, const void* k, const void* v, void* out,
                                   sage_dtype_t dtype, int B, int H, int N, int D, int causal,
                                   float sm_scale, void* workspace, size_t ws_bytes, void* stream);

/*
 * The whole forward on bf16 tensors with a library-owned workspace taken from the
 * stream-ordered allocator (cudaMallocAsync / cudaFreeAsync on `stream`).
 */
sage_status_t sage_fp4_attn_fwd(const void* q, const void* k, const void* v, void* out, int B,
                                int H, int N, int D, int causal, float sm_scale, void* stream);

/*
 * The whole forward (steps 1-4) for callers that cannot allocate device memory. No
 * passage of the method corresponds to it: it exists for callers that may not call
 * cudaMalloc or any allocating library routine (engines that own a fixed memory pool,
 * plugin hosts that forbid allocation while executing, threads without an initialised
 * allocator). It allocates nothing: the caller passes q, k, v and out as for
 * sage_fp4_attn_fwd_ex, and the scratch lives in a 16 MiB file-scope device array that
 * every GPU which loads this library holds until the process exits.
 *   - Limit: sage_fp4_workspace_bytes(B, H, N, D) must be <= 16 MiB (for example
 *     B*H = 16, N = 4096, D = 128); larger problems return SAGE_ERR_UNSUPPORTED before
 *     anything is launched.
 *   - The first call on a device looks up the array's device address (with that device
 *     current) and caches it; make that first call before any stream capture. The cache
 *     lives as long as the process: do not use this entry point on a device after
 *     cudaDeviceReset() or any other teardown of its primary context (the cached address
 *     would belong to the destroyed context).
 *   - Every call shares the one array, which keeps the last call's contents. Nothing in
 *     it has to start at zero (each call writes every byte it later reads), but calls
 *     that overlap on the GPU (different streams, or different host threads, on the same
 *     device) race on it and corrupt each other's results: serialize them.
 */
sage_status_t sage_fp4_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                        sage_dtype_t dtype, int B, int H, int N, int D, int causal,
                                        float sm_scale, void* stream);

/*
 * S = sm_scale * Q^ K^^T (dequantized FP4 operands, FP32 accumulation) for every query
 * and key of the quantized inputs: s_out is [B*H, Np, Np] float32. The tensor-core
 * contraction of step 3 on its own, exported so that it can be checked in isolation.
 */
sage_status_t sage_fp4_qk_scores(const uint8_t* q_fp4, const uint8_t* q_sf, const uint8_t* k_fp4,
                                 const uint8_t* k_sf, float* s_out, int B, int H, int N, int D,
                                 float sm_scale, void* stream);

/*
 * Read and clear the device error word the kernels set when a bounded wait runs out.
 * Synchronizes `stream`. *word receives the raw bits (0 = none); returns SAGE_OK when
 * the word was 0, SAGE_ERR_TIMEOUT when a wait ran out, SAGE_ERR_CUDA on a CUDA error.
 */
sage_status_t sage_fp4_get_device_error(uint32_t* word, void* stream);

/*
 * Text of the last CUDA error that made a call on this host thread return SAGE_ERR_CUDA
 * (empty if none). Static thread-local storage, valid until the next failing call.
 */
const char* sage_fp4_last_cuda_error(void);

/*
 * Test switch for the error path (0 = normal operation, the default). Bit 0: the
 * attention kernel's copy warp issues no loads, so every wait of the other roles runs
 * out after the bound set below; the kernel then drains, frees its tensor memory and
 * returns, and sage_fp4_get_device_error() reports SAGE_ERR_TIMEOUT. Bit 1 (bounds-checked
 * build only, else SAGE_ERR_UNSUPPORTED): the attention kernels take the output's extent
 * as 0, so every output store fails its check, is skipped and reported (SAGE_ERR_BOUNDS).
 * Nothing faults and nothing waits without bound. Applies to launches made after the
 * call; other bits are rejected with SAGE_ERR_INVALID_ARG.
 */
sage_status_t sage_fp4_set_debug_flags(uint32_t flags);

/*
 * Rate probe of the FP4 tensor cores the method runs on (SageAttention3 abstract, "FP4
 * Tensor Cores in Blackwell GPUs"): the block-scaled FP4 instruction both attention
 * contractions use (tcgen05.mma kind::mxf4nvf4, block 16, E2M1 operands, UE4M3 scales,
 * M = 128, N = n, K = 64). Launches `ctas` CTAs of one per SM; each issues `iters`
 * products back to back from operands resident in its shared memory and waits (bounded)
 * for them. The caller times the launch (for instance with CUDA events on `stream`);
 * it performs 2 * 128 * n * 64 * iters * ctas operations. n must be 64 or 128, iters and
 * ctas positive (ctas <= 65535), else SAGE_ERR_INVALID_ARG. Reads and writes no caller
 * memory; the products themselves are discarded.
 */
sage_status_t sage_fp4_mma_rate(int n, int iters, int ctas, void* stream);

/*
 * 1 when this library is the bounds-checked build (libsage_fp4_checks.so, compiled with
 * SAGE_CHECKS): every computed global index of the quantization and attention kernels --
 * input rows, quantized codes and scale tiles, statistics, TMA rows, the output -- is
 * tested against the extents the problem implies before the access; a failure sets a bit
 * of the device error word (sage_fp4_get_device_error returns SAGE_ERR_BOUNDS), raises the
 * CTA's abort flag where the kernel has one, and skips the access (no trap). 0 for the
 * regular build, where the checks compile to nothing. A debugging stand-in for a memory
 * checker; slower than the regular build.
 */
int sage_fp4_bounds_checked(void);

/*
 * Bound on every in-kernel wait, in nanoseconds (default 2e9; 0 restores the default).
 * Applies to launches made after the call.
 */
sage_status_t sage_fp4_set_wait_timeout_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_FP4_H */
