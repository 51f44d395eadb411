// Host launchers for the templated kernels, each compiled in its own translation unit.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "tq.h"

namespace tq {

// Launch `k` with programmatic stream serialization: it may start (and run what precedes
// its pdl_wait()) while the previous kernel in the stream finishes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

struct DecodeParams;
struct UmmaQuantParams;
struct SplitGemmParams;

// Launch decode_attn_kernel for (key format, key bits, value format, value bits) at D = 128.
// Returns cudaErrorNotSupported (without launching) for a combination that is not built.
// MSE / PROD keys run the bulk-copy staged kernel (decode_tma.cuh), spectral keys the
// direct-load kernel (decode.cuh).  `status`/`lim`: device status word and wait limit.
cudaError_t launch_decode(const DecodeParams& p, int kfmt, int kb, int vfmt, int vb, dim3 grid,
                          size_t smem, cudaStream_t stream, int* status, long long lim);
cudaError_t launch_decode_mse(const DecodeParams& p, int kb, int vb, dim3 grid, size_t smem, cudaStream_t s,
                              int* status, long long lim);
cudaError_t launch_decode_prod(const DecodeParams& p, int kb, int vb, dim3 grid, size_t smem, cudaStream_t s,
                               int* status, long long lim);
cudaError_t launch_decode_spec(const DecodeParams& p, int kb, int vb, dim3 grid, size_t smem, cudaStream_t s);
cudaError_t launch_decode_spec_tma(const DecodeParams& p, dim3 grid, cudaStream_t s, int* status, long long lim);
// Values quantized as prod (MSE-stage bits 1..4, m = 128): MSE / PROD keys.
cudaError_t launch_decode_vprod(const DecodeParams& p, int kfmt, int kb, int vb, dim3 grid, cudaStream_t s,
                                int* status, long long lim);
// Causal query blocks (prefill): MSE / PROD keys (bits of the MSE stage 1..4), MSE values.
cudaError_t launch_decode_causal(const DecodeParams& p, int kfmt, int kb, int vb, dim3 grid, cudaStream_t s,
                                 int* status, long long lim);

// Tensor-core quantize (d = 128, 16-bit input, MSE bits 1..4).
cudaError_t launch_umma_quantize(const CUtensorMap& map, const UmmaQuantParams& p, int bits, int grid,
                                 cudaStream_t stream);
// Split-precision product for wide vectors: maps = {A_hi, A_lo, B_hi, B_lo}; epi 0 writes
// codes (bits 1..4) and the QJL residual, epi 1 the sign words.
cudaError_t launch_split_gemm(const CUtensorMap* maps, const SplitGemmParams& p, int epi, int bits, int grid,
                              cudaStream_t s);
// Tensor-core estimator operands: [a | b] rows as bf16 hi + lo; records decoded to
// [c[code] | coef * gamma * (2s - 1)] rows as bf16 hi + lo.
cudaError_t launch_split_cat(const float* a, int da, const float* b, int db, int64_t rows, uint16_t* hi,
                             uint16_t* lo, cudaStream_t s, const int* sym = nullptr, const float* centroids = nullptr);
cudaError_t launch_expand_records(const uint32_t* codes, int code_words, const uint32_t* signs, int sign_words,
                                  const float* rnorms, const float* centroids, float coef, int64_t n, int d, int m,
                                  int bits, uint16_t* hi, uint16_t* lo, int* sym_flag, cudaStream_t s);
// fp32 rows -> bf16 hi + lo parts (and row norms when norms != nullptr).
cudaError_t launch_split_rows(const float* x, int64_t rows, int d, uint16_t* hi, uint16_t* lo, float* norms,
                              cudaStream_t s);
// Outlier split (32 channels at b0 bits + 96 at b1 bits, (3, 2) or (4, 3)) as one
// tensor-core pass over 16-bit rows of 128 channels.
cudaError_t launch_umma_quantize_split(const CUtensorMap& map, const UmmaQuantParams& p, int b0, int b1, int grid,
                                       cudaStream_t s);
// Operands of the tensor-core estimator over outlier-split records: per group the rotated
// (and S-projected, PROD) queries and the records, concatenated along K (see score_split_tc.cu).
struct SplitScoreGroups {
  int n;                                   // groups
  int d[TQ_MAX_GROUPS], m[TQ_MAX_GROUPS];  // MSE-part and QJL-part widths (m = 0 for MSE)
  int bits[TQ_MAX_GROUPS];                 // MSE-stage bits (0: no codes)
  int code_words[TQ_MAX_GROUPS], sign_words[TQ_MAX_GROUPS];
  const float* qr[TQ_MAX_GROUPS];          // [nq][d_g] (the block of queries of this pass)
  const float* qu[TQ_MAX_GROUPS];          // [nq][m_g]
  const uint32_t* codes[TQ_MAX_GROUPS];
  const uint32_t* signs[TQ_MAX_GROUPS];
  const float* norms[TQ_MAX_GROUPS];
  const float* rnorms[TQ_MAX_GROUPS];
  const float* centroids[TQ_MAX_GROUPS];
  float coef[TQ_MAX_GROUPS];               // sqrt(pi/2) / m_g
};
cudaError_t launch_split_score_queries(const SplitScoreGroups& G, int64_t nq, int K, uint16_t* qh, uint16_t* ql,
                                       cudaStream_t s);
cudaError_t launch_split_score_records(const SplitScoreGroups& G, int64_t n, int K, uint16_t* rh, uint16_t* rl,
                                       float* ones, cudaStream_t s);
// Split-cache decode on the tensor cores: two MSE groups per record, 32 rotated dims at 3
// bits then 96 at 2 bits (keys and values), GQA groups of at most 4 heads.
struct SplitMmaParams;
cudaError_t launch_decode_split_mma(const SplitMmaParams& p, int grid, cudaStream_t s, int* status, long long lim);
// TurboQuant-prod with m = d = 128: the rotation and the QJL projection on the tensor cores
cudaError_t launch_umma_quantize_prod(const CUtensorMap& map, const UmmaQuantParams& p, int mse_bits, int grid,
                                      cudaStream_t s);

}  // namespace tq
