// Operands of the tensor-core estimator for outlier-split records (TurboQuant review,
// Method: a split record's estimate is the sum of its groups' estimates).  Each group g
// contributes d_g columns (MSE part) and m_g columns (QJL part of a PROD group) to one
// contraction of width K = sum_g (d_g + m_g):
//   query row   [Pi_g q[cols_g] | S_g Pi_g q[cols_g]]                  over the groups
//   record row  [||k_g|| c_g[code] | ||k_g|| sqrt(pi/2)/m_g gamma_g (2s - 1)]   over the groups
// so their inner product is the summed estimate; the group norms ride in the record row
// (the product's column scale is 1).  Both rows are written as bf16 hi + lo parts.
#include <cuda_bf16.h>

#include "launchers.h"

namespace tq {
namespace {

__device__ __forceinline__ void split_bf16(float v, uint16_t& h, uint16_t& l) {
  const __nv_bfloat16 bh = __float2bfloat16_rn(v);
  h = __bfloat16_as_ushort(bh);
  l = __bfloat16_as_ushort(__float2bfloat16_rn(v - __bfloat162float(bh)));
}

// Which group part column k of a row falls in: returns the group and sets the offset
// within the part and whether it is the QJL part.
__device__ __forceinline__ int split_col(const SplitScoreGroups& G, int k, int& j, bool& qjl) {
  int off = 0;
  for (int g = 0; g < G.n; ++g) {
    if (k < off + G.d[g]) { j = k - off; qjl = false; return g; }
    off += G.d[g];
    if (k < off + G.m[g]) { j = k - off; qjl = true; return g; }
    off += G.m[g];
  }
  j = 0;
  qjl = false;
  return -1;
}

__global__ void __launch_bounds__(256) split_queries_kernel(const SplitScoreGroups G, int64_t nq, int K,
                                                            uint16_t* __restrict__ hi, uint16_t* __restrict__ lo) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (i >= nq * K) return;
  const int64_t r = i / K;
  const int k = static_cast<int>(i - r * K);
  int j;
  bool qjl;
  const int g = split_col(G, k, j, qjl);
  float v = 0.f;
  if (g >= 0) v = qjl ? G.qu[g][r * G.m[g] + j] : G.qr[g][r * G.d[g] + j];
  split_bf16(v, hi[i], lo[i]);
}

// One warp per record, lanes over the K columns.
__global__ void __launch_bounds__(256) split_records_kernel(const SplitScoreGroups G, int64_t n, int K,
                                                            uint16_t* __restrict__ hi, uint16_t* __restrict__ lo,
                                                            float* __restrict__ ones) {
  const int lane = threadIdx.x & 31;
  const int64_t rec = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (rec >= n) return;
  if (lane == 0) ones[rec] = 1.f;
  for (int k = lane; k < K; k += 32) {
    int j;
    bool qjl;
    const int g = split_col(G, k, j, qjl);
    float v = 0.f;
    if (g >= 0) {
      const float nrm = __ldg(G.norms[g] + rec);
      if (qjl) {
        const bool pos = (__ldg(G.signs[g] + rec * G.sign_words[g] + (j >> 5)) >> (j & 31)) & 1u;
        const float a = nrm * G.coef[g] * __ldg(G.rnorms[g] + rec);
        v = pos ? a : -a;
      } else if (G.bits[g] > 0) {
        const int b = G.bits[g], pos = j * b;
        const uint32_t* w = G.codes[g] + rec * G.code_words[g];
        uint32_t code = __ldg(w + (pos >> 5)) >> (pos & 31);
        if ((pos & 31) + b > 32) code |= __ldg(w + (pos >> 5) + 1) << (32 - (pos & 31));
        v = nrm * __ldg(G.centroids[g] + (code & ((1u << b) - 1u)));
      }
    }
    split_bf16(v, hi[rec * K + k], lo[rec * K + k]);
  }
}

}  // namespace

cudaError_t launch_split_score_queries(const SplitScoreGroups& G, int64_t nq, int K, uint16_t* qh, uint16_t* ql,
                                       cudaStream_t s) {
  const int64_t tq = nq * K;
  split_queries_kernel<<<static_cast<unsigned>((tq + 255) / 256), 256, 0, s>>>(G, nq, K, qh, ql);
  return cudaGetLastError();
}

cudaError_t launch_split_score_records(const SplitScoreGroups& G, int64_t n, int K, uint16_t* rh, uint16_t* rl,
                                       float* ones, cudaStream_t s) {
  split_records_kernel<<<static_cast<unsigned>((n + 7) / 8), 256, 0, s>>>(G, n, K, rh, rl, ones);
  return cudaGetLastError();
}

}  // namespace tq
