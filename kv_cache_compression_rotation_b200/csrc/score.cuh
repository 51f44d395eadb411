// Inner-product estimates of queries against packed records, dense or top-k.
//
// TurboQuant review, "Validation"/"Results": the quantizer also serves exhaustive
// inner-product search; the estimate per (query, record) is the same one attention
// uses, without the softmax.  This kernel computes it on CUDA cores in fp32:
// one thread per record, QT queries per pass with the rotated queries in shared
// memory, codes decoded on the fly from the record's word stream.
#pragma once

#include "device_common.cuh"

namespace tq {

constexpr int kScoreThreads = 128;
constexpr int kScoreQT = 8;

struct ScoreParams {
  int kind, d, bmse, m;
  const uint32_t* codes;
  int code_words;
  const uint32_t* signs;
  int sign_words;
  const float* norms;
  const float* rnorms;
  const float* centroids;
  // spectral
  int k_top, tail_bits, qjl, head_words;
  int top_bits[TQ_MAX_TOP];
  const float* dim_sigma;
  const float* unit_c;
  float coef;                 // sqrt(pi/2)/m (prod) or sqrt(pi/2)/k (spectral)
  // rotated queries
  const float* qr;            // [nq][d]  rot @ q
  const float* qu;            // [nq][m]  S @ (rot @ q)   (prod / spectral qjl)
  int qu_stride;
  int64_t nq, n;
  float* out;                 // [nq][n]
  int accumulate;             // 1: add the estimates to out (split groups after the first)
};

__global__ void __launch_bounds__(kScoreThreads) score_dense_kernel(ScoreParams p) {
  extern __shared__ __align__(16) float ssm[];
  const int d = p.d;
  float* sq = ssm;                         // [QT][d]
  float* su = sq + kScoreQT * d;           // [QT][qu_stride]
  float* cb = su + kScoreQT * p.qu_stride; // centroids (mse/prod: 2^b)
  const int64_t v = static_cast<int64_t>(blockIdx.x) * kScoreThreads + threadIdx.x;
  const int64_t q0 = static_cast<int64_t>(blockIdx.y) * kScoreQT;
  const int nqb = static_cast<int>(min(static_cast<int64_t>(kScoreQT), p.nq - q0));
  for (int i = threadIdx.x; i < kScoreQT * d; i += kScoreThreads) {
    const int qq = i / d;
    sq[i] = qq < nqb ? p.qr[(q0 + qq) * d + (i - qq * d)] : 0.f;
  }
  for (int i = threadIdx.x; i < kScoreQT * p.qu_stride; i += kScoreThreads) {
    const int qq = i / p.qu_stride;
    su[i] = (qq < nqb && p.qu) ? p.qu[(q0 + qq) * p.qu_stride + (i - qq * p.qu_stride)] : 0.f;
  }
  if (p.kind != TQ_KIND_SPECTRAL && p.bmse > 0)
    for (int i = threadIdx.x; i < (1 << p.bmse); i += kScoreThreads) cb[i] = p.centroids[i];
  __syncthreads();
  if (v >= p.n) return;
  float acc[kScoreQT];
#pragma unroll
  for (int i = 0; i < kScoreQT; ++i) acc[i] = 0.f;
  const uint32_t* rec = p.codes + v * p.code_words;
  if (p.kind == TQ_KIND_SPECTRAL) {
    int pos = 0;
    for (int j = 0; j < d; ++j) {
      int b, bp;
      if (j < p.k_top) { b = p.top_bits[j]; bp = pos; pos += b; }
      else { b = p.tail_bits; bp = 32 * p.head_words + j * b; }
      if (b == 0) continue;
      const float c = p.dim_sigma[j] * __ldg(p.unit_c + unit_c_off(b) + stream_bits(rec, bp, b));
#pragma unroll
      for (int i = 0; i < kScoreQT; ++i) acc[i] = fmaf(sq[i * d + j], c, acc[i]);
    }
    if (p.qjl) {
      const float gmm = p.rnorms[v] * p.coef;
      for (int i2 = 0; i2 < p.k_top; ++i2) {
        const float s = stream_bits(rec, pos + i2, 1) ? 1.f : -1.f;
#pragma unroll
        for (int i = 0; i < kScoreQT; ++i) acc[i] = fmaf(gmm * s, su[i * p.qu_stride + i2], acc[i]);
      }
    }
  } else {
    const int b = p.bmse;
    if (b > 0) {
      for (int j = 0; j < d; ++j) {
        const float c = cb[stream_bits(rec, j * b, b)];
#pragma unroll
        for (int i = 0; i < kScoreQT; ++i) acc[i] = fmaf(sq[i * d + j], c, acc[i]);
      }
    }
    if (p.kind == TQ_KIND_PROD) {
      const uint32_t* sg = p.signs + v * p.sign_words;
      float a2[kScoreQT];
#pragma unroll
      for (int i = 0; i < kScoreQT; ++i) a2[i] = 0.f;
      for (int r = 0; r < p.m; ++r) {
        const float s = ((__ldg(sg + (r >> 5)) >> (r & 31)) & 1u) ? 1.f : -1.f;
#pragma unroll
        for (int i = 0; i < kScoreQT; ++i) a2[i] = fmaf(s, su[i * p.qu_stride + r], a2[i]);
      }
      const float gm = p.rnorms[v] * p.coef;
#pragma unroll
      for (int i = 0; i < kScoreQT; ++i) acc[i] = fmaf(gm, a2[i], acc[i]);
    }
    const float nu = p.norms[v];
#pragma unroll
    for (int i = 0; i < kScoreQT; ++i) acc[i] *= nu;
  }
  for (int i = 0; i < nqb; ++i) {
    float* o = p.out + (q0 + i) * p.n + v;
    *o = p.accumulate ? *o + acc[i] : acc[i];
  }
}

// Rotated queries for scoring: qr = rot @ q, qu = S @ qr (prod) or S_top @ qr_top.
// Query element j of row r is q[r * ldq + (cols ? cols[j] : j)] (the split's gather; a
// column outside 0..ldq-1 reads column 0 and reports TQ_ERR_INVALID_ARG to *status).
__global__ void __launch_bounds__(128) score_qprep_kernel(const void* q, int dtype, int d, int kind,
                                                          const float* rot, const float* S, int m,
                                                          int k_top, float* qr, float* qu, int qu_stride,
                                                          int64_t ldq, const int32_t* cols, int* status) {
  extern __shared__ __align__(16) float qsm2[];
  float* qin = qsm2;
  float* qo = qin + d;
  const int64_t r = blockIdx.x;
  for (int j = threadIdx.x; j < d; j += 128) {
    int64_t col = j;
    if (cols) {
      col = __ldg(cols + j);
      if (col < 0 || col >= ldq) {
        report_status(status, TQ_ERR_INVALID_ARG);
        col = 0;
      }
    }
    qin[j] = load_elem(q, dtype, r * ldq + col);
  }
  __syncthreads();
  for (int j = threadIdx.x; j < d; j += 128) {
    float a = 0.f;
    for (int k = 0; k < d; ++k) a = fmaf(__ldg(rot + static_cast<int64_t>(j) * d + k), qin[k], a);
    qo[j] = a;
    qr[r * d + j] = a;
  }
  __syncthreads();
  if (!qu) return;
  for (int i = threadIdx.x; i < qu_stride; i += 128) {
    float a = 0.f;
    if (kind == TQ_KIND_PROD && i < m) {
      for (int k = 0; k < d; ++k) a = fmaf(__ldg(S + static_cast<int64_t>(i) * d + k), qo[k], a);
    } else if (kind == TQ_KIND_SPECTRAL && i < k_top) {
      for (int k = 0; k < k_top; ++k) a = fmaf(__ldg(S + i * k_top + k), qo[k], a);
    }
    qu[r * qu_stride + i] = a;
  }
}

// Top-k of one dense score row per CTA: each thread keeps a sorted list of its best K
// (descending score, ascending id), then the lists are merged pairwise in shared memory.
template <int K>
__global__ void __launch_bounds__(128) topk_kernel(const float* scores, int64_t n, int k,
                                                   int64_t row0, float* out_s, int32_t* out_i) {
  __shared__ float ss[128][K];
  __shared__ int32_t si[128][K];
  const int64_t r = blockIdx.x;
  const float* row = scores + r * n;
  float bs[K];
  int32_t bi[K];
#pragma unroll
  for (int i = 0; i < K; ++i) { bs[i] = -INFINITY; bi[i] = 0x7fffffff; }
  for (int64_t j = threadIdx.x; j < n; j += 128) {
    const float s = row[j];
    const int32_t id = static_cast<int32_t>(j);
    // better(s,id) than the current last entry?
    if (s > bs[K - 1] || (s == bs[K - 1] && id < bi[K - 1])) {
      float cs = s;
      int32_t ci = id;
#pragma unroll
      for (int i = 0; i < K; ++i) {
        const bool better = cs > bs[i] || (cs == bs[i] && ci < bi[i]);
        if (better) {
          const float ts = bs[i]; const int32_t ti = bi[i];
          bs[i] = cs; bi[i] = ci; cs = ts; ci = ti;
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < K; ++i) { ss[threadIdx.x][i] = bs[i]; si[threadIdx.x][i] = bi[i]; }
  __syncthreads();
  for (int stride = 64; stride > 0; stride >>= 1) {
    if (threadIdx.x < stride) {
      const int a = threadIdx.x, b = threadIdx.x + stride;
      float ms[K];
      int32_t mi[K];
      int ia = 0, ib = 0;
#pragma unroll
      for (int i = 0; i < K; ++i) {
        const bool takeA = ss[a][ia] > ss[b][ib] || (ss[a][ia] == ss[b][ib] && si[a][ia] < si[b][ib]);
        if (takeA) { ms[i] = ss[a][ia]; mi[i] = si[a][ia]; ++ia; }
        else { ms[i] = ss[b][ib]; mi[i] = si[b][ib]; ++ib; }
      }
#pragma unroll
      for (int i = 0; i < K; ++i) { ss[a][i] = ms[i]; si[a][i] = mi[i]; }
    }
    __syncthreads();
  }
  if (threadIdx.x < k) {
    out_s[(row0 + r) * k + threadIdx.x] = ss[0][threadIdx.x];
    out_i[(row0 + r) * k + threadIdx.x] = si[0][threadIdx.x];
  }
}

// y[i][j] = sum_k A[j][k] x[i][k] for queries i < nx and rows j < rows (A fp32 [rows][d], x
// [nx][ldx] in the given dtype, d a multiple of 128): the query rotation and projection of the
// tensor-core estimator.  Block (x, y) takes queries kMvQ x .. (in shared memory) and rows
// kMvRows y .., one warp per row at a time: the lanes read the row with coalesced 16-byte
// loads and reduce the kMvQ dot products with shuffles.
constexpr int kMvQ = 8, kMvRows = 32;
__global__ void __launch_bounds__(128) rows_matvec_kernel(const float* __restrict__ A, int rows, int d,
                                                          const void* x, int dtype, int64_t nx, int64_t ldx,
                                                          float* __restrict__ y, int64_t ldy) {
  extern __shared__ __align__(16) float xs[];      // [kMvQ][d]
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kMvQ;
  for (int e = threadIdx.x; e < kMvQ * d; e += 128) {
    const int qi = e / d, k = e - qi * d;
    xs[e] = (i0 + qi < nx) ? load_elem(x, dtype, (i0 + qi) * ldx + k) : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float4* xs4 = reinterpret_cast<const float4*>(xs);
#pragma unroll 1
  for (int jj = 0; jj < kMvRows / 4; ++jj) {
    const int j = blockIdx.y * kMvRows + warp * (kMvRows / 4) + jj;
    if (j >= rows) break;
    const float4* a4 = reinterpret_cast<const float4*>(A + static_cast<int64_t>(j) * d);
    float acc[kMvQ];
#pragma unroll
    for (int qi = 0; qi < kMvQ; ++qi) acc[qi] = 0.f;
    for (int k4 = lane; k4 < d / 4; k4 += 32) {
      const float4 a = __ldg(a4 + k4);
#pragma unroll
      for (int qi = 0; qi < kMvQ; ++qi) {
        const float4 v = xs4[qi * (d / 4) + k4];
        acc[qi] = fmaf(a.x, v.x, fmaf(a.y, v.y, fmaf(a.z, v.z, fmaf(a.w, v.w, acc[qi]))));
      }
    }
    float mine = 0.f;                               // lane qi keeps query qi's sum
#pragma unroll
    for (int qi = 0; qi < kMvQ; ++qi) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[qi] += __shfl_xor_sync(0xffffffffu, acc[qi], o);
      if (lane == qi) mine = acc[qi];
    }
    if (lane < kMvQ && i0 + lane < nx) y[(i0 + lane) * ldy + j] = mine;
  }
}

// Top-K of row segments: CTA (s, r) takes candidates [s L, min((s + 1) L, len)) of row r,
// scores from `scores` and ids from `ids` (or the positions when ids is null), and writes its
// best k_out in the order of the whole search (descending score, ascending id) to
// out[((out_row0 + r) * gridDim.x + s) * k_out ..].  Run over the dense rows in segments and
// then once over the segments' K candidates, it gives the same top-k as one pass over the row
// (every member of the row's top-k is in its segment's top-K).
template <int K>
__global__ void __launch_bounds__(128) topk_seg_kernel(const float* scores, const int32_t* ids, int64_t len,
                                                       int64_t seg, int k_out, float* out_s, int32_t* out_i,
                                                       int64_t out_row0) {
  __shared__ float ss[128][K];
  __shared__ int32_t si[128][K];
  const int64_t r = blockIdx.y, b = static_cast<int64_t>(blockIdx.x) * seg;
  const int64_t e = min(len, b + seg);
  const float* row = scores + r * len;
  const int32_t* idr = ids ? ids + r * len : nullptr;
  float bs[K];
  int32_t bi[K];
#pragma unroll
  for (int i = 0; i < K; ++i) { bs[i] = -INFINITY; bi[i] = 0x7fffffff; }
  for (int64_t j = b + threadIdx.x; j < e; j += 128) {
    const float s = row[j];
    const int32_t id = idr ? idr[j] : static_cast<int32_t>(j);
    if (s > bs[K - 1] || (s == bs[K - 1] && id < bi[K - 1])) {
      float cs = s;
      int32_t ci = id;
#pragma unroll
      for (int i = 0; i < K; ++i) {
        const bool better = cs > bs[i] || (cs == bs[i] && ci < bi[i]);
        if (better) {
          const float ts = bs[i]; const int32_t ti = bi[i];
          bs[i] = cs; bi[i] = ci; cs = ts; ci = ti;
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < K; ++i) { ss[threadIdx.x][i] = bs[i]; si[threadIdx.x][i] = bi[i]; }
  __syncthreads();
  for (int stride = 64; stride > 0; stride >>= 1) {
    if (threadIdx.x < stride) {
      const int a = threadIdx.x, c = threadIdx.x + stride;
      float ms[K];
      int32_t mi[K];
      int ia = 0, ic = 0;
#pragma unroll
      for (int i = 0; i < K; ++i) {
        const bool takeA = ss[a][ia] > ss[c][ic] || (ss[a][ia] == ss[c][ic] && si[a][ia] < si[c][ic]);
        if (takeA) { ms[i] = ss[a][ia]; mi[i] = si[a][ia]; ++ia; }
        else { ms[i] = ss[c][ic]; mi[i] = si[c][ic]; ++ic; }
      }
#pragma unroll
      for (int i = 0; i < K; ++i) { ss[a][i] = ms[i]; si[a][i] = mi[i]; }
    }
    __syncthreads();
  }
  if (threadIdx.x < k_out) {
    const int64_t o = ((out_row0 + r) * gridDim.x + blockIdx.x) * k_out + threadIdx.x;
    out_s[o] = ss[0][threadIdx.x];
    out_i[o] = si[0][threadIdx.x];
  }
}

}  // namespace tq
