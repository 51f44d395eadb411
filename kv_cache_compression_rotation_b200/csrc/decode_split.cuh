// Decode attention over an outlier-channel split cache (CUDA cores).
//
// TurboQuant review, Method: for the KV-cache experiments the channels are split into
// groups, each quantized by its own TurboQuant instance.  Attention then reads a key
// through the sum of its groups' estimates and a value through the sum of its groups'
// reconstructions:
//
//   logit_i = scale * sum_g ||k_i,g|| <Pi_g q[cols_g], c_g[code_i,g]>
//   out[cols_g] = Pi_g^T sum_i p_i ||v_i,g|| c_g[code_i,g]          (p = softmax(logit))
//
// score_qprep_kernel (score.cuh) forms each key group's gathered, rotated query;
// split_decode_kernel runs one CTA of 4 warps per (batch * kv-head, context chunk), a
// warp per token at a time, lanes over the concatenated rotated coordinates, online
// softmax in the log2 domain, and the per-warp P.V accumulators in shared memory;
// split_combine_kernel merges the chunks and applies each value group's Pi_g^T,
// scattering to the group's channels.  Key groups are MSE or PROD instances: a PROD group
// adds its QJL term sqrt(pi/2)/m_g ||r|| <S_g Pi_g q[cols_g], 2s - 1> to the group's
// estimate (times ||k_g||); value groups are MSE.
#pragma once

#include "device_common.cuh"

namespace tq {

constexpr int kSplitDecThreads = 128;
constexpr int kSplitMaxD = 256;        // full vector width
constexpr int kSplitMaxG = 8;          // query heads per kv-head

struct SplitDecodeParams {
  int B, Hq, Hkv, G, d;                // d = full width (sum of the group widths)
  int64_t Nmax;
  int chunk_len, n_chunks;
  const int32_t* seq_lens;
  int nkg, nvg;
  int kd[TQ_MAX_GROUPS], kbits[TQ_MAX_GROUPS], kwords[TQ_MAX_GROUPS], koff[TQ_MAX_GROUPS];
  const uint32_t* kcodes[TQ_MAX_GROUPS];
  const float* knorms[TQ_MAX_GROUPS];
  const float* kcent[TQ_MAX_GROUPS];
  const float* qr[TQ_MAX_GROUPS];      // [B*Hq][kd[g]]: Pi_g q[cols_g]
  // PROD key groups (km = 0 for MSE): kbits is the MSE stage's width (0: no codes)
  int km[TQ_MAX_GROUPS], ksw[TQ_MAX_GROUPS], kuoff[TQ_MAX_GROUPS], mu;   // mu = sum of km
  const uint32_t* ksigns[TQ_MAX_GROUPS];
  const float* krnorms[TQ_MAX_GROUPS];
  const float* qu[TQ_MAX_GROUPS];      // [B*Hq][km[g]]: S_g Pi_g q[cols_g]
  float kcoef[TQ_MAX_GROUPS];          // sqrt(pi/2) / m_g
  int vd[TQ_MAX_GROUPS], vbits[TQ_MAX_GROUPS], vwords[TQ_MAX_GROUPS], voff[TQ_MAX_GROUPS];
  const uint32_t* vcodes[TQ_MAX_GROUPS];
  const float* vnorms[TQ_MAX_GROUPS];
  const float* vcent[TQ_MAX_GROUPS];
  float logit_scale;                   // scale * log2(e)
  float* part_ml;                      // [B*Hq][n_chunks][2]  (max, sum) in the log2 domain
  float* part_o;                       // [B*Hq][n_chunks][d]  value groups concatenated
};

// Shared memory (floats): q'[G][d] | key codebooks [4][256] | value codebooks [4][256] |
// per-warp max [4][G], sum [4][G] | per-warp P.V [4][G][d] | S q'[G][mu] (PROD key groups)
__host__ __device__ inline size_t split_decode_smem(int G, int d, int mu = 0) {
  return (static_cast<size_t>(G) * d + 2 * TQ_MAX_GROUPS * 256 + 2 * 4 * G + 4 * static_cast<size_t>(G) * d +
          static_cast<size_t>(G) * mu) * 4;
}

__global__ void __launch_bounds__(kSplitDecThreads) split_decode_kernel(const SplitDecodeParams p) {
  extern __shared__ __align__(16) float sdsm[];
  const int G = p.G, d = p.d;
  float* sq = sdsm;
  float* cbk = sq + G * d;
  float* cbv = cbk + TQ_MAX_GROUPS * 256;
  float* wm = cbv + TQ_MAX_GROUPS * 256;
  float* wl = wm + 4 * G;
  float* wo = wl + 4 * G;
  float* su = wo + 4 * G * d;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.Hkv, hk = bh - b * p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row0 = static_cast<int64_t>(b) * p.Hq + static_cast<int64_t>(hk) * G;   // first query row

  for (int i = tid; i < G * d; i += kSplitDecThreads) {
    const int h = i / d, j = i - h * d;
    float v = 0.f;
    for (int g = 0; g < p.nkg; ++g)
      if (j >= p.koff[g] && j < p.koff[g] + p.kd[g]) v = p.qr[g][(row0 + h) * p.kd[g] + (j - p.koff[g])];
    sq[i] = v;
  }
  for (int i = tid; i < G * p.mu; i += kSplitDecThreads) {
    const int h = i / p.mu, j = i - h * p.mu;
    float v = 0.f;
    for (int g = 0; g < p.nkg; ++g)
      if (p.km[g] && j >= p.kuoff[g] && j < p.kuoff[g] + p.km[g]) v = p.qu[g][(row0 + h) * p.km[g] + (j - p.kuoff[g])];
    su[i] = v;
  }
  for (int i = tid; i < TQ_MAX_GROUPS * 256; i += kSplitDecThreads) {
    const int g = i >> 8, e = i & 255;
    cbk[i] = (g < p.nkg && p.kbits[g] > 0 && e < (1 << p.kbits[g])) ? p.kcent[g][e] : 0.f;
    cbv[i] = (g < p.nvg && e < (1 << p.vbits[g])) ? p.vcent[g][e] : 0.f;
  }
  for (int i = tid; i < 4 * G * d; i += kSplitDecThreads) wo[i] = 0.f;
  __syncthreads();

  const int len = static_cast<int>(min(static_cast<int64_t>(p.seq_lens[b]), p.Nmax));
  const int t0 = chunk * p.chunk_len, t1 = min(len, t0 + p.chunk_len);
  float m[kSplitMaxG], l[kSplitMaxG];
#pragma unroll
  for (int h = 0; h < kSplitMaxG; ++h) { m[h] = -INFINITY; l[h] = 0.f; }
  float* my_o = wo + warp * G * d;
  for (int t = t0 + warp; t < t1; t += 4) {
    const int64_t rec = static_cast<int64_t>(bh) * p.Nmax + t;
    float s[kSplitMaxG];
#pragma unroll
    for (int h = 0; h < kSplitMaxG; ++h) s[h] = 0.f;
    for (int g = 0; g < p.nkg; ++g) {
      const float nk = p.knorms[g][rec];
      if (p.kbits[g] > 0) {
        const uint32_t* w = p.kcodes[g] + rec * p.kwords[g];
        for (int jj = lane; jj < p.kd[g]; jj += 32) {
          const float c = nk * cbk[g * 256 + stream_bits(w, jj * p.kbits[g], p.kbits[g])];
          const int j = p.koff[g] + jj;
#pragma unroll
          for (int h = 0; h < kSplitMaxG; ++h)
            if (h < G) s[h] = fmaf(sq[h * d + j], c, s[h]);
        }
      }
      if (p.km[g]) {
        // QJL term: ||k_g|| sqrt(pi/2)/m ||r|| sum_i (S q')_i (2 s_i - 1)
        const uint32_t* sw = p.ksigns[g] + rec * p.ksw[g];
        const float f = nk * p.kcoef[g] * p.krnorms[g][rec];
        for (int i = lane; i < p.km[g]; i += 32) {
          const float c = ((sw[i >> 5] >> (i & 31)) & 1u) ? f : -f;
          const int j = p.kuoff[g] + i;
#pragma unroll
          for (int h = 0; h < kSplitMaxG; ++h)
            if (h < G) s[h] = fmaf(su[h * p.mu + j], c, s[h]);
        }
      }
    }
    float f[kSplitMaxG], pr[kSplitMaxG];
#pragma unroll
    for (int h = 0; h < kSplitMaxG; ++h) {
      f[h] = 1.f;
      pr[h] = 0.f;
      if (h < G) {
        const float lg = warp_sum(s[h]) * p.logit_scale;
        const float mn = fmaxf(m[h], lg);
        f[h] = exp2f(m[h] - mn);                 // 0 on the first token (m = -inf)
        pr[h] = exp2f(lg - mn);
        l[h] = l[h] * f[h] + pr[h];
        m[h] = mn;
      }
    }
    for (int g = 0; g < p.nvg; ++g) {
      const uint32_t* w = p.vcodes[g] + rec * p.vwords[g];
      const float nv = p.vnorms[g][rec];
      for (int jj = lane; jj < p.vd[g]; jj += 32) {
        const float c = nv * cbv[g * 256 + stream_bits(w, jj * p.vbits[g], p.vbits[g])];
        const int j = p.voff[g] + jj;
#pragma unroll
        for (int h = 0; h < kSplitMaxG; ++h)
          if (h < G) my_o[h * d + j] = fmaf(my_o[h * d + j], f[h], pr[h] * c);
      }
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < kSplitMaxG; ++h)
      if (h < G) { wm[warp * G + h] = m[h]; wl[warp * G + h] = l[h]; }
  }
  __syncthreads();
  // merge the 4 warps: (max, sum) and the rescaled P.V sums, one partial per head and chunk
  for (int i = tid; i < G * d; i += kSplitDecThreads) {
    const int h = i / d, j = i - h * d;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w * G + h]);
    float L = 0.f, o = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float mw = wm[w * G + h];
      const float e = mw == -INFINITY ? 0.f : exp2f(mw - M);
      L += e * wl[w * G + h];
      o += e * wo[(w * G + h) * d + j];
    }
    const int64_t pi = (row0 + h) * p.n_chunks + chunk;
    if (j == 0) { p.part_ml[pi * 2] = M; p.part_ml[pi * 2 + 1] = L; }
    p.part_o[pi * d + j] = o;
  }
}

struct SplitCombineParams {
  int rows, d, n_chunks, nvg;
  int vd[TQ_MAX_GROUPS], voff[TQ_MAX_GROUPS];
  const float* vrot[TQ_MAX_GROUPS];    // [vd][vd] row-major, y = Pi x
  const int32_t* vcols[TQ_MAX_GROUPS];
  int* status;
  const float* part_ml;
  const float* part_o;
  float* out;                          // [rows][d]
};

// One CTA per query row: log-sum-exp merge of the chunks, then out[cols_g] = Pi_g^T o'_g / L.
__global__ void __launch_bounds__(128) split_combine_kernel(const SplitCombineParams p) {
  extern __shared__ __align__(16) float csm2[];
  float* ow = csm2;                    // [n_chunks] chunk weights
  float* ov = ow + p.n_chunks;         // [d] merged o'
  __shared__ float sL;
  const int64_t r = blockIdx.x;
  const int tid = threadIdx.x;
  const float* ml = p.part_ml + r * p.n_chunks * 2;
  if (tid < 32) {
    float M = -INFINITY;
    for (int c = tid; c < p.n_chunks; c += 32) M = fmaxf(M, ml[c * 2]);
    M = warp_max(M);
    float L = 0.f;
    for (int c = tid; c < p.n_chunks; c += 32) {
      const float mc = ml[c * 2];
      const float e = mc == -INFINITY ? 0.f : exp2f(mc - M);
      ow[c] = e;
      L += e * ml[c * 2 + 1];
    }
    L = warp_sum(L);
    if (tid == 0) sL = L;
  }
  __syncthreads();
  const float invL = sL > 0.f ? 1.f / sL : 0.f;
  for (int j = tid; j < p.d; j += 128) {
    float a = 0.f;
    for (int c = 0; c < p.n_chunks; ++c) a = fmaf(ow[c], p.part_o[(r * p.n_chunks + c) * p.d + j], a);
    ov[j] = a * invL;
  }
  __syncthreads();
  for (int g = 0; g < p.nvg; ++g) {
    const int dg = p.vd[g];
    for (int j = tid; j < dg; j += 128) {
      float a = 0.f;
      for (int k = 0; k < dg; ++k) a = fmaf(__ldg(p.vrot[g] + static_cast<int64_t>(k) * dg + j), ov[p.voff[g] + k], a);
      int col = __ldg(p.vcols[g] + j);
      if (col < 0 || col >= p.d) {
        report_status(p.status, TQ_ERR_INVALID_ARG);
        continue;
      }
      p.out[r * p.d + col] = a;
    }
  }
}

}  // namespace tq
