// Query preparation and chunk combine for decode attention (see decode.cuh).
#pragma once

#include "decode.cuh"

namespace tq {

// One CTA per query row: q' = scale * rot @ q, then the second operand, both
// normalized to max-abs 1 (the scales go to qs) so half-precision MMA operands neither
// overflow nor lose relative precision.
__global__ void __launch_bounds__(128) qprep_kernel(QPrepParams p) {
  extern __shared__ __align__(16) float qsm[];
  float* qin = qsm;              // [D]
  float* qr = qin + p.D;         // [D]
  float* q2 = qr + p.D;          // [max(D,16)]
  __shared__ float red[2][4];
  const int r = blockIdx.x, tid = threadIdx.x, D = p.D;
  for (int j = tid; j < D; j += 128) qin[j] = load_elem(p.q, p.dtype, static_cast<int64_t>(r) * D + j);
  __syncthreads();
  for (int j = tid; j < D; j += 128) {
    float a = 0.f;
    for (int k = 0; k < D; ++k) a = fmaf(__ldg(p.rot + j * D + k), qin[k], a);
    qr[j] = a * p.scale;
  }
  __syncthreads();
  const int n2 = p.qb_stride;
  for (int i = tid; i < n2; i += 128) {
    float a = 0.f;
    if (p.kind == TQ_KIND_PROD) {
      if (i < p.m) for (int k = 0; k < D; ++k) a = fmaf(__ldg(p.S + i * D + k), qr[k], a);
    } else if (p.kind == TQ_KIND_SPECTRAL) {
      if (i < p.k_top) a = qr[i] * p.dim_sigma[i];
      else if (i >= 8 && i < 8 + p.k_top && p.qjl) {
        const int ii = i - 8;
        for (int k = 0; k < p.k_top; ++k) a = fmaf(__ldg(p.S + ii * p.k_top + k), qr[k], a);
        a *= p.spec_coef;
      }
    }
    q2[i] = a;
  }
  __syncthreads();
  if (p.kind == TQ_KIND_SPECTRAL)
    for (int j = tid; j < D; j += 128) qr[j] = (j < p.k_top) ? 0.f : qr[j] * p.dim_sigma[j];
  __syncthreads();
  float ma = 0.f, mb = 0.f;
  for (int j = tid; j < D; j += 128) ma = fmaxf(ma, fabsf(qr[j]));
  for (int i = tid; i < n2; i += 128) mb = fmaxf(mb, fabsf(q2[i]));
  ma = warp_max(ma); mb = warp_max(mb);
  if ((tid & 31) == 0) { red[0][tid >> 5] = ma; red[1][tid >> 5] = mb; }
  __syncthreads();
  ma = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
  mb = fmaxf(fmaxf(red[1][0], red[1][1]), fmaxf(red[1][2], red[1][3]));
  const float sa = ma > 0.f ? ma : 1.f, sb = mb > 0.f ? mb : 1.f;
  for (int j = tid; j < D; j += 128) p.qa[static_cast<int64_t>(r) * D + j] = qr[j] / sa;
  for (int i = tid; i < n2; i += 128) p.qb[static_cast<int64_t>(r) * n2 + i] = q2[i] / sb;
  if (tid == 0) { p.qs[r * 2] = sa; p.qs[r * 2 + 1] = sb; }
}

// Log-sum-exp merge of the chunk partials, then o = rot_V^T o' / L.
__global__ void __launch_bounds__(128) combine_kernel(CombineParams p) {
  extern __shared__ __align__(16) float csm[];
  float* ov = csm;                  // [D]
  __shared__ float sM, sL;
  const int r = blockIdx.x, tid = threadIdx.x, D = p.D;
  const float* ml = p.part_ml + static_cast<int64_t>(r) * p.n_chunks * 2;
  if (tid < 32) {
    float M = -INFINITY;
    for (int c = tid; c < p.n_chunks; c += 32) M = fmaxf(M, ml[c * 2]);
    M = warp_max(M);
    float L = 0.f;
    for (int c = tid; c < p.n_chunks; c += 32) {
      const float mc = ml[c * 2];
      if (mc != -INFINITY) L += exp2f(mc - M) * ml[c * 2 + 1];
    }
    L = warp_sum(L);
    if (tid == 0) { sM = M; sL = L; }
  }
  __syncthreads();
  const float M = sM, invL = sL > 0.f ? 1.f / sL : 0.f;
  for (int j = tid; j < D; j += 128) {
    float a = 0.f;
    for (int c = 0; c < p.n_chunks; ++c) {
      const float mc = ml[c * 2];
      if (mc != -INFINITY) a += exp2f(mc - M) * p.part_o[(static_cast<int64_t>(r) * p.n_chunks + c) * D + j];
    }
    if (p.v_sigma) a *= p.v_sigma[j];
    ov[j] = a * invL;
  }
  __syncthreads();
  for (int k = tid; k < D; k += 128) {
    float a = 0.f;
    for (int j = 0; j < D; ++j) a = fmaf(ov[j], __ldg(p.rot_v + j * D + k), a);
    p.out[static_cast<int64_t>(r) * D + k] = a;
  }
}

}  // namespace tq
