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
  pdl_trigger();   // the decode kernel may launch; it waits for this grid before reading q'
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
  pdl_wait();      // the partials come from the decode kernel before this one
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

// ---- d = 128 versions: 8 query rows per CTA of 256 threads ----

// ys[r][j] = scale * sum_k M[j][k] xs[r][k] for 8 rows r and 128 outputs j (M row-major,
// 128 x 128; xs, ys in shared memory).  Warp w produces j in [16 w, 16 w + 16); lane l
// holds xs[r][4 l .. 4 l + 3].  Each group of 4 outputs x 8 rows is 32 partial dot products
// per lane, summed across the warp by a halving exchange that leaves total l in lane l.
__device__ __forceinline__ void matvec8x128(const float* __restrict__ M, const float* xs, float* ys, float scale,
                                            int warp, int lane) {
  float4 xv[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) xv[r] = *reinterpret_cast<const float4*>(xs + r * 128 + 4 * lane);
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    float v[32];
#pragma unroll
    for (int d = 0; d < 4; ++d) {
      const float4 m = __ldg(reinterpret_cast<const float4*>(M + (16 * warp + 4 * pass + d) * 128 + 4 * lane));
#pragma unroll
      for (int r = 0; r < 8; ++r)
        v[d * 8 + r] = fmaf(m.w, xv[r].w, fmaf(m.z, xv[r].z, fmaf(m.y, xv[r].y, m.x * xv[r].x)));
    }
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) {
      const bool up = (lane & sh) != 0;
#pragma unroll
      for (int i = 0; i < sh; ++i) {
        const float send = up ? v[i] : v[i + sh];
        const float keep = up ? v[i + sh] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, sh);
      }
    }
    // lane l now holds the total of value l = 8 d + r
    ys[(lane & 7) * 128 + 16 * warp + 4 * pass + (lane >> 3)] = v[0] * scale;
  }
}

// qprep_kernel with d = 128 (same outputs, every key kind).
__global__ void __launch_bounds__(256) qprep128_kernel(QPrepParams p) {
  __shared__ __align__(16) float xs[8 * 128], ys[8 * 128], us[8 * 128];
  const int r0 = blockIdx.x * 8, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();   // the decode kernel may launch; it waits for this grid before reading q'
  for (int i = tid; i < 8 * 128; i += 256) {
    const int r = i >> 7, j = i & 127;
    xs[i] = (r0 + r < p.rows) ? load_elem(p.q, p.dtype, static_cast<int64_t>(r0 + r) * 128 + j) : 0.f;
  }
  __syncthreads();
  matvec8x128(p.rot, xs, ys, p.scale, warp, lane);
  __syncthreads();
  const bool prod = p.kind == TQ_KIND_PROD;
  if (prod) {
    matvec8x128(p.S, ys, us, 1.f, warp, lane);
    __syncthreads();
  }
  const int r = r0 + warp;                         // warp w normalizes row w
  if (r >= p.rows) return;
  if (p.kind == TQ_KIND_SPECTRAL) {
    // qa: sigma_j q'_j on the tail dims (0 on the top dims); qb slots 0..7: sigma_j q'_j of
    // the top dims, slots 8..15: coef * (S q'_top)_i (QJL)
    const float* y = ys + warp * 128;
    float a4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = 4 * lane + i;
      a4[i] = j < p.k_top ? 0.f : y[j] * __ldg(p.dim_sigma + j);
    }
    float ma = fmaxf(fmaxf(fabsf(a4[0]), fabsf(a4[1])), fmaxf(fabsf(a4[2]), fabsf(a4[3])));
    ma = warp_max(ma);
    const float sa = ma > 0.f ? ma : 1.f;
    reinterpret_cast<float4*>(p.qa + static_cast<int64_t>(r) * 128)[lane] =
        make_float4(a4[0] / sa, a4[1] / sa, a4[2] / sa, a4[3] / sa);
    float bv = 0.f;                                 // lane i < 16: slot i
    if (lane < p.k_top) bv = y[lane] * __ldg(p.dim_sigma + lane);
    else if (lane >= 8 && lane < 8 + p.k_top && p.qjl) {
      const int ii = lane - 8;
      for (int k = 0; k < p.k_top; ++k) bv = fmaf(__ldg(p.S + ii * p.k_top + k), y[k], bv);
      bv *= p.spec_coef;
    }
    if (lane >= 16) bv = 0.f;
    float mb = warp_max(fabsf(bv));
    const float sb = mb > 0.f ? mb : 1.f;
    if (lane < p.qb_stride) p.qb[static_cast<int64_t>(r) * p.qb_stride + lane] = bv / sb;
    if (lane == 0) { p.qs[r * 2] = sa; p.qs[r * 2 + 1] = sb; }
    return;
  }
  const float4 a = *reinterpret_cast<const float4*>(ys + warp * 128 + 4 * lane);
  float ma = fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w)));
  ma = warp_max(ma);
  const float sa = ma > 0.f ? ma : 1.f;
  reinterpret_cast<float4*>(p.qa + static_cast<int64_t>(r) * 128)[lane] =
      make_float4(a.x / sa, a.y / sa, a.z / sa, a.w / sa);
  float sb = 1.f;
  const int n2 = p.qb_stride;
  if (prod) {                                       // n2 = m = 128
    const float4 u = *reinterpret_cast<const float4*>(us + warp * 128 + 4 * lane);
    float mb = fmaxf(fmaxf(fabsf(u.x), fabsf(u.y)), fmaxf(fabsf(u.z), fabsf(u.w)));
    mb = warp_max(mb);
    sb = mb > 0.f ? mb : 1.f;
    reinterpret_cast<float4*>(p.qb + static_cast<int64_t>(r) * n2)[lane] =
        make_float4(u.x / sb, u.y / sb, u.z / sb, u.w / sb);
  } else {
    for (int i = lane; i < n2; i += 32) p.qb[static_cast<int64_t>(r) * n2 + i] = 0.f;
  }
  if (lane == 0) { p.qs[r * 2] = sa; p.qs[r * 2 + 1] = sb; }
}

// combine_kernel with d = 128: 2 rows per CTA of 256 threads (many CTAs: the step is a
// few microseconds of dependent loads); dynamic shared memory holds the chunk weights
// 2^(m_c - M) / L of the 2 rows ([2][n_chunks] floats).
__global__ void __launch_bounds__(256) combine128_kernel(CombineParams p) {
  constexpr int R = 2;
  extern __shared__ __align__(16) float cw[];       // [R][n_chunks] weights, then rot_V [128][128]
  __shared__ __align__(16) float ov[R * 128];      // o' per row
  const int r0 = blockIdx.x * R, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nch = p.n_chunks;
  // rot_V is an input, not a decode result: its copy into shared memory is issued before
  // the wait for the decode kernel and lands while that kernel drains
  float* rv = cw + ((R * nch + 3) & ~3);
  const uint32_t rv_s = static_cast<uint32_t>(__cvta_generic_to_shared(rv));
  if ((reinterpret_cast<uintptr_t>(p.rot_v) & 15u) == 0) {
    for (int i = tid; i < 128 * 128 / 4; i += 256)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(rv_s + 16u * i), "l"(p.rot_v + 4 * i) : "memory");
  } else {
    for (int i = tid; i < 128 * 128; i += 256)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(rv_s + 4u * i), "l"(p.rot_v + i) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  pdl_wait();      // the partials come from the decode kernel before this one
  if (warp < R) {
    float* w = cw + warp * nch;
    const int r = r0 + warp;
    if (r < p.rows) {
      const float* ml = p.part_ml + static_cast<int64_t>(r) * nch * 2;
      float M = -INFINITY;
      for (int c = lane; c < nch; c += 32) M = fmaxf(M, ml[c * 2]);
      M = warp_max(M);
      float L = 0.f;
      for (int c = lane; c < nch; c += 32) {
        const float mc = ml[c * 2];
        const float e = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
        w[c] = e;
        L += e * ml[c * 2 + 1];
      }
      L = warp_sum(L);
      const float invL = L > 0.f ? 1.f / L : 0.f;
      for (int c = lane; c < nch; c += 32) w[c] *= invL;
    } else {
      for (int c = lane; c < nch; c += 32) w[c] = 0.f;
    }
  }
  __syncthreads();
  const int rr = tid >> 7, k = tid & 127;           // thread: row rr, dim k
  const int r = r0 + rr;
  {
    float a = 0.f;
    if (r < p.rows) {
      const float* w = cw + rr * nch;
      const float* po = p.part_o + static_cast<int64_t>(r) * nch * 128 + k;
#pragma unroll 8
      for (int c = 0; c < nch; ++c) a = fmaf(w[c], __ldg(po + c * 128), a);
      if (p.v_sigma) a *= p.v_sigma[k];
    }
    ov[rr * 128 + k] = a;
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  float o = 0.f;
#pragma unroll 8
  for (int j = 0; j < 128; ++j) o = fmaf(ov[rr * 128 + j], rv[j * 128 + k], o);
  if (r < p.rows) p.out[static_cast<int64_t>(r) * 128 + k] = o;
}

}  // namespace tq
