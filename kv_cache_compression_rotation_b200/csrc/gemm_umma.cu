// Instantiations of the split-precision tensor-core product (wide-vector quantize).
#include "gemm_umma.cuh"
#include "launchers.h"

namespace tq {
namespace {

// Elementwise split of fp32 rows into bf16 hi + lo parts, with the row norm: one warp per
// row (x [rows][d], d a multiple of 8; also used for Pi and S with norms = nullptr).
__global__ void __launch_bounds__(256) split_rows_kernel(const float* __restrict__ x, int64_t rows, int d,
                                                         uint16_t* __restrict__ hi, uint16_t* __restrict__ lo,
                                                         float* __restrict__ norms) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float4* src = reinterpret_cast<const float4*>(x + row * d);
  uint2* dh = reinterpret_cast<uint2*>(hi + row * d);
  uint2* dl = reinterpret_cast<uint2*>(lo + row * d);
  float ss = 0.f;
  for (int i = lane; i < d / 4; i += 32) {
    const float4 v = __ldg(src + i);
    const float a[4] = {v.x, v.y, v.z, v.w};
    uint32_t h[2], l[2];
#pragma unroll
    for (int k = 0; k < 4; k += 2) {
      const __nv_bfloat162 hb = __floats2bfloat162_rn(a[k], a[k + 1]);
      const float2 back = __bfloat1622float2(hb);
      const __nv_bfloat162 lb = __floats2bfloat162_rn(a[k] - back.x, a[k + 1] - back.y);
      h[k >> 1] = *reinterpret_cast<const uint32_t*>(&hb);
      l[k >> 1] = *reinterpret_cast<const uint32_t*>(&lb);
      ss = fmaf(a[k], a[k], fmaf(a[k + 1], a[k + 1], ss));
    }
    dh[i] = make_uint2(h[0], h[1]);
    dl[i] = make_uint2(l[0], l[1]);
  }
  if (norms) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) norms[row] = sqrtf(ss);
  }
}


template <int EPI, int B, int TN>
cudaError_t go_tn(const CUtensorMap* maps, const SplitGemmParams& p, int grid, cudaStream_t s) {
  auto k = split_gemm_kernel<EPI, B, TN>;
  const uint32_t smem = gemm_smem_bytes(TN);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  k<<<grid, kGemmThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], p);
  return cudaGetLastError();
}

// N tiles of 256 columns, or of 128 when N is not a multiple of 256
template <int EPI, int B>
cudaError_t go(const CUtensorMap* maps, const SplitGemmParams& p, int grid, cudaStream_t s) {
  return gemm_tile_n(p.N) == 256 ? go_tn<EPI, B, 256>(maps, p, grid, s) : go_tn<EPI, B, 128>(maps, p, grid, s);
}

// Queries for the tensor-core estimator: row r of [qr | qu] (fp32, d + m columns) as bf16
// hi + lo parts.  While *sym is nonzero (records expanded as +-1 in units of c[1]) the qr
// columns carry that centroid.
__global__ void __launch_bounds__(256) split_cat_kernel(const float* __restrict__ a, int da,
                                                        const float* __restrict__ b, int db, int64_t rows,
                                                        uint16_t* __restrict__ hi, uint16_t* __restrict__ lo,
                                                        const int* sym, const float* centroids) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int k = da + db;
  if (i >= rows * k) return;
  const int64_t r = i / k;
  const int c = static_cast<int>(i - r * k);
  const float sa = (sym && *sym) ? __ldg(centroids + 1) : 1.f;
  const float v = c < da ? a[r * da + c] * sa : b[r * db + (c - da)];
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  hi[i] = __bfloat16_as_ushort(h);
  lo[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v - __bfloat162float(h)));
}

// Records for the tensor-core estimator: row i = [c[code_i] (d) | coef * gamma_i * (2 s_i - 1) (m)]
// as bf16 hi + lo parts (one warp per record; B code bits, LSB-first stream).
template <int B>
__global__ void __launch_bounds__(256) expand_records_kernel(const uint32_t* __restrict__ codes, int code_words,
                                                             const uint32_t* __restrict__ signs, int sign_words,
                                                             const float* __restrict__ rnorms,
                                                             const float* __restrict__ centroids, float coef,
                                                             int64_t n, int d, int m, uint16_t* __restrict__ hi,
                                                             uint16_t* __restrict__ lo) {
  const int lane = threadIdx.x & 31;
  const int64_t rec = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (rec >= n) return;
  const int k = d + m;
  const uint32_t* cw = codes + rec * code_words;
  uint16_t* h = hi + rec * k;
  uint16_t* l = lo + rec * k;
  for (int j = lane; j < d; j += 32) {
    const int pos = j * B, w = pos >> 5, sh = pos & 31;
    uint32_t code = cw[w] >> sh;
    if (sh + B > 32) code |= cw[w + 1] << (32 - sh);
    const float v = __ldg(centroids + (code & ((1u << B) - 1u)));
    const __nv_bfloat16 vh = __float2bfloat16_rn(v);
    h[j] = __bfloat16_as_ushort(vh);
    l[j] = __bfloat16_as_ushort(__float2bfloat16_rn(v - __bfloat162float(vh)));
  }
  if (m > 0) {
    const float g = coef * rnorms[rec];
    const __nv_bfloat16 gh = __float2bfloat16_rn(g);
    const __nv_bfloat16 gl = __float2bfloat16_rn(g - __bfloat162float(gh));
    const uint16_t ph = __bfloat16_as_ushort(gh), pl = __bfloat16_as_ushort(gl);
    const uint32_t* sw = signs + rec * sign_words;
    for (int i = lane; i < m; i += 32) {
      const bool pos = (sw[i >> 5] >> (i & 31)) & 1u;
      // -x flips the sign bit of a bf16 (gamma >= 0)
      h[d + i] = pos ? ph : static_cast<uint16_t>(ph ^ 0x8000u);
      l[d + i] = pos ? pl : static_cast<uint16_t>(pl ^ 0x8000u);
    }
  }
}

// The same records, 8 consecutive values per lane and step with one 16-byte store of each
// part: d and m multiples of 8, hi and lo 16-byte aligned.  The hi / lo rounding is that of
// expand_records_kernel value by value.  1-bit codes with c[0] = -c[1] (sym_flag given):
// the d code columns are written as exactly +-1 (units of c[1], which the queries then
// carry) with no lo part, and *sym_flag = 1 tells the query split and the product so.
template <int B>
__global__ void __launch_bounds__(256) expand_records8_kernel(const uint32_t* __restrict__ codes, int code_words,
                                                              const uint32_t* __restrict__ signs, int sign_words,
                                                              const float* __restrict__ rnorms,
                                                              const float* __restrict__ centroids, float coef,
                                                              int64_t n, int d, int m, uint16_t* __restrict__ hi,
                                                              uint16_t* __restrict__ lo, int* sym_flag) {
  constexpr uint32_t kMask = (1u << B) - 1u;
  __shared__ float cs[1 << B];
  if (threadIdx.x < (1u << B)) cs[threadIdx.x] = __ldg(centroids + threadIdx.x);
  __syncthreads();
  const bool sym = B == 1 && sym_flag != nullptr && cs[0] == -cs[1];
  if (sym_flag && blockIdx.x == 0 && threadIdx.x == 0) *sym_flag = sym ? 1 : 0;
  const int lane = threadIdx.x & 31;
  const int64_t rec = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (rec >= n) return;
  const int64_t k = d + m;
  const uint32_t* cw = codes + rec * code_words;
  uint4* h = reinterpret_cast<uint4*>(hi + rec * k);
  uint4* l = reinterpret_cast<uint4*>(lo + rec * k);
  for (int gi = lane; gi < d / 8; gi += 32) {
    // codes of dims 8 gi .. 8 gi + 7: 8 B bits from bit 8 gi B of the stream
    const int pos = gi * 8 * B, w = pos >> 5, sh = pos & 31;
    uint32_t bits = cw[w] >> sh;
    if (sh + 8 * B > 32) bits |= cw[w + 1] << (32 - sh);
    if (sym) {
      // bf16 -1 is 0xBF80; code 1 (+1) clears the sign bit
      uint32_t hv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        hv[j] = 0xBF80BF80u ^ (((bits >> (2 * j)) & 1u) << 15) ^ (((bits >> (2 * j + 1)) & 1u) << 31);
      h[gi] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      continue;
    }
    uint32_t hv[4], lv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = cs[(bits >> (2 * j * B)) & kMask];
      const float b = cs[(bits >> ((2 * j + 1) * B)) & kMask];
      const __nv_bfloat162 hb = __floats2bfloat162_rn(a, b);
      const float2 back = __bfloat1622float2(hb);
      const __nv_bfloat162 lb = __floats2bfloat162_rn(a - back.x, b - back.y);
      hv[j] = *reinterpret_cast<const uint32_t*>(&hb);
      lv[j] = *reinterpret_cast<const uint32_t*>(&lb);
    }
    h[gi] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    l[gi] = make_uint4(lv[0], lv[1], lv[2], lv[3]);
  }
  if (m > 0) {
    const float g = coef * rnorms[rec];
    const __nv_bfloat16 gh = __float2bfloat16_rn(g);
    const __nv_bfloat16 gl = __float2bfloat16_rn(g - __bfloat162float(gh));
    const uint32_t ph = __bfloat16_as_ushort(gh), pl = __bfloat16_as_ushort(gl);
    const uint32_t ph2 = ph | (ph << 16), pl2 = pl | (pl << 16);
    // byte gi of the sign words holds signs 8 gi .. 8 gi + 7 (LSB first)
    const unsigned char* sb = reinterpret_cast<const unsigned char*>(signs + rec * sign_words);
    uint4* h2 = reinterpret_cast<uint4*>(hi + rec * k + d);
    uint4* l2 = reinterpret_cast<uint4*>(lo + rec * k + d);
    for (int gi = lane; gi < m / 8; gi += 32) {
      const uint32_t ns = ~static_cast<uint32_t>(sb[gi]);   // set bit: a negative sign
      uint32_t hv[4], lv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // -x flips the sign bit of a bf16 (gamma >= 0): bit 15 of the low half, 31 of the high
        const uint32_t flip = (((ns >> (2 * j)) & 1u) << 15) | (((ns >> (2 * j + 1)) & 1u) << 31);
        hv[j] = ph2 ^ flip;
        lv[j] = pl2 ^ flip;
      }
      h2[gi] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      l2[gi] = make_uint4(lv[0], lv[1], lv[2], lv[3]);
    }
  }
}

}  // namespace

cudaError_t launch_split_cat(const float* a, int da, const float* b, int db, int64_t rows, uint16_t* hi,
                             uint16_t* lo, cudaStream_t s, const int* sym, const float* centroids) {
  const int64_t total = rows * (da + db);
  split_cat_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(a, da, b, db, rows, hi, lo, sym,
                                                                                centroids);
  return cudaGetLastError();
}

cudaError_t launch_expand_records(const uint32_t* codes, int code_words, const uint32_t* signs, int sign_words,
                                  const float* rnorms, const float* centroids, float coef, int64_t n, int d, int m,
                                  int bits, uint16_t* hi, uint16_t* lo, int* sym_flag, cudaStream_t s) {
  const unsigned blocks = static_cast<unsigned>((n + 7) / 8);
  const bool vec = d % 8 == 0 && m % 8 == 0 && ((reinterpret_cast<uintptr_t>(hi) | reinterpret_cast<uintptr_t>(lo)) & 15u) == 0;
  if (vec) {
    switch (bits) {
      case 1: expand_records8_kernel<1><<<blocks, 256, 0, s>>>(codes, code_words, signs, sign_words, rnorms, centroids, coef, n, d, m, hi, lo, sym_flag); break;
      case 2: expand_records8_kernel<2><<<blocks, 256, 0, s>>>(codes, code_words, signs, sign_words, rnorms, centroids, coef, n, d, m, hi, lo, sym_flag); break;
      case 3: expand_records8_kernel<3><<<blocks, 256, 0, s>>>(codes, code_words, signs, sign_words, rnorms, centroids, coef, n, d, m, hi, lo, sym_flag); break;
      case 4: expand_records8_kernel<4><<<blocks, 256, 0, s>>>(codes, code_words, signs, sign_words, rnorms, centroids, coef, n, d, m, hi, lo, sym_flag); break;
      default: return cudaErrorNotSupported;
    }
    return cudaGetLastError();
  }
  // the value-by-value kernel always writes both parts
  if (sym_flag) {
    const cudaError_t e = cudaMemsetAsync(sym_flag, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
  }
  switch (bits) {
    case 1: expand_records_kernel<1><<<blocks, 256, 0, s>>>(codes, code_words, signs, sign_words, rnorms, centroids, coef, n, d, m, hi, lo); break;
    case 2: expand_records_kernel<2><<<blocks, 256, 0, s>>>(codes, code_words, signs, sign_words, rnorms, centroids, coef, n, d, m, hi, lo); break;
    case 3: expand_records_kernel<3><<<blocks, 256, 0, s>>>(codes, code_words, signs, sign_words, rnorms, centroids, coef, n, d, m, hi, lo); break;
    case 4: expand_records_kernel<4><<<blocks, 256, 0, s>>>(codes, code_words, signs, sign_words, rnorms, centroids, coef, n, d, m, hi, lo); break;
    default: return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

cudaError_t launch_split_gemm(const CUtensorMap* maps, const SplitGemmParams& p, int epi, int bits, int grid,
                              cudaStream_t s) {
  if (epi == GEMM_EPI_SIGNS) return go<GEMM_EPI_SIGNS, 1>(maps, p, grid, s);
  if (epi == GEMM_EPI_SCORE) return go<GEMM_EPI_SCORE, 1>(maps, p, grid, s);
  switch (bits) {
    case 1: return go<GEMM_EPI_QUANT, 1>(maps, p, grid, s);
    case 2: return go<GEMM_EPI_QUANT, 2>(maps, p, grid, s);
    case 3: return go<GEMM_EPI_QUANT, 3>(maps, p, grid, s);
    case 4: return go<GEMM_EPI_QUANT, 4>(maps, p, grid, s);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t launch_split_rows(const float* x, int64_t rows, int d, uint16_t* hi, uint16_t* lo, float* norms,
                              cudaStream_t s) {
  split_rows_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(x, rows, d, hi, lo, norms);
  return cudaGetLastError();
}

}  // namespace tq
