// General-shape quantize / dequantize kernels on CUDA cores (any d up to 2048).
//
// These cover every descriptor the ABI accepts; the tensor-core kernel
// (quantize_umma.cuh) takes over for the shapes it supports.  One CTA handles a
// tile of TV vectors held in shared memory as fp32:
//   1. load x (fp32 / bf16 / fp16) and reduce ||x|| per vector (TurboQuant review,
//      Limitations: norms stored separately; the codebook sees x/||x||);
//   2. y = rot @ x, one output coordinate per thread, scaled by 1/||x||;
//   3. code_j = #{k : t_k < y_j} by binary search over the boundaries;
//   4. pack codes LSB-first into the record's word stream;
//   5. (prod) r = y - c[code], ||r||, signs of S r packed by warp ballot;
//      (spectral) per-dimension codebooks, QJL on the top-k residual.
#pragma once

#include "device_common.cuh"

namespace tq {

constexpr int kSimtThreads = 256;

struct SimtQuantParams {
  const void* x;
  int dtype;
  int64_t n;
  int d;
  int kind;
  const float* rot;
  const float* S;
  int m;              // QJL rows (prod) / k_top (spectral with qjl) / 0
  const float* centroids;
  const float* boundaries;
  int bmse;           // MSE code bits (prod: bits-1)
  // spectral
  int k_top, tail_bits, qjl;
  int top_bits[TQ_MAX_TOP];
  const float* dim_sigma;
  const float* unit_c;
  const float* unit_t;
  // outputs
  uint32_t* codes;
  int code_words;
  uint32_t* signs;
  int sign_words;
  float* norms;
  float* rnorms;
  int tv;             // vectors per CTA
  // input gather: element j of vector v is x[v * ld + (cols ? cols[j] : j)]; a column
  // outside 0..ld-1 reads column 0 and reports TQ_ERR_INVALID_ARG to *status
  int64_t ld;
  const int32_t* cols;
  int* status;
  // output rows: record v goes to slot orow(v) (paged append: vector v = b * Hkv + h is the
  // newest token seq_lens[b] - 1 of (b, h), placed through the block table)
  const int32_t* pg_table;    // [B][pg_max] page ids, or nullptr (record v at slot v)
  const int32_t* pg_seq;      // [B] token counts including the appended one
  int pg_size, pg_max, pg_hkv;
  int64_t pg_num;
};

// Record slot of output vector v; -1 when the block table or the length is out of range
// (reported as TQ_ERR_INVALID_ARG by the caller of this function, and nothing is written).
__device__ __forceinline__ int64_t simt_out_row(const SimtQuantParams& p, int64_t v) {
  if (!p.pg_table) return v;
  const int b = static_cast<int>(v / p.pg_hkv), h = static_cast<int>(v - static_cast<int64_t>(b) * p.pg_hkv);
  const int t = p.pg_seq[b] - 1;
  if (t < 0 || t >= p.pg_size * p.pg_max) return -1;
  const int pg = p.pg_table[static_cast<int64_t>(b) * p.pg_max + t / p.pg_size];
  if (pg < 0 || pg >= p.pg_num) return -1;
  return (static_cast<int64_t>(pg) * p.pg_hkv + h) * p.pg_size + t % p.pg_size;
}

__device__ __forceinline__ void spectral_dim_book(const SimtQuantParams& p, int j, int* bits,
                                                  float* sig) {
  *bits = j < p.k_top ? p.top_bits[j] : p.tail_bits;
  *sig = p.dim_sigma[j];
}

// Tiled product on CUDA cores: out[v][j] = scale_v * sum_k A[v][k] M[j][k] for v < 8 * VPT
// rows of A (shared memory, row stride lda, zero-padded to a multiple of 32 columns) and
// j < mrows rows of M (global, row-major [mrows][d]).  M is staged through shared memory
// in 32-column chunks of 128 rows (Ms, [32][kMsStride], transposed); thread (ty, tx) owns
// rows ty * VPT .. + VPT - 1 and outputs tx + 32 q of each 128-row block.
constexpr int kMsStride = 132;

template <int VPT>
__device__ __forceinline__ void tile_gemm(const float* A, int lda, const float* __restrict__ M, int mrows, int d,
                                          float* out, int ldo, const float* rowscale, float* Ms) {
  const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
  const int dp = (d + 31) & ~31;
  for (int jb = 0; jb < mrows; jb += 128) {
    float acc[VPT][4];
#pragma unroll
    for (int v = 0; v < VPT; ++v)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[v][q] = 0.f;
    for (int k0 = 0; k0 < dp; k0 += 32) {
      __syncthreads();                              // Ms is free
      for (int i = tid; i < 32 * 128; i += kSimtThreads) {
        const int jj = i >> 5, kk = i & 31, row = jb + jj, col = k0 + kk;
        Ms[kk * kMsStride + jj] = (row < mrows && col < d) ? __ldg(M + static_cast<int64_t>(row) * d + col) : 0.f;
      }
      __syncthreads();
#pragma unroll 2
      for (int kk = 0; kk < 32; kk += 4) {
        float4 a[VPT];
#pragma unroll
        for (int v = 0; v < VPT; ++v) a[v] = *reinterpret_cast<const float4*>(A + (ty * VPT + v) * lda + k0 + kk);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          float b[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) b[q] = Ms[(kk + k4) * kMsStride + tx + 32 * q];
#pragma unroll
          for (int v = 0; v < VPT; ++v) {
            const float av = k4 == 0 ? a[v].x : (k4 == 1 ? a[v].y : (k4 == 2 ? a[v].z : a[v].w));
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[v][q] = fmaf(av, b[q], acc[v][q]);
          }
        }
      }
    }
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const float sc = rowscale ? rowscale[ty * VPT + v] : 1.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = jb + tx + 32 * q;
        if (j < mrows) out[(ty * VPT + v) * ldo + j] = acc[v][q] * sc;
      }
    }
  }
  __syncthreads();
}

// Shared memory: xs[tv][dp] f32 | ys[tv][yp] f32 | Ms[32][kMsStride] f32 | nu[tv] | inv[tv] |
// gam[tv] | code8[tv][d] u8, with dp = d and yp = max(d, m) rounded up to 32 (zero padding).
__global__ void __launch_bounds__(kSimtThreads)
simt_quantize_kernel(SimtQuantParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int d = p.d, tv = p.tv;
  const int dp = (d + 31) & ~31, yp = (max(d, p.m) + 31) & ~31;
  float* xs = reinterpret_cast<float*>(smem);
  float* ys = xs + tv * dp;
  float* Ms = ys + tv * yp;
  float* nu = Ms + 32 * kMsStride;
  float* inv = nu + tv;
  float* gam = inv + tv;
  uint8_t* code8 = reinterpret_cast<uint8_t*>(gam + tv);
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * tv;
  const int nv = static_cast<int>(min(static_cast<int64_t>(tv), p.n - v0));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int i = tid; i < tv * dp; i += kSimtThreads) {
    const int v = i / dp, k = i - v * dp;
    float xv = 0.f;
    if (v < nv && k < d) {
      int64_t col = k;
      if (p.cols) {
        col = __ldg(p.cols + k);
        if (col < 0 || col >= p.ld) {
          report_status(p.status, TQ_ERR_INVALID_ARG);
          col = 0;
        }
      }
      xv = load_elem(p.x, p.dtype, (v0 + v) * p.ld + col);
    }
    xs[i] = xv;
  }
  __syncthreads();
  for (int v = warp; v < tv; v += kSimtThreads / 32) {
    float s = 0.f;
    for (int k = lane; k < d; k += 32) s += xs[v * dp + k] * xs[v * dp + k];
    s = warp_sum(s);
    if (lane == 0) {
      const float r = sqrtf(s);
      nu[v] = r;
      inv[v] = (p.kind == TQ_KIND_SPECTRAL) ? 1.f : (r > 0.f ? 1.f / r : 0.f);
    }
  }
  __syncthreads();
  // y = rot @ x (per vector), scaled to the unit sphere for mse / prod
  switch (tv / 8) {
    case 1: tile_gemm<1>(xs, dp, p.rot, d, d, ys, yp, inv, Ms); break;
    case 2: tile_gemm<2>(xs, dp, p.rot, d, d, ys, yp, inv, Ms); break;
    case 3: tile_gemm<3>(xs, dp, p.rot, d, d, ys, yp, inv, Ms); break;
    default: tile_gemm<4>(xs, dp, p.rot, d, d, ys, yp, inv, Ms); break;
  }
  // scalar codes (and residual for prod / spectral-qjl, kept in xs)
  for (int i = tid; i < tv * d; i += kSimtThreads) {
    const int v = i / d, j = i - v * d;
    const float y = ys[v * yp + j];
    int c = 0;
    float chat = 0.f;
    if (p.kind == TQ_KIND_SPECTRAL) {
      int b; float sg;
      spectral_dim_book(p, j, &b, &sg);
      if (b > 0) {
        const float* t = p.unit_t + unit_t_off(b);
        const int nb = (1 << b) - 1;
        int lo = 0, hi = nb;   // #{k : sg * t_k < y}
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (sg * __ldg(t + mid) < y) lo = mid + 1; else hi = mid;
        }
        c = lo;
        chat = sg * __ldg(p.unit_c + unit_c_off(b) + c);
      }
    } else if (p.bmse > 0) {
      c = count_below(p.boundaries, (1 << p.bmse) - 1, y);
      chat = __ldg(p.centroids + c);
    }
    code8[i] = static_cast<uint8_t>(c);
    xs[v * dp + j] = y - chat;   // residual (x no longer needed; padding stays 0)
  }
  __syncthreads();
  // pack code words
  if (p.kind == TQ_KIND_SPECTRAL) {
    const int k = p.k_top, tb = p.tail_bits;
    int head_bits = 0;
    for (int j = 0; j < k; ++j) head_bits += p.top_bits[j];
    const int hw = (head_bits + (p.qjl ? k : 0) + 31) >> 5;
    const int tw = words_for(d, tb);
    for (int i = tid; i < tv * tw; i += kSimtThreads) {
      const int v = i / tw, w = i - v * tw;
      if (v >= nv) continue;
      uint32_t word = 0;
      const int j0 = max(k, (32 * w) / tb), j1 = min(d - 1, (32 * w + 31) / tb);
      for (int j = j0; j <= j1; ++j) {
        const int pos = j * tb - 32 * w;
        const uint64_t c = code8[v * d + j];
        if (pos >= 0) word |= static_cast<uint32_t>(c << pos);
        else word |= static_cast<uint32_t>(c >> (-pos));
      }
      const int64_t o = simt_out_row(p, v0 + v);
      if (o >= 0) p.codes[o * p.code_words + hw + w] = word;
    }
    if (tid < tv && tid < nv) {
      const int v = tid;
      float proj[TQ_MAX_TOP];
      float g2 = 0.f;
      if (p.qjl) {
        for (int i = 0; i < k; ++i) g2 += xs[v * dp + i] * xs[v * dp + i];
        for (int i = 0; i < k; ++i) {
          float a = 0.f;
          for (int kk = 0; kk < k; ++kk) a = fmaf(__ldg(p.S + i * k + kk), xs[v * dp + kk], a);
          proj[i] = a;
        }
      }
      uint64_t head[2] = {0ull, 0ull};   // up to 8*8 + 8 = 72 bits; hw <= 3 words
      uint32_t extra = 0;
      int pos = 0;
      auto put = [&](uint32_t val, int nb) {
        for (int bb = 0; bb < nb; ++bb, ++pos) {
          const uint32_t bit = (val >> bb) & 1u;
          if (pos < 64) head[0] |= static_cast<uint64_t>(bit) << pos;
          else if (pos < 128) head[1] |= static_cast<uint64_t>(bit) << (pos - 64);
          else extra |= bit << (pos - 128);
        }
      };
      for (int j = 0; j < k; ++j) put(code8[v * d + j], p.top_bits[j]);
      if (p.qjl)
        for (int i = 0; i < k; ++i) put(proj[i] >= 0.f ? 1u : 0u, 1);
      const int64_t orow = simt_out_row(p, v0 + v);
      if (orow >= 0) {
        uint32_t* dst = p.codes + orow * p.code_words;
        for (int w = 0; w < hw; ++w) {
          const uint64_t src = head[w >> 1];
          dst[w] = static_cast<uint32_t>((w & 1) ? (src >> 32) : src);
        }
        if (p.qjl && p.rnorms) p.rnorms[orow] = sqrtf(g2);
      }
      (void)extra;
    }
    return;
  }
  const int b = p.bmse;
  if (b > 0) {
    const int W = p.code_words;
    for (int i = tid; i < tv * W; i += kSimtThreads) {
      const int v = i / W, w = i - v * W;
      if (v >= nv) continue;
      uint32_t word = 0;
      const int j0 = (32 * w) / b, j1 = min(d - 1, (32 * w + 31) / b);
      for (int j = j0; j <= j1; ++j) {
        const int pos = j * b - 32 * w;
        const uint64_t c = code8[v * d + j];
        if (pos >= 0) word |= static_cast<uint32_t>(c << pos);
        else word |= static_cast<uint32_t>(c >> (-pos));
      }
      const int64_t o = simt_out_row(p, v0 + v);
      if (o >= 0) p.codes[o * W + w] = word;
    }
  }
  if (tid < nv) {
    const int64_t o = simt_out_row(p, v0 + tid);
    if (o < 0) report_status(p.status, TQ_ERR_INVALID_ARG);
    else if (p.norms) p.norms[o] = nu[tid];
  }
  if (p.kind != TQ_KIND_PROD) return;
  // prod: gamma = ||r||, then S r for the tile (tiled product) and its signs by warp ballot
  for (int v = warp; v < tv; v += kSimtThreads / 32) {
    float s = 0.f;
    for (int k = lane; k < d; k += 32) s += xs[v * dp + k] * xs[v * dp + k];
    s = warp_sum(s);
    if (lane == 0) gam[v] = sqrtf(s);
  }
  __syncthreads();
  if (tid < nv && p.rnorms) {
    const int64_t o = simt_out_row(p, v0 + tid);
    if (o >= 0) p.rnorms[o] = gam[tid];
  }
  switch (tv / 8) {
    case 1: tile_gemm<1>(xs, dp, p.S, p.m, d, ys, yp, nullptr, Ms); break;
    case 2: tile_gemm<2>(xs, dp, p.S, p.m, d, ys, yp, nullptr, Ms); break;
    case 3: tile_gemm<3>(xs, dp, p.S, p.m, d, ys, yp, nullptr, Ms); break;
    default: tile_gemm<4>(xs, dp, p.S, p.m, d, ys, yp, nullptr, Ms); break;
  }
  for (int v = warp; v < nv; v += kSimtThreads / 32) {
    for (int ib = 0; ib < p.m; ib += 32) {
      const int i = ib + lane;
      const unsigned bits = __ballot_sync(0xffffffffu, i < p.m && ys[v * yp + min(i, p.m - 1)] >= 0.f);
      const int64_t o = simt_out_row(p, v0 + v);
      if (lane == 0 && o >= 0) p.signs[o * p.sign_words + (ib >> 5)] = bits;
    }
  }
}

struct DequantParams {
  int kind, d, bmse, m;
  const float* rot;
  const float* S;
  const float* centroids;
  const uint32_t* codes;
  int code_words;
  const uint32_t* signs;
  int sign_words;
  const float* norms;
  const float* rnorms;
  int k_top, tail_bits, qjl;
  int top_bits[TQ_MAX_TOP];
  const float* dim_sigma;
  const float* unit_c;
  float* out;
  int64_t n;
};

// x_hat[v][k] = sum_j c_hat[v][j] rot[j][k]; one CTA per vector.
__global__ void __launch_bounds__(kSimtThreads) dequant_kernel(DequantParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  float* yh = reinterpret_cast<float*>(smem);
  const int64_t v = blockIdx.x;
  const int d = p.d, tid = threadIdx.x;
  const uint32_t* rec = p.codes + v * p.code_words;
  if (p.kind == TQ_KIND_SPECTRAL) {
    int head_bits = 0;
    for (int j = 0; j < p.k_top; ++j) head_bits += p.top_bits[j];
    const int hw = (head_bits + (p.qjl ? p.k_top : 0) + 31) >> 5;
    for (int j = tid; j < d; j += kSimtThreads) {
      int b, pos;
      if (j < p.k_top) {
        b = p.top_bits[j];
        pos = 0;
        for (int jj = 0; jj < j; ++jj) pos += p.top_bits[jj];
      } else {
        b = p.tail_bits;
        pos = 32 * hw + j * b;
      }
      float c = 0.f;
      if (b > 0) c = p.dim_sigma[j] * __ldg(p.unit_c + unit_c_off(b) + stream_bits(rec, pos, b));
      yh[j] = c;
    }
  } else {
    const float nu = p.norms[v];
    for (int j = tid; j < d; j += kSimtThreads) {
      float c = p.bmse > 0 ? __ldg(p.centroids + stream_bits(rec, j * p.bmse, p.bmse)) : 0.f;
      yh[j] = c * nu;
    }
    if (p.kind == TQ_KIND_PROD) {
      __syncthreads();
      // add sqrt(pi/2)/m * gamma * S^T (2s - 1), scaled by nu
      const float coef = 1.2533141373155003f / p.m * p.rnorms[v] * nu;
      const uint32_t* sg = p.signs + v * p.sign_words;
      for (int j = tid; j < d; j += kSimtThreads) {
        float a = 0.f;
        for (int i = 0; i < p.m; ++i) {
          const float s = ((sg[i >> 5] >> (i & 31)) & 1u) ? 1.f : -1.f;
          a = fmaf(s, __ldg(p.S + static_cast<int64_t>(i) * d + j), a);
        }
        yh[j] += coef * a;
      }
    }
  }
  __syncthreads();
  for (int k = tid; k < d; k += kSimtThreads) {
    float a = 0.f;
    for (int j = 0; j < d; ++j) a = fmaf(yh[j], __ldg(p.rot + static_cast<int64_t>(j) * d + k), a);
    p.out[v * d + k] = a;
  }
}

}  // namespace tq
