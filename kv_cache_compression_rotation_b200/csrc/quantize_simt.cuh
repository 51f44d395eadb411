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
};

__device__ __forceinline__ void spectral_dim_book(const SimtQuantParams& p, int j, int* bits,
                                                  float* sig) {
  *bits = j < p.k_top ? p.top_bits[j] : p.tail_bits;
  *sig = p.dim_sigma[j];
}

// Shared memory: xs[tv][d] f32 | ys[tv][d] f32 | code8[tv][d] u8 | nu[tv] | inv[tv] | gam[tv]
__global__ void __launch_bounds__(kSimtThreads)
simt_quantize_kernel(SimtQuantParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int d = p.d, tv = p.tv;
  float* xs = reinterpret_cast<float*>(smem);
  float* ys = xs + tv * d;
  float* nu = ys + tv * d;
  float* inv = nu + tv;
  float* gam = inv + tv;
  uint8_t* code8 = reinterpret_cast<uint8_t*>(gam + tv);
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * tv;
  const int nv = static_cast<int>(min(static_cast<int64_t>(tv), p.n - v0));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int i = tid; i < tv * d; i += kSimtThreads) {
    const int v = i / d;
    xs[i] = v < nv ? load_elem(p.x, p.dtype, (v0 + v) * d + (i - v * d)) : 0.f;
  }
  __syncthreads();
  for (int v = warp; v < tv; v += kSimtThreads / 32) {
    float s = 0.f;
    for (int k = lane; k < d; k += 32) s += xs[v * d + k] * xs[v * d + k];
    s = warp_sum(s);
    if (lane == 0) {
      const float r = sqrtf(s);
      nu[v] = r;
      inv[v] = (p.kind == TQ_KIND_SPECTRAL) ? 1.f : (r > 0.f ? 1.f / r : 0.f);
    }
  }
  __syncthreads();
  // y = rot @ x (per vector), scaled to the unit sphere for mse / prod
  for (int j = tid; j < d; j += kSimtThreads) {
    const float* rrow = p.rot + static_cast<int64_t>(j) * d;
    for (int vb = 0; vb < tv; vb += 8) {
      float acc[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] = 0.f;
      for (int k = 0; k < d; ++k) {
        const float r = __ldg(rrow + k);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (vb + u < tv) acc[u] = fmaf(r, xs[(vb + u) * d + k], acc[u]);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (vb + u < tv) ys[(vb + u) * d + j] = acc[u] * inv[vb + u];
    }
  }
  __syncthreads();
  // scalar codes (and residual for prod / spectral-qjl, kept in xs)
  for (int i = tid; i < tv * d; i += kSimtThreads) {
    const int j = i % d;
    const float y = ys[i];
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
    xs[i] = y - chat;   // residual (x no longer needed)
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
      p.codes[(v0 + v) * p.code_words + hw + w] = word;
    }
    if (tid < tv && tid < nv) {
      const int v = tid;
      float proj[TQ_MAX_TOP];
      float g2 = 0.f;
      if (p.qjl) {
        for (int i = 0; i < k; ++i) g2 += xs[v * d + i] * xs[v * d + i];
        for (int i = 0; i < k; ++i) {
          float a = 0.f;
          for (int kk = 0; kk < k; ++kk) a = fmaf(__ldg(p.S + i * k + kk), xs[v * d + kk], a);
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
      uint32_t* dst = p.codes + (v0 + v) * p.code_words;
      for (int w = 0; w < hw; ++w) {
        const uint64_t src = head[w >> 1];
        dst[w] = static_cast<uint32_t>((w & 1) ? (src >> 32) : src);
      }
      if (p.qjl && p.rnorms) p.rnorms[v0 + v] = sqrtf(g2);
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
      p.codes[(v0 + v) * W + w] = word;
    }
  }
  if (tid < nv && p.norms) p.norms[v0 + tid] = nu[tid];
  if (p.kind != TQ_KIND_PROD) return;
  // prod: gamma = ||r||, signs of S r by warp ballot (32 rows of S per warp step)
  for (int v = warp; v < tv; v += kSimtThreads / 32) {
    float s = 0.f;
    for (int k = lane; k < d; k += 32) s += xs[v * d + k] * xs[v * d + k];
    s = warp_sum(s);
    if (lane == 0) gam[v] = sqrtf(s);
  }
  __syncthreads();
  if (tid < nv && p.rnorms) p.rnorms[v0 + tid] = gam[tid];
  for (int ib = warp * 32; ib < p.m; ib += kSimtThreads) {
    const int i = ib + lane;
    const float* srow = p.S + static_cast<int64_t>(min(i, p.m - 1)) * d;
    for (int v = 0; v < nv; ++v) {
      float a = 0.f;
      for (int k = 0; k < d; ++k) a = fmaf(__ldg(srow + k), xs[v * d + k], a);
      const unsigned bits = __ballot_sync(0xffffffffu, i < p.m && a >= 0.f);
      if (lane == 0) p.signs[(v0 + v) * p.sign_words + (ib >> 5)] = bits;
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
