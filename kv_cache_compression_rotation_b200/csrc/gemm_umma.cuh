// Split-precision tensor-core product for fp32 vectors (d a multiple of 128, e.g. 128 or 1536):
//
//   C[M x N] = A[M x K] . B[N x K]^T   with A = A_hi + A_lo and B = B_hi + B_lo in bf16,
//   accumulated as A_hi B_hi + A_hi B_lo + A_lo B_hi in fp32 (tensor memory).
//
// The dropped A_lo B_lo term and the bf16 splits leave every entry within ~2^-17 of the
// fp32 product's scale, so a rotated coordinate of a unit vector is exact far inside the
// 1e-5 decision band (TurboQuant review, "Method": y = Pi x / ||x||, then per-coordinate
// Lloyd-Max codes; the QJL variant projects the residual with S).  Rows of A are vectors
// (128 per tile), N is cut into TN-wide chunks (256, or 128 when N is not a multiple of
// 256), K runs in 64-wide stages.
//
// Roles in a persistent CTA (one per SM), 192 threads:
//   warp 0      TMA producer: A_hi, A_lo (128 x 64) and B_hi, B_lo (TN x 64) per stage
//   warp 1      TMEM allocator (512 columns: two TN-column accumulators) and MMA issuer
//   warps 2-5   epilogue: one row per thread, the TN accumulator columns of a tile
// Epilogues:
//   QUANT  y = acc / ||x||: codes against the Lloyd-Max boundaries, packed LSB-first into
//          the record's stream; with a QJL stage, the residual r = y - c[code] as bf16
//          hi + lo (the A operand of the next product) and the tile's part of ||r||^2
//   SIGNS  bit i of the record's sign words = [(S r)_i >= 0]; the first column chunk also
//          writes ||r|| from the parts
//   SCORE  out[row][col] = col_scale[col] * acc (inner-product estimates of queries against
//          decoded records: rows are queries, columns records; the last column tile is
//          partial)
// Every mbarrier wait is bounded (TQ_ERR_TIMEOUT, drain, free TMEM, exit).
#pragma once

#include <cuda.h>

#include "quantize_umma.cuh"

namespace tq {

constexpr int kGemmThreads = 192;
constexpr int kGemmStages = 2;
constexpr int kGemmTileM = 128;
constexpr int kGemmTileK = 64;
constexpr uint32_t kGemmAStage = kGemmTileM * kGemmTileK * 2;     // 16 KB per part
__host__ __device__ constexpr uint32_t gemm_b_stage(int tn) { return static_cast<uint32_t>(tn) * kGemmTileK * 2; }
__host__ __device__ constexpr uint32_t gemm_stage_bytes(int tn) { return 2 * kGemmAStage + 2 * gemm_b_stage(tn); }
__host__ __device__ constexpr uint32_t gemm_smem_bytes(int tn) {
  return 1024 + kGemmStages * gemm_stage_bytes(tn) + 256 + 512 * 4;
}

enum : int { GEMM_EPI_QUANT = 0, GEMM_EPI_SIGNS = 1, GEMM_EPI_SCORE = 2 };

// Column tile of a product with N output columns (the SCORE epilogue takes any N).
__host__ __device__ constexpr int gemm_tile_n(int n) { return n % 256 == 0 || n > 4096 ? 256 : 128; }

struct SplitGemmParams {
  int64_t M;               // rows (vectors)
  int N, K;                // output columns and contraction length (multiples of TN and 64)
  int* status;
  long long wait_limit;
  // QUANT
  const float* rnorm_x;    // [M] ||x|| (0 for a zero row)
  const float* boundaries; // [2^B - 1]
  const float* centroids;  // [2^B]
  uint32_t* codes;         // [M][code_words]
  int code_words;
  uint16_t* r_hi;          // [M][K] bf16 residual parts (QJL stage), or nullptr
  uint16_t* r_lo;
  float* r2_part;          // [M][N / TN] parts of ||r||^2
  float* norms;            // [M] record norms (written once, by column chunk 0)
  // SIGNS
  uint32_t* signs;         // [M][N / 32]
  float* rnorms;           // [M] ||r||
  const float* r2_in;      // [M][n_chunks of the residual] parts of ||r||^2
  int r2_chunks;
  // SCORE
  float* out;              // [M][ldo]
  int64_t ldo;
  const float* col_scale;  // [N]
  // SCORE: while *lo_skip_flag is nonzero the B lo part is zero in columns [0, lo_skip_k) of
  // K (records exactly +-1 there), so those lo loads and their products are not issued
  const int* lo_skip_flag;
  int lo_skip_k;           // multiple of 64
};

// Instruction descriptor: D f32, A/B bf16, both K-major, M = 128, N = tn.
__device__ __forceinline__ uint32_t idesc_m128_bf16(uint32_t tn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((tn >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d_g(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}

template <int EPI, int B, int TN>
__global__ void __launch_bounds__(kGemmThreads, 1)
split_gemm_kernel(const __grid_constant__ CUtensorMap a_hi, const __grid_constant__ CUtensorMap a_lo,
                  const __grid_constant__ CUtensorMap b_hi, const __grid_constant__ CUtensorMap b_lo,
                  const SplitGemmParams p) {
  constexpr int NS = kGemmStages;
  constexpr uint32_t kGemmBStage = gemm_b_stage(TN), kGemmStageBytes = gemm_stage_bytes(TN);
  constexpr int kGemmTileN = TN;
  constexpr int NCH = TN / 32;                   // 32-column chunks of a tile
  constexpr int NB = (1 << B) - 1;
  extern __shared__ unsigned char gsm_raw[];
  const uint32_t raw = smem_u32(gsm_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sm = gsm_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + NS * kGemmStageBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (NS + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * NS + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * NS + 2 + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* tab = reinterpret_cast<float*>(sm + NS * kGemmStageBytes + 256);   // boundaries [NB], centroids [NB+1]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m_tiles = (p.M + kGemmTileM - 1) / kGemmTileM;
  const int n_tiles = (p.N + kGemmTileN - 1) / kGemmTileN;
  const int64_t n_work = m_tiles * n_tiles;
  const int k_steps = p.K / kGemmTileK;
  // first K column whose B lo part is read (a flag written by the record expansion)
  const int k_lo0 = (EPI == GEMM_EPI_SCORE && p.lo_skip_flag && *p.lo_skip_flag) ? p.lo_skip_k : 0;

  if constexpr (EPI == GEMM_EPI_QUANT) {
    if (tid < NB) tab[tid] = __ldg(p.boundaries + tid);
    if (tid < NB + 1) tab[NB + tid] = __ldg(p.centroids + tid);
  }
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull_bar(b), 1); mbar_init(tempty_bar(b), 128); }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_slot)), "r"(512) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long lim = p.wait_limit;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;                                  // stage uses issued
      int issued = 0;
      bool stop = false;
      for (int64_t w = blockIdx.x; w < n_work && !stop; w += gridDim.x) {
        const int row = static_cast<int>((w / n_tiles) * kGemmTileM);
        const int col = static_cast<int>((w % n_tiles) * kGemmTileN);
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = it % NS, use = it / NS;
          if (use > 0 && !mbar_wait(empty_bar(s), (use - 1) & 1, lim, p.status, abort_flag)) { stop = true; break; }
          const uint32_t st = base + s * kGemmStageBytes;
          const int k0 = ks * kGemmTileK;
          const bool lo = k0 >= k_lo0;
          mbar_expect_tx(full_bar(s), lo ? kGemmStageBytes : kGemmStageBytes - kGemmBStage);
          tma_load_2d_g(st, &a_hi, k0, row, full_bar(s));
          tma_load_2d_g(st + kGemmAStage, &a_lo, k0, row, full_bar(s));
          tma_load_2d_g(st + 2 * kGemmAStage, &b_hi, k0, col, full_bar(s));
          if (lo) tma_load_2d_g(st + 2 * kGemmAStage + kGemmBStage, &b_lo, k0, col, full_bar(s));
          ++issued;
        }
      }
      // drain: every issued stage lands before the CTA can exit
      for (int j = max(0, issued - NS); j < issued; ++j)
        for (long long i = 0; !mbar_try(full_bar(j % NS), (j / NS) & 1) && i < kDrainLimit; ++i) {}
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_m128_bf16(TN);
      int it = 0, t = 0;                           // stage uses, tiles
      bool stop = false;
      for (int64_t w = blockIdx.x; w < n_work && !stop; w += gridDim.x, ++t) {
        const int buf = t & 1, j = t >> 1;
        if (j > 0 && !mbar_wait(tempty_bar(buf), (j - 1) & 1, lim, p.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t td = tmem_base + buf * TN;
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = it % NS;
          if (!mbar_wait(full_bar(s), (it / NS) & 1, lim, p.status, abort_flag)) { stop = true; break; }
          tc_fence_after();
          const uint32_t st = base + s * kGemmStageBytes;
          const uint32_t ah = st, al = st + kGemmAStage, bh = st + 2 * kGemmAStage, bl = bh + kGemmBStage;
          const bool lo = ks * kGemmTileK >= k_lo0;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t ko = kk * 32;
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            umma_f16(td, sw128_desc(ah + ko), sw128_desc(bh + ko), idesc, acc);
            if (lo) umma_f16(td, sw128_desc(ah + ko), sw128_desc(bl + ko), idesc, 1u);
            umma_f16(td, sw128_desc(al + ko), sw128_desc(bh + ko), idesc, 1u);
          }
          umma_commit(empty_bar(s));
        }
        if (stop) break;
        umma_commit(tfull_bar(buf));
      }
      // the tensor core finishes everything issued before tensor memory is freed
      if (t > 0) {
        const int last = t - 1;
        for (long long i = 0; !mbar_try(tfull_bar(last & 1), (last >> 1) & 1) && i < kDrainLimit; ++i) {}
      }
    }
  } else {
    const int lanebase = 32 * (warp & 3);          // TMEM lanes this warp may access
    const int r = lanebase + lane;                 // row within the tile
    int t = 0;
    for (int64_t w = blockIdx.x; w < n_work; w += gridDim.x, ++t) {
      const int buf = t & 1, j = t >> 1;
      if (!mbar_wait(tfull_bar(buf), j & 1, lim, p.status, abort_flag)) break;
      tc_fence_after();
      const int64_t v = (w / n_tiles) * kGemmTileM + r;
      const int nt = static_cast<int>(w % n_tiles);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(lanebase) << 16) + buf * TN;
      if constexpr (EPI == GEMM_EPI_QUANT) {
        const float nx = v < p.M ? __ldg(p.rnorm_x + v) : 0.f;
        const float inv = nx > 0.f ? 1.f / nx : 0.f;   // a zero row keeps y = 0
        float g2 = 0.f;
#pragma unroll 1
        for (int c = 0; c < NCH; ++c) {                  // 32 columns at a time
          float y[32];
          tmem_ld32(taddr + 32 * c, y);
          tmem_wait_ld();
          uint32_t wc[B];
#pragma unroll
          for (int q = 0; q < B; ++q) wc[q] = 0u;
          uint32_t hw[16], lw[16];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float u = y[i] * inv;
            uint32_t code = 0u;
#pragma unroll
            for (int k = 0; k < NB; ++k) code += u > tab[k] ? 1u : 0u;
            const int pos = i * B;
            wc[pos >> 5] |= code << (pos & 31);
            if ((pos & 31) + B > 32) wc[(pos >> 5) + 1] |= code >> (32 - (pos & 31));
            if (p.r_hi) {
              const float rr = u - tab[NB + code];
              g2 = fmaf(rr, rr, g2);
              const __nv_bfloat16 h = __float2bfloat16_rn(rr);
              const __nv_bfloat16 l = __float2bfloat16_rn(rr - __bfloat162float(h));
              const uint32_t hb = __bfloat16_as_ushort(h), lb = __bfloat16_as_ushort(l);
              if (i & 1) { hw[i >> 1] |= hb << 16; lw[i >> 1] |= lb << 16; }
              else { hw[i >> 1] = hb; lw[i >> 1] = lb; }
            }
          }
          if (v < p.M) {
            const int col0 = nt * kGemmTileN + 32 * c;
            uint32_t* dst = p.codes + v * p.code_words + (col0 * B) / 32;
#pragma unroll
            for (int q = 0; q < B; ++q) dst[q] = wc[q];
            if (p.r_hi) {
              uint4* rh = reinterpret_cast<uint4*>(p.r_hi + v * p.K + col0);
              uint4* rl = reinterpret_cast<uint4*>(p.r_lo + v * p.K + col0);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                rh[q] = make_uint4(hw[4 * q], hw[4 * q + 1], hw[4 * q + 2], hw[4 * q + 3]);
                rl[q] = make_uint4(lw[4 * q], lw[4 * q + 1], lw[4 * q + 2], lw[4 * q + 3]);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(buf));
        if (v < p.M) {
          if (p.r2_part) p.r2_part[v * n_tiles + nt] = g2;
          if (nt == 0 && p.norms) p.norms[v] = nx;
        }
      } else if constexpr (EPI == GEMM_EPI_SCORE) {
#pragma unroll 1
        for (int c = 0; c < NCH; ++c) {
          float z[32];
          tmem_ld32(taddr + 32 * c, z);
          tmem_wait_ld();
          const int64_t col0 = static_cast<int64_t>(nt) * kGemmTileN + 32 * c;
          if (v < p.M && col0 < p.N) {
            float* dst = p.out + v * p.ldo + col0;
            if (col0 + 32 <= p.N && (p.ldo & 3) == 0) {
#pragma unroll
              for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(dst + i) =
                    make_float4(z[i] * __ldg(p.col_scale + col0 + i), z[i + 1] * __ldg(p.col_scale + col0 + i + 1),
                                z[i + 2] * __ldg(p.col_scale + col0 + i + 2), z[i + 3] * __ldg(p.col_scale + col0 + i + 3));
            } else {
              for (int i = 0; i < 32 && col0 + i < p.N; ++i) dst[i] = z[i] * __ldg(p.col_scale + col0 + i);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(buf));
      } else {
        uint32_t sw[NCH];
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          float z[32];
          tmem_ld32(taddr + 32 * c, z);
          tmem_wait_ld();
          uint32_t bits = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) bits |= (z[i] >= 0.f ? 1u : 0u) << i;
          sw[c] = bits;
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(buf));
        if (v < p.M) {
          uint4* dst = reinterpret_cast<uint4*>(p.signs + v * (p.N / 32) + nt * NCH);
#pragma unroll
          for (int q = 0; q < NCH / 4; ++q) dst[q] = make_uint4(sw[4 * q], sw[4 * q + 1], sw[4 * q + 2], sw[4 * q + 3]);
          if (nt == 0) {
            float g2 = 0.f;
            for (int q = 0; q < p.r2_chunks; ++q) g2 += p.r2_in[v * p.r2_chunks + q];
            p.rnorms[v] = sqrtf(g2);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512) : "memory");
  }
}

}  // namespace tq
