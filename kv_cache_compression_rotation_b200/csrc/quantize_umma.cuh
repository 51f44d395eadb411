// Tensor-core quantize for d = 128, 16-bit input: TMA -> tcgen05.mma (TMEM) -> epilogue.
//
// TurboQuant review, "Method": y = Pi x / ||x||, then each coordinate is coded against
// the Lloyd-Max boundaries.  The rotation is the only dense contraction of the path:
//   Y[128 vectors x 128] = X[128 x 128] . Pi^T,   accumulated in TMEM (fp32).
// Pi is fp32; the input is exact in bf16 (or fp16), so Pi is split as Pi_hi + Pi_lo
// (both in the input's 16-bit type) and the tile takes two MMAs per k-step into the same
// accumulator.  The split keeps every rotated coordinate within about 2^-17 ||x|| of
// the fp32 product, far inside the 1e-5 decision band around a boundary.
//
// Roles in a persistent CTA (one per SM), 320 threads:
//   warp 0      TMA producer: 128-row tiles of x into a 4-stage ring (128B swizzle)
//   warp 1      TMEM allocator and single-thread MMA issuer (2 accumulator buffers)
//   warps 2-5   epilogue group 0 (even tiles), warps 6-9 group 1 (odd tiles):
//               one vector per thread: tcgen05.ld the row, ||y||, then per coordinate
//               u = y / ||y|| and its code, packed LSB-first; store record + norm.
// Code assignment (b >= 2): [-R, R) with R = 1.25 t_max is cut into 32 equal cells,
// narrower than the smallest gap between boundaries, so each cell holds at most one
// boundary.  Lane g of every warp keeps cell g's entry: the boundary inside it (or a
// huge value) with the number of boundaries below the cell in its 4 low mantissa bits
// (a perturbation below 1e-6 of a unit-scale boundary).  A coordinate's code is then
// one FFMA to find its cell, one warp shuffle to fetch the entry and one compare:
// code = (#boundaries below the cell) + (u > boundary in the cell).  A codebook whose
// gaps are narrower than the cells falls back to counting all boundaries.
// ||y|| equals ||x|| up to the orthogonality of the fp32 Pi (~1e-7 relative).
// TurboQuant-prod (PRODK instantiation, m = d = 128): the (b-1)-bit MSE stage as above,
// then the QJL projection of the unit-scale residual r = u - c[code] is a second tensor-
// core product Z[128 x 128] = R . S^T.  The epilogue writes r as fp16 hi + lo parts into
// tensor memory, where it is the A operand (S hi + lo in shared memory is B); the three
// products R_hi S_hi + R_hi S_lo + R_lo S_hi keep every projection within ~1e-6 ||S_i|| ||r||
// of the fp32 value, far inside the 1e-5 ||S_i|| sign band.  Tensor memory: one Y
// accumulator (128 columns, handed back as soon as an epilogue group has read its row),
// one Z accumulator (128) and one R_hi | R_lo block per epilogue group (2 x 128), 512 in
// all; the groups overlap their code and residual arithmetic and meet only on Y and Z.
// Every mbarrier wait is bounded; on timeout the CTA records TQ_ERR_TIMEOUT, drains
// what it issued, frees TMEM and exits.
#pragma once

#include <cuda.h>

#include "device_common.cuh"

namespace tq {

constexpr int kUmmaThreads = 320;
constexpr int kUmmaStages = 4;
constexpr int kUmmaTileRows = 128;
constexpr int kUmmaD = 128;
constexpr uint32_t kXStageBytes = kUmmaTileRows * kUmmaD * 2;      // 32 KB
constexpr uint32_t kPiBytes = kUmmaD * kUmmaD * 2;                 // 32 KB per half
// Drains (copies and MMAs this CTA already issued) always complete on their own; their
// bound is fixed and independent of the test-adjustable wait limit.
constexpr long long kDrainLimit = 1ll << 28;
// 32 cells over [-R, R): f in [0, 1] maps to floor(f * kCellSpan) in 0..31
constexpr float kCellSpan = 31.9999f;
// spectral tables: per top dim up to 63 thresholds and 64 centroids (top bits <= 6), S (<= 8 x 8)
constexpr int kSpecMaxTopBits = 6;
constexpr uint32_t kSpecTabBytes = (TQ_MAX_TOP * 64 * 2 + 64) * 4;
constexpr uint32_t kUmmaSmemBytes = 1024 /*align slack*/ + 2 * kPiBytes + kUmmaStages * kXStageBytes + 256 + kSpecTabBytes;
// prod: Pi hi + lo and S hi + lo (fp16), a 3-stage ring, barriers and the centroid table
constexpr int kProdStages = 3;
constexpr uint32_t kUmmaProdSmemBytes = 1024 + 4 * kPiBytes + kProdStages * kXStageBytes + 256 + 64 * 4;

struct UmmaQuantParams {
  const float* rot;        // [128*128] fp32
  const float* boundaries; // [2^b - 1]
  int64_t n;
  int is_f16;              // 0 bf16, 1 fp16
  uint32_t* codes;         // [n][W]
  float* norms;            // [n]
  int* status;
  long long wait_limit;
  // spectral records (1-bit tail): top dims 0..k_top-1 with their own bits, QJL on them
  int k_top, qjl;
  int top_bits[TQ_MAX_TOP];
  const float* dim_sigma;  // [128]
  const float* unit_c;     // standard-normal codebooks (concatenated by bits)
  const float* unit_t;
  const float* S;          // [k_top*k_top] (qjl)
  float* rnorms;           // [n] (qjl)
  // rotations with entries +-pm1_scale: one exact +-1 MMA operand, no low-order term
  int pm1;
  float pm1_scale;         // 1/sqrt(d) as fp32
  // prod (m = 128): S [128*128] fp32 is the field S above; MSE-stage centroids, sign words
  const float* centroids;  // [2^B]
  uint32_t* signs;         // [n][4]
  // outlier split (B1 instantiation): rot is Pi_0 [32*32] of the channels cols0, rot1 Pi_1
  // [96*96] of cols1; group 0 records (B bits) go to codes / norms, group 1 (B1 bits) to
  // codes1 / norms1
  const float* rot1;
  const int32_t* cols0;
  const int32_t* cols1;
  const float* boundaries1;
  uint32_t* codes1;        // [n][3 * B1]
  float* norms1;           // [n]
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait; returns false (and records a timeout) if the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long limit, int* status,
                                          volatile int* abort_flag) {
  if (limit < 0) {                 // test hook: every bounded wait expires at once
    report_status(status, kDevTimeout);
    *abort_flag = 1;
    return false;
  }
  for (long long i = 0;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if (i >= limit || *abort_flag) {
      report_status(status, kDevTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}

// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzle layout
// (8-row x 128-byte atoms, 1024 B apart).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);          // start address
  desc |= static_cast<uint64_t>(1u) << 16;                          // leading byte offset (unused)
  desc |= static_cast<uint64_t>(1024u >> 4) << 32;                  // stride byte offset
  desc |= static_cast<uint64_t>(1u) << 46;                          // descriptor version
  desc |= static_cast<uint64_t>(2u) << 61;                          // 128-byte swizzle
  return desc;
}

// Instruction descriptor: D f32, A/B bf16 or f16, both K-major, M = 128, N = 128.
__device__ __forceinline__ uint32_t idesc_m128n128(int is_f16) {
  const uint32_t ab = is_f16 ? 0u : 1u;
  return (1u << 4) | (ab << 7) | (ab << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// Same, with the A operand read from tensor memory (M rows = lanes, K 16-bit elements
// packed two per 32-bit column).
__device__ __forceinline__ void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n"
      ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// B packed words of one 32-coordinate chunk (the chunk starts 4 * B bytes into the record).
template <int B>
__device__ __forceinline__ void store_words(uint32_t* dst, const uint32_t (&w)[B]) {
  if constexpr (B == 4) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (B == 2) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else {
#pragma unroll
    for (int i = 0; i < B; ++i) dst[i] = w[i];
  }
}

// SPEC: spectral records instead of MSE codes (B unused): z = rot x without normalization;
// tail dims take 1 bit, code (z_j > 0) (the 1-bit standard-normal boundary is 0); the top
// dims are coded against sigma_j times their unit codebooks and get the QJL signs of
// S (z_top - c_top); record = head word + 4 tail words (+ ||z_top - c_top||).
// B1 > 0: the outlier-channel split of the KV experiments (TurboQuant review, Method) as
// one pass over the full 128-channel rows: the operand is the block rotation whose rows
// 0..31 are Pi_0 scattered over the channels cols0 and rows 32..127 Pi_1 over cols1, so
// Y = [Pi_0 x[cols0] | Pi_1 x[cols1]] (the zero entries add nothing); each group is then
// coded with its own norm ||y_g|| = ||x[cols_g]||, boundaries and width (B, then B1 bits).
template <int B, bool SPEC, bool PRODK = false, int B1 = 0>
__global__ void __launch_bounds__(kUmmaThreads, 1)
umma_quantize_kernel(const __grid_constant__ CUtensorMap xmap, const UmmaQuantParams p) {
  constexpr int K = 1 << B;
  constexpr int NB = K - 1;
  constexpr int W = kUmmaD * B / 32;             // code words per vector
  // spectral codes compare raw (unnormalized) coordinates with boundaries at 0, where the
  // data is densest: Pi takes three 16-bit terms (hi + lo + lo2, ~2^-26 relative) instead of
  // two, and the ring one stage less so the shared memory stays the same
  constexpr int NT = SPEC ? 3 : 2;
  constexpr int NS = SPEC ? 3 : (PRODK ? kProdStages : kUmmaStages);
  // 32 KB operand blocks before the ring: Pi terms, and for prod S hi + lo
  constexpr int NPI = PRODK ? 4 : NT;
  static_assert(PRODK || NT * kPiBytes + NS * kXStageBytes == 2 * kPiBytes + kUmmaStages * kXStageBytes, "smem");
  static_assert(!PRODK || 1024 + NPI * kPiBytes + NS * kXStageBytes + 256 + 64 * 4 <= kUmmaProdSmemBytes, "smem");
  constexpr uint32_t kTmemCols = PRODK ? 512u : 256u;
  // prod tensor-memory columns: Y 0..127, Z 128..255, R_hi of group b at 256 + 128 b, R_lo 64 after
  constexpr uint32_t kZcol = 128u, kR = 256u;
  extern __shared__ unsigned char usm_raw[];
  const uint32_t raw = smem_u32(usm_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sm = usm_raw + (base - raw);
  const uint32_t pi_hi = base, pi_lo = base + kPiBytes, pi_lo2 = base + 2 * kPiBytes;
  const uint32_t s_hi = base + 2 * kPiBytes, s_lo = base + 3 * kPiBytes;   // prod only
  const uint32_t xs0 = base + NPI * kPiBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + NPI * kPiBytes + NS * kXStageBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (NS + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * NS + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * NS + 2 + b); };
  // prod: R of group b written (count 128), Z of group b's tile committed (1), Z read
  // (count 128).  Y is one buffer: its full barrier is the group's tfull (each group waits
  // only for its own tiles, so a parity wait never passes on a phase of the other group),
  // its empty barrier tempty(0), waited in tile order by the MMA warp alone.
  auto rfull_bar = [&](int b) { return bar0 + 8u * (2 * NS + 4 + b); };
  auto zfull_bar = [&](int b) { return bar0 + 8u * (2 * NS + 6 + b); };
  auto zempty_bar = [&]() { return bar0 + 8u * (2 * NS + 8); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + (PRODK ? 10 : 4));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* tsm = reinterpret_cast<float*>(tmem_slot + 2);   // boundaries [NB]
  // spectral: thresholds [top dim][64], centroids [top dim][64], S [64]
  float* sthr = reinterpret_cast<float*>(sm + NPI * kPiBytes + NS * kXStageBytes + 256);
  float* pcen = sthr;                                     // prod: MSE-stage centroids [2^B]
  float* scen = sthr + TQ_MAX_TOP * 64;
  float* sS = scen + TQ_MAX_TOP * 64;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (p.n + kUmmaTileRows - 1) / kUmmaTileRows;

  // split: the block rotation is zero outside the scattered group rows
  if constexpr (B1 > 0) {
    for (int i = tid; i < static_cast<int>(2 * kPiBytes / 4); i += kUmmaThreads) reinterpret_cast<uint32_t*>(sm)[i] = 0u;
    __syncthreads();
  }
  // Pi_hi / Pi_lo in the swizzled K-major layout: row = output dim n, k = input dim.
  for (int i = tid; i < (B1 > 0 ? 32 * 32 + 96 * 96 : kUmmaD * kUmmaD); i += kUmmaThreads) {
    int nrow = i >> 7, k = i & 127;
    float v;
    if constexpr (B1 > 0) {
      // row r of Pi_0 (first 1024 entries) or of Pi_1, entry j -> channel cols_g[j]
      int j, col;
      if (i < 32 * 32) {
        nrow = i >> 5; j = i & 31;
        col = __ldg(p.cols0 + j);
        v = __ldg(p.rot + i);
      } else {
        const int i2 = i - 32 * 32, r = i2 / 96;
        nrow = 32 + r; j = i2 - r * 96;
        col = __ldg(p.cols1 + j);
        v = __ldg(p.rot1 + i2);
      }
      if (col < 0 || col >= kUmmaD) {           // a channel out of range contributes nothing
        report_status(p.status, TQ_ERR_INVALID_ARG);
        continue;
      }
      k = col;
    } else {
      v = __ldg(p.rot + i);
    }
    if (p.pm1) {
      // the +-1 pattern is exact in both 16-bit types; the scale is applied to the norm
      if (fabsf(v) != p.pm1_scale) report_status(p.status, TQ_ERR_INVALID_ARG);
      v = v < 0.f ? -1.f : 1.f;
    }
    uint16_t hi, lo, lo2;
    if (p.is_f16) {
      const __half h = __float2half_rn(v);
      const __half l = __float2half_rn(v - __half2float(h));
      const __half l2 = __float2half_rn(v - __half2float(h) - __half2float(l));
      hi = __half_as_ushort(h); lo = __half_as_ushort(l); lo2 = __half_as_ushort(l2);
    } else {
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
      const __nv_bfloat16 l2 = __float2bfloat16_rn(v - __bfloat162float(h) - __bfloat162float(l));
      hi = __bfloat16_as_ushort(h); lo = __bfloat16_as_ushort(l); lo2 = __bfloat16_as_ushort(l2);
    }
    const int kb = k >> 6, kk = k & 63;
    const uint32_t off = kb * (kUmmaD * 128) + nrow * 128 + ((((kk >> 3) ^ (nrow & 7))) << 4) + (kk & 7) * 2;
    *reinterpret_cast<uint16_t*>(sm + off) = hi;
    *reinterpret_cast<uint16_t*>(sm + kPiBytes + off) = lo;
    if (NT == 3) *reinterpret_cast<uint16_t*>(sm + 2 * kPiBytes + off) = lo2;
  }
  if constexpr (SPEC) {
    for (int i = tid; i < p.k_top * 64; i += kUmmaThreads) {
      const int j = i >> 6, k = i & 63, b = p.top_bits[j];
      const float sg = __ldg(p.dim_sigma + j);
      sthr[i] = k < (1 << b) - 1 ? sg * __ldg(p.unit_t + unit_t_off(b) + k) : 3.0e38f;
      scen[i] = k < (1 << b) ? sg * __ldg(p.unit_c + unit_c_off(b) + k) : 0.f;
    }
    if (p.qjl && tid < p.k_top * p.k_top) sS[tid] = __ldg(p.S + tid);
  } else {
    if (tid < NB) tsm[tid] = __ldg(p.boundaries + tid);
    if (B1 > 0 && tid < (1 << B1) - 1) sthr[tid] = __ldg(p.boundaries1 + tid);
  }
  if constexpr (PRODK) {
    // S_hi / S_lo (fp16) in the same swizzled K-major layout: row = projection i, k = dim
    for (int i = tid; i < kUmmaD * kUmmaD; i += kUmmaThreads) {
      const int nrow = i >> 7, k = i & 127;
      const float v = __ldg(p.S + i);
      const __half h = __float2half_rn(v);
      const __half l = __float2half_rn(v - __half2float(h));
      const int kb = k >> 6, kk = k & 63;
      const uint32_t off = kb * (kUmmaD * 128) + nrow * 128 + ((((kk >> 3) ^ (nrow & 7))) << 4) + (kk & 7) * 2;
      *reinterpret_cast<uint16_t*>(sm + 2 * kPiBytes + off) = __half_as_ushort(h);
      *reinterpret_cast<uint16_t*>(sm + 3 * kPiBytes + off) = __half_as_ushort(l);
    }
    if (tid < K) pcen[tid] = __ldg(p.centroids + tid);
  }
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull_bar(b), 1); mbar_init(tempty_bar(b), 128); }
    if (PRODK) {
      for (int b = 0; b < 2; ++b) { mbar_init(rfull_bar(b), 128); mbar_init(zfull_bar(b), 1); }
      mbar_init(zempty_bar(), 128);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // generic-proxy writes of Pi must be visible to the tensor-core (async) proxy
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long lim = p.wait_limit;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      int issued = 0;
      for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
        const int s = it % NS, use = it / NS;
        if (use > 0 && !mbar_wait(empty_bar(s), (use - 1) & 1, lim, p.status, abort_flag)) break;
        mbar_expect_tx(full_bar(s), kXStageBytes);
        const uint32_t dst = xs0 + s * kXStageBytes;
        const int row = static_cast<int>(tile * kUmmaTileRows);
        tma_load_2d(dst, &xmap, 0, row, full_bar(s));
        tma_load_2d(dst + kXStageBytes / 2, &xmap, 64, row, full_bar(s));
        ++issued;
      }
      // drain: every issued stage must land before the CTA can exit
      for (int j = max(0, issued - NS); j < issued; ++j) {
        const int s = j % NS, use = j / NS;
        for (long long i = 0; !mbar_try(full_bar(s), use & 1) && i < kDrainLimit; ++i) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_m128n128(p.is_f16);
      // prod: Z(t) = R(t) . S^T once the epilogue of tile t has written R(t) and tile t - 1's
      // Z has been read (three fp16 products: R_hi S_hi + R_hi S_lo + R_lo S_hi)
      int zt = 0;                                   // next tile whose Z is issued
      auto issue_z = [&]() {
        const int zb = zt & 1;
        if (!mbar_wait(rfull_bar(zb), (zt >> 1) & 1, lim, p.status, abort_flag)) return false;
        if (zt > 0 && !mbar_wait(zempty_bar(), (zt - 1) & 1, lim, p.status, abort_flag)) return false;
        tc_fence_after();
        const uint32_t zidesc = idesc_m128n128(1);
        const uint32_t zd = tmem_base + kZcol, ra = tmem_base + kR + zb * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t boff = (kk >> 2) * (kPiBytes / 2) + (kk & 3) * 32;
          umma_f16_ts(zd, ra + kk * 8, sw128_desc(s_hi + boff), zidesc, kk > 0 ? 1u : 0u);
          umma_f16_ts(zd, ra + kk * 8, sw128_desc(s_lo + boff), zidesc, 1u);
          umma_f16_ts(zd, ra + 64 + kk * 8, sw128_desc(s_hi + boff), zidesc, 1u);
        }
        umma_commit(zfull_bar(zb));
        ++zt;
        return true;
      };
      int it = 0;                                   // rotations issued
      bool zok = true;
      for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        // prod: one Y accumulator (buffer 0, a phase per tile); otherwise two, by tile parity
        const int s = it % NS, buf = PRODK ? 0 : (it & 1), j = PRODK ? it : (it >> 1);
        if (j > 0 && !mbar_wait(tempty_bar(buf), (j - 1) & 1, lim, p.status, abort_flag)) break;
        if (!mbar_wait(full_bar(s), (it / NS) & 1, lim, p.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t xa = xs0 + s * kXStageBytes;
        const uint32_t td = tmem_base + buf * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * (kXStageBytes / 2) + (kk & 3) * 32;
          const uint32_t poff = (kk >> 2) * (kPiBytes / 2) + (kk & 3) * 32;
          umma_f16(td, sw128_desc(xa + koff), sw128_desc(pi_hi + poff), idesc, kk > 0 ? 1u : 0u);
          if (!p.pm1) umma_f16(td, sw128_desc(xa + koff), sw128_desc(pi_lo + poff), idesc, 1u);
          if (NT == 3) umma_f16(td, sw128_desc(xa + koff), sw128_desc(pi_lo2 + poff), idesc, 1u);
        }
        umma_commit(empty_bar(s));
        umma_commit(tfull_bar(PRODK ? (it & 1) : buf));
        ++it;
        // the previous tile's projection, issued behind this tile's rotation
        if (PRODK && it > 1 && !(zok = issue_z())) break;
      }
      if (PRODK && zok && zt < it) zok = issue_z();      // the last tile
      // wait for the tensor core to finish everything issued before TMEM is freed
      if (it > 0) {
        const int last = it - 1;
        for (long long i = 0; !mbar_try(tfull_bar(last & 1), (last >> 1) & 1) && i < kDrainLimit; ++i) {}
      }
      if (PRODK && zt > 0)
        for (long long i = 0; !mbar_try(zfull_bar((zt - 1) & 1), ((zt - 1) >> 1) & 1) && i < kDrainLimit; ++i) {}
    }
  } else {
    const int grp = (warp - 2) >> 2;                   // 0: warps 2-5, 1: warps 6-9
    const int lanebase = 32 * (warp & 3);              // TMEM lanes this warp may access
    const int r = lanebase + lane;                     // row within the tile
    float thr[NB];
    // cell table (identical in every warp): lane g holds the entry of cell g
    bool use_cells = false;
    float cell_scale = 0.f;
    uint32_t cell_entry = 0u;
    if (NB >= 3) {
      const float R = 1.25f * tsm[NB - 1];
      float min_gap = 3.0e38f;
      for (int k = 0; k + 1 < NB; ++k) min_gap = fminf(min_gap, tsm[k + 1] - tsm[k]);
      const float width = 2.f * R / kCellSpan;
      use_cells = R > 0.f && width < 0.9f * min_gap;
      cell_scale = 0.5f / R;
      const float a = (static_cast<float>(lane) / kCellSpan - 0.5f) * 2.f * R;
      const float b = (static_cast<float>(lane + 1) / kCellSpan - 0.5f) * 2.f * R;
      uint32_t base_code = 0u;
      float inside = 3.0e38f;
      for (int k = 0; k < NB; ++k) {
        if (tsm[k] < a) ++base_code;
        else if (tsm[k] < b || lane == 31) inside = fminf(inside, tsm[k]);
      }
      // the boundary is kept in the cell coordinate f = u / (2R) + 1/2 (in [0, 1]), where
      // the code assignment compares it with f directly
      const float inside_f = inside < 1.0e38f ? fmaf(inside, 0.5f / R, 0.5f) : 3.0e38f;
      cell_entry = (__float_as_uint(inside_f) & ~15u) | base_code;
    }
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int buf = it & 1;
      if (buf != grp) continue;
      const int j = it >> 1;
      if (!mbar_wait(tfull_bar(buf), j & 1, lim, p.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(lanebase) << 16) + (PRODK ? 0u : buf * 128u);
      const int64_t v = tile * kUmmaTileRows + r;
      if constexpr (PRODK) {
        // the whole row comes out of tensor memory at once and Y goes straight back to the
        // MMA warp (the next tile's rotation runs while this group computes)
        float y[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(taddr + 32 * c, y[c]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(tempty_bar(0));
        float2 s2[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 v2 = make_float2(y[c][i], y[c][i + 1]);
            s2[(i >> 1) & 3] = __ffma2_rn(v2, v2, s2[(i >> 1) & 3]);
          }
        }
        const float ny = sqrtf(((s2[0].x + s2[0].y) + (s2[1].x + s2[1].y)) + ((s2[2].x + s2[2].y) + (s2[3].x + s2[3].y)));
        const float inv = ny > 0.f ? 1.f / ny : 1.f;
        const float fs = inv * cell_scale;
        const float ccen = lane < K ? pcen[lane] : 0.f;   // centroid of code `lane`
        // this group's R columns were last read by its previous tile's projection, which
        // completed before that tile's Z was read
        const uint32_t rowaddr = tmem_base + (static_cast<uint32_t>(lanebase) << 16);
        const uint32_t rcol = rowaddr + kR + buf * 128;
        float2 g2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t wc[B], hw[16], lw[16];
#pragma unroll
          for (int w = 0; w < B; ++w) wc[w] = 0u;
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            uint32_t code[2];
            if (use_cells) {
              const float2 f2 = make_float2(__saturatef(fmaf(y[c][i], fs, 0.5f)), __saturatef(fmaf(y[c][i + 1], fs, 0.5f)));
              const float2 gg = __ffma2_rz(f2, make_float2(kCellSpan, kCellSpan), make_float2(8388608.0f, 8388608.0f));
              const uint32_t e0 = __shfl_sync(0xffffffffu, cell_entry, __float_as_int(gg.x));
              const uint32_t e1 = __shfl_sync(0xffffffffu, cell_entry, __float_as_int(gg.y));
              const float2 d2 = __ffma2_rn(f2, make_float2(-1.f, -1.f), make_float2(__uint_as_float(e0), __uint_as_float(e1)));
              code[0] = (e0 & 15u) + (__float_as_uint(d2.x) >> 31);
              code[1] = (e1 & 15u) + (__float_as_uint(d2.y) >> 31);
            } else {
              uint32_t c0 = 0u, c1 = 0u;
#pragma unroll
              for (int k = 0; k < NB; ++k) {
                c0 += y[c][i] * inv > tsm[k] ? 1u : 0u;
                c1 += y[c][i + 1] * inv > tsm[k] ? 1u : 0u;
              }
              code[0] = c0; code[1] = c1;
            }
            // unit-scale residual r = u - c[code] and its fp16 hi + lo parts (the A operand)
            const float ch0 = __shfl_sync(0xffffffffu, ccen, static_cast<int>(code[0]));
            const float ch1 = __shfl_sync(0xffffffffu, ccen, static_cast<int>(code[1]));
            const float2 rr = __ffma2_rn(make_float2(y[c][i], y[c][i + 1]), make_float2(inv, inv), make_float2(-ch0, -ch1));
            g2 = __ffma2_rn(rr, rr, g2);
            // hi = half2(r), lo = half2(r - hi): one paired conversion each, one packed FMA
            const __half2 h2 = __floats2half2_rn(rr.x, rr.y);
            const float2 back = __half22float2(h2);
            const float2 res = __ffma2_rn(back, make_float2(-1.f, -1.f), rr);
            const __half2 l2 = __floats2half2_rn(res.x, res.y);
            hw[i >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
            lw[i >> 1] = *reinterpret_cast<const uint32_t*>(&l2);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int pos = (i + h) * B;
              wc[pos >> 5] += code[h] << (pos & 31);
              if ((pos & 31) + B > 32) wc[(pos >> 5) + 1] += code[h] >> (32 - (pos & 31));
            }
          }
          tmem_st16(rcol + 16 * c, hw);
          tmem_st16(rcol + 64 + 16 * c, lw);
          if (v < p.n) store_words<B>(p.codes + v * W + c * B, wc);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(rfull_bar(buf));
        if (v < p.n) {
          p.norms[v] = ny;
          p.rnorms[v] = sqrtf(g2.x + g2.y);
        }
        // sign bits of the projection, (S r)_i >= 0
        if (!mbar_wait(zfull_bar(buf), j & 1, lim, p.status, abort_flag)) break;
        tc_fence_after();
        uint32_t sw[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float z[32];
          tmem_ld32(rowaddr + kZcol + 32 * c, z);
          tmem_wait_ld();
          uint32_t wbits = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) wbits |= (z[i] >= 0.f ? 1u : 0u) << i;
          sw[c] = wbits;
        }
        tc_fence_before();
        mbar_arrive(zempty_bar());                      // Z is free for the next tile
        if (v < p.n) *reinterpret_cast<uint4*>(p.signs + v * 4) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
        continue;
      }
      if constexpr (SPEC) {
        const int kt = p.k_top;
        uint32_t tail[4];
        float ztop[TQ_MAX_TOP];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float z[32];
          tmem_ld32(taddr + 32 * c, z);
          tmem_wait_ld();
          uint32_t wbits = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) wbits |= (z[i] > 0.f ? 1u : 0u) << i;
          if (c == 0) {
#pragma unroll
            for (int j = 0; j < TQ_MAX_TOP; ++j) ztop[j] = z[j];
            wbits &= ~((1u << kt) - 1u);                // top dims carry no tail code
          }
          tail[c] = wbits;
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(buf));
        uint32_t head = 0u;
        int pos = 0;
        float rr[TQ_MAX_TOP];
        float g2 = 0.f;
#pragma unroll
        for (int j = 0; j < TQ_MAX_TOP; ++j) {
          rr[j] = 0.f;
          if (j < kt) {
            const int b = p.top_bits[j];
            uint32_t cnt = 0u;
            for (int k = 0; k < (1 << b) - 1; ++k) cnt += ztop[j] > sthr[j * 64 + k] ? 1u : 0u;
            head |= cnt << pos;
            pos += b;
            rr[j] = ztop[j] - scen[j * 64 + cnt];
            g2 = fmaf(rr[j], rr[j], g2);
          }
        }
        if (p.qjl) {
#pragma unroll
          for (int i = 0; i < TQ_MAX_TOP; ++i) {
            if (i < kt) {
              float a = 0.f;
#pragma unroll
              for (int k = 0; k < TQ_MAX_TOP; ++k)
                if (k < kt) a = fmaf(sS[i * kt + k], rr[k], a);
              head |= (a >= 0.f ? 1u : 0u) << (pos + i);
            }
          }
        }
        if (v < p.n) {
          uint32_t* dst = p.codes + v * 5;
          dst[0] = head;
          dst[1] = tail[0]; dst[2] = tail[1]; dst[3] = tail[2]; dst[4] = tail[3];
          if (p.qjl) p.rnorms[v] = sqrtf(g2);
        }
        continue;
      }
      if constexpr (B1 > 0) {
        // split: group 0 = chunk 0 (B bits), group 1 = chunks 1..3 (B1 bits), each coded
        // against its own norm times its boundaries (unnormalized coordinates)
        constexpr int NB1 = (1 << B1) - 1;
        float y[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(taddr + 32 * c, y[c]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(tempty_bar(buf));
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 32; ++i) s0[i & 3] = fmaf(y[0][i], y[0][i], s0[i & 3]);
#pragma unroll
        for (int c = 1; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) s1[i & 3] = fmaf(y[c][i], y[c][i], s1[i & 3]);
        const float n0 = sqrtf((s0[0] + s0[1]) + (s0[2] + s0[3])), n1 = sqrtf((s1[0] + s1[1]) + (s1[2] + s1[3]));
        float th0[NB], th1[NB1];
#pragma unroll
        for (int k = 0; k < NB; ++k) th0[k] = (n0 > 0.f ? n0 : 1.f) * tsm[k];   // a zero group codes u = 0
#pragma unroll
        for (int k = 0; k < NB1; ++k) th1[k] = (n1 > 0.f ? n1 : 1.f) * sthr[k];
        {
          uint32_t wc[B];
#pragma unroll
          for (int w = 0; w < B; ++w) wc[w] = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            uint32_t cnt = 0u;
#pragma unroll
            for (int k = 0; k < NB; ++k) cnt += y[0][i] > th0[k] ? 1u : 0u;
            const int pos = i * B;
            wc[pos >> 5] |= cnt << (pos & 31);
            if ((pos & 31) + B > 32) wc[(pos >> 5) + 1] |= cnt >> (32 - (pos & 31));
          }
          if (v < p.n) store_words<B>(p.codes + v * B, wc);
        }
#pragma unroll
        for (int c = 1; c < 4; ++c) {
          uint32_t wc[B1];
#pragma unroll
          for (int w = 0; w < B1; ++w) wc[w] = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            uint32_t cnt = 0u;
#pragma unroll
            for (int k = 0; k < NB1; ++k) cnt += y[c][i] > th1[k] ? 1u : 0u;
            const int pos = i * B1;
            wc[pos >> 5] |= cnt << (pos & 31);
            if ((pos & 31) + B1 > 32) wc[(pos >> 5) + 1] |= cnt >> (32 - (pos & 31));
          }
          if (v < p.n) store_words<B1>(p.codes1 + v * (3 * B1) + (c - 1) * B1, wc);
        }
        if (v < p.n) { p.norms[v] = n0; p.norms1[v] = n1; }
        continue;
      }
      uint32_t* dst = p.codes + v * W;
      if (use_cells) {
        // the whole row comes out of TMEM in one go (128 registers), so the accumulator
        // buffer goes back to the MMA warp before any of the arithmetic below
        float y[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(taddr + 32 * c, y[c]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(tempty_bar(buf));
        // pass 1: ||y|| over the whole row, two coordinates per packed FMA (four independent
        // pairs of partial sums keep the FMA pipe busy)
        float2 s2[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 v2 = make_float2(y[c][i], y[c][i + 1]);
            s2[(i >> 1) & 3] = __ffma2_rn(v2, v2, s2[(i >> 1) & 3]);
          }
        }
        const float ny = sqrtf(((s2[0].x + s2[0].y) + (s2[1].x + s2[1].y)) + ((s2[2].x + s2[2].y) + (s2[3].x + s2[3].y)));
        const float nu = p.pm1 ? ny * p.pm1_scale : ny;  // ||x|| (the +-1 product is sqrt(d) Pi x)
        const float inv = ny > 0.f ? 1.f / ny : 1.f;     // a zero row keeps u = 0
        // pass 2: codes of 32 coordinates at a time, B packed words per chunk (the code
        // fields are disjoint, so they are added into the words)
        const float fs = inv * cell_scale;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t wc[B];
#pragma unroll
          for (int w = 0; w < B; ++w) wc[w] = 0u;
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            // two coordinates at a time: the cell index and the boundary difference go through
            // packed FMAs (the same roundings as the scalar forms)
            const float2 f2 = make_float2(__saturatef(fmaf(y[c][i], fs, 0.5f)), __saturatef(fmaf(y[c][i + 1], fs, 0.5f)));
            const float2 g2 = __ffma2_rz(f2, make_float2(kCellSpan, kCellSpan), make_float2(8388608.0f, 8388608.0f));
            const uint32_t e0 = __shfl_sync(0xffffffffu, cell_entry, __float_as_int(g2.x));
            const uint32_t e1 = __shfl_sync(0xffffffffu, cell_entry, __float_as_int(g2.y));
            // + 1 when f lies above the cell's boundary: the sign bit of (boundary - f)
            const float2 d2 = __ffma2_rn(f2, make_float2(-1.f, -1.f), make_float2(__uint_as_float(e0), __uint_as_float(e1)));
            const uint32_t code[2] = {(e0 & 15u) + (__float_as_uint(d2.x) >> 31), (e1 & 15u) + (__float_as_uint(d2.y) >> 31)};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int pos = (i + h) * B;
              wc[pos >> 5] += code[h] << (pos & 31);
              if ((pos & 31) + B > 32) wc[(pos >> 5) + 1] += code[h] >> (32 - (pos & 31));
            }
          }
          if (v < p.n) store_words<B>(dst + c * B, wc);
        }
        if (v < p.n) p.norms[v] = nu;
      } else {
        // thresholds against the unnormalized row: TMEM is read twice, 32 columns at a time
        float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; c += 2) {
          float va[32], vb[32];
          tmem_ld32(taddr + 32 * c, va);
          tmem_ld32(taddr + 32 * (c + 1), vb);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            ss[i & 3] = fmaf(va[i], va[i], ss[i & 3]);
            ss[(i + 2) & 3] = fmaf(vb[i], vb[i], ss[(i + 2) & 3]);
          }
        }
        const float ny = sqrtf((ss[0] + ss[1]) + (ss[2] + ss[3]));
        const float nu = p.pm1 ? ny * p.pm1_scale : ny;
        const float nthr = ny > 0.f ? ny : 1.f;
#pragma unroll
        for (int k = 0; k < NB; ++k) thr[k] = nthr * tsm[k];
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float y[32];
          tmem_ld32(taddr + 32 * c, y);
          tmem_wait_ld();
          uint32_t wc[B];
#pragma unroll
          for (int w = 0; w < B; ++w) wc[w] = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            int cnt = 0;
#pragma unroll
            for (int k = 0; k < NB; ++k) cnt += (y[i] > thr[k]) ? 1 : 0;
            const int pos = i * B;
            wc[pos >> 5] |= static_cast<uint32_t>(cnt) << (pos & 31);
            if ((pos & 31) + B > 32) wc[(pos >> 5) + 1] |= static_cast<uint32_t>(cnt) >> (32 - (pos & 31));
          }
          if (v < p.n) store_words<B>(dst + c * B, wc);
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(buf));
        if (v < p.n) p.norms[v] = nu;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols) : "memory");
  }
}

}  // namespace tq
