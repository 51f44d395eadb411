// Decode attention straight from the packed TurboQuant cache.
//
// TurboQuant review, "Problem": attention reads the KV cache only through query-key
// inner products.  So the step is  logit_i = scale * est(q, k_i),  p = softmax(logit),
// o = sum_i p_i v_hat_i, computed without ever materializing k_hat or v_hat in memory:
//
//   query prep   q' = scale * log2(e) * Pi_K q (and u = S q' for prod), once per head
//   decode       split over the context: each CTA owns one (batch, kv-head, chunk) and
//                streams the chunk's packed records.  Per 16-key unit a warp
//                  - turns pairs of codes into half2 codebook values with a lookup table
//                    in shared memory (one 32-bit load per two codes, replicated per lane
//                    so a warp's 32 lookups hit 32 distinct banks),
//                  - scores the unit with mma.sync m16n8k16 (rows = query heads of the
//                    GQA group, columns = keys, k = head dims),
//                  - runs an online softmax in the log2 domain,
//                  - accumulates p * ||v|| * c[code_v] with a second mma.sync in the
//                    rotated value domain.
//                The CTA's four warps merge their (max, sum, o') and write one partial.
//   combine      log-sum-exp merge of the chunks, then o = Pi_V^T o' once per head.
//
// Precision: every half-precision MMA operand that is not a table entry is split as
// hi + lo (two MMAs into the same fp32 accumulator), and the table entries are c_k / s
// with a shared scale s chosen so that each entry rounds to within ~1e-4 of c_k / s;
// products are scaled back by s in fp32.  Without these, half-precision rounding of
// q', p and c alone moves the attention output by ~1e-3 of its largest entry.
//
// Dimension mapping: the mma k index is a permutation of the head dims chosen so that
// each thread reads one contiguous slice of a record; the query operand uses the same
// permutation, so the inner product is unchanged.
#pragma once

#include "device_common.cuh"

namespace tq {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;

enum : int { KFMT_MSE = 0, KFMT_PROD = 1, KFMT_SPEC = 2 };
enum : int { VFMT_MSE = 0, VFMT_PROD = 1, VFMT_SPEC = 2 };

struct DecodeParams {
  int B, Hq, Hkv, G;
  int64_t Nmax;
  int chunk_len, n_chunks;
  const int32_t* seq_lens;
  // keys
  const uint32_t* kcodes;
  int k_words;          // words per key record
  int k_code_off;       // word offset of the code stream used by the main MMA (spectral: head words)
  const uint32_t* ksigns;
  int k_sign_words;
  const float* knorms;
  const float* krnorms;
  // values
  const uint32_t* vcodes;
  int v_words;
  int v_code_off;
  const float* vnorms;
  // codebooks for the lookup tables (device fp32)
  const float* kc;      // K main codebook [2^KB]
  const float* vc;      // V main codebook [2^VB]
  // spectral head description (k_top <= 8)
  int k_top_k, k_qjl, v_top;
  int k_top_bits[TQ_MAX_TOP];
  int v_top_bits[TQ_MAX_TOP];
  const float* unit_c;  // concatenated standard-normal codebooks (spectral)
  // query-prep outputs
  const float* qa;      // [B*Hq][D] main operand, normalized
  const float* qb;      // [B*Hq][QB] second operand (prod: u = S q'; spectral: 16 head slots)
  const float* qs;      // [B*Hq][2] scales of qa and qb
  int qb_stride;
  float qjl_coef;       // prod: sqrt(pi/2)/m
  float k_scale, v_scale; // shared scales of the half-precision codebook tables (entries c/s)
  // partial results
  float* part_ml;       // [B*Hq][n_chunks][2]
  float* part_o;        // [B*Hq][n_chunks][D]
  // paged pool (block_table != nullptr): token t of (b, kv-head h) is record
  // (block_table[b * max_pages + t / page] * Hkv + h) * page + t % page of every array
  const int32_t* block_table;
  int page, max_pages;
  int64_t num_pages;
  // causal query rows (prefill): row r = (b * Hq_rows + ...) sees tokens t < q_pos[b * T + r % T] + 1
  const int32_t* q_pos;
  int T;
  // values quantized as prod: sign words [recs][4], gamma [recs], S [128*128], sqrt(pi/2)/m
  const uint32_t* vsigns;
  const float* vrnorms;
  const float* vS;
  float v_coef;
};

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// hi = half(lo_v, hi_v) and lo = half of the rounding residuals.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 back = __half22float2(h);
  // x - back in one packed FMA (the product by -1 is exact, so the rounding is the add's)
  const float2 r = __ffma2_rn(back, make_float2(-1.f, -1.f), make_float2(x0, x1));
  const __half2 l = __floats2half2_rn(r.x, r.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Per-thread slice of a record: `NW` words starting at bit `base` of the record's stream,
// re-aligned so that bit 0 of seg[0] is bit `base`.  GLOBAL selects the read-only global
// load path; otherwise `rec` points into shared memory.
template <int NW, bool GLOBAL = true>
__device__ __forceinline__ void load_slice(const uint32_t* rec, int rec_words, int base,
                                           bool valid, uint32_t (&seg)[NW]) {
  const int w0 = base >> 5, sh = base & 31;
  uint32_t w[NW + 1];
#pragma unroll
  for (int i = 0; i <= NW; ++i) {
    const int wi = w0 + i;
    const bool use = valid && wi < rec_words && (i < NW || sh != 0);
    if constexpr (GLOBAL) w[i] = use ? __ldg(rec + wi) : 0u;
    else w[i] = use ? rec[wi] : 0u;
  }
#pragma unroll
  for (int i = 0; i < NW; ++i) seg[i] = __funnelshift_r(w[i], w[i + 1], sh);
}

// 2*B-bit field at bit position `pos` of a realigned slice (`pos` folds to a constant
// inside the unrolled loops that call this).
template <int B, int NW>
__device__ __forceinline__ uint32_t pair_at(const uint32_t (&seg)[NW], int pos) {
  const int wi = pos >> 5, sh = pos & 31;
  constexpr uint32_t mask = (1u << (2 * B)) - 1u;
  if (sh + 2 * B <= 32 || wi + 1 >= NW) return (seg[wi] >> sh) & mask;
  return __funnelshift_r(seg[wi], seg[wi + 1], sh) & mask;
}

template <int B, int NW>
__device__ __forceinline__ uint32_t field_at(const uint32_t (&seg)[NW], int pos) {
  const int wi = pos >> 5, sh = pos & 31;
  uint32_t v = seg[wi] >> sh;
  if (sh + B > 32 && wi + 1 < NW) v |= seg[wi + 1] << (32 - sh);
  return v & ((1u << B) - 1u);
}

// Head field of a spectral record (<= 72 bits in at most 3 words).
__device__ __forceinline__ uint32_t head_field(const uint32_t* h, int pos, int nb) {
  if (nb <= 0) return 0u;
  const int wi = pos >> 5, sh = pos & 31;
  uint64_t v = h[wi];
  if (sh + nb > 32) v |= static_cast<uint64_t>(h[wi + 1]) << 32;
  return static_cast<uint32_t>((v >> sh) & ((1ull << nb) - 1ull));
}

template <int D, int KF, int KB, int VF, int VB>
__global__ void __launch_bounds__(kDecThreads)
decode_attn_kernel(const DecodeParams p) {
  static_assert(D == 64 || D == 128, "head dim");
  constexpr int KST = D / 16;                 // mma k-steps over the head dims
  constexpr int TDK = D / 4;                  // key dims per thread (4 threads per key)
  constexpr int NWK = (TDK * KB + 31) / 32;   // words in a thread's key slice
  constexpr int TDV = D / 8;                  // value dims per thread (8 threads per key)
  constexpr int NWV = (TDV * VB + 31) / 32;
  constexpr int NT = D / 8;                   // P.V n-tiles
  constexpr int KLUT = 1 << (2 * KB), VLUT = 1 << (2 * VB);
  extern __shared__ __align__(16) uint32_t dsm[];
  uint32_t* lutk = dsm;                       // [KLUT][32]
  uint32_t* lutv = lutk + KLUT * 32;          // [VLUT][32]
  uint32_t* luts = lutv + VLUT * 32;          // [4][32]  (+-1 pairs for QJL signs)
  __half* uhalf = reinterpret_cast<__half*>(luts + 4 * 32);   // [510] unit codebooks (spectral)
  float* mrg = reinterpret_cast<float*>(dsm);   // merge area, aliases the tables after the loop

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int bh = blockIdx.y, chunk = blockIdx.x;
  const int bb = bh / p.Hkv, hk = bh - bb * p.Hkv;
  const int len = static_cast<int>(min(static_cast<int64_t>(p.seq_lens[bb]), p.Nmax));
  const int k0 = chunk * p.chunk_len;
  const int k1 = min(len, k0 + p.chunk_len);

  for (int i = tid; i < KLUT * 32; i += kDecThreads) {
    const int e = i >> 5;
    lutk[i] = pack_half2(__ldg(p.kc + (e & ((1 << KB) - 1))) / p.k_scale, __ldg(p.kc + (e >> KB)) / p.k_scale);
  }
  for (int i = tid; i < VLUT * 32; i += kDecThreads) {
    const int e = i >> 5;
    lutv[i] = pack_half2(__ldg(p.vc + (e & ((1 << VB) - 1))) / p.v_scale, __ldg(p.vc + (e >> VB)) / p.v_scale);
  }
  if (tid < 128) {
    const int e = tid >> 5;
    luts[tid] = pack_half2((e & 1) ? 1.f : -1.f, (e & 2) ? 1.f : -1.f);
  }
  if constexpr (KF == KFMT_SPEC || VF == VFMT_SPEC) {
    for (int i = tid; i < 510; i += kDecThreads) {
      const float v = __ldg(p.unit_c + i);
      const __half h = __float2half_rn(v);
      uhalf[i] = h;
      uhalf[510 + i] = __float2half_rn(v - __half2float(h));
    }
  }
  __syncthreads();

  // ---- query operands (rows g and g+8 of the GQA group) ----
  const int G = p.G;
  const int row0 = g, row1 = g + 8;
  const bool r0ok = row0 < G, r1ok = row1 < G;
  const int64_t qrow0 = static_cast<int64_t>(bb) * p.Hq + hk * G + row0;
  const int64_t qrow1 = static_cast<int64_t>(bb) * p.Hq + hk * G + row1;
  uint32_t qa[KST][4], ql[KST][4];   // hi and lo halves of the query operand
#pragma unroll
  for (int s = 0; s < KST; ++s) {
    const int dm = t * TDK + 4 * s;
    float a[4] = {0.f, 0.f, 0.f, 0.f}, b[4] = {0.f, 0.f, 0.f, 0.f};
    if (r0ok) for (int i = 0; i < 4; ++i) a[i] = p.qa[qrow0 * D + dm + i];
    if (r1ok) for (int i = 0; i < 4; ++i) b[i] = p.qa[qrow1 * D + dm + i];
    split_pair(a[0], a[1], qa[s][0], ql[s][0]);
    split_pair(b[0], b[1], qa[s][1], ql[s][1]);
    split_pair(a[2], a[3], qa[s][2], ql[s][2]);
    split_pair(b[2], b[3], qa[s][3], ql[s][3]);
  }
  uint32_t qb[KST][4], qbl[KST][4];   // prod: QJL operand (hi, lo) with the same permutation
  uint32_t qx[4], qxl[4];              // spectral: the extra head k-step (hi, lo)
  if constexpr (KF == KFMT_PROD) {
#pragma unroll
    for (int s = 0; s < KST; ++s) {
      const int dm = t * TDK + 4 * s;
      float a[4] = {0.f, 0.f, 0.f, 0.f}, c[4] = {0.f, 0.f, 0.f, 0.f};
      if (r0ok) for (int i = 0; i < 4; ++i) a[i] = p.qb[qrow0 * p.qb_stride + dm + i];
      if (r1ok) for (int i = 0; i < 4; ++i) c[i] = p.qb[qrow1 * p.qb_stride + dm + i];
      split_pair(a[0], a[1], qb[s][0], qbl[s][0]);
      split_pair(c[0], c[1], qb[s][1], qbl[s][1]);
      split_pair(a[2], a[3], qb[s][2], qbl[s][2]);
      split_pair(c[2], c[3], qb[s][3], qbl[s][3]);
    }
  }
  if constexpr (KF == KFMT_SPEC) {
    float a[4] = {0.f, 0.f, 0.f, 0.f}, c[4] = {0.f, 0.f, 0.f, 0.f};
    const int sl[4] = {2 * t, 2 * t + 1, 8 + 2 * t, 9 + 2 * t};
    if (r0ok) for (int i = 0; i < 4; ++i) a[i] = p.qb[qrow0 * p.qb_stride + sl[i]];
    if (r1ok) for (int i = 0; i < 4; ++i) c[i] = p.qb[qrow1 * p.qb_stride + sl[i]];
    split_pair(a[0], a[1], qx[0], qxl[0]);
    split_pair(c[0], c[1], qx[1], qxl[1]);
    split_pair(a[2], a[3], qx[2], qxl[2]);
    split_pair(c[2], c[3], qx[3], qxl[3]);
  }
  const float sa0 = r0ok ? p.qs[qrow0 * 2] * p.k_scale : 0.f, sa1 = r1ok ? p.qs[qrow1 * 2] * p.k_scale : 0.f;
  const float sb0 = r0ok ? p.qs[qrow0 * 2 + 1] : 0.f, sb1 = r1ok ? p.qs[qrow1 * 2 + 1] : 0.f;

  // spectral head layout (bit offsets of the top dims inside the head words)
  int kpos[TQ_MAX_TOP], vpos[TQ_MAX_TOP];
  int kq_pos = 0;
  if constexpr (KF == KFMT_SPEC) {
    int acc = 0;
    for (int j = 0; j < TQ_MAX_TOP; ++j) { kpos[j] = acc; acc += (j < p.k_top_k) ? p.k_top_bits[j] : 0; }
    kq_pos = acc;
  }
  if constexpr (VF == VFMT_SPEC) {
    int acc = 0;
    for (int j = 0; j < TQ_MAX_TOP; ++j) { vpos[j] = acc; acc += (j < p.v_top) ? p.v_top_bits[j] : 0; }
  }

  // ---- running state ----
  float o[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float oh[4] = {0.f, 0.f, 0.f, 0.f};       // spectral value head dims
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  const int64_t rec0 = static_cast<int64_t>(bh) * p.Nmax;
  for (int u0 = k0 + warp * 16; u0 < k1; u0 += kDecWarps * 16) {
    // keys this thread touches: score B operand -> keys u0+g, u0+8+g; C/P keys -> u0+2t(+1), u0+8+2t(+1)
    const int kA = u0 + g, kB = u0 + 8 + g;
    const int kc[4] = {u0 + 2 * t, u0 + 2 * t + 1, u0 + 8 + 2 * t, u0 + 9 + 2 * t};
    uint32_t ks0[NWK], ks1[NWK];
    load_slice<NWK>(p.kcodes + (rec0 + kA) * p.k_words + p.k_code_off, p.k_words - p.k_code_off,
                    t * TDK * KB, kA < k1, ks0);
    load_slice<NWK>(p.kcodes + (rec0 + kB) * p.k_words + p.k_code_off, p.k_words - p.k_code_off,
                    t * TDK * KB, kB < k1, ks1);
    float kn[4], vn[4], gm[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool ok = kc[i] < k1;
      kn[i] = (KF != KFMT_SPEC && ok) ? __ldg(p.knorms + rec0 + kc[i]) : 1.f;
      vn[i] = (VF != VFMT_SPEC && ok) ? __ldg(p.vnorms + rec0 + kc[i]) : 1.f;
      gm[i] = (KF == KFMT_PROD && ok) ? __ldg(p.krnorms + rec0 + kc[i]) : 0.f;
    }
    uint32_t vs[4][NWV];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      load_slice<NWV>(p.vcodes + (rec0 + kc[i]) * p.v_words + p.v_code_off, p.v_words - p.v_code_off,
                      g * TDV * VB, kc[i] < k1, vs[i]);

    // ---- scores ----
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t(&ks)[NWK] = nt ? ks1 : ks0;
#pragma unroll
      for (int s = 0; s < KST; ++s) {
        const uint32_t b0 = lutk[(pair_at<KB, NWK>(ks, 4 * s * KB) << 5) + lane];
        const uint32_t b1 = lutk[(pair_at<KB, NWK>(ks, (4 * s + 2) * KB) << 5) + lane];
        mma16816(acc, qa[s][0], qa[s][1], qa[s][2], qa[s][3], b0, b1);
        mma16816(acc, ql[s][0], ql[s][1], ql[s][2], ql[s][3], b0, b1);
      }
      float acc2[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (KF == KFMT_PROD) {
        const int key = nt ? kB : kA;
        const uint32_t sw = key < k1 ? __ldg(p.ksigns + (rec0 + key) * p.k_sign_words + t * (TDK / 32)) : 0u;
        static_assert(KF != KFMT_PROD || TDK == 32, "prod signs need d = 128");
#pragma unroll
        for (int s = 0; s < KST; ++s) {
          const uint32_t b0 = luts[(((sw >> (4 * s)) & 3u) << 5) + lane];
          const uint32_t b1 = luts[(((sw >> (4 * s + 2)) & 3u) << 5) + lane];
          mma16816(acc2, qb[s][0], qb[s][1], qb[s][2], qb[s][3], b0, b1);
          mma16816(acc2, qbl[s][0], qbl[s][1], qbl[s][2], qbl[s][3], b0, b1);
        }
      }
      if constexpr (KF == KFMT_SPEC) {
        // extra k-step: slots 2t,2t+1 = head dims, slots 8+2t,9+2t = QJL signs times gamma
        const int key = nt ? kB : kA;
        uint32_t hw[3] = {0u, 0u, 0u};
        float gk = 0.f;
        if (key < k1) {
          const uint32_t* rec = p.kcodes + (rec0 + key) * p.k_words;
          for (int i = 0; i < 3 && i < p.k_code_off; ++i) hw[i] = __ldg(rec + i);
          if (p.k_qjl) gk = __ldg(p.krnorms + rec0 + key);
        }
        float hv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int j = 2 * t + i;
          if (j < p.k_top_k) {
            const int nb = p.k_top_bits[j];
            if (nb > 0) {
              const int e = unit_c_off(nb) + head_field(hw, kpos[j], nb);
              hv[i] = __half2float(uhalf[e]) + __half2float(uhalf[510 + e]);
            }
            if (p.k_qjl) hv[2 + i] = head_field(hw, kq_pos + j, 1) ? gk : -gk;
          }
        }
        uint32_t bh0, bl0, bh1, bl1;
        split_pair(hv[0], hv[1], bh0, bl0);
        split_pair(hv[2], hv[3], bh1, bl1);
        mma16816(acc2, qx[0], qx[1], qx[2], qx[3], bh0, bh1);
        mma16816(acc2, qxl[0], qxl[1], qxl[2], qxl[3], bh0, bh1);
        mma16816(acc2, qx[0], qx[1], qx[2], qx[3], bl0, bl1);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int ci = nt * 2 + (i & 1);        // which of kc[] this column is
        const float sa = (i < 2) ? sa0 : sa1, sb = (i < 2) ? sb0 : sb1;
        float v;
        if constexpr (KF == KFMT_PROD) v = kn[ci] * (sa * acc[i] + p.qjl_coef * gm[ci] * sb * acc2[i]);
        else if constexpr (KF == KFMT_SPEC) v = sa * acc[i] + sb * acc2[i];
        else v = kn[ci] * sa * acc[i];
        sc[nt][i] = (kc[ci] < k1) ? v : -INFINITY;
      }
    }
    // ---- online softmax (log2 domain), rows g (c0,c1) and g+8 (c2,c3) ----
    float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
    float mx1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    if (mn0 > m0) {
      const float f = exp2f(m0 - mn0);
      l0 *= f;
#pragma unroll
      for (int i = 0; i < NT; ++i) { o[i][0] *= f; o[i][1] *= f; }
      oh[0] *= f; oh[1] *= f;
      m0 = mn0;
    }
    if (G > 8 && mn1 > m1) {
      const float f = exp2f(m1 - mn1);
      l1 *= f;
#pragma unroll
      for (int i = 0; i < NT; ++i) { o[i][2] *= f; o[i][3] *= f; }
      oh[2] *= f; oh[3] *= f;
      m1 = mn1;
    }
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      pr[nt][0] = r0ok ? exp2f(sc[nt][0] - m0) : 0.f;
      pr[nt][1] = r0ok ? exp2f(sc[nt][1] - m0) : 0.f;
      pr[nt][2] = (G > 8 && r1ok) ? exp2f(sc[nt][2] - m1) : 0.f;
      pr[nt][3] = (G > 8 && r1ok) ? exp2f(sc[nt][3] - m1) : 0.f;
      l0 += pr[nt][0] + pr[nt][1];
      l1 += pr[nt][2] + pr[nt][3];
    }
    // A operand of P.V: p * ||v|| as half (rows g, g+8; keys 2t,2t+1 | 8+2t,9+2t)
    uint32_t pa0, pa1, pa2, pa3, pl0, pl1, pl2, pl3;
    split_pair(pr[0][0] * vn[0], pr[0][1] * vn[1], pa0, pl0);
    split_pair(pr[0][2] * vn[0], pr[0][3] * vn[1], pa1, pl1);
    split_pair(pr[1][0] * vn[2], pr[1][1] * vn[3], pa2, pl2);
    split_pair(pr[1][2] * vn[2], pr[1][3] * vn[3], pa3, pl3);
    // ---- P.V in the rotated domain ----
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const uint32_t e01 = field_at<VB, NWV>(vs[0], i * VB) | (field_at<VB, NWV>(vs[1], i * VB) << VB);
      const uint32_t e23 = field_at<VB, NWV>(vs[2], i * VB) | (field_at<VB, NWV>(vs[3], i * VB) << VB);
      const uint32_t b0 = lutv[(e01 << 5) + lane], b1 = lutv[(e23 << 5) + lane];
      mma16816(o[i], pa0, pa1, pa2, pa3, b0, b1);
      mma16816(o[i], pl0, pl1, pl2, pl3, b0, b1);
    }
    if constexpr (VF == VFMT_SPEC) {
      // head dims of the values: n-tile slot g = head dim g
      float hv[4] = {0.f, 0.f, 0.f, 0.f};
      if (g < p.v_top) {
        const int nb = p.v_top_bits[g];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (kc[i] < k1 && nb > 0) {
            const uint32_t* rec = p.vcodes + (rec0 + kc[i]) * p.v_words;
            uint32_t hw[3] = {0u, 0u, 0u};
            for (int w = 0; w < 3 && w < p.v_code_off; ++w) hw[w] = __ldg(rec + w);
            const int e = unit_c_off(nb) + head_field(hw, vpos[g], nb);
            hv[i] = (__half2float(uhalf[e]) + __half2float(uhalf[510 + e])) / p.v_scale;
          }
        }
      }
      uint32_t bh0, bl0, bh1, bl1;
      split_pair(hv[0], hv[1], bh0, bl0);
      split_pair(hv[2], hv[3], bh1, bl1);
      mma16816(oh, pa0, pa1, pa2, pa3, bh0, bh1);
      mma16816(oh, pl0, pl1, pl2, pl3, bh0, bh1);
      mma16816(oh, pa0, pa1, pa2, pa3, bl0, bl1);
    }
  }

  // ---- merge the warps of this CTA (the tables are dead from here on) ----
  __syncthreads();
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  float* wm = mrg + warp * 16 * (D + 2);      // [16 rows][m, l, o'[D]]
  if (t == 0) {
    wm[row0 * (D + 2)] = m0; wm[row0 * (D + 2) + 1] = l0;
    wm[row1 * (D + 2)] = m1; wm[row1 * (D + 2) + 1] = l1;
  }
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    // column n = 2t (+1) of n-tile i is value dim n*TDV + i
    wm[row0 * (D + 2) + 2 + (2 * t) * TDV + i] = o[i][0];
    wm[row0 * (D + 2) + 2 + (2 * t + 1) * TDV + i] = o[i][1];
    wm[row1 * (D + 2) + 2 + (2 * t) * TDV + i] = o[i][2];
    wm[row1 * (D + 2) + 2 + (2 * t + 1) * TDV + i] = o[i][3];
  }
  __syncwarp();
  if constexpr (VF == VFMT_SPEC) {
    // head dims j < v_top come from the head accumulator (columns 2t, 2t+1)
    if (2 * t < p.v_top) { wm[row0 * (D + 2) + 2 + 2 * t] = oh[0]; wm[row1 * (D + 2) + 2 + 2 * t] = oh[2]; }
    if (2 * t + 1 < p.v_top) { wm[row0 * (D + 2) + 3 + 2 * t] = oh[1]; wm[row1 * (D + 2) + 3 + 2 * t] = oh[3]; }
  }
  __syncthreads();
  for (int r = 0; r < G; ++r) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, mrg[w * 16 * (D + 2) + r * (D + 2)]);
    float f[kDecWarps];
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float mw = mrg[w * 16 * (D + 2) + r * (D + 2)];
      f[w] = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
      L += f[w] * mrg[w * 16 * (D + 2) + r * (D + 2) + 1];
    }
    const int64_t qi = static_cast<int64_t>(bb) * p.Hq + hk * G + r;
    const int64_t pi = qi * p.n_chunks + chunk;
    if (tid == 0) { p.part_ml[pi * 2] = M; p.part_ml[pi * 2 + 1] = L; }
    for (int j = tid; j < D; j += kDecThreads) {
      float a = 0.f;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) a += f[w] * mrg[w * 16 * (D + 2) + r * (D + 2) + 2 + j];
      p.part_o[pi * D + j] = a * p.v_scale;
    }
  }
}

// Dynamic shared memory of decode_attn_kernel<D, *, KB, *, VB>.
inline size_t decode_smem_bytes(int D, int kb, int vb) {
  const size_t tables = (static_cast<size_t>(1u << (2 * kb)) + (1u << (2 * vb)) + 4) * 32 * 4 + 2048;
  const size_t merge = static_cast<size_t>(kDecWarps) * 16 * (D + 2) * 4;
  return tables > merge ? tables : merge;
}

struct QPrepParams {
  const void* q;
  int dtype;
  int rows, D, kind;
  float scale;               // softmax scale * log2(e)
  const float* rot;          // K rotation [D*D]
  const float* S;            // prod [m*D] / spectral [k*k]
  int m;
  const float* dim_sigma;    // spectral
  int k_top, qjl;
  float spec_coef;           // sqrt(pi/2)/k
  float* qa;                 // [rows][D]
  float* qb;                 // [rows][qb_stride]
  float* qs;                 // [rows][2]
  int qb_stride;
};

struct CombineParams {
  int rows, D, n_chunks;
  const float* part_ml;
  const float* part_o;
  const float* rot_v;       // [D*D]
  const float* v_sigma;     // spectral values: per-dim scale, else NULL
  float* out;               // [rows][D]
};

}  // namespace tq
