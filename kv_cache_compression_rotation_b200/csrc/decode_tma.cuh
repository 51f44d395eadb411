// Decode attention with bulk-copy (TMA engine) staging of the packed cache, d = 128.
//
// Computes, for MSE or PROD keys and MSE values, the same step as decode_attn_kernel
// (decode.cuh): logit = scale * est(q, k_i), online softmax, o' = sum p ||v|| c[code_v].
//
// Streaming.  Persistent CTAs (one per SM) walk work items (batch * kv-head, head block,
// context chunk).  One producer warp copies each item in stages of 16 tokens per consumer warp with
// cp.async.bulk (key codes, value codes, norms; prod adds sign words and residual norms)
// into a 4-deep shared-memory ring; 11 (prod: 7) consumer warps each take 16 tokens of a stage,
// pull their record slices into registers, release the stage and compute.
//
// Math per 16-token unit, all on mma.sync m16n8k16 (fp16 in, fp32 accumulate):
//   scores  S[16 tokens x 8 heads] = K_hat[16 x 128] . Q'^T     (A = table-decoded keys)
//   P       exp2(S - m) * ||v||, transposed in registers with movmatrix
//   values  O'^T[128 dims x 8 heads] += V_hat^T[128 x 16] . P^T (A = table-decoded values)
// Tokens and value dims sit on the MMA's M side (16 rows), the query heads of the GQA
// group on N (8 columns), so a 4-head group fills half of each MMA instead of a quarter.
// Table decoding: one 32-bit shared load turns a pair of codes into half2 codebook values
// (table replicated per lane, so a warp's 32 loads hit 32 banks).
// Precision: the query operand and P are split hi + lo (two MMAs into one accumulator),
// table entries are c / s with a searched shared scale s (see tq_lut_scale).
// Token order inside a unit: score row r holds token r/2 + 4 (r mod 2) + 8 (r / 8)
// (rows 0..7) which spreads a warp's value-slice loads over both halves of the banks;
// the k-index of P^T follows the score rows through the transpose.
// All waits are bounded (TQ_ERR_TIMEOUT on expiry); a CTA that times out drains the
// copies it issued before it exits.
#pragma once

#include "decode.cuh"

namespace tq {

// Consumer warps per CTA: MSE keys fit 11 (plus the producer: 12 warps of <= 168
// registers fill the register file); PROD keys need more registers and run 7.
__host__ __device__ constexpr int tma_consumers(int kf) { return kf == KFMT_PROD ? 7 : 11; }
__host__ __device__ constexpr int tma_stage_tokens(int kf) { return tma_consumers(kf) * 16; }
constexpr int kTmaStages = 4;
constexpr int kTmaHeadBlock = 8;     // query heads per work item (MMA N)

__device__ __forceinline__ uint32_t tma_smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool tma_mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool tma_mbar_wait(uint32_t bar, uint32_t parity, long long limit, int* status,
                                              volatile int* abort_flag) {
  for (long long i = 0;; ++i) {
    if (tma_mbar_try(bar, parity)) return true;
    if (i >= limit || *abort_flag) {
      report_status(status, kDevTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// Transpose of an 8x8 matrix of halves held one row-pair per thread (mma fragment layout).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

struct TmaStageLayout {
  uint32_t kcodes, vcodes, knorm, vnorm, ksign, krn, bytes;
};

// Byte offsets of the arrays of one stage (all 16-byte aligned).
__host__ __device__ inline TmaStageLayout tma_stage_layout(int kw, int vw, int kf, int ksw) {
  const int st = tma_stage_tokens(kf);
  TmaStageLayout L{};
  uint32_t o = 0;
  L.kcodes = o; o += st * kw * 4;
  L.vcodes = o; o += st * vw * 4;
  L.knorm = o; o += (st + 4) * 4;
  L.vnorm = o; o += (st + 4) * 4;
  L.ksign = o; o += (kf == KFMT_PROD) ? st * ksw * 4 : 0;
  L.krn = o; o += (kf == KFMT_PROD) ? (st + 4) * 4 : 0;
  L.bytes = o;
  return L;
}

inline size_t decode_tma_smem_bytes(int kb, int vb, int kf, int ksw) {
  const size_t ne = static_cast<size_t>(1u << (2 * (kb > vb ? kb : vb)));
  const size_t tables = (ne * 64 + 4 * 32) * 4;
  const TmaStageLayout L = tma_stage_layout(128 * kb / 32, 128 * vb / 32, kf, ksw);
  const size_t merge = static_cast<size_t>(tma_consumers(kf)) * kTmaHeadBlock * (128 + 2) * 4;
  return tables + static_cast<size_t>(kTmaStages) * L.bytes + merge + 2 * kTmaStages * 8 + 64 + 16;
}

// Head blocks per GQA group (work items split groups larger than 8 heads).
__host__ __device__ inline int tma_head_blocks(int G) { return (G + kTmaHeadBlock - 1) / kTmaHeadBlock; }

// Explicit shared-space loads (32-bit shared addresses): the stage and table reads must
// be LDS, never generic loads through the global path.
__device__ __forceinline__ uint32_t tab_ld(uint32_t tab, uint32_t off) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(tab + off));
  return v;
}
__device__ __forceinline__ uint32_t sld32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ float sldf(uint32_t a) { return __uint_as_float(sld32(a)); }

// Slice of NW words of a record in shared memory starting at word w0 (aligned slices).
template <int NW>
__device__ __forceinline__ void sld_words(uint32_t a, bool valid, uint32_t (&w)[NW]) {
  if constexpr (NW == 4) {
    uint32_t x0 = 0, x1 = 0, x2 = 0, x3 = 0;
    if (valid) asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3) : "r"(a) : "memory");
    w[0] = x0; w[1] = x1; w[2] = x2; w[3] = x3;
  } else if constexpr (NW == 2) {
    uint32_t x0 = 0, x1 = 0;
    if (valid) asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(x0), "=r"(x1) : "r"(a) : "memory");
    w[0] = x0; w[1] = x1;
  } else {
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = valid ? sld32(a + 4 * i) : 0u;
  }
}

// General slice (any bit offset): NW words starting at bit `base` of the record at `rec`.
template <int NW>
__device__ __forceinline__ void sld_slice(uint32_t rec, int rec_words, int base, bool valid, uint32_t (&seg)[NW]) {
  const int w0 = base >> 5, sh = base & 31;
  if (sh == 0 && (w0 * 4) % (NW == 4 ? 16 : (NW == 2 ? 8 : 4)) == 0) {
    sld_words<NW>(rec + 4 * w0, valid, seg);
    return;
  }
  uint32_t w[NW + 1];
#pragma unroll
  for (int i = 0; i <= NW; ++i) {
    const int wi = w0 + i;
    w[i] = (valid && wi < rec_words && (i < NW || sh != 0)) ? sld32(rec + 4 * wi) : 0u;
  }
#pragma unroll
  for (int i = 0; i < NW; ++i) seg[i] = __funnelshift_r(w[i], w[i + 1], sh);
}

// Byte k of w as table entry index, combined with this lane's byte offset `lo8` (< 256).
__device__ __forceinline__ uint32_t tab_off(uint32_t w, uint32_t lo8, int k) {
  return __byte_perm(w, lo8, 0x7604u | (static_cast<uint32_t>(k) << 4));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int KF, int KB, int VB>
__global__ void __launch_bounds__((tma_consumers(KF) + 1) * 32, 1)
decode_tma_kernel(const DecodeParams p, int* status, long long wait_lim) {
  constexpr int kTmaConsumerWarps = tma_consumers(KF);
  constexpr int kTmaThreads = (kTmaConsumerWarps + 1) * 32;
  constexpr int kTmaStageTokens = tma_stage_tokens(KF);
  constexpr int D = 128;
  constexpr int KST = D / 16;                 // mma k-steps over the key dims
  constexpr int TDK = D / 4;                  // key dims per thread
  constexpr int NWK = (TDK * KB + 31) / 32;
  constexpr int TDV = D / 8;                  // value dims per thread
  constexpr int NWV = (TDV * VB + 31) / 32;
  constexpr int MT = D / 16;                  // P.V M-tiles (16 dims each)
  constexpr int KLUT = 1 << (2 * KB), VLUT = 1 << (2 * VB);
  constexpr int KW = D * KB / 32, VW = D * VB / 32;     // record words
  constexpr int KSW = 4;                                // prod sign words (m = 128)
  constexpr int HB = kTmaHeadBlock;
  constexpr int CONSUMERS = kTmaConsumerWarps * 32;
  constexpr int NE = KLUT > VLUT ? KLUT : VLUT;        // table entries
  extern __shared__ __align__(128) uint32_t tsm_[];
  // table entry e is 256 B: the key value pair for lanes 0..31, then the value pair; a
  // lookup address is (e << 8) | (lane * 4) [+ 128], one byte permute from the code word
  const uint32_t tab = tma_smem_u32(tsm_);
  uint32_t* luts = tsm_ + NE * 64;
  const uint32_t luts_a = tma_smem_u32(luts);
  unsigned char* stage0 = reinterpret_cast<unsigned char*>(luts + 4 * 32);
  const TmaStageLayout SL = tma_stage_layout(KW, VW, KF, KSW);
  float* mrg = reinterpret_cast<float*>(stage0 + static_cast<size_t>(kTmaStages) * SL.bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(mrg + kTmaConsumerWarps * HB * (D + 2));
  int* nb_count = reinterpret_cast<int*>(bars + 2 * kTmaStages);   // [kTmaStages] tokens with staged norms
  int* nb_off = nb_count + kTmaStages;                                 // [kTmaStages] their offset in the stage
  volatile int* abort_flag = nb_off + kTmaStages;
  volatile int* consumers_stop = abort_flag + 1;   // uniform exit decision of the consumer warps
  const uint32_t bar0 = tma_smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kTmaStages + s); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.G;
  const int nhb = tma_head_blocks(G);
  const int n_items = p.B * p.Hkv * nhb * p.n_chunks;
  const int64_t total_recs = static_cast<int64_t>(p.B) * p.Hkv * p.Nmax;
  // item -> (bh, head block, chunk, token range)
  auto item_range = [&](int item, int& bh, int& hblk, int& chunk, int& k0, int& k1) {
    chunk = item % p.n_chunks;
    const int rest = item / p.n_chunks;
    hblk = rest % nhb;
    bh = rest / nhb;
    const int bb = bh / p.Hkv;
    const int len = static_cast<int>(min(static_cast<int64_t>(p.seq_lens[bb]), p.Nmax));
    k0 = chunk * p.chunk_len;
    k1 = min(len, k0 + p.chunk_len);
  };

  if (tid == 0) {
    for (int s = 0; s < kTmaStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(full_bar(s)), "r"(1));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty_bar(s)), "r"(kTmaConsumerWarps));
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < NE * 64; i += kTmaThreads) {
    const int e = i >> 6;
    uint32_t val = 0u;
    if ((i & 32) == 0) {
      if (e < KLUT)
        val = pack_half2(__ldg(p.kc + (e & ((1 << KB) - 1))) / p.k_scale, __ldg(p.kc + (e >> KB)) / p.k_scale);
    } else if (e < VLUT) {
      val = pack_half2(__ldg(p.vc + (e & ((1 << VB) - 1))) / p.v_scale, __ldg(p.vc + (e >> VB)) / p.v_scale);
    }
    tsm_[i] = val;
  }
  if (tid < 128) {
    const int e = tid >> 5;
    luts[tid] = pack_half2((e & 1) ? 1.f : -1.f, (e & 2) ? 1.f : -1.f);
  }
  __syncthreads();

  if (warp == kTmaConsumerWarps) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int gs = 0;                                   // global stage counter of this CTA
      bool stop = false;
      for (int item = blockIdx.x; item < n_items && !stop; item += gridDim.x) {
        int bh, hblk, chunk, k0, k1;
        item_range(item, bh, hblk, chunk, k0, k1);
        const int64_t rec0 = static_cast<int64_t>(bh) * p.Nmax;
        for (int t0 = k0; t0 < k1; t0 += kTmaStageTokens, ++gs) {
          const int s = gs % kTmaStages, use = gs / kTmaStages;
          if (use > 0 && !tma_mbar_wait(empty_bar(s), (use - 1) & 1, wait_lim, status, abort_flag)) {
            stop = true;
            break;
          }
          const int cnt = min(kTmaStageTokens, k1 - t0);
          // norms are 4 B per token and a bulk copy moves 16-byte aligned multiples of
          // 16 B: start at the aligned token below the stage and cover whole groups of 4
          // tokens, never past the end of the array; leftovers are read directly
          const int64_t r = rec0 + t0;
          const int off = static_cast<int>(r & 3);
          int nn = (off + cnt + 3) & ~3;
          if (r - off + nn > total_recs) nn = (off + cnt) & ~3;
          nb_count[s] = max(0, nn - off);
          nb_off[s] = off;
          uint32_t bytes = cnt * (KW + VW) * 4 + 2 * nn * 4;
          if (KF == KFMT_PROD) bytes += cnt * KSW * 4 + nn * 4;
          const uint32_t fb = full_bar(s);
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(fb), "r"(bytes) : "memory");
          const uint32_t sb = tma_smem_u32(stage0 + static_cast<size_t>(s) * SL.bytes);
          bulk_g2s(sb + SL.kcodes, p.kcodes + r * KW, cnt * KW * 4, fb);
          bulk_g2s(sb + SL.vcodes, p.vcodes + r * VW, cnt * VW * 4, fb);
          if (nn > 0) {
            bulk_g2s(sb + SL.knorm, p.knorms + (r - off), nn * 4, fb);
            bulk_g2s(sb + SL.vnorm, p.vnorms + (r - off), nn * 4, fb);
          }
          if (KF == KFMT_PROD) {
            bulk_g2s(sb + SL.ksign, p.ksigns + r * KSW, cnt * KSW * 4, fb);
            if (nn > 0) bulk_g2s(sb + SL.krn, p.krnorms + (r - off), nn * 4, fb);
          }
        }
      }
      // drain: the copies this CTA issued land before it may exit
      for (int j = max(0, gs - kTmaStages); j < gs; ++j)
        for (long long i = 0; !tma_mbar_try(full_bar(j % kTmaStages), (j / kTmaStages) & 1) && i < (1ll << 28); ++i) {}
    }
    return;
  }

  // ---------------- consumers ----------------
  // score-tile row g holds token pg of the unit, row g + 8 token 8 + pg
  const int pg = (g >> 1) + 4 * (g & 1);
  // value-operand k-indices 2t, 2t+1, 2t+8, 2t+9 are the tokens of score rows 2t, 2t+1, ...
  const int kv[4] = {t, t + 4, 8 + t, 12 + t};
  const uint32_t klo = static_cast<uint32_t>(lane) * 4u, vlo = klo + 128u;
  int gs = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    int bh, hblk, chunk, k0, k1;
    item_range(item, bh, hblk, chunk, k0, k1);
    const int bb = bh / p.Hkv, hk = bh - bb * p.Hkv;
    const int64_t rec0 = static_cast<int64_t>(bh) * p.Nmax;
    const int h0 = hblk * HB;                         // first head of this block in the group
    const int nh = min(HB, G - h0);
    const int64_t qbase = static_cast<int64_t>(bb) * p.Hq + hk * G + h0;
    // query operand (B of the score MMA): column g = head h0 + g
    const bool hok = g < nh;
    uint32_t qh[KST][2], ql[KST][2];
#pragma unroll
    for (int s = 0; s < KST; ++s) {
      const int dm = t * TDK + 4 * s;
      float a[4] = {0.f, 0.f, 0.f, 0.f};
      if (hok) for (int i = 0; i < 4; ++i) a[i] = p.qa[(qbase + g) * D + dm + i];
      split_pair(a[0], a[1], qh[s][0], ql[s][0]);
      split_pair(a[2], a[3], qh[s][1], ql[s][1]);
    }
    uint32_t qb[KST][2];
    if constexpr (KF == KFMT_PROD) {
#pragma unroll
      for (int s = 0; s < KST; ++s) {
        const int dm = t * TDK + 4 * s;
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        if (hok) for (int i = 0; i < 4; ++i) a[i] = p.qb[(qbase + g) * p.qb_stride + dm + i];
        qb[s][0] = pack_half2(a[0], a[1]);
        qb[s][1] = pack_half2(a[2], a[3]);
      }
    }
    // this thread's score columns are heads 2t, 2t+1 of the block
    const bool c0ok = 2 * t < nh, c1ok = 2 * t + 1 < nh;
    const float sa0 = c0ok ? p.qs[(qbase + 2 * t) * 2] * p.k_scale : 0.f;
    const float sa1 = c1ok ? p.qs[(qbase + 2 * t + 1) * 2] * p.k_scale : 0.f;
    const float sb0 = c0ok ? p.qs[(qbase + 2 * t) * 2 + 1] * p.qjl_coef : 0.f;
    const float sb1 = c1ok ? p.qs[(qbase + 2 * t + 1) * 2 + 1] * p.qjl_coef : 0.f;

    float o[MT][4];
#pragma unroll
    for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // heads 2t, 2t+1

    for (int t0 = k0; t0 < k1; t0 += kTmaStageTokens, ++gs) {
      const int s = gs % kTmaStages;
      if (!tma_mbar_wait(full_bar(s), (gs / kTmaStages) & 1, wait_lim, status, abort_flag)) break;
      const uint32_t sb = tma_smem_u32(stage0) + static_cast<uint32_t>(s) * SL.bytes;
      const int cnt = min(kTmaStageTokens, k1 - t0);
      const int nn = nb_count[s], noff = nb_off[s];
      const int u0 = warp * 16;                      // first token of this warp's unit (stage-local)
      // ---- pull this warp's slices out of the stage ----
      const int ka = u0 + pg, kb2 = u0 + 8 + pg;     // tokens of score rows g, g + 8
      const bool oka = ka < cnt, okb = kb2 < cnt;
      uint32_t ks0[NWK], ks1[NWK];
      sld_slice<NWK>(sb + SL.kcodes + ka * KW * 4, KW, t * TDK * KB, oka, ks0);
      sld_slice<NWK>(sb + SL.kcodes + kb2 * KW * 4, KW, t * TDK * KB, okb, ks1);
      auto norm_of = [&](uint32_t staged, const float* global, int lk, bool ok) {
        return ok ? (lk < nn ? sldf(staged + 4 * (noff + lk)) : __ldg(global + rec0 + t0 + lk)) : 0.f;
      };
      const float kn0 = norm_of(sb + SL.knorm, p.knorms, ka, oka), kn1 = norm_of(sb + SL.knorm, p.knorms, kb2, okb);
      const float vn0 = norm_of(sb + SL.vnorm, p.vnorms, ka, oka), vn1 = norm_of(sb + SL.vnorm, p.vnorms, kb2, okb);
      float gm0 = 0.f, gm1 = 0.f;
      uint32_t sw0 = 0u, sw1 = 0u;
      if constexpr (KF == KFMT_PROD) {
        gm0 = norm_of(sb + SL.krn, p.krnorms, ka, oka);
        gm1 = norm_of(sb + SL.krn, p.krnorms, kb2, okb);
        sw0 = oka ? sld32(sb + SL.ksign + (ka * KSW + t) * 4) : 0u;
        sw1 = okb ? sld32(sb + SL.ksign + (kb2 * KSW + t) * 4) : 0u;
      }
      uint32_t vs[4][NWV];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int lk = u0 + kv[i];
        sld_slice<NWV>(sb + SL.vcodes + lk * VW * 4, VW, g * TDV * VB, lk < cnt, vs[i]);
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty_bar(s)) : "memory");
      if (u0 >= cnt) continue;

      // ---- scores: S[16 tokens x 8 heads] ----
      float acc[4] = {0.f, 0.f, 0.f, 0.f}, accl[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s2 = 0; s2 < KST; ++s2) {
        uint32_t a0, a1, a2, a3;
        if constexpr (KB == 4) {
          // dims (4 s2, 4 s2 + 1) are byte 2 (s2 % 2) of word s2 / 2; (+2, +3) the next byte
          const uint32_t w0 = ks0[s2 >> 1], w1 = ks1[s2 >> 1];
          const int k = 2 * (s2 & 1);
          a0 = tab_ld(tab, tab_off(w0, klo, k));
          a1 = tab_ld(tab, tab_off(w1, klo, k));
          a2 = tab_ld(tab, tab_off(w0, klo, k + 1));
          a3 = tab_ld(tab, tab_off(w1, klo, k + 1));
        } else {
          a0 = tab_ld(tab, (pair_at<KB, NWK>(ks0, 4 * s2 * KB) << 8) | klo);
          a1 = tab_ld(tab, (pair_at<KB, NWK>(ks1, 4 * s2 * KB) << 8) | klo);
          a2 = tab_ld(tab, (pair_at<KB, NWK>(ks0, (4 * s2 + 2) * KB) << 8) | klo);
          a3 = tab_ld(tab, (pair_at<KB, NWK>(ks1, (4 * s2 + 2) * KB) << 8) | klo);
        }
        mma16816(acc, a0, a1, a2, a3, qh[s2][0], qh[s2][1]);
        mma16816(accl, a0, a1, a2, a3, ql[s2][0], ql[s2][1]);
      }
      float acc2[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (KF == KFMT_PROD) {
#pragma unroll
        for (int s2 = 0; s2 < KST; ++s2) {
          const uint32_t a0 = tab_ld(luts_a, ((((sw0 >> (4 * s2)) & 3u) << 5) + lane) * 4);
          const uint32_t a1 = tab_ld(luts_a, ((((sw1 >> (4 * s2)) & 3u) << 5) + lane) * 4);
          const uint32_t a2 = tab_ld(luts_a, ((((sw0 >> (4 * s2 + 2)) & 3u) << 5) + lane) * 4);
          const uint32_t a3 = tab_ld(luts_a, ((((sw1 >> (4 * s2 + 2)) & 3u) << 5) + lane) * 4);
          mma16816(acc2, a0, a1, a2, a3, qb[s2][0], qb[s2][1]);
        }
      }
      // acc[0], acc[1]: token row g, heads 2t, 2t+1; acc[2], acc[3]: token row g + 8
      float sc[4];
      {
        const float kr[4] = {kn0, kn0, kn1, kn1};
        const float gr[4] = {gm0, gm0, gm1, gm1};
        const float sa[4] = {sa0, sa1, sa0, sa1}, sbq[4] = {sb0, sb1, sb0, sb1};
        const bool ok[4] = {oka, oka, okb, okb};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float v = sa[i] * (acc[i] + accl[i]);
          if constexpr (KF == KFMT_PROD) v += gr[i] * sbq[i] * acc2[i];
          sc[i] = ok[i] ? kr[i] * v : -INFINITY;
        }
      }
      // ---- online softmax per head (log2 domain), reduced over the 8 token rows ----
      float mx0 = fmaxf(sc[0], sc[2]), mx1 = fmaxf(sc[1], sc[3]);
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      if (mn0 > m0 || mn1 > m1) {
        const float f0 = ex2(m0 - mn0), f1 = ex2(m1 - mn1);
        l0 *= f0;
        l1 *= f1;
#pragma unroll
        for (int i = 0; i < MT; ++i) { o[i][0] *= f0; o[i][2] *= f0; o[i][1] *= f1; o[i][3] *= f1; }
        m0 = mn0;
        m1 = mn1;
      }
      const float p00 = c0ok ? ex2(sc[0] - m0) : 0.f, p01 = c1ok ? ex2(sc[1] - m1) : 0.f;
      const float p10 = c0ok ? ex2(sc[2] - m0) : 0.f, p11 = c1ok ? ex2(sc[3] - m1) : 0.f;
      l0 += p00 + p10;
      l1 += p01 + p11;
      // P^T (16 tokens x 8 heads) as the B operand: transpose the two 8x8 halves
      uint32_t pth, ptl, pbh, pbl;
      split_pair(p00 * vn0, p01 * vn0, pth, ptl);
      split_pair(p10 * vn1, p11 * vn1, pbh, pbl);
      const uint32_t b0h = movmatrix_t(pth), b1h = movmatrix_t(pbh);
      const uint32_t b0l = movmatrix_t(ptl), b1l = movmatrix_t(pbl);
      // ---- O'^T[128 dims x 8 heads] += V_hat^T . P^T ----
      // M-tile i: row g = dim TDV g + i (first word of the slice), row g + 8 = dim TDV g + 8 + i
      if constexpr (VB == 4) {
        // byte j of lo (hi) holds the codes of one token pair for dim 2j (2j + 1) of a word
        uint32_t lo[2][2], hi[2][2];   // [token pair][word]
#pragma unroll
        for (int w = 0; w < 2; ++w) {
#pragma unroll
          for (int kp = 0; kp < 2; ++kp) {
            const uint32_t x = vs[2 * kp][w], y = vs[2 * kp + 1][w];
            lo[kp][w] = (x & 0x0F0F0F0Fu) | ((y << 4) & 0xF0F0F0F0u);
            hi[kp][w] = ((x >> 4) & 0x0F0F0F0Fu) | (y & 0xF0F0F0F0u);
          }
        }
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          const int k = i >> 1;
          const uint32_t a0 = tab_ld(tab, tab_off((i & 1) ? hi[0][0] : lo[0][0], vlo, k));
          const uint32_t a1 = tab_ld(tab, tab_off((i & 1) ? hi[0][1] : lo[0][1], vlo, k));
          const uint32_t a2 = tab_ld(tab, tab_off((i & 1) ? hi[1][0] : lo[1][0], vlo, k));
          const uint32_t a3 = tab_ld(tab, tab_off((i & 1) ? hi[1][1] : lo[1][1], vlo, k));
          mma16816(o[i], a0, a1, a2, a3, b0h, b1h);
          mma16816(o[i], a0, a1, a2, a3, b0l, b1l);
        }
      } else {
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          const uint32_t e00 = field_at<VB, NWV>(vs[0], i * VB) | (field_at<VB, NWV>(vs[1], i * VB) << VB);
          const uint32_t e01 = field_at<VB, NWV>(vs[0], (8 + i) * VB) | (field_at<VB, NWV>(vs[1], (8 + i) * VB) << VB);
          const uint32_t e10 = field_at<VB, NWV>(vs[2], i * VB) | (field_at<VB, NWV>(vs[3], i * VB) << VB);
          const uint32_t e11 = field_at<VB, NWV>(vs[2], (8 + i) * VB) | (field_at<VB, NWV>(vs[3], (8 + i) * VB) << VB);
          const uint32_t a0 = tab_ld(tab, (e00 << 8) | vlo), a1 = tab_ld(tab, (e01 << 8) | vlo);
          const uint32_t a2 = tab_ld(tab, (e10 << 8) | vlo), a3 = tab_ld(tab, (e11 << 8) | vlo);
          mma16816(o[i], a0, a1, a2, a3, b0h, b1h);
          mma16816(o[i], a0, a1, a2, a3, b0l, b1l);
        }
      }
    }

    // ---- merge this item across the consumer warps (named barrier 1) ----
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
    }
    float* wm = mrg + warp * HB * (D + 2);          // [head][m, l, o'[D]]
    if (g == 0) {
      wm[(2 * t) * (D + 2)] = m0; wm[(2 * t) * (D + 2) + 1] = l0;
      wm[(2 * t + 1) * (D + 2)] = m1; wm[(2 * t + 1) * (D + 2) + 1] = l1;
    }
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      wm[(2 * t) * (D + 2) + 2 + TDV * g + i] = o[i][0];
      wm[(2 * t + 1) * (D + 2) + 2 + TDV * g + i] = o[i][1];
      wm[(2 * t) * (D + 2) + 2 + TDV * g + 8 + i] = o[i][2];
      wm[(2 * t + 1) * (D + 2) + 2 + TDV * g + 8 + i] = o[i][3];
    }
    asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
    for (int idx = tid; idx < nh * D; idx += CONSUMERS) {
      const int r = idx / D, j = idx - r * D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kTmaConsumerWarps; ++w) M = fmaxf(M, mrg[(w * HB + r) * (D + 2)]);
      float a = 0.f, L = 0.f;
#pragma unroll
      for (int w = 0; w < kTmaConsumerWarps; ++w) {
        const float* row = mrg + (w * HB + r) * (D + 2);
        const float f = (row[0] == -INFINITY) ? 0.f : exp2f(row[0] - M);
        L += f * row[1];
        a += f * row[2 + j];
      }
      const int64_t qi = qbase + r;
      const int64_t pi = qi * p.n_chunks + chunk;
      if (j == 0) { p.part_ml[pi * 2] = M; p.part_ml[pi * 2 + 1] = L; }
      p.part_o[pi * D + j] = a * p.v_scale;
    }
    // every consumer warp takes the same exit decision: one thread samples the abort
    // flag between the two barriers (a warp that timed out still reaches both)
    if (tid == 0) *consumers_stop = *abort_flag;
    asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
    if (*consumers_stop) break;
  }
}

}  // namespace tq
