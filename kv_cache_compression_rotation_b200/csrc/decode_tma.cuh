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
//   scores  S[16 tokens x 8 columns] = K_hat[16 x 128] . Q'^T     (A = table-decoded keys)
//   P       exp2(S - m) * ||v||, transposed in registers with movmatrix
//   values  O'^T[128 dims x 8 columns] += V_hat^T[128 x 16] . P^T (A = table-decoded values)
// Tokens and value dims sit on the MMA's M side (16 rows), the query heads on N.  For GQA
// groups of at most 4 heads the 8 columns are 4 heads x (hi, lo) parts of the split
// operands (see PK below); larger groups take 8 heads per work item.
// Table decoding: one 32-bit shared load turns a pair of codes into half2 codebook values
// (table replicated per lane, so a warp's 32 loads hit 32 banks; the table sits at a
// 64 KB-aligned shared address, so one byte permute of the code word is the address).
// Precision: the query operand and P are split hi + lo (one accumulator), table entries
// are c / s with a searched shared scale s (see tq_lut_scale).
// Token order inside a unit: score rows r and r + 8 hold tokens tau(r) and 8 + tau(r), with
// tau = [0, 5, 1, 4, 2, 7, 3, 6]: the two rows a quarter-warp reads in one 16-byte key
// slice load are tokens of opposite parity (64-byte records: opposite bank halves), and
// the four tokens a half-warp reads in one value slice load cover both halves twice;
// the k-index of P^T follows the score rows through the transpose.
// Scheduling: the cross-row max runs only when a score of the warp exceeds its running
// max (warp vote), and the value half of unit i - 1 is issued next to the key half of
// unit i, so table loads, MMAs and softmax arithmetic of two units interleave.
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
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
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

// Shared memory of one CTA.  The lookup table must start at a 64 KB-aligned shared
// address (a byte permute then forms the complete lookup address); the small arrays
// (merge buffer, sign table, barriers) sit in the gap below it when they fit, so the
// request covers a gap of up to 64 KB plus the table and the stage ring.
__host__ __device__ inline uint32_t tma_table_bytes(int kb, int vb) {
  return (1u << (2 * (kb > vb ? kb : vb))) * 256u;
}
__host__ __device__ inline uint32_t tma_misc_bytes(int kf) {
  const uint32_t merge = static_cast<uint32_t>(tma_consumers(kf)) * 8u * (128u + 2u) * 4u;
  return merge + 4u * 32u * 4u + 2u * 4u * 8u + 64u;
}
inline size_t decode_tma_smem_bytes(int kb, int vb, int kf, int ksw) {
  const TmaStageLayout L = tma_stage_layout(128 * kb / 32, 128 * vb / 32, kf, ksw);
  return 65536 + tma_table_bytes(kb, vb) + 4 * static_cast<size_t>(L.bytes);
}

// Head blocks per GQA group (work items split groups larger than 8 heads).
__host__ __device__ inline int tma_head_blocks(int G) { return (G + kTmaHeadBlock - 1) / kTmaHeadBlock; }

// Explicit shared-space loads (32-bit shared addresses): the stage and table reads must
// be LDS, never generic loads through the global path.
__device__ __forceinline__ uint32_t tab_ld(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
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

// PK (packed columns, GQA groups of at most 4 heads): MMA column c < 4 carries the hi part
// of head c, column c + 4 its lo part.  The score MMA then yields hi and lo products in one
// instruction (summed across lanes t and t ^ 2), and P's hi / lo split rides in the same
// columns of the value MMA (summed in the merge).  Without PK the 8 columns are 8 heads and
// the hi / lo parts take separate MMAs.
template <int KF, int KB, int VB, bool PK>
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
  constexpr int HB = PK ? 4 : kTmaHeadBlock;            // query heads per work item
  constexpr int CONSUMERS = kTmaConsumerWarps * 32;
  constexpr int NE = KLUT > VLUT ? KLUT : VLUT;        // table entries
  constexpr uint32_t TAB = static_cast<uint32_t>(NE) * 256u;
  extern __shared__ __align__(128) unsigned char tsm_[];

  // ---- shared layout: table at a 64 KB-aligned address ----
  // Table entry e is 256 B: the key value pair for lanes 0..31, then the value pair.  With the
  // table base B (a multiple of 64 KB), the lookup address of a code pair byte x for this lane
  // is B | x << 8 | lane * 4 [+ 128]: one byte permute, no add.
  const TmaStageLayout SL = tma_stage_layout(KW, VW, KF, KSW);
  const uint32_t base = tma_smem_u32(tsm_);
  uint32_t dyn;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
  const uint32_t gap = (0u - base) & 0xFFFFu;
  const uint32_t tabA = base + gap;
  const uint32_t stageA = tabA + TAB;
  const uint32_t miscA = gap >= tma_misc_bytes(KF) ? base : stageA + kTmaStages * SL.bytes;
  const uint32_t endA = max(stageA + kTmaStages * SL.bytes, miscA + tma_misc_bytes(KF));
  if (endA > base + dyn) {                        // the request did not cover this layout
    if (threadIdx.x == 0) report_status(status, TQ_ERR_UNSUPPORTED);
    return;
  }
  auto gen = [&](uint32_t a) { return tsm_ + (a - base); };   // generic pointer of a shared address
  uint32_t* tab_g = reinterpret_cast<uint32_t*>(gen(tabA));
  float* mrg = reinterpret_cast<float*>(gen(miscA));             // [warp][8 columns][m, l, o'[D]]
  const uint32_t mrg_bytes = kTmaConsumerWarps * 8 * (D + 2) * 4;
  uint32_t* luts = reinterpret_cast<uint32_t*>(gen(miscA + mrg_bytes));
  const uint32_t luts_a = miscA + mrg_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gen(miscA + mrg_bytes + 512));
  int* nb_count = reinterpret_cast<int*>(bars + 2 * kTmaStages);   // [kTmaStages] tokens with staged norms
  int* nb_off = nb_count + kTmaStages;                                 // [kTmaStages] their offset in the stage
  volatile int* abort_flag = nb_off + kTmaStages;
  volatile int* consumers_stop = abort_flag + 1;   // uniform exit decision of the consumer warps
  const uint32_t bar0 = tma_smem_u32(bars);
  const uint32_t nb_a = tma_smem_u32(nb_count);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kTmaStages + s); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.G;
  const int nhb = PK ? 1 : tma_head_blocks(G);
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
    tab_g[i] = val;
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
          const uint32_t sb = stageA + static_cast<uint32_t>(s) * SL.bytes;
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
  const int pg = (g & 1) ? ((g >> 1) ^ 5) : (g >> 1);
  // value-operand k-indices 2t, 2t+1, 2t+8, 2t+9 are the tokens of score rows 2t, 2t+1, ...
  const int kv[4] = {t, t ^ 5, 8 + t, 8 + (t ^ 5)};
  const uint32_t klo = tabA | static_cast<uint32_t>(lane) * 4u, vlo = klo + 128u;
  // MMA column of this lane's B operand (g) and of its accumulators (2t, 2t + 1)
  const int qcol = PK ? (g & 3) : g;               // head (in the block) of B column g
  const bool qlo = PK && g >= 4;                  // B column g carries a lo part
  const int h0 = PK ? 2 * (t & 1) : 2 * t;         // heads of accumulator columns 2t, 2t + 1
  const bool plo = PK && t >= 2;                  // accumulator columns 2t, 2t + 1 are lo parts
  int gs = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    int bh, hblk, chunk, k0, k1;
    item_range(item, bh, hblk, chunk, k0, k1);
    const int bb = bh / p.Hkv, hk = bh - bb * p.Hkv;
    const int64_t rec0 = static_cast<int64_t>(bh) * p.Nmax;
    const int hb0 = hblk * HB;                        // first head of this block in the group
    const int nh = min(HB, G - hb0);
    const int64_t qbase = static_cast<int64_t>(bb) * p.Hq + hk * G + hb0;
    // query operand (B of the score MMA)
    const bool hok = qcol < nh;
    uint32_t qh[KST][2], ql[PK ? 1 : KST][2];
#pragma unroll
    for (int s = 0; s < KST; ++s) {
      const int dm = t * TDK + 4 * s;
      float a[4] = {0.f, 0.f, 0.f, 0.f};
      if (hok) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p.qa + (qbase + qcol) * D + dm));
        a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
      }
      uint32_t h01, l01, h23, l23;
      split_pair(a[0], a[1], h01, l01);
      split_pair(a[2], a[3], h23, l23);
      if constexpr (PK) {
        qh[s][0] = qlo ? l01 : h01;
        qh[s][1] = qlo ? l23 : h23;
      } else {
        qh[s][0] = h01; qh[s][1] = h23;
        ql[s][0] = l01; ql[s][1] = l23;
      }
    }
    uint32_t qb[KST][2];
    if constexpr (KF == KFMT_PROD) {
#pragma unroll
      for (int s = 0; s < KST; ++s) {
        const int dm = t * TDK + 4 * s;
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        if (hok) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(p.qb + (qbase + qcol) * p.qb_stride + dm));
          a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
        }
        if constexpr (PK) {
          uint32_t h01, l01, h23, l23;
          split_pair(a[0], a[1], h01, l01);
          split_pair(a[2], a[3], h23, l23);
          qb[s][0] = qlo ? l01 : h01;
          qb[s][1] = qlo ? l23 : h23;
        } else {
          qb[s][0] = pack_half2(a[0], a[1]);
          qb[s][1] = pack_half2(a[2], a[3]);
        }
      }
    }
    // this thread's score columns are heads h0, h0 + 1 of the block
    const bool c0ok = h0 < nh, c1ok = h0 + 1 < nh;
    const float sa0 = c0ok ? p.qs[(qbase + h0) * 2] * p.k_scale : 0.f;
    const float sa1 = c1ok ? p.qs[(qbase + h0 + 1) * 2] * p.k_scale : 0.f;
    const float sb0 = c0ok ? p.qs[(qbase + h0) * 2 + 1] * p.qjl_coef : 0.f;
    const float sb1 = c1ok ? p.qs[(qbase + h0 + 1) * 2 + 1] * p.qjl_coef : 0.f;

    float o[MT][4];
#pragma unroll
    for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // heads h0, h0 + 1
    // Software pipeline: the value half of unit i - 1 (its value slices and P operand,
    // kept here) is issued next to the key half of unit i.  A zero P makes the first
    // pass a no-op, so the loop body has no branch around it.
    uint32_t pvs[4][NWV];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int w = 0; w < NWV; ++w) pvs[i][w] = 0u;
    uint32_t pb0h = 0u, pb1h = 0u, pb0l = 0u, pb1l = 0u;
    // O'^T[128 dims x 8 columns] += V_hat^T . P^T for the pending unit
    // M-tile i: row g = dim TDV g + i (first word of the slice), row g + 8 = dim TDV g + 8 + i
    auto value_half = [&]() {
      if constexpr (VB == 4) {
        // byte j of lo (hi) holds the codes of one token pair for dim 2j (2j + 1) of a word
        uint32_t lo[2][2], hi[2][2];   // [token pair][word]
#pragma unroll
        for (int w = 0; w < 2; ++w) {
#pragma unroll
          for (int kp = 0; kp < 2; ++kp) {
            const uint32_t x = pvs[2 * kp][w], y = pvs[2 * kp + 1][w];
            lo[kp][w] = (x & 0x0F0F0F0Fu) | ((y << 4) & 0xF0F0F0F0u);
            hi[kp][w] = ((x >> 4) & 0x0F0F0F0Fu) | (y & 0xF0F0F0F0u);
          }
        }
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          const int k = i >> 1;
          const uint32_t a0 = tab_ld(tab_off((i & 1) ? hi[0][0] : lo[0][0], vlo, k));
          const uint32_t a1 = tab_ld(tab_off((i & 1) ? hi[0][1] : lo[0][1], vlo, k));
          const uint32_t a2 = tab_ld(tab_off((i & 1) ? hi[1][0] : lo[1][0], vlo, k));
          const uint32_t a3 = tab_ld(tab_off((i & 1) ? hi[1][1] : lo[1][1], vlo, k));
          mma16816(o[i], a0, a1, a2, a3, pb0h, pb1h);
          if constexpr (!PK) mma16816(o[i], a0, a1, a2, a3, pb0l, pb1l);
        }
      } else {
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          const uint32_t e00 = field_at<VB, NWV>(pvs[0], i * VB) | (field_at<VB, NWV>(pvs[1], i * VB) << VB);
          const uint32_t e01 = field_at<VB, NWV>(pvs[0], (8 + i) * VB) | (field_at<VB, NWV>(pvs[1], (8 + i) * VB) << VB);
          const uint32_t e10 = field_at<VB, NWV>(pvs[2], i * VB) | (field_at<VB, NWV>(pvs[3], i * VB) << VB);
          const uint32_t e11 = field_at<VB, NWV>(pvs[2], (8 + i) * VB) | (field_at<VB, NWV>(pvs[3], (8 + i) * VB) << VB);
          const uint32_t a0 = tab_ld((e00 << 8) | vlo), a1 = tab_ld((e01 << 8) | vlo);
          const uint32_t a2 = tab_ld((e10 << 8) | vlo), a3 = tab_ld((e11 << 8) | vlo);
          mma16816(o[i], a0, a1, a2, a3, pb0h, pb1h);
          if constexpr (!PK) mma16816(o[i], a0, a1, a2, a3, pb0l, pb1l);
        }
      }
    };

    for (int t0 = k0; t0 < k1; t0 += kTmaStageTokens, ++gs) {
      const int s = gs % kTmaStages;
      if (!tma_mbar_wait(full_bar(s), (gs / kTmaStages) & 1, wait_lim, status, abort_flag)) break;
      const uint32_t sb = stageA + static_cast<uint32_t>(s) * SL.bytes;
      const int cnt = min(kTmaStageTokens, k1 - t0);
      const int nn = static_cast<int>(sld32(nb_a + 4u * s)), noff = static_cast<int>(sld32(nb_a + 4u * (kTmaStages + s)));
      const int u0 = warp * 16;                      // first token of this warp's unit (stage-local)
      // ---- pull this warp's slices out of the stage ----
      const int ka = u0 + pg, kb2 = u0 + 8 + pg;     // tokens of score rows g, g + 8
      bool oka = true, okb = true;
      uint32_t ks0[NWK], ks1[NWK];
      float kn0, kn1, vn0, vn1;
      float gm0 = 0.f, gm1 = 0.f;
      uint32_t sw0 = 0u, sw1 = 0u;
      uint32_t vs[4][NWV];
      if (cnt == kTmaStageTokens && nn >= cnt) {
        // a whole stage with every norm staged (all but the last stage of a chunk): no
        // per-token checks
        sld_slice<NWK>(sb + SL.kcodes + ka * KW * 4, KW, t * TDK * KB, true, ks0);
        sld_slice<NWK>(sb + SL.kcodes + kb2 * KW * 4, KW, t * TDK * KB, true, ks1);
        kn0 = sldf(sb + SL.knorm + 4 * (noff + ka)); kn1 = sldf(sb + SL.knorm + 4 * (noff + kb2));
        vn0 = sldf(sb + SL.vnorm + 4 * (noff + ka)); vn1 = sldf(sb + SL.vnorm + 4 * (noff + kb2));
        if constexpr (KF == KFMT_PROD) {
          gm0 = sldf(sb + SL.krn + 4 * (noff + ka));
          gm1 = sldf(sb + SL.krn + 4 * (noff + kb2));
          sw0 = sld32(sb + SL.ksign + (ka * KSW + t) * 4);
          sw1 = sld32(sb + SL.ksign + (kb2 * KSW + t) * 4);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
          sld_slice<NWV>(sb + SL.vcodes + (u0 + kv[i]) * VW * 4, VW, g * TDV * VB, true, vs[i]);
      } else {
        oka = ka < cnt;
        okb = kb2 < cnt;
        sld_slice<NWK>(sb + SL.kcodes + ka * KW * 4, KW, t * TDK * KB, oka, ks0);
        sld_slice<NWK>(sb + SL.kcodes + kb2 * KW * 4, KW, t * TDK * KB, okb, ks1);
        auto norm_of = [&](uint32_t staged, const float* global, int lk, bool ok) {
          return ok ? (lk < nn ? sldf(staged + 4 * (noff + lk)) : __ldg(global + rec0 + t0 + lk)) : 0.f;
        };
        kn0 = norm_of(sb + SL.knorm, p.knorms, ka, oka); kn1 = norm_of(sb + SL.knorm, p.knorms, kb2, okb);
        vn0 = norm_of(sb + SL.vnorm, p.vnorms, ka, oka); vn1 = norm_of(sb + SL.vnorm, p.vnorms, kb2, okb);
        if constexpr (KF == KFMT_PROD) {
          gm0 = norm_of(sb + SL.krn, p.krnorms, ka, oka);
          gm1 = norm_of(sb + SL.krn, p.krnorms, kb2, okb);
          sw0 = oka ? sld32(sb + SL.ksign + (ka * KSW + t) * 4) : 0u;
          sw1 = okb ? sld32(sb + SL.ksign + (kb2 * KSW + t) * 4) : 0u;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int lk = u0 + kv[i];
          sld_slice<NWV>(sb + SL.vcodes + lk * VW * 4, VW, g * TDV * VB, lk < cnt, vs[i]);
        }
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty_bar(s)) : "memory");
      if (u0 >= cnt) continue;

      // ---- scores: S[16 tokens x 8 columns], two accumulator chains (even / odd k-steps) ----
      float acc[4] = {0.f, 0.f, 0.f, 0.f}, accb[4] = {0.f, 0.f, 0.f, 0.f};
      float accl[4] = {0.f, 0.f, 0.f, 0.f}, acclb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s2 = 0; s2 < KST; ++s2) {
        uint32_t a0, a1, a2, a3;
        if constexpr (KB == 4) {
          // dims (4 s2, 4 s2 + 1) are byte 2 (s2 % 2) of word s2 / 2; (+2, +3) the next byte
          const uint32_t w0 = ks0[s2 >> 1], w1 = ks1[s2 >> 1];
          const int k = 2 * (s2 & 1);
          a0 = tab_ld(tab_off(w0, klo, k));
          a1 = tab_ld(tab_off(w1, klo, k));
          a2 = tab_ld(tab_off(w0, klo, k + 1));
          a3 = tab_ld(tab_off(w1, klo, k + 1));
        } else {
          a0 = tab_ld((pair_at<KB, NWK>(ks0, 4 * s2 * KB) << 8) | klo);
          a1 = tab_ld((pair_at<KB, NWK>(ks1, 4 * s2 * KB) << 8) | klo);
          a2 = tab_ld((pair_at<KB, NWK>(ks0, (4 * s2 + 2) * KB) << 8) | klo);
          a3 = tab_ld((pair_at<KB, NWK>(ks1, (4 * s2 + 2) * KB) << 8) | klo);
        }
        if (s2 & 1) {
          mma16816(accb, a0, a1, a2, a3, qh[s2][0], qh[s2][1]);
          if constexpr (!PK) mma16816(acclb, a0, a1, a2, a3, ql[s2][0], ql[s2][1]);
        } else {
          mma16816(acc, a0, a1, a2, a3, qh[s2][0], qh[s2][1]);
          if constexpr (!PK) mma16816(accl, a0, a1, a2, a3, ql[s2][0], ql[s2][1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] += accb[i] + (accl[i] + acclb[i]);
      float acc2[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (KF == KFMT_PROD) {
#pragma unroll
        for (int s2 = 0; s2 < KST; ++s2) {
          const uint32_t a0 = tab_ld(luts_a + ((((sw0 >> (4 * s2)) & 3u) << 5) + lane) * 4);
          const uint32_t a1 = tab_ld(luts_a + ((((sw1 >> (4 * s2)) & 3u) << 5) + lane) * 4);
          const uint32_t a2 = tab_ld(luts_a + ((((sw0 >> (4 * s2 + 2)) & 3u) << 5) + lane) * 4);
          const uint32_t a3 = tab_ld(luts_a + ((((sw1 >> (4 * s2 + 2)) & 3u) << 5) + lane) * 4);
          mma16816(acc2, a0, a1, a2, a3, qb[s2][0], qb[s2][1]);
        }
      }
      value_half();                                  // unit i - 1 (independent of the scores)
      if constexpr (PK) {
        // columns c and c + 4 hold the hi and lo products of one head: lanes t and t ^ 2
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 2);
          if constexpr (KF == KFMT_PROD) acc2[i] += __shfl_xor_sync(0xffffffffu, acc2[i], 2);
        }
      }
      // acc[0], acc[1]: token row g, heads h0, h0 + 1; acc[2], acc[3]: token row g + 8
      float sc[4];
      {
        const float kr[4] = {kn0, kn0, kn1, kn1};
        const float gr[4] = {gm0, gm0, gm1, gm1};
        const float sa[4] = {sa0, sa1, sa0, sa1}, sbq[4] = {sb0, sb1, sb0, sb1};
        const bool ok[4] = {oka, oka, okb, okb};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float v = sa[i] * acc[i];
          if constexpr (KF == KFMT_PROD) v += gr[i] * sbq[i] * acc2[i];
          sc[i] = ok[i] ? kr[i] * v : -INFINITY;
        }
      }
      // ---- online softmax per head (log2 domain), reduced over the 8 token rows; the
      // reduction runs only when some score of the warp exceeds its running maximum ----
      if (__any_sync(0xffffffffu, sc[0] > m0 || sc[2] > m0 || sc[1] > m1 || sc[3] > m1)) {
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
      }
      const float p00 = c0ok ? ex2(sc[0] - m0) : 0.f, p01 = c1ok ? ex2(sc[1] - m1) : 0.f;
      const float p10 = c0ok ? ex2(sc[2] - m0) : 0.f, p11 = c1ok ? ex2(sc[3] - m1) : 0.f;
      l0 += p00 + p10;
      l1 += p01 + p11;
      // P^T (16 tokens x 8 columns) as the B operand of the next value half: transpose the
      // two 8x8 halves
      uint32_t pth, ptl, pbh, pbl;
      split_pair(p00 * vn0, p01 * vn0, pth, ptl);
      split_pair(p10 * vn1, p11 * vn1, pbh, pbl);
      if constexpr (PK) {
        pb0h = movmatrix_t(plo ? ptl : pth);
        pb1h = movmatrix_t(plo ? pbl : pbh);
      } else {
        pb0h = movmatrix_t(pth); pb1h = movmatrix_t(pbh);
        pb0l = movmatrix_t(ptl); pb1l = movmatrix_t(pbl);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int w = 0; w < NWV; ++w) pvs[i][w] = vs[i][w];
    }
    value_half();                                    // the last unit of the item

    // ---- merge this item across the consumer warps (named barrier 1) ----
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
    }
    float* wm = mrg + warp * 8 * (D + 2);           // [column][m, l, o'[D]]
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
      for (int w = 0; w < kTmaConsumerWarps; ++w) M = fmaxf(M, mrg[(w * 8 + r) * (D + 2)]);
      float a = 0.f, L = 0.f;
#pragma unroll
      for (int w = 0; w < kTmaConsumerWarps; ++w) {
        const float* row = mrg + (w * 8 + r) * (D + 2);
        const float f = (row[0] == -INFINITY) ? 0.f : exp2f(row[0] - M);
        L += f * row[1];
        float ov = row[2 + j];
        if constexpr (PK) ov += row[4 * (D + 2) + 2 + j];      // the lo column of head r
        a += f * ov;
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
