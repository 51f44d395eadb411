// Decode attention with bulk-copy (TMA engine) staging of the packed cache, d = 128.
//
// Computes, for MSE or PROD keys and MSE values, the same step as decode_attn_kernel
// (decode.cuh): logit = scale * est(q, k_i), online softmax, o' = sum p ||v|| c[code_v].
//
// Streaming.  Persistent CTAs (one per SM) walk work items (batch * kv-head, head block,
// context chunk).  One producer warp copies each item in stages of 16 tokens per consumer
// warp and unit with cp.async.bulk (key codes, value codes, norms; prod adds sign words and
// residual norms) into a shared-memory ring (2 or 4 deep, see the work split below); 11
// (prod: 7) consumer warps each take one or two 16-token units of a stage, pull their record
// slices into registers, release the stage and compute.
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
// 1-bit codes (TurboQuant-mse b=1, the MSE stage of b=2 prod, spectral 1-bit tails) take
// a whole byte per lookup instead: one 128-bit load returns 8 decoded values, the A
// registers of two key k-steps (the byte holds 8 consecutive dims of one token), or all
// four A registers of a value M-tile (the byte holds one dim of the 4 tokens of the lane's
// two rows, bit-transposed per unit); those entries keep 8 lane slots of 16 bytes, which a
// 128-bit load of 32 lanes reads in four conflict-free passes.
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

// Work split.  With packed columns (GQA groups of at most 4 heads) every consumer warp takes
// two 16-token units of a stage (11 consumer warps, 2 stages of 352 tokens: more warps to
// interleave measured faster than a deeper ring, 8 warps x 3 stages of 256 tokens); otherwise
// one unit (11 consumer warps for MSE keys, 4 stages).  PROD keys need more registers and run
// 7 consumer warps.  Plus one producer warp.
#ifndef TQ_DEC_PK_NC
#define TQ_DEC_PK_NC 11
#endif
#ifndef TQ_DEC_PK_U
#define TQ_DEC_PK_U 2
#endif
#ifndef TQ_DEC_PK_NS
#define TQ_DEC_PK_NS 2
#endif
// Ring depth for MSE keys and values with packed columns.  Three stages fit (the half-size
// merge buffer and one stage below the 64 KB-aligned table, two after it) but measured no
// faster than two at the 128k-token shapes: the consumers' instruction stream sets the time.
#ifndef TQ_DEC_PK_NS_MSE
#define TQ_DEC_PK_NS_MSE 2
#endif
__host__ __device__ constexpr int tma_units(bool pk) { return pk ? TQ_DEC_PK_U : 1; }
__host__ __device__ constexpr int tma_consumers(int kf, bool pk) { return kf == KFMT_PROD ? 7 : (pk ? TQ_DEC_PK_NC : 11); }
__host__ __device__ constexpr int tma_stage_tokens(int kf, bool pk) { return tma_consumers(kf, pk) * 16 * tma_units(pk); }
__host__ __device__ constexpr int tma_stages(int kf, bool pk, bool vpr) {
  return pk ? ((kf == KFMT_MSE && !vpr) ? TQ_DEC_PK_NS_MSE : TQ_DEC_PK_NS) : 4;
}
static_assert(TQ_DEC_PK_NS >= 2 && TQ_DEC_PK_NS <= 4 && TQ_DEC_PK_NS_MSE >= 2 && TQ_DEC_PK_NS_MSE <= 4,
              "decode ring depth");
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
  if (limit < 0) {                 // test hook: every bounded wait expires at once
    report_status(status, kDevTimeout);
    *abort_flag = 1;
    return false;
  }
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
  uint32_t kcodes, vcodes, knorm, vnorm, ksign, krn, vsign, vrn, bytes;
};

// Byte offsets of the arrays of one stage (all 16-byte aligned).
__host__ __device__ inline TmaStageLayout tma_stage_layout(int kw, int vw, int kf, int ksw, bool pk, bool vpr = false) {
  const int st = tma_stage_tokens(kf, pk);
  TmaStageLayout L{};
  uint32_t o = 0;
  // spectral records (20 bytes) are staged from the 16-byte boundary below the stage's first
  // record: slack for the partial 16-byte blocks at both ends
  const int slack = (kf == KFMT_SPEC) ? 32 : 0;
  L.kcodes = o; o += st * kw * 4 + slack;
  L.vcodes = o; o += st * vw * 4 + slack;
  L.knorm = o; o += (kf == KFMT_SPEC) ? 0 : (st + 4) * 4;
  L.vnorm = o; o += (kf == KFMT_SPEC) ? 0 : (st + 4) * 4;
  L.ksign = o; o += (kf == KFMT_PROD) ? st * ksw * 4 : 0;
  L.krn = o; o += (kf == KFMT_PROD || kf == KFMT_SPEC) ? (st + 4) * 4 : 0;
  L.vsign = o; o += vpr ? st * 4 * 4 : 0;          // values as prod: 4 sign words and gamma
  L.vrn = o; o += vpr ? (st + 4) * 4 : 0;
  L.bytes = o;
  return L;
}

// Shared memory of one CTA.  The lookup table must start at a 64 KB-aligned shared
// address (a byte permute then forms the complete lookup address).  The small arrays
// (merge buffer, sign table, barriers) and as many stages as fit go into the gap below
// the table, the rest after it; the kernel checks the layout against the allocation.
__host__ __device__ inline uint32_t tma_table_bytes(int kb, int vb) {
  // 1-bit codes index the table by whole bytes
  return (kb <= 2 || vb <= 2) ? 65536u : (1u << (2 * (kb > vb ? kb : vb))) * 256u;
}
__host__ __device__ constexpr uint32_t tma_merge_rows(bool pk) { return pk ? 4u : 8u; }
// Floats per merge row: m, l and o'[128] for the spectral and values-as-prod merge; l and
// half of o' for the others, whose merge runs in two halves of the dims.
__host__ __device__ constexpr uint32_t tma_merge_row_floats(int kf, bool vpr) {
  return (kf == KFMT_SPEC || vpr) ? 128u + 2u : 64u + 1u;
}
__host__ __device__ inline uint32_t tma_misc_bytes(int kf, bool pk, bool vpr = false) {
  const uint32_t merge = static_cast<uint32_t>(tma_consumers(kf, pk)) * tma_merge_rows(pk) * tma_merge_row_floats(kf, vpr) * 4u;
  // values as prod: the merged sign-domain sums of up to 8 rows
  const uint32_t v = merge + 4u * 32u * 4u + 2u * 4u * 8u + 2u * 4u * 4u + 16u + 1024u * 4u + 8u + (vpr ? 8u * 128u * 4u : 0u);
  return (v + 127u) & ~127u;
}
// words of one record: the code stream, plus the head word of a spectral record
__host__ __device__ constexpr int tma_record_words(int bits, int kf) { return 128 * bits / 32 + (kf == KFMT_SPEC ? 1 : 0); }
inline size_t decode_tma_smem_bytes(int kb, int vb, int kf, bool pk, bool vpr = false) {
  const TmaStageLayout L = tma_stage_layout(tma_record_words(kb, kf), tma_record_words(vb, kf), kf, 4, pk, vpr);
  const size_t want = 65536 + tma_table_bytes(kb, vb) + static_cast<size_t>(tma_stages(kf, pk, vpr)) * L.bytes +
                      tma_misc_bytes(kf, pk, vpr);
  return want < 232448 ? want : 232448;
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
// Bits [pos, pos + W) of a word slice moved to bit `to`, the rest cleared.  pos and to are
// compile-time after unrolling, so this is one shift (a funnel shift across two words) and
// a mask that folds into the OR forming the table address.
template <int W, int NW>
__device__ __forceinline__ uint32_t field_to(const uint32_t (&seg)[NW], int pos, int to) {
  const int wi = pos >> 5, sh = pos & 31;
  constexpr uint32_t m = (1u << W) - 1u;
  if (sh + W > 32 && wi + 1 < NW) return (__funnelshift_r(seg[wi], seg[wi + 1], sh) << to) & (m << to);
  const uint32_t x = seg[wi];
  return (sh >= to ? (x >> (sh - to)) : (x << (to - sh))) & (m << to);
}

// 64-bit table load (2-bit entries).
__device__ __forceinline__ uint2 tab_ld64(uint32_t addr) {
  uint2 v;
  asm("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
// 128-bit table load (1-bit entries).
__device__ __forceinline__ uint4 tab_ld128(uint32_t addr) {
  uint4 v;
  asm("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

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
// CZ (prefill): query row r only sees tokens below its causal limit q_pos[b * T + r % T] + 1;
// a work item stops at the largest limit of its rows.
// VPR: values quantized as TurboQuant-prod (VB = bits of their MSE stage, m = d = 128 sign
// bits and gamma per value).  The unbiased reconstruction adds sqrt(pi/2)/m gamma S^T (2s-1)
// to c[code] (rotated domain), so the step also accumulates the sign-domain sum
// a = sum_i p_i ||v_i|| gamma_i (2 s_i - 1) with a third MMA per unit (A = the +-1 signs), and
// the merge of an item folds sqrt(pi/2)/m S^T a into its partial o'.
template <int KF, int KB, int VB, bool PK, bool CZ = false, bool VPR = false>
__global__ void __launch_bounds__((tma_consumers(KF, PK) + 1) * 32, 1)
decode_tma_kernel(const DecodeParams p, int* status, long long wait_lim) {
  constexpr int NC = tma_consumers(KF, PK);   // consumer warps
  constexpr int U = tma_units(PK);            // 16-token units per consumer warp per stage
  constexpr int NS = tma_stages(KF, PK, VPR);  // ring stages
  constexpr int kTmaThreads = (NC + 1) * 32;
  constexpr int kTmaStageTokens = tma_stage_tokens(KF, PK);
  constexpr int D = 128;
  constexpr int KST = D / 16;                 // mma k-steps over the key dims
  constexpr int TDK = D / 4;                  // key dims per thread
  constexpr int NWK = (TDK * KB + 31) / 32;
  constexpr int TDV = D / 8;                  // value dims per thread
  constexpr int NWV = (TDV * VB + 31) / 32;
  constexpr int MT = D / 16;                  // P.V M-tiles (16 dims each)
  constexpr int KLUT = 1 << (2 * KB), VLUT = 1 << (2 * VB);
  constexpr bool SP = KF == KFMT_SPEC;                 // spectral keys and values (1-bit tails)
  constexpr int KW = tma_record_words(KB, KF), VW = tma_record_words(VB, KF);   // record words
  constexpr int TOFF = SP ? 32 : 0;                    // bit offset of the code stream in a record
  constexpr int KSW = 4;                                // prod sign words (m = 128)
  constexpr int HB = PK ? 4 : kTmaHeadBlock;            // query heads per work item
  constexpr int RW = static_cast<int>(tma_merge_rows(PK));   // merge rows per warp
  constexpr int CONSUMERS = NC * 32;
  constexpr int NE = (KB <= 2 || VB <= 2) ? 256 : (KLUT > VLUT ? KLUT : VLUT);   // table entries
  constexpr uint32_t TAB = static_cast<uint32_t>(NE) * 256u;
  extern __shared__ __align__(128) unsigned char tsm_[];

  // ---- shared layout: table at a 64 KB-aligned address ----
  // Table entry e is 256 B: the key value pair for lanes 0..31, then the value pair.  With the
  // table base B (a multiple of 64 KB), the lookup address of a code pair byte x for this lane
  // is B | x << 8 | lane * 4 [+ 128]: one byte permute, no add.
  const TmaStageLayout SL = tma_stage_layout(KW, VW, KF, KSW, PK, VPR);
  const uint32_t base = tma_smem_u32(tsm_);
  uint32_t dyn;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
  const uint32_t gap = (0u - base) & 0xFFFFu;
  const uint32_t tabA = base + gap;
  // first fit: misc block, then each stage, into the gap; the rest after the table
  uint32_t gap_used = 0u, after = tabA + TAB;
  auto place = [&](uint32_t bytes) {
    if (gap_used + bytes <= gap) { const uint32_t a0 = base + gap_used; gap_used += bytes; return a0; }
    const uint32_t a0 = after;
    after += bytes;
    return a0;
  };
  const uint32_t miscA = place(tma_misc_bytes(KF, PK, VPR));
  // equal-size stages: the first st_gap of them sit back to back in the gap, the rest back
  // to back after the table
  uint32_t st_first = 0u, st_after = 0u;
  int st_gap = 0;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const uint32_t a = place(SL.bytes);
    if (i == 0) st_first = a;
    if (a < tabA) ++st_gap;
    else if (i == st_gap) st_after = a;
  }
  if (after > base + dyn) {                       // the request did not cover this layout
    if (threadIdx.x == 0) report_status(status, TQ_ERR_UNSUPPORTED);
    return;
  }
  auto stage_addr = [&](int st) {
    return st < st_gap ? st_first + static_cast<uint32_t>(st) * SL.bytes
                       : st_after + static_cast<uint32_t>(st - st_gap) * SL.bytes;
  };
  auto gen = [&](uint32_t a) { return tsm_ + (a - base); };   // generic pointer of a shared address
  uint32_t* tab_g = reinterpret_cast<uint32_t*>(gen(tabA));
  float* mrg = reinterpret_cast<float*>(gen(miscA));             // [warp][RW rows][merge row]
  const uint32_t mrg_bytes = NC * RW * tma_merge_row_floats(KF, VPR) * 4;
  uint32_t* luts = reinterpret_cast<uint32_t*>(gen(miscA + mrg_bytes));
  const uint32_t luts_a = miscA + mrg_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gen(miscA + mrg_bytes + 512));
  int* nb_count = reinterpret_cast<int*>(bars + 2 * NS);   // [NS] tokens with staged norms
  int* nb_off = nb_count + NS;                              // [NS] their offset in the stage
  volatile int* abort_flag = nb_off + NS;
  volatile int* consumers_stop = abort_flag + 1;   // uniform exit decision of the consumer warps
  // spectral unit codebooks [512]: the 510 entries, then zeros (the entry of a dim with no
  // top code); for values the same divided by the value table scale
  float* utab = reinterpret_cast<float*>(const_cast<int*>(consumers_stop) + 2);
  float* utabv = utab + 512;
  float* asum = utabv + 512;                       // values as prod: merged sign-domain sums [8][128]
  const uint32_t bar0 = tma_smem_u32(bars);
  const uint32_t nb_a = tma_smem_u32(nb_count);
  auto full_bar = [&](int st) { return bar0 + 8u * st; };
  auto empty_bar = [&](int st) { return bar0 + 8u * (NS + st); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.G;
  const int nhb = PK ? 1 : tma_head_blocks(G);
  const int n_items = p.B * p.Hkv * nhb * p.n_chunks;
  const int64_t total_recs = static_cast<int64_t>(p.B) * p.Hkv * p.Nmax;
  // causal limit of query row r (prefill)
  auto row_limit = [&](int bb, int64_t r) { return p.q_pos[bb * p.T + static_cast<int>(r % p.T)] + 1; };
  // item -> (bh, head block, chunk, token range)
  auto item_range = [&](int item, int& bh, int& hblk, int& chunk, int& k0, int& k1) {
    chunk = item % p.n_chunks;
    const int rest = item / p.n_chunks;
    hblk = rest % nhb;
    bh = rest / nhb;
    const int bb = bh / p.Hkv;
    int len = static_cast<int>(min(static_cast<int64_t>(p.seq_lens[bb]), p.Nmax));
    if constexpr (CZ) {
      // no token past the block's largest causal limit is visible to any of its rows
      const int hb = PK ? 4 : kTmaHeadBlock;
      const int64_t r0 = static_cast<int64_t>(bb) * p.Hq + (bh - bb * p.Hkv) * G + hblk * hb;
      int mx = 0;
      for (int c = 0; c < min(hb, G - hblk * hb); ++c) mx = max(mx, row_limit(bb, r0 + c));
      len = min(len, mx);
    }
    k0 = chunk * p.chunk_len;
    k1 = min(len, k0 + p.chunk_len);
  };

  if (tid == 0) {
    for (int st = 0; st < NS; ++st) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(full_bar(st)), "r"(1));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty_bar(st)), "r"(NC));
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // entries c / s: one reciprocal per thread, a product per value (the table is up to 64 KB,
  // refilled by every CTA; the product is within an fp32 ulp of the quotient, far below
  // the entries' fp16 rounding)
  const float kinv = 1.f / p.k_scale, vinv = 1.f / p.v_scale;
  for (int i = tid; i < NE * 64; i += kTmaThreads) {
    const int e = i >> 6, j = i & 3;               // j: word of a 16-byte slot (1-bit entries)
    uint32_t val = 0u;
    if ((i & 32) == 0) {
      if constexpr (KB == 1) {
        // byte e = codes of 8 consecutive dims: word j holds dims 2j, 2j + 1
        val = pack_half2(__ldg(p.kc + ((e >> (2 * j)) & 1)) * kinv,
                         __ldg(p.kc + ((e >> (2 * j + 1)) & 1)) * kinv);
      } else if constexpr (KB == 2) {
        // byte e = codes of 4 consecutive dims: word i & 1 holds dims (0, 1) or (2, 3)
        const int w = i & 1;
        val = pack_half2(__ldg(p.kc + ((e >> (4 * w)) & 3)) * kinv,
                         __ldg(p.kc + ((e >> (4 * w + 2)) & 3)) * kinv);
      } else if (e < KLUT) {
        val = pack_half2(__ldg(p.kc + (e & ((1 << KB) - 1))) * kinv, __ldg(p.kc + (e >> KB)) * kinv);
      }
    } else {
      if constexpr (VB == 1) {
        // byte e: bits 0-3 = one dim of the lane's 4 tokens (row g), bits 4-7 = row g + 8;
        // words = A registers a0 (row g, tokens 0, 1), a1 (row g + 8), a2 (row g, tokens 2, 3), a3
        const int b = (j == 0) ? 0 : (j == 1) ? 4 : (j == 2) ? 2 : 6;
        val = pack_half2(__ldg(p.vc + ((e >> b) & 1)) * vinv, __ldg(p.vc + ((e >> (b + 1)) & 1)) * vinv);
      } else if constexpr (VB == 2) {
        // byte e: bits 0-3 = one dim of a token pair (row g), bits 4-7 = row g + 8: words =
        // A registers of the pair in rows g and g + 8
        const int w = i & 1;
        val = pack_half2(__ldg(p.vc + ((e >> (4 * w)) & 3)) * vinv,
                         __ldg(p.vc + ((e >> (4 * w + 2)) & 3)) * vinv);
      } else if (e < VLUT) {
        val = pack_half2(__ldg(p.vc + (e & ((1 << VB) - 1))) * vinv, __ldg(p.vc + (e >> VB)) * vinv);
      }
    }
    tab_g[i] = val;
  }
  if (tid < 128) {
    const int e = tid >> 5;
    luts[tid] = pack_half2((e & 1) ? 1.f : -1.f, (e & 2) ? 1.f : -1.f);
  }
  if constexpr (SP)
    for (int i = tid; i < 512; i += kTmaThreads) {
      const float c = i < 510 ? __ldg(p.unit_c + i) : 0.f;
      utab[i] = c;
      utabv[i] = c / p.v_scale;
    }
  __syncthreads();
  pdl_trigger();   // the chunk combine may launch; it waits for this grid to complete

  if (warp == NC) {
    // ---------------- producer ----------------
    // Bulk copies need 16-byte aligned sources, destinations and sizes.  MSE and PROD records
    // are multiples of 16 bytes; spectral records (20 bytes) are copied word by word by the
    // whole producer warp instead, and only their gamma array goes by bulk copy.
    static_assert(SP || ((KW * 4) % 16 == 0 && (VW * 4) % 16 == 0), "record size");
    if (SP || lane == 0) {
      int gs = 0;                                   // global stage counter of this CTA
      bool stop = false;
      for (int item = blockIdx.x; item < n_items && !stop; item += gridDim.x) {
        int bh, hblk, chunk, k0, k1;
        item_range(item, bh, hblk, chunk, k0, k1);
        const int64_t rec0 = static_cast<int64_t>(bh) * p.Nmax;
        for (int t0 = k0; t0 < k1; t0 += kTmaStageTokens, ++gs) {
          const int st = gs % NS, use = gs / NS;
          bool free_ok = true;
          if (use > 0 && lane == 0) free_ok = tma_mbar_wait(empty_bar(st), (use - 1) & 1, wait_lim, status, abort_flag);
          if constexpr (SP) free_ok = __shfl_sync(0xffffffffu, free_ok, 0);
          if (!free_ok) {
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
          const uint32_t fb = full_bar(st);
          const uint32_t sb = stage_addr(st);
          // spectral: the records' bytes [b0, b1) go from the 16-byte boundary below b0 by bulk
          // copy up to the last 16-byte boundary inside the array; the few words past it
          // (the array's last records) are copied by the warp's lanes
          uint32_t sp_bytes = 0u;
          int64_t ka0 = 0, kbe = 0, va0 = 0, vbe = 0;
          if constexpr (SP) {
            const int64_t kb0 = r * KW * 4, kb1 = (r + cnt) * KW * 4, kend = total_recs * KW * 4;
            const int64_t vb0 = r * VW * 4, vb1 = (r + cnt) * VW * 4, vend = total_recs * VW * 4;
            ka0 = kb0 & ~15ll;
            kbe = min((kb1 + 15) & ~15ll, kend & ~15ll);
            va0 = vb0 & ~15ll;
            vbe = min((vb1 + 15) & ~15ll, vend & ~15ll);
            sp_bytes = static_cast<uint32_t>((kbe - ka0) + (vbe - va0));
            const unsigned char* kg = reinterpret_cast<const unsigned char*>(p.kcodes);
            const unsigned char* vg = reinterpret_cast<const unsigned char*>(p.vcodes);
            for (int64_t b = kbe + 4 * lane; b < kb1; b += 128)
              *reinterpret_cast<uint32_t*>(gen(sb + SL.kcodes + static_cast<uint32_t>(b - ka0))) =
                  __ldg(reinterpret_cast<const uint32_t*>(kg + b));
            for (int64_t b = vbe + 4 * lane; b < vb1; b += 128)
              *reinterpret_cast<uint32_t*>(gen(sb + SL.vcodes + static_cast<uint32_t>(b - va0))) =
                  __ldg(reinterpret_cast<const uint32_t*>(vg + b));
            __syncwarp();
          }
          if (!SP && p.block_table) {
            // paged pool: the stage is cut at page boundaries and each piece copied from its
            // page (pages hold a multiple of 16 tokens and stages start on multiples of 16, so
            // every piece is 16-byte aligned; norms are copied in whole groups of 4, which the
            // page holds)
            if (lane == 0) {
              const int bb = bh / p.Hkv, hk = bh - bb * p.Hkv;
              nb_count[st] = cnt;
              nb_off[st] = 0;
              uint32_t bytes = 0u;
              for (int tt = t0; tt < t0 + cnt;) {
                const int seg = min(t0 + cnt, (tt / p.page + 1) * p.page) - tt, nseg = (seg + 3) & ~3;
                bytes += seg * (KW + VW) * 4 + 2 * nseg * 4;
                if (KF == KFMT_PROD) bytes += seg * KSW * 4 + nseg * 4;
                if (VPR) bytes += seg * 16 + nseg * 4;
                tt += seg;
              }
              asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(fb), "r"(bytes) : "memory");
              for (int tt = t0; tt < t0 + cnt;) {
                const int pi = tt / p.page, seg = min(t0 + cnt, (pi + 1) * p.page) - tt, nseg = (seg + 3) & ~3;
                int pg = p.block_table[static_cast<int64_t>(bb) * p.max_pages + pi];
                if (pg < 0 || pg >= p.num_pages) {            // a bad page id reads page 0
                  report_status(status, TQ_ERR_INVALID_ARG);
                  pg = 0;
                }
                const int64_t rr = (static_cast<int64_t>(pg) * p.Hkv + hk) * p.page + (tt - pi * p.page);
                const uint32_t so = static_cast<uint32_t>(tt - t0);
                bulk_g2s(sb + SL.kcodes + so * KW * 4, p.kcodes + rr * KW, seg * KW * 4, fb);
                bulk_g2s(sb + SL.vcodes + so * VW * 4, p.vcodes + rr * VW, seg * VW * 4, fb);
                bulk_g2s(sb + SL.knorm + so * 4, p.knorms + rr, nseg * 4, fb);
                bulk_g2s(sb + SL.vnorm + so * 4, p.vnorms + rr, nseg * 4, fb);
                if (KF == KFMT_PROD) {
                  bulk_g2s(sb + SL.ksign + so * KSW * 4, p.ksigns + rr * KSW, seg * KSW * 4, fb);
                  bulk_g2s(sb + SL.krn + so * 4, p.krnorms + rr, nseg * 4, fb);
                }
                if (VPR) {
                  bulk_g2s(sb + SL.vsign + so * 16, p.vsigns + rr * 4, seg * 16, fb);
                  bulk_g2s(sb + SL.vrn + so * 4, p.vrnorms + rr, nseg * 4, fb);
                }
                tt += seg;
              }
            }
            continue;
          }
          if (lane == 0) {
            nb_count[st] = max(0, nn - off);
            nb_off[st] = off;
            uint32_t bytes = SP ? sp_bytes : cnt * (KW + VW) * 4 + 2 * nn * 4;
            if (KF == KFMT_PROD) bytes += cnt * KSW * 4 + nn * 4;
            if (VPR) bytes += cnt * 16 + nn * 4;
            if (SP && p.krnorms) bytes += nn * 4;
            // the arrival releases the word copies above (spectral) and expects the bulk bytes
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(fb), "r"(bytes) : "memory");
            if (!SP) {
              bulk_g2s(sb + SL.kcodes, p.kcodes + r * KW, cnt * KW * 4, fb);
              bulk_g2s(sb + SL.vcodes, p.vcodes + r * VW, cnt * VW * 4, fb);
              if (nn > 0) {
                bulk_g2s(sb + SL.knorm, p.knorms + (r - off), nn * 4, fb);
                bulk_g2s(sb + SL.vnorm, p.vnorms + (r - off), nn * 4, fb);
              }
            }
            if (SP) {
              if (kbe > ka0)
                bulk_g2s(sb + SL.kcodes, reinterpret_cast<const unsigned char*>(p.kcodes) + ka0,
                         static_cast<uint32_t>(kbe - ka0), fb);
              if (vbe > va0)
                bulk_g2s(sb + SL.vcodes, reinterpret_cast<const unsigned char*>(p.vcodes) + va0,
                         static_cast<uint32_t>(vbe - va0), fb);
            }
            if (SP && p.krnorms && nn > 0) bulk_g2s(sb + SL.krn, p.krnorms + (r - off), nn * 4, fb);
            if (KF == KFMT_PROD) {
              bulk_g2s(sb + SL.ksign, p.ksigns + r * KSW, cnt * KSW * 4, fb);
              if (nn > 0) bulk_g2s(sb + SL.krn, p.krnorms + (r - off), nn * 4, fb);
            }
            if (VPR) {
              bulk_g2s(sb + SL.vsign, p.vsigns + r * 4, cnt * 16, fb);
              if (nn > 0) bulk_g2s(sb + SL.vrn, p.vrnorms + (r - off), nn * 4, fb);
            }
          }
        }
      }
      // drain: the copies this CTA issued land before it may exit
      if (lane == 0)
        for (int j = max(0, gs - NS); j < gs; ++j)
          for (long long i = 0; !tma_mbar_try(full_bar(j % NS), (j / NS) & 1) && i < (1ll << 28); ++i) {}
    }
    return;
  }

  // ---------------- consumers ----------------
  // score-tile row g holds token pg of the unit, row g + 8 token 8 + pg
  const int pg = (g & 1) ? ((g >> 1) ^ 5) : (g >> 1);
  // value-operand k-indices 2t, 2t+1, 2t+8, 2t+9 are the tokens of score rows 2t, 2t+1, ...
  const int kv[4] = {t, t ^ 5, 8 + t, 8 + (t ^ 5)};
  const uint32_t klo = tabA | static_cast<uint32_t>(lane) * 4u, vlo = klo + 128u;
  // 16-byte slots of the 1-bit entries: 8 per half row
  const uint32_t k1lo = tabA | (static_cast<uint32_t>(lane & 7) << 4), v1lo = k1lo + 128u;
  // 8-byte slots of the 2-bit entries: 16 per half row (a 64-bit load of 32 lanes takes two
  // passes, so 16 slots keep it conflict-free)
  const uint32_t k2lo = tabA | (static_cast<uint32_t>(lane & 15) << 3), v2lo = k2lo + 128u;
  // MMA column of this lane's B operand (g) and of its accumulators (2t, 2t + 1)
  const int qcol = PK ? (g & 3) : g;               // head (in the block) of B column g
  const bool qlo = PK && g >= 4;                  // B column g carries a lo part
  const int h0 = PK ? 2 * (t & 1) : 2 * t;         // heads of accumulator columns 2t, 2t + 1
  const bool plo = PK && t >= 2;                  // accumulator columns 2t, 2t + 1 are lo parts
  // spectral head words: this lane scores top dims 2t, 2t + 1 and QJL signs 2t, 2t + 1 of its
  // key rows, and carries top value dim g (bit position, width, codebook offset; 0 = none)
  // (branch-free: a dim without a top code reads the zero entry with an empty mask, a sign
  // outside the QJL dims is scaled by 0)
  int kh_pos[2] = {0, 0}, kh_nb[2] = {0, 0}, kh_off[2] = {510, 510}, ks_pos[2] = {0, 0};
  uint32_t kh_mask[2] = {0u, 0u};
  float ks_f[2] = {0.f, 0.f};
  int vh_pos = 0, vh_nb = 0, vh_off = 510;
  uint32_t vh_mask = 0u;
  if constexpr (SP) {
    // static indices only (a dynamically indexed array would live in local memory)
    int acc = 0;
#pragma unroll
    for (int j = 0; j < TQ_MAX_TOP; ++j) {
      const int b = j < p.k_top_k ? p.k_top_bits[j] : 0;
      if (j == 2 * t) { kh_pos[0] = acc; kh_nb[0] = b; }
      if (j == 2 * t + 1) { kh_pos[1] = acc; kh_nb[1] = b; }
      acc += b;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      kh_off[i] = kh_nb[i] ? unit_c_off(kh_nb[i]) : 510;
      kh_mask[i] = kh_nb[i] ? (1u << kh_nb[i]) - 1u : 0u;
      ks_pos[i] = acc + 2 * t + i;
      ks_f[i] = (p.k_qjl && 2 * t + i < p.k_top_k) ? 1.f : 0.f;
    }
    acc = 0;
#pragma unroll
    for (int j = 0; j < TQ_MAX_TOP; ++j) {
      const int b = j < p.v_top ? p.v_top_bits[j] : 0;
      if (j == g) { vh_pos = acc; vh_nb = b; }
      acc += b;
    }
    vh_off = vh_nb ? unit_c_off(vh_nb) : 510;
    vh_mask = vh_nb ? (1u << vh_nb) - 1u : 0u;
  }
  // the prepared queries come from the kernel before this one (the producer's copies of the
  // cache do not depend on it and are already under way)
  pdl_wait();
  int gs = 0;
  int ipar = 0;                                   // parity of this CTA's item count (merge buffers)
  for (int item = blockIdx.x; item < n_items; item += gridDim.x, ipar ^= 1) {
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
    for (int k = 0; k < KST; ++k) {
      const int dm = t * TDK + 4 * k;
      float a[4] = {0.f, 0.f, 0.f, 0.f};
      if (hok) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p.qa + (qbase + qcol) * D + dm));
        a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
      }
      uint32_t h01, l01, h23, l23;
      split_pair(a[0], a[1], h01, l01);
      split_pair(a[2], a[3], h23, l23);
      if constexpr (PK) {
        qh[k][0] = qlo ? l01 : h01;
        qh[k][1] = qlo ? l23 : h23;
      } else {
        qh[k][0] = h01; qh[k][1] = h23;
        ql[k][0] = l01; ql[k][1] = l23;
      }
    }
    uint32_t qb[KST][2], qbl[PK ? 1 : KST][2];     // QJL operand (hi; lo without packed columns)
    if constexpr (KF == KFMT_PROD) {
#pragma unroll
      for (int k = 0; k < KST; ++k) {
        const int dm = t * TDK + 4 * k;
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        if (hok) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(p.qb + (qbase + qcol) * p.qb_stride + dm));
          a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
        }
        if constexpr (PK) {
          uint32_t h01, l01, h23, l23;
          split_pair(a[0], a[1], h01, l01);
          split_pair(a[2], a[3], h23, l23);
          qb[k][0] = qlo ? l01 : h01;
          qb[k][1] = qlo ? l23 : h23;
        } else {
          split_pair(a[0], a[1], qb[k][0], qbl[k][0]);
          split_pair(a[2], a[3], qb[k][1], qbl[k][1]);
        }
      }
    }
    // spectral head slots (B of the head MMA): slots 2t, 2t + 1 (top dims) and 2t + 8, 2t + 9
    // (QJL) of column g
    uint32_t qhb[2] = {0u, 0u};
    if constexpr (SP) {
      float a[4] = {0.f, 0.f, 0.f, 0.f};
      if (hok) {
        const float* qr = p.qb + (qbase + qcol) * p.qb_stride;
        a[0] = qr[2 * t]; a[1] = qr[2 * t + 1]; a[2] = qr[2 * t + 8]; a[3] = qr[2 * t + 9];
      }
      uint32_t h01, l01, h23, l23;
      split_pair(a[0], a[1], h01, l01);
      split_pair(a[2], a[3], h23, l23);
      qhb[0] = (PK && qlo) ? l01 : h01;
      qhb[1] = (PK && qlo) ? l23 : h23;
    }
    // this thread's score columns are heads h0, h0 + 1 of the block
    const bool c0ok = h0 < nh, c1ok = h0 + 1 < nh;
    int lim0 = 0x7fffffff, lim1 = 0x7fffffff;      // causal limits of those rows (prefill)
    if constexpr (CZ) {
      if (c0ok) lim0 = row_limit(bb, qbase + h0);
      if (c1ok) lim1 = row_limit(bb, qbase + h0 + 1);
    }
    const float sa0 = c0ok ? p.qs[(qbase + h0) * 2] * p.k_scale : 0.f;
    const float sa1 = c1ok ? p.qs[(qbase + h0 + 1) * 2] * p.k_scale : 0.f;
    const float sb0 = c0ok ? p.qs[(qbase + h0) * 2 + 1] * (SP ? 1.f : p.qjl_coef) : 0.f;
    const float sb1 = c1ok ? p.qs[(qbase + h0 + 1) * 2 + 1] * (SP ? 1.f : p.qjl_coef) : 0.f;

    float o[MT][4];
#pragma unroll
    for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    // values as prod: sign-domain sums, row g = sign index TDV g + i, row g + 8 = TDV g + 8 + i
    float os[VPR ? MT : 1][4];
#pragma unroll
    for (int i = 0; i < (VPR ? MT : 1); ++i) os[i][0] = os[i][1] = os[i][2] = os[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // heads h0, h0 + 1
    float oh[4] = {0.f, 0.f, 0.f, 0.f};   // spectral: top value dim g (columns 2t, 2t + 1)

    for (int t0 = k0; t0 < k1; t0 += kTmaStageTokens, ++gs) {
      const int st = gs % NS;
      if (!tma_mbar_wait(full_bar(st), (gs / NS) & 1, wait_lim, status, abort_flag)) break;
      const uint32_t sb = stage_addr(st);
      const int cnt = min(kTmaStageTokens, k1 - t0);
      const int nn = static_cast<int>(sld32(nb_a + 4u * st)), noff = static_cast<int>(sld32(nb_a + 4u * (NS + st)));
      const int w0 = warp * 16 * U;                  // first token of this warp (stage-local)
      // spectral code arrays start at the 16-byte boundary below the stage's first record
      const uint32_t kcb = sb + SL.kcodes + (SP ? static_cast<uint32_t>(((rec0 + t0) * KW * 4) & 15) : 0u);
      const uint32_t vcb = sb + SL.vcodes + (SP ? static_cast<uint32_t>(((rec0 + t0) * VW * 4) & 15) : 0u);
      // ---- pull this warp's slices out of the stage ----
      bool ok[U][2];
      uint32_t ks[U][2][NWK];
      float kn[U][2], vn[U][2], gm[U][2];
      uint32_t sw[U][2];
      uint32_t vs[U][4][NWV];
      uint32_t hk[U][2], hv[U][4];                   // spectral head words (keys by row, values by k-index)
      // values as prod: this thread's 16 sign bits (signs TDV g ..) of the value-operand tokens,
      // and gamma of the score-row tokens
      uint32_t vsw[VPR ? U : 1][4];
      float vgm[VPR ? U : 1][2];
      if (cnt == kTmaStageTokens && nn >= cnt) {
        // a whole stage with every norm staged (all but the last stage of a chunk): no
        // per-token checks
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int tk = w0 + 16 * u + 8 * h + pg;     // token of score row g + 8 h
            ok[u][h] = true;
            sld_slice<NWK>(kcb + tk * KW * 4, KW, TOFF + t * TDK * KB, true, ks[u][h]);
            kn[u][h] = SP ? 1.f : sldf(sb + SL.knorm + 4 * (noff + tk));
            vn[u][h] = SP ? 1.f : sldf(sb + SL.vnorm + 4 * (noff + tk));
            gm[u][h] = 0.f;
            sw[u][h] = 0u;
            if constexpr (SP) {
              hk[u][h] = sld32(kcb + tk * KW * 4);
              if (p.k_qjl) gm[u][h] = sldf(sb + SL.krn + 4 * (noff + tk));
            }
            if constexpr (KF == KFMT_PROD) {
              gm[u][h] = sldf(sb + SL.krn + 4 * (noff + tk));
              sw[u][h] = sld32(sb + SL.ksign + (tk * KSW + t) * 4);
            }
            if constexpr (VPR) vgm[u][h] = sldf(sb + SL.vrn + 4 * (noff + tk));
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            sld_slice<NWV>(vcb + (w0 + 16 * u + kv[i]) * VW * 4, VW, TOFF + g * TDV * VB, true, vs[u][i]);
            if constexpr (SP) hv[u][i] = sld32(vcb + (w0 + 16 * u + kv[i]) * VW * 4);
            if constexpr (VPR)
              vsw[u][i] = (sld32(sb + SL.vsign + ((w0 + 16 * u + kv[i]) * 4 + (g >> 1)) * 4) >> (16 * (g & 1))) & 0xFFFFu;
          }
        }
      } else {
        auto norm_of = [&](uint32_t staged, const float* global, int lk, bool okk) {
          return okk ? (lk < nn ? sldf(staged + 4 * (noff + lk)) : __ldg(global + rec0 + t0 + lk)) : 0.f;
        };
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int tk = w0 + 16 * u + 8 * h + pg;
            const bool okk = tk < cnt;
            ok[u][h] = okk;
            sld_slice<NWK>(kcb + tk * KW * 4, KW, TOFF + t * TDK * KB, okk, ks[u][h]);
            kn[u][h] = SP ? 1.f : norm_of(sb + SL.knorm, p.knorms, tk, okk);
            vn[u][h] = SP ? 1.f : norm_of(sb + SL.vnorm, p.vnorms, tk, okk);
            gm[u][h] = 0.f;
            sw[u][h] = 0u;
            if constexpr (SP) {
              hk[u][h] = okk ? sld32(kcb + tk * KW * 4) : 0u;
              if (p.k_qjl) gm[u][h] = norm_of(sb + SL.krn, p.krnorms, tk, okk);
            }
            if constexpr (KF == KFMT_PROD) {
              gm[u][h] = norm_of(sb + SL.krn, p.krnorms, tk, okk);
              sw[u][h] = okk ? sld32(sb + SL.ksign + (tk * KSW + t) * 4) : 0u;
            }
            if constexpr (VPR) vgm[u][h] = norm_of(sb + SL.vrn, p.vrnorms, tk, okk);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int lk = w0 + 16 * u + kv[i];
            sld_slice<NWV>(vcb + lk * VW * 4, VW, TOFF + g * TDV * VB, lk < cnt, vs[u][i]);
            if constexpr (SP) hv[u][i] = lk < cnt ? sld32(vcb + lk * VW * 4) : 0u;
            if constexpr (VPR)
              vsw[u][i] = lk < cnt ? (sld32(sb + SL.vsign + (lk * 4 + (g >> 1)) * 4) >> (16 * (g & 1))) & 0xFFFFu : 0u;
          }
        }
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty_bar(st)) : "memory");
      if (w0 >= cnt) continue;

      // ---- scores: per unit S[16 tokens x 8 columns], two accumulator chains ----
      float sc[U][4];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, accb[4] = {0.f, 0.f, 0.f, 0.f};
        float accl[4] = {0.f, 0.f, 0.f, 0.f}, acclb[4] = {0.f, 0.f, 0.f, 0.f};
        // 1-bit keys: byte j of a row's 32-dim slice decodes k-steps 2j and 2j + 1 at once
        uint32_t kq[KB == 1 ? 2 : 1][KB == 1 ? KST : 1][2];
        if constexpr (KB == 1) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < KST / 2; ++j) {
              const uint4 r = tab_ld128(__byte_perm(ks[u][h][0], k1lo, 0x7604u | (static_cast<uint32_t>(j) << 4)));
              kq[h][2 * j][0] = r.x; kq[h][2 * j][1] = r.y;
              kq[h][2 * j + 1][0] = r.z; kq[h][2 * j + 1][1] = r.w;
            }
        }
#pragma unroll
        for (int k = 0; k < KST; ++k) {
          uint32_t a0, a1, a2, a3;
          if constexpr (KB == 1) {
            a0 = kq[0][k][0]; a1 = kq[1][k][0]; a2 = kq[0][k][1]; a3 = kq[1][k][1];
          } else if constexpr (KB == 2) {
            // dims 4k .. 4k + 3 of a row are byte k % 4 of word k / 4: one 64-bit lookup per row
            const uint32_t sel = 0x7604u | (static_cast<uint32_t>(k & 3) << 4);
            const uint2 r0 = tab_ld64(__byte_perm(ks[u][0][k >> 2], k2lo, sel));
            const uint2 r1 = tab_ld64(__byte_perm(ks[u][1][k >> 2], k2lo, sel));
            a0 = r0.x; a2 = r0.y; a1 = r1.x; a3 = r1.y;
          } else if constexpr (KB == 4) {
            // dims (4 k, 4 k + 1) are byte 2 (k % 2) of word k / 2; (+2, +3) the next byte
            const uint32_t w0c = ks[u][0][k >> 1], w1c = ks[u][1][k >> 1];
            const int bsel = 2 * (k & 1);
            a0 = tab_ld(tab_off(w0c, klo, bsel));
            a1 = tab_ld(tab_off(w1c, klo, bsel));
            a2 = tab_ld(tab_off(w0c, klo, bsel + 1));
            a3 = tab_ld(tab_off(w1c, klo, bsel + 1));
          } else {
            // the code pair's 2 KB bits placed straight at the entry index bits 8..
            a0 = tab_ld(field_to<2 * KB, NWK>(ks[u][0], 4 * k * KB, 8) | klo);
            a1 = tab_ld(field_to<2 * KB, NWK>(ks[u][1], 4 * k * KB, 8) | klo);
            a2 = tab_ld(field_to<2 * KB, NWK>(ks[u][0], (4 * k + 2) * KB, 8) | klo);
            a3 = tab_ld(field_to<2 * KB, NWK>(ks[u][1], (4 * k + 2) * KB, 8) | klo);
          }
          if (k & 1) {
            mma16816(accb, a0, a1, a2, a3, qh[k][0], qh[k][1]);
            if constexpr (!PK) mma16816(acclb, a0, a1, a2, a3, ql[k][0], ql[k][1]);
          } else {
            mma16816(acc, a0, a1, a2, a3, qh[k][0], qh[k][1]);
            if constexpr (!PK) mma16816(accl, a0, a1, a2, a3, ql[k][0], ql[k][1]);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += PK ? accb[i] : accb[i] + (accl[i] + acclb[i]);
        float acc2[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (KF == KFMT_PROD) {
#pragma unroll
          for (int k = 0; k < KST; ++k) {
            const uint32_t a0 = tab_ld(luts_a + ((((sw[u][0] >> (4 * k)) & 3u) << 5) + lane) * 4);
            const uint32_t a1 = tab_ld(luts_a + ((((sw[u][1] >> (4 * k)) & 3u) << 5) + lane) * 4);
            const uint32_t a2 = tab_ld(luts_a + ((((sw[u][0] >> (4 * k + 2)) & 3u) << 5) + lane) * 4);
            const uint32_t a3 = tab_ld(luts_a + ((((sw[u][1] >> (4 * k + 2)) & 3u) << 5) + lane) * 4);
            mma16816(acc2, a0, a1, a2, a3, qb[k][0], qb[k][1]);
            if constexpr (!PK) mma16816(acc2, a0, a1, a2, a3, qbl[k][0], qbl[k][1]);
          }
        }
        if constexpr (SP) {
          // head slots of the spectral keys, one extra k-step: slots 2t, 2t+1 hold the top-dim
          // codebook values, slots 2t+8, 2t+9 the QJL signs times gamma (split hi + lo)
          float hvv[2][4];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t w = hk[u][h];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              hvv[h][i] = utab[kh_off[i] + ((w >> kh_pos[i]) & kh_mask[i])];
              hvv[h][2 + i] = (((w >> ks_pos[i]) & 1u) ? gm[u][h] : -gm[u][h]) * ks_f[i];
            }
          }
          uint32_t ah[4], al[4];
          split_pair(hvv[0][0], hvv[0][1], ah[0], al[0]);
          split_pair(hvv[1][0], hvv[1][1], ah[1], al[1]);
          split_pair(hvv[0][2], hvv[0][3], ah[2], al[2]);
          split_pair(hvv[1][2], hvv[1][3], ah[3], al[3]);
          mma16816(acc2, ah[0], ah[1], ah[2], ah[3], qhb[0], qhb[1]);
          mma16816(acc2, al[0], al[1], al[2], al[3], qhb[0], qhb[1]);
        }
        if constexpr (PK) {
          // columns c and c + 4 hold the hi and lo products of one head: lanes t and t ^ 2
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 2);
            if constexpr (KF == KFMT_PROD || SP) acc2[i] += __shfl_xor_sync(0xffffffffu, acc2[i], 2);
          }
        }
        // acc[0], acc[1]: token row g, heads h0, h0 + 1; acc[2], acc[3]: token row g + 8
        // (one packed two-lane FMA per row and step)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float2 v = __fmul2_rn(make_float2(sa0, sa1), make_float2(acc[2 * h], acc[2 * h + 1]));
          if constexpr (KF == KFMT_PROD)
            v = __ffma2_rn(__fmul2_rn(make_float2(gm[u][h], gm[u][h]), make_float2(sb0, sb1)),
                           make_float2(acc2[2 * h], acc2[2 * h + 1]), v);
          if constexpr (SP) v = __ffma2_rn(make_float2(sb0, sb1), make_float2(acc2[2 * h], acc2[2 * h + 1]), v);
          v = __fmul2_rn(make_float2(kn[u][h], kn[u][h]), v);
          if constexpr (CZ) {
            const int tok = t0 + w0 + 16 * u + 8 * h + pg;     // absolute token of score row g + 8 h
            sc[u][2 * h] = (ok[u][h] && tok < lim0) ? v.x : -INFINITY;
            sc[u][2 * h + 1] = (ok[u][h] && tok < lim1) ? v.y : -INFINITY;
          } else {
            sc[u][2 * h] = ok[u][h] ? v.x : -INFINITY;
            sc[u][2 * h + 1] = ok[u][h] ? v.y : -INFINITY;
          }
        }
      }
      // ---- online softmax per head (log2 domain) over the warp's tokens; the row
      // reduction runs only when some score of the warp exceeds its running maximum ----
      bool up = false;
#pragma unroll
      for (int u = 0; u < U; ++u) up = up || sc[u][0] > m0 || sc[u][2] > m0 || sc[u][1] > m1 || sc[u][3] > m1;
      if (__any_sync(0xffffffffu, up)) {
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          mx0 = fmaxf(mx0, fmaxf(sc[u][0], sc[u][2]));
          mx1 = fmaxf(mx1, fmaxf(sc[u][1], sc[u][3]));
        }
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        if (mn0 > m0 || mn1 > m1) {
          // (causal rows: a row still fully masked keeps max -inf and nothing to rescale)
          const float f0 = (CZ && m0 == -INFINITY) ? 0.f : ex2(m0 - mn0);
          const float f1 = (CZ && m1 == -INFINITY) ? 0.f : ex2(m1 - mn1);
          l0 *= f0;
          l1 *= f1;
          const float2 f01 = make_float2(f0, f1);
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            const float2 a = __fmul2_rn(make_float2(o[i][0], o[i][1]), f01);
            const float2 b = __fmul2_rn(make_float2(o[i][2], o[i][3]), f01);
            o[i][0] = a.x; o[i][1] = a.y; o[i][2] = b.x; o[i][3] = b.y;
          }
          if constexpr (SP) { oh[0] *= f0; oh[1] *= f1; }
          if constexpr (VPR) {
#pragma unroll
            for (int i = 0; i < MT; ++i) {
              const float2 a = __fmul2_rn(make_float2(os[i][0], os[i][1]), f01);
              const float2 b = __fmul2_rn(make_float2(os[i][2], os[i][3]), f01);
              os[i][0] = a.x; os[i][1] = a.y; os[i][2] = b.x; os[i][3] = b.y;
            }
          }
          m0 = mn0;
          m1 = mn1;
        }
      }
      // a causal row whose tokens of this warp are all masked keeps max -inf: its
      // probabilities are exp2(-inf - 0) = 0, not exp2(-inf + inf)
      const float ms0 = (CZ && m0 == -INFINITY) ? 0.f : m0, ms1 = (CZ && m1 == -INFINITY) ? 0.f : m1;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float2 nm = make_float2(-ms0, -ms1);
        const float2 d0 = __fadd2_rn(make_float2(sc[u][0], sc[u][1]), nm);
        const float2 d1 = __fadd2_rn(make_float2(sc[u][2], sc[u][3]), nm);
        const float p00 = c0ok ? ex2(d0.x) : 0.f, p01 = c1ok ? ex2(d0.y) : 0.f;
        const float p10 = c0ok ? ex2(d1.x) : 0.f, p11 = c1ok ? ex2(d1.y) : 0.f;
        const float2 l01 = __fadd2_rn(make_float2(l0, l1), __fadd2_rn(make_float2(p00, p01), make_float2(p10, p11)));
        l0 = l01.x;
        l1 = l01.y;
        // P^T (16 tokens x 8 columns) as the B operand: transpose the two 8x8 halves
        uint32_t pth, ptl, pbh, pbl;
        const float2 pv0 = __fmul2_rn(make_float2(p00, p01), make_float2(vn[u][0], vn[u][0]));
        const float2 pv1 = __fmul2_rn(make_float2(p10, p11), make_float2(vn[u][1], vn[u][1]));
        split_pair(pv0.x, pv0.y, pth, ptl);
        split_pair(pv1.x, pv1.y, pbh, pbl);
        uint32_t b0h, b1h, b0l = 0u, b1l = 0u;
        if constexpr (PK) {
          b0h = movmatrix_t(plo ? ptl : pth);
          b1h = movmatrix_t(plo ? pbl : pbh);
        } else {
          b0h = movmatrix_t(pth); b1h = movmatrix_t(pbh);
          b0l = movmatrix_t(ptl); b1l = movmatrix_t(pbl);
        }
        if constexpr (SP) {
          // top value dims: an extra M-tile whose row g is top dim g (rows g + 8 unused), k =
          // the unit's tokens; values in the units of the table entries (c / v_scale)
          float tv4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            tv4[i] = utabv[vh_off + ((hv[u][i] >> vh_pos) & vh_mask)];
          uint32_t vh0, vl0, vh2, vl2;
          split_pair(tv4[0], tv4[1], vh0, vl0);
          split_pair(tv4[2], tv4[3], vh2, vl2);
          float ohx[4] = {oh[0], oh[1], 0.f, 0.f};
          mma16816(ohx, vh0, 0u, vh2, 0u, b0h, b1h);
          mma16816(ohx, vl0, 0u, vl2, 0u, b0h, b1h);
          if constexpr (!PK) {
            mma16816(ohx, vh0, 0u, vh2, 0u, b0l, b1l);
            mma16816(ohx, vl0, 0u, vl2, 0u, b0l, b1l);
          }
          oh[0] = ohx[0];
          oh[1] = ohx[1];
        }
        if constexpr (VPR) {
          // ---- A^T[128 signs x 8 columns] += (2 s - 1)^T . (P gamma)^T ----
          // weights p ||v|| gamma of the score rows, split and transposed like P
          const float2 pw0 = __fmul2_rn(pv0, make_float2(vgm[u][0], vgm[u][0]));
          const float2 pw1 = __fmul2_rn(pv1, make_float2(vgm[u][1], vgm[u][1]));
          uint32_t wth, wtl, wbh, wbl;
          split_pair(pw0.x, pw0.y, wth, wtl);
          split_pair(pw1.x, pw1.y, wbh, wbl);
          uint32_t c0h, c1h, c0l = 0u, c1l = 0u;
          if constexpr (PK) {
            c0h = movmatrix_t(plo ? wtl : wth);
            c1h = movmatrix_t(plo ? wbl : wbh);
          } else {
            c0h = movmatrix_t(wth); c1h = movmatrix_t(wbh);
            c0l = movmatrix_t(wtl); c1l = movmatrix_t(wbl);
          }
          // bit j of token kv[0] (kv[2]) at bit 2 j, of kv[1] (kv[3]) at bit 2 j + 1: the A entry
          // pair of rows (sign i, tokens k, k + 1) is a 2-bit index into the +-1 pair table
          auto spread = [](uint32_t v) {
            v = (v | (v << 8)) & 0x00FF00FFu;
            v = (v | (v << 4)) & 0x0F0F0F0Fu;
            v = (v | (v << 2)) & 0x33333333u;
            return (v | (v << 1)) & 0x55555555u;
          };
          const uint32_t z01 = spread(vsw[u][0]) | (spread(vsw[u][1]) << 1);
          const uint32_t z23 = spread(vsw[u][2]) | (spread(vsw[u][3]) << 1);
          const uint32_t lane4 = luts_a + static_cast<uint32_t>(lane) * 4u;
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            const uint32_t a0 = tab_ld(lane4 + ((z01 >> (2 * i)) & 3u) * 128u);
            const uint32_t a1 = tab_ld(lane4 + ((z01 >> (16 + 2 * i)) & 3u) * 128u);
            const uint32_t a2 = tab_ld(lane4 + ((z23 >> (2 * i)) & 3u) * 128u);
            const uint32_t a3 = tab_ld(lane4 + ((z23 >> (16 + 2 * i)) & 3u) * 128u);
            mma16816(os[i], a0, a1, a2, a3, c0h, c1h);
            if constexpr (!PK) mma16816(os[i], a0, a1, a2, a3, c0l, c1l);
          }
        }
        // ---- O'^T[128 dims x 8 columns] += V_hat^T . P^T ----
        // M-tile i: row g = dim TDV g + i (first word of the slice), row g + 8 = dim TDV g + 8 + i
        if constexpr (VB == 4) {
          // byte j of lo (hi) holds the codes of one token pair for dim 2j (2j + 1) of a word
          uint32_t lo[2][2], hi[2][2];   // [token pair][word]
#pragma unroll
          for (int w = 0; w < 2; ++w) {
#pragma unroll
            for (int kp = 0; kp < 2; ++kp) {
              const uint32_t x = vs[u][2 * kp][w], y = vs[u][2 * kp + 1][w];
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
            mma16816(o[i], a0, a1, a2, a3, b0h, b1h);
            if constexpr (!PK) mma16816(o[i], a0, a1, a2, a3, b0l, b1l);
          }
        } else if constexpr (VB == 2) {
          // interleave the 2-bit codes of a token pair: byte i of z (zl: i < 4, zh: i >= 4)
          // holds dim i of both tokens (bits 0-3) and dim 8 + i (bits 4-7), one 64-bit
          // lookup per pair and M-tile
          auto spread = [](uint32_t x) {           // 2-bit fields j = 0..3 of a byte -> bits 8j
            x = (x | (x << 12)) & 0x000F000Fu;
            return (x | (x << 6)) & 0x03030303u;
          };
          uint32_t zl[2], zh[2];
#pragma unroll
          for (int pr = 0; pr < 2; ++pr) {
            const uint32_t a = vs[u][2 * pr][0], b = vs[u][2 * pr + 1][0];
            zl[pr] = spread(a & 0xFFu) | (spread(b & 0xFFu) << 2) | (spread((a >> 16) & 0xFFu) << 4) |
                     (spread((b >> 16) & 0xFFu) << 6);
            zh[pr] = spread((a >> 8) & 0xFFu) | (spread((b >> 8) & 0xFFu) << 2) | (spread(a >> 24) << 4) |
                     (spread(b >> 24) << 6);
          }
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            const uint32_t sel = 0x7604u | (static_cast<uint32_t>(i & 3) << 4);
            const uint2 r0 = tab_ld64(__byte_perm(i < 4 ? zl[0] : zh[0], v2lo, sel));
            const uint2 r1 = tab_ld64(__byte_perm(i < 4 ? zl[1] : zh[1], v2lo, sel));
            mma16816(o[i], r0.x, r0.y, r1.x, r1.y, b0h, b1h);
            if constexpr (!PK) mma16816(o[i], r0.x, r0.y, r1.x, r1.y, b0l, b1l);
          }
        } else if constexpr (VB == 1) {
          // bit-transpose the 4 tokens' 16-dim slices: byte i of zl (i < 4) / zh holds dim i
          // (bits 0-3, one per token) and dim 8 + i (bits 4-7) of the M-tile's two rows
          auto spread4 = [](uint32_t x) { return (x * 0x00204081u) & 0x01010101u; };   // bit k -> 8k
          uint32_t zl = 0u, zh = 0u;
#pragma unroll
          for (int tau = 0; tau < 4; ++tau) {
            const uint32_t sv = vs[u][tau][0];
            zl |= (spread4(sv & 15u) << tau) | (spread4((sv >> 8) & 15u) << (4 + tau));
            zh |= (spread4((sv >> 4) & 15u) << tau) | (spread4((sv >> 12) & 15u) << (4 + tau));
          }
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            const uint4 r = tab_ld128(__byte_perm(i < 4 ? zl : zh, v1lo, 0x7604u | (static_cast<uint32_t>(i & 3) << 4)));
            mma16816(o[i], r.x, r.y, r.z, r.w, b0h, b1h);
            if constexpr (!PK) mma16816(o[i], r.x, r.y, r.z, r.w, b0l, b1l);
          }
        } else {
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            // entry index (code of the first token | code of the second << VB) at bits 8..
            auto vaddr = [&](const uint32_t (&x)[NWV], const uint32_t (&y)[NWV], int pos) {
              return field_to<VB, NWV>(x, pos, 8) | field_to<VB, NWV>(y, pos, 8 + VB) | vlo;
            };
            const uint32_t a0 = tab_ld(vaddr(vs[u][0], vs[u][1], i * VB));
            const uint32_t a1 = tab_ld(vaddr(vs[u][0], vs[u][1], (8 + i) * VB));
            const uint32_t a2 = tab_ld(vaddr(vs[u][2], vs[u][3], i * VB));
            const uint32_t a3 = tab_ld(vaddr(vs[u][2], vs[u][3], (8 + i) * VB));
            mma16816(o[i], a0, a1, a2, a3, b0h, b1h);
            if constexpr (!PK) mma16816(o[i], a0, a1, a2, a3, b0l, b1l);
          }
        }
      }
    }

    // ---- merge this item across the consumer warps (named barrier 1) ----
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
    }
    if constexpr (PK) {
      // fold the lo columns (lanes t ^ 2) into the hi columns: lanes t < 2 keep heads 2t, 2t+1
#pragma unroll
      for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[i][j] += __shfl_xor_sync(0xffffffffu, o[i][j], 2);
    }
    if constexpr (!SP && !VPR) {
      // Each warp publishes its row maxima m_w, then scales its own partial (l, o') by
      // 2^(m_w - M) in registers (M = the row maximum over the warps), so the item's partial
      // is a plain sum over the warps in a fixed order.  The maxima go to a buffer per item
      // parity: a warp may publish the next item's while a slower one still reads these.
      static_assert(2 * NC * RW <= 1024, "merge maxima fit the spectral codebook area");
      float* mb = utab + ipar * (NC * RW);          // [warp][RW rows]
      const bool wr = !PK || t < 2;                 // lanes holding rows 2t, 2t + 1
      if (wr && g == 0) {
        mb[warp * RW + 2 * t] = m0;
        mb[warp * RW + 2 * t + 1] = m1;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
      // one exit decision for every consumer warp, sampled between the two barriers (a warp
      // that timed out still reaches both) and read after the second
      if (tid == 0) *consumers_stop = *abort_flag;
      // the partials go through the buffer in two halves of the dims: half hf holds dims
      // TDV g + 8 hf + i (i < 8) of every lane group g at local index 8 g + i, after l
      constexpr int HW = D / 2 + 1;
      float* wm = mrg + warp * RW * HW;              // [row][l, o' half]
      float2 f = make_float2(0.f, 0.f);
      if (wr) {
        float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
        for (int w = 0; w < NC; ++w) {
          M0 = fmaxf(M0, mb[w * RW + 2 * t]);
          M1 = fmaxf(M1, mb[w * RW + 2 * t + 1]);
        }
        // a row this warp never saw (causal masking) keeps max -inf and weight 0
        f = make_float2(m0 == -INFINITY ? 0.f : ex2(m0 - M0), m1 == -INFINITY ? 0.f : ex2(m1 - M1));
        if (g == 0) {
          wm[(2 * t) * HW] = l0 * f.x;
          wm[(2 * t + 1) * HW] = l1 * f.y;
        }
      }
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        if (hf) asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");   // first half read
        if (wr) {
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            const float2 x = __fmul2_rn(make_float2(o[i][2 * hf], o[i][2 * hf + 1]), f);
            wm[(2 * t) * HW + 1 + 8 * g + i] = x.x;
            wm[(2 * t + 1) * HW + 1 + 8 * g + i] = x.y;
          }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
        for (int idx = tid; idx < nh * (D / 2); idx += CONSUMERS) {
          const int r = idx / (D / 2), jl = idx - r * (D / 2);
          const int j = TDV * (jl >> 3) + 8 * hf + (jl & 7);
          float s0 = 0.f, s1 = 0.f;                  // two chains over the warps
#pragma unroll
          for (int w = 0; w < NC; w += 2) {
            s0 += mrg[(w * RW + r) * HW + 1 + jl];
            if (w + 1 < NC) s1 += mrg[((w + 1) * RW + r) * HW + 1 + jl];
          }
          const int64_t pi = (qbase + r) * p.n_chunks + chunk;
          if (hf == 0 && jl == 0) {
            float M = -INFINITY, L = 0.f;
#pragma unroll
            for (int w = 0; w < NC; ++w) {
              M = fmaxf(M, mb[w * RW + r]);
              L += mrg[(w * RW + r) * HW];
            }
            p.part_ml[pi * 2] = M;
            p.part_ml[pi * 2 + 1] = L;
          }
          p.part_o[pi * D + j] = (s0 + s1) * p.v_scale;
        }
      }
      // the next writes of mrg come after the next item's first barrier, which every thread
      // reaches only after this loop
      if (*consumers_stop) break;
    } else {
      float* wm = mrg + warp * RW * (D + 2);           // [row][m, l, o'[D]]
      if (!PK || t < 2) {
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
      }
      if constexpr (SP) {
        // the top value dims come from the head M-tile, not from the (zero) tail codes
        if constexpr (PK) {
          oh[0] += __shfl_xor_sync(0xffffffffu, oh[0], 2);
          oh[1] += __shfl_xor_sync(0xffffffffu, oh[1], 2);
        }
        __syncwarp();
        if ((!PK || t < 2) && vh_nb) {
          wm[(2 * t) * (D + 2) + 2 + g] = oh[0];
          wm[(2 * t + 1) * (D + 2) + 2 + g] = oh[1];
        }
      }
      asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
      for (int idx = tid; idx < nh * D; idx += CONSUMERS) {
        const int r = idx / D, j = idx - r * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NC; ++w) M = fmaxf(M, mrg[(w * RW + r) * (D + 2)]);
        float a = 0.f, L = 0.f;
#pragma unroll
        for (int w = 0; w < NC; ++w) {
          const float* row = mrg + (w * RW + r) * (D + 2);
          const float f = (row[0] == -INFINITY) ? 0.f : exp2f(row[0] - M);
          L += f * row[1];
          a += f * row[2 + j];
        }
        const int64_t qi = qbase + r;
        const int64_t pi = qi * p.n_chunks + chunk;
        if (j == 0) { p.part_ml[pi * 2] = M; p.part_ml[pi * 2 + 1] = L; }
        p.part_o[pi * D + j] = a * p.v_scale;
      }
      if constexpr (VPR) {
        // fold sqrt(pi/2)/m S^T a into the partial: merge the warps' sign-domain sums with the
        // same chunk weights, then one matrix-vector product per row with S from global memory
        if constexpr (PK) {
#pragma unroll
          for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) os[i][j] += __shfl_xor_sync(0xffffffffu, os[i][j], 2);
        }
        asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");   // every warp has read mrg
        if (!PK || t < 2) {
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            wm[(2 * t) * (D + 2) + 2 + TDV * g + i] = os[i][0];
            wm[(2 * t + 1) * (D + 2) + 2 + TDV * g + i] = os[i][1];
            wm[(2 * t) * (D + 2) + 2 + TDV * g + 8 + i] = os[i][2];
            wm[(2 * t + 1) * (D + 2) + 2 + TDV * g + 8 + i] = os[i][3];
          }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
        for (int idx = tid; idx < nh * D; idx += CONSUMERS) {
          const int r = idx / D, j = idx - r * D;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < NC; ++w) M = fmaxf(M, mrg[(w * RW + r) * (D + 2)]);
          float a = 0.f;
#pragma unroll
          for (int w = 0; w < NC; ++w) {
            const float* row = mrg + (w * RW + r) * (D + 2);
            const float f = (row[0] == -INFINITY) ? 0.f : exp2f(row[0] - M);
            a += f * row[2 + j];
          }
          asum[r * D + j] = a;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
        for (int idx = tid; idx < nh * D; idx += CONSUMERS) {
          const int r = idx / D, j = idx - r * D;
          float c = 0.f;
#pragma unroll 8
          for (int i = 0; i < D; ++i) c = fmaf(__ldg(p.vS + i * D + j), asum[r * D + i], c);
          const int64_t pi = (qbase + r) * p.n_chunks + chunk;
          p.part_o[pi * D + j] += p.v_coef * c;
        }
      }
      // every consumer warp takes the same exit decision: one thread samples the abort
      // flag between the two barriers (a warp that timed out still reaches both)
      if (tid == 0) *consumers_stop = *abort_flag;
      asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
      if (*consumers_stop) break;
    }
  }
}

}  // namespace tq
