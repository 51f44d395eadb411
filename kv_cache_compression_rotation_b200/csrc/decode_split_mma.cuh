// Decode attention over an outlier-channel split cache on the tensor cores (d = 128).
//
// TurboQuant review, Method: for the KV experiments the channels split into an outlier
// group and the rest, each quantized by its own TurboQuant instance (2.5 bits: 32 channels
// at 3 bits and 96 at 2 bits).  A key's estimate is the sum of its groups' estimates and a
// value's reconstruction the concatenation of its groups' reconstructions:
//
//   logit_i = scale * sum_g ||k_i,g|| <Pi_g q[cols_g], c_g[code_i,g]>
//   o'_g    = sum_i p_i ||v_i,g|| c_g[code_i,g]          (rotated domain, per value group)
//
// This kernel is the packed-table decode of decode_tma_kernel rearranged so that every
// tensor-core step touches a single group: the concatenated rotated coordinates (group 0
// first, D0 of them, then group 1) are cut into 16-wide k-steps (scores) and M-tiles
// (values) that never straddle the boundary.  Each group then has its own accumulator
// (scores: summed with the group's norm; values: the P operand carries the group's norm),
// its own lookup table and its own bit width, and every lane runs the same instructions.
//
//   scores  lane (g, t) holds, per k-step, the 4 consecutive codes of dims 16k + 4t .. + 3
//           of its two token rows (an 8-bit field at 2 bits, 12 bits at 3);
//   values  lane g holds 2 dims of each M-tile of a group, all from the run of D_g / 8
//           consecutive dims g * D_g / 8 .. of that group, for its 4 tokens; the codes of
//           two tokens are interleaved so that one table index serves a token pair.
//
// Tables (entries c / s with the group's searched scale s):
//   2 bits  one byte = 4 codes -> two half2 (8 bytes): 256 entries of 256 bytes, 16 lane
//           slots for keys then 16 for values (a 64-bit load of 32 lanes takes two passes,
//           so 16 slots keep it conflict-free); one byte permute forms the address
//   3 bits  one 6-bit pair -> half2: 64 entries of 256 bytes (32 lane slots each side)
//
// Streaming is that of decode_tma_kernel: persistent CTAs over (batch * kv-head, context
// chunk) items, a producer warp copying stages of 32 tokens per consumer warp (the four
// record arrays and four norm arrays) into a ring with bulk copies, consumer warps of two
// 16-token units each, mma.sync m16n8k16 with packed hi / lo query columns (GQA groups of at most 4 heads),
// an online softmax in the log2 domain, and a cross-warp merge per item into chunk partials
// that split_combine_kernel merges (with each value group's Pi_g^T and channel scatter).
// Every wait is bounded (TQ_ERR_TIMEOUT); a CTA that times out drains its copies.
#pragma once

#include "decode_tma.cuh"

namespace tq {

// 11 consumer warps and the producer: 3 warps per scheduler (measured faster than 8 or 10
// consumer warps with a 3-deep ring)
#ifndef TQ_SPLIT_NC
#define TQ_SPLIT_NC 11
#endif
#ifndef TQ_SPLIT_NS
#define TQ_SPLIT_NS 2
#endif
constexpr int kSmNC = TQ_SPLIT_NC;                // consumer warps
constexpr int kSmU = 2;                           // 16-token units per consumer warp and stage
constexpr int kSmNS = TQ_SPLIT_NS;                // ring stages
static_assert(kSmNS >= 2 && kSmNS <= 4, "split decode ring depth");
constexpr int kSmStage = kSmNC * 16 * kSmU;       // tokens per stage
constexpr int kSmThreads = (kSmNC + 1) * 32;
constexpr int kSmRows = 4;                        // query heads per item (packed columns)

struct SplitMmaParams {
  int B, Hq, Hkv, G;                              // G = Hq / Hkv <= 4
  int64_t Nmax;                                   // multiple of 4
  int chunk_len, n_chunks;                        // chunk_len: multiple of the stage
  const int32_t* seq_lens;
  const uint32_t* kc[2];                          // key records per group [B*Hkv*Nmax][words]
  const float* kn[2];
  const uint32_t* vc[2];
  const float* vn[2];
  const float* kcent[2];                          // codebooks (2^bits entries)
  const float* vcent[2];
  float kscale[2], vscale[2];                     // table scales
  const float* qr[2];                             // [B*Hq][D_g] rotated key-group queries
  float logit_scale;                              // scale * log2(e)
  float* part_ml;                                 // [B*Hq][n_chunks][2]
  float* part_o;                                  // [B*Hq][n_chunks][128]
};

__host__ __device__ constexpr int sm_words(int dg, int b) { return dg * b / 32; }
__host__ __device__ constexpr uint32_t sm_table_bytes(int b) { return b == 2 ? 65536u : 16384u; }
__host__ __device__ constexpr uint32_t sm_stage_bytes(int d0, int b0, int b1) {
  return static_cast<uint32_t>(kSmStage) * (2u * 4u * (sm_words(d0, b0) + sm_words(128 - d0, b1)) + 16u);
}
__host__ __device__ constexpr uint32_t sm_misc_bytes() {
  return (kSmNC * kSmRows * (128u + 2u) * 4u + 2u * kSmNS * 8u + 64u + 2u * kSmNC * kSmRows * 4u + 127u) & ~127u;
}
inline size_t decode_split_mma_smem(int d0, int b0, int b1) {
  const size_t want = 65536 + sm_table_bytes(b0) + sm_table_bytes(b1) + static_cast<size_t>(kSmNS) *
                      sm_stage_bytes(d0, b0, b1) + sm_misc_bytes();
  return want < 232448 ? want : 232448;
}

// 64-bit shared load (two half2 table halves).
__device__ __forceinline__ void lds64(uint32_t a, uint32_t& x, uint32_t& y) {
  asm("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(x), "=r"(y) : "r"(a));
}

// Where the lane's 12-bit key field of 3-bit k-step kl starts (bit 48 kl + 12 t): word jb =
// 48 kl / 32 or the one after it (up), at bit s of that word.  When it starts in word jb + 1
// it ends there too (s + 12 <= 32), so the field is always the funnel of (jb or jb + 1, jb + 1).
struct Field3 {
  bool up;
  uint32_t s;
};
__device__ __forceinline__ Field3 field3(int kl, int t) {
  const int pos = 48 * kl + 12 * t, jb = (48 * kl) >> 5;
  return Field3{(pos >> 5) > jb, static_cast<uint32_t>(pos & 31)};
}

// Key operand of one k-step for one token row: the lane's 4-code field of local k-step kl
// (dims 16 kl + 4t .. + 3 of its group) -> (dims 0,1) and (dims 2,3) as half2.
template <int B, int W>
__device__ __forceinline__ void key_pairs(const uint32_t (&w)[W], int kl, uint32_t sel, uint32_t tlo, Field3 f,
                                          uint32_t& lo, uint32_t& hi) {
  if constexpr (B == 2) {
    // byte t of word kl holds the 4 codes: one 64-bit lookup
    lds64(__byte_perm(w[kl], tlo, sel), lo, hi);
  } else {
    static_assert(B == 3, "key field width");
    const int jb = (48 * kl) >> 5;
    const uint32_t x = __funnelshift_r(f.up ? w[jb + 1] : w[jb], w[jb + 1], f.s);
    // the two 6-bit pair indices placed at the entry bits 8..13
    lo = tab_ld(tlo | ((x << 8) & 0x3F00u));
    hi = tab_ld(tlo | ((x << 2) & 0x3F00u));
  }
}

template <int D0, int B0, int B1>
__global__ void __launch_bounds__(kSmThreads, 1)
decode_split_mma_kernel(const SplitMmaParams p, int* status, long long wait_lim) {
  constexpr int D1 = 128 - D0;
  constexpr int W0 = sm_words(D0, B0), W1 = sm_words(D1, B1);
  constexpr int KS0 = D0 / 16, KS1 = D1 / 16;     // k-steps (scores) = M-tiles (values) per group
  constexpr int L0 = D0 / 8, L1 = D1 / 8;         // value dims per lane and group
  constexpr int NS = kSmNS, NC = kSmNC, U = kSmU, D = 128;
  constexpr int CONSUMERS = NC * 32;
  static_assert(D0 % 16 == 0 && D0 > 0 && D0 < 128, "group widths");
  static_assert(B0 == 3 && B1 == 2, "instantiated for the 3-bit outlier / 2-bit rest split");
  static_assert(W0 * 32 == D0 * B0 && W1 * 32 == D1 * B1, "whole words per group record");
  static_assert(L0 * B0 + 11 <= 32 && L1 * B1 <= 32, "value fields fit a word (group 0 shifted by up to 11)");
  static_assert(L1 % 4 == 0, "2-bit value runs of whole bytes");
  extern __shared__ __align__(128) unsigned char ssm_[];

  // ---- shared layout: the 2-bit table at a 64 KB boundary, the 3-bit one after it ----
  const uint32_t SB = sm_stage_bytes(D0, B0, B1);
  const uint32_t base = tma_smem_u32(ssm_);
  uint32_t dyn;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
  const uint32_t gap = (0u - base) & 0xFFFFu;
  const uint32_t t2A = base + gap;                // 2-bit table (64 KB)
  const uint32_t t3A = t2A + 65536u;              // 3-bit table (16 KB)
  uint32_t gap_used = 0u, after = t3A + 16384u;
  auto place = [&](uint32_t bytes) {
    if (gap_used + bytes <= gap) { const uint32_t a0 = base + gap_used; gap_used += bytes; return a0; }
    const uint32_t a0 = after;
    after += bytes;
    return a0;
  };
  const uint32_t miscA = place(sm_misc_bytes());
  uint32_t st_first = 0u, st_after = 0u;
  int st_gap = 0;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const uint32_t a = place(SB);
    if (i == 0) st_first = a;
    if (a < t2A) ++st_gap;
    else if (i == st_gap) st_after = a;
  }
  if (after > base + dyn) {
    if (threadIdx.x == 0) report_status(status, TQ_ERR_UNSUPPORTED);
    return;
  }
  auto stage_addr = [&](int st) {
    return st < st_gap ? st_first + static_cast<uint32_t>(st) * SB : st_after + static_cast<uint32_t>(st - st_gap) * SB;
  };
  auto gen = [&](uint32_t a) { return ssm_ + (a - base); };
  // stage arrays (byte offsets)
  constexpr uint32_t oK0 = 0, oK1 = oK0 + kSmStage * W0 * 4, oV0 = oK1 + kSmStage * W1 * 4,
                     oV1 = oV0 + kSmStage * W0 * 4, oKN0 = oV1 + kSmStage * W1 * 4, oKN1 = oKN0 + kSmStage * 4,
                     oVN0 = oKN1 + kSmStage * 4, oVN1 = oVN0 + kSmStage * 4;
  float* mrg = reinterpret_cast<float*>(gen(miscA));             // [warp][4 rows][m, l, o'[128]]
  uint64_t* bars = reinterpret_cast<uint64_t*>(gen(miscA + NC * kSmRows * (D + 2) * 4));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * NS);
  volatile int* consumers_stop = abort_flag + 1;
  int* cnt_st = const_cast<int*>(consumers_stop) + 1;             // [NS] tokens of each stage
  float* mxb = reinterpret_cast<float*>(gen(miscA + NC * kSmRows * (D + 2) * 4 + 2 * NS * 8 + 64));   // [2][warp][4] maxima
  const uint32_t bar0 = tma_smem_u32(bars);
  auto full_bar = [&](int st) { return bar0 + 8u * st; };
  auto empty_bar = [&](int st) { return bar0 + 8u * (NS + st); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.G;
  const int n_items = p.B * p.Hkv * p.n_chunks;

  if (tid == 0) {
    for (int st = 0; st < NS; ++st) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(full_bar(st)), "r"(1));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty_bar(st)), "r"(NC));
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // tables: the 2-bit one of group 1 (16 slots of 8 bytes each side), the 3-bit one of group 0
  {
    uint32_t* t2 = reinterpret_cast<uint32_t*>(gen(t2A));
    const float ik = 1.f / p.kscale[1], iv = 1.f / p.vscale[1];
    for (int i = tid; i < 256 * 64; i += kSmThreads) {
      const int e = i >> 6, w = i & 63;          // 64 words per entry: K slots 0..31, V slots 32..63
      const bool val = w >= 32;
      const float* c = val ? p.vcent[1] : p.kcent[1];
      const float s = val ? iv : ik;
      const int half = w & 1;                    // word 0: codes 0, 1; word 1: codes 2, 3
      const int c0 = (e >> (4 * half)) & 3, c1 = (e >> (4 * half + 2)) & 3;
      t2[i] = pack_half2(__ldg(c + c0) * s, __ldg(c + c1) * s);
    }
    uint32_t* t3 = reinterpret_cast<uint32_t*>(gen(t3A));
    const float jk = 1.f / p.kscale[0], jv = 1.f / p.vscale[0];
    for (int i = tid; i < 64 * 64; i += kSmThreads) {
      const int e = i >> 6, w = i & 63;
      const bool val = w >= 32;
      const float* c = val ? p.vcent[0] : p.kcent[0];
      const float s = val ? jv : jk;
      t3[i] = pack_half2(__ldg(c + (e & 7)) * s, __ldg(c + (e >> 3)) * s);
    }
  }
  __syncthreads();
  pdl_trigger();

  auto item_range = [&](int item, int& bh, int& chunk, int& k0, int& k1) {
    chunk = item % p.n_chunks;
    bh = item / p.n_chunks;
    const int bb = bh / p.Hkv;
    const int len = static_cast<int>(min(static_cast<int64_t>(p.seq_lens[bb]), p.Nmax));
    k0 = chunk * p.chunk_len;
    k1 = min(len, k0 + p.chunk_len);
  };

  if (warp == NC) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int gs = 0;
      bool stop = false;
      for (int item = blockIdx.x; item < n_items && !stop; item += gridDim.x) {
        int bh, chunk, k0, k1;
        item_range(item, bh, chunk, k0, k1);
        const int64_t rec0 = static_cast<int64_t>(bh) * p.Nmax;
        for (int t0 = k0; t0 < k1; t0 += kSmStage, ++gs) {
          const int st = gs % NS, use = gs / NS;
          if (use > 0 && !tma_mbar_wait(empty_bar(st), (use - 1) & 1, wait_lim, status, abort_flag)) {
            stop = true;
            break;
          }
          const int cnt = min(kSmStage, k1 - t0);
          // whole groups of 4 records: 16-byte aligned sources and sizes (rows start on
          // multiples of 4 records, Nmax is one), never past the row
          const int c4 = (cnt + 3) & ~3;
          const int64_t r = rec0 + t0;
          const uint32_t fb = full_bar(st), sb = stage_addr(st);
          cnt_st[st] = cnt;
          const uint32_t bytes = static_cast<uint32_t>(c4) * (2u * 4u * (W0 + W1) + 16u);
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(fb), "r"(bytes) : "memory");
          bulk_g2s(sb + oK0, p.kc[0] + r * W0, c4 * W0 * 4, fb);
          bulk_g2s(sb + oK1, p.kc[1] + r * W1, c4 * W1 * 4, fb);
          bulk_g2s(sb + oV0, p.vc[0] + r * W0, c4 * W0 * 4, fb);
          bulk_g2s(sb + oV1, p.vc[1] + r * W1, c4 * W1 * 4, fb);
          bulk_g2s(sb + oKN0, p.kn[0] + r, c4 * 4, fb);
          bulk_g2s(sb + oKN1, p.kn[1] + r, c4 * 4, fb);
          bulk_g2s(sb + oVN0, p.vn[0] + r, c4 * 4, fb);
          bulk_g2s(sb + oVN1, p.vn[1] + r, c4 * 4, fb);
        }
      }
      for (int j = max(0, gs - NS); j < gs; ++j)
        for (long long i = 0; !tma_mbar_try(full_bar(j % NS), (j / NS) & 1) && i < (1ll << 28); ++i) {}
    }
    return;
  }

  // ---------------- consumers ----------------
  const int qcol = g & 3;                          // head of B column g
  const bool qlo = g >= 4;                         // B column g carries a lo part
  const int h0 = 2 * (t & 1);                      // heads of accumulator columns 2t, 2t + 1
  const bool plo = t >= 2;                         // accumulator columns 2t, 2t + 1 are lo parts
  const int kv[4] = {2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9};   // value k-index -> token of the unit
  const uint32_t sel_t = 0x7604u | (static_cast<uint32_t>(t) << 4);
  const uint32_t k2lo = t2A | (static_cast<uint32_t>(lane & 15) << 3), v2lo = k2lo + 128u;
  const uint32_t k3lo = t3A | (static_cast<uint32_t>(lane) << 2), v3lo = k3lo + 128u;
  // value runs of this lane: group 0 dims L0 g .., group 1 dims L1 g ..
  const int vw0 = (L0 * B0 * g) >> 5, vs0 = (L0 * B0 * g) & 31;
  const int vw1 = (L1 * B1 * g) >> 5, vs1 = (L1 * B1 * g) & 31;
  const int vw0n = min(vw0 + 1, W0 - 1), vw1n = min(vw1 + 1, W1 - 1);
  constexpr uint32_t M0 = (1u << (L0 * B0)) - 1u;
  constexpr uint32_t M1 = L1 * B1 == 32 ? 0xFFFFFFFFu : (1u << (L1 * B1)) - 1u;
  const float lk0 = p.logit_scale * p.kscale[0], lk1 = p.logit_scale * p.kscale[1];
  Field3 f3[KS0];
#pragma unroll
  for (int k = 0; k < KS0; ++k) f3[k] = field3(k, t);

  pdl_wait();
  int gs = 0, ipar = 0;                          // ipar: parity of this CTA's item count
  for (int item = blockIdx.x; item < n_items; item += gridDim.x, ipar ^= 1) {
    int bh, chunk, k0, k1;
    item_range(item, bh, chunk, k0, k1);
    const int bb = bh / p.Hkv, hk = bh - bb * p.Hkv;
    const int nh = min(kSmRows, G);
    const int64_t qbase = static_cast<int64_t>(bb) * p.Hq + static_cast<int64_t>(hk) * G;
    // query operand: k-step k covers dims 16k + 4t .. + 3 (group 0 for k < KS0), times the
    // group's logit factor (scale log2(e) and its table scale), so that a score row is the
    // two groups' accumulators weighted by the token's norms alone
    const bool hok = qcol < nh;
    uint32_t qh[8][2];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float a[4] = {0.f, 0.f, 0.f, 0.f};
      if (hok) {
        const float* src = k < KS0 ? p.qr[0] + (qbase + qcol) * D0 + 16 * k + 4 * t
                                   : p.qr[1] + (qbase + qcol) * D1 + 16 * (k - KS0) + 4 * t;
        const float4 v = __ldg(reinterpret_cast<const float4*>(src));
        const float f = k < KS0 ? lk0 : lk1;
        a[0] = v.x * f; a[1] = v.y * f; a[2] = v.z * f; a[3] = v.w * f;
      }
      uint32_t h01, l01, h23, l23;
      split_pair(a[0], a[1], h01, l01);
      split_pair(a[2], a[3], h23, l23);
      qh[k][0] = qlo ? l01 : h01;
      qh[k][1] = qlo ? l23 : h23;
    }
    const bool c0ok = h0 < nh, c1ok = h0 + 1 < nh;
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int t0 = k0; t0 < k1; t0 += kSmStage, ++gs) {
      const int st = gs % NS;
      if (!tma_mbar_wait(full_bar(st), (gs / NS) & 1, wait_lim, status, abort_flag)) break;
      const uint32_t sb = stage_addr(st);
      const int cnt = static_cast<int>(sld32(tma_smem_u32(cnt_st + st)));
      const int w0 = warp * 16 * U;
      // ---- this warp's slices (no per-token checks when the warp's tokens are all in the stage) ----
      const bool whole = w0 + 16 * U <= cnt;
      bool ok[U][2];
      uint32_t kw0[U][2][W0], kw1[U][2][W1];
      float kn0[U][2], kn1[U][2], vn0[U][2], vn1[U][2];
      uint32_t f0[U][4], f1[U][4];                 // value runs of the unit's tokens kv[i]
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int tk = w0 + 16 * u + 8 * h + g;
          ok[u][h] = whole || tk < cnt;
#pragma unroll
          for (int j = 0; j < W0; ++j) kw0[u][h][j] = sld32(sb + oK0 + (tk * W0 + j) * 4);
          static_assert(W1 % 2 == 0, "8-byte aligned group-1 records");
#pragma unroll
          for (int j = 0; j < W1; j += 2) {
            uint32_t x, y;
            asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(x), "=r"(y) : "r"(sb + oK1 + (tk * W1 + j) * 4) : "memory");
            kw1[u][h][j] = x;
            kw1[u][h][j + 1] = y;
          }
          if (whole) {
            kn0[u][h] = sldf(sb + oKN0 + 4 * tk);
            kn1[u][h] = sldf(sb + oKN1 + 4 * tk);
            vn0[u][h] = sldf(sb + oVN0 + 4 * tk);
            vn1[u][h] = sldf(sb + oVN1 + 4 * tk);
          } else {
            kn0[u][h] = ok[u][h] ? sldf(sb + oKN0 + 4 * tk) : 0.f;
            kn1[u][h] = ok[u][h] ? sldf(sb + oKN1 + 4 * tk) : 0.f;
            vn0[u][h] = ok[u][h] ? sldf(sb + oVN0 + 4 * tk) : 0.f;
            vn1[u][h] = ok[u][h] ? sldf(sb + oVN1 + 4 * tk) : 0.f;
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tk = w0 + 16 * u + kv[i];
          const uint32_t r0 = sb + oV0 + tk * W0 * 4, r1 = sb + oV1 + tk * W1 * 4;
          // codes of group 0 at bit 8 (tokens kv 0, 2) or 11 (kv 1, 3): the pair index of a dim
          // is then two masked shifts of the pair's words
          f0[u][i] = (__funnelshift_r(sld32(r0 + 4 * vw0), sld32(r0 + 4 * vw0n), vs0) & M0) << (i & 1 ? 11 : 8);
          f1[u][i] = __funnelshift_r(sld32(r1 + 4 * vw1), sld32(r1 + 4 * vw1n), vs1) & M1;
        }
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty_bar(st)) : "memory");
      if (w0 >= cnt) continue;

      // ---- scores of both units: group 0 k-steps into acc0, group 1 into acc1 / acc2 ----
      float sc[U][4];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < KS0; ++k) {
          uint32_t a0, a1, a2, a3;
          key_pairs<B0, W0>(kw0[u][0], k, sel_t, k3lo, f3[k], a0, a2);
          key_pairs<B0, W0>(kw0[u][1], k, sel_t, k3lo, f3[k], a1, a3);
          mma16816(acc0, a0, a1, a2, a3, qh[k][0], qh[k][1]);
        }
#pragma unroll
        for (int k = 0; k < KS1; ++k) {
          uint32_t a0, a1, a2, a3;
          key_pairs<B1, W1>(kw1[u][0], k, sel_t, k2lo, Field3{}, a0, a2);
          key_pairs<B1, W1>(kw1[u][1], k, sel_t, k2lo, Field3{}, a1, a3);
          if (k & 1) mma16816(acc2, a0, a1, a2, a3, qh[KS0 + k][0], qh[KS0 + k][1]);
          else mma16816(acc1, a0, a1, a2, a3, qh[KS0 + k][0], qh[KS0 + k][1]);
        }
        // row h: ||k_0|| acc0 + ||k_1|| acc1 on this lane's hi or lo columns, then the
        // partner lane's half (lanes t and t ^ 2 hold the same token rows)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 s1 = __fadd2_rn(make_float2(acc1[2 * h], acc1[2 * h + 1]), make_float2(acc2[2 * h], acc2[2 * h + 1]));
          float2 v = __ffma2_rn(make_float2(kn0[u][h], kn0[u][h]), make_float2(acc0[2 * h], acc0[2 * h + 1]),
                                __fmul2_rn(make_float2(kn1[u][h], kn1[u][h]), s1));
          v.x += __shfl_xor_sync(0xffffffffu, v.x, 2);
          v.y += __shfl_xor_sync(0xffffffffu, v.y, 2);
          sc[u][2 * h] = ok[u][h] ? v.x : -INFINITY;
          sc[u][2 * h + 1] = ok[u][h] ? v.y : -INFINITY;
        }
      }
      // ---- online softmax (log2 domain), one maximum check per stage ----
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
          const float2 f = make_float2(ex2(m0 - mn0), ex2(m1 - mn1));
          l0 *= f.x;
          l1 *= f.y;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 x = __fmul2_rn(make_float2(o[i][0], o[i][1]), f);
            const float2 y = __fmul2_rn(make_float2(o[i][2], o[i][3]), f);
            o[i][0] = x.x; o[i][1] = x.y; o[i][2] = y.x; o[i][3] = y.y;
          }
          m0 = mn0;
          m1 = mn1;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float2 nm = make_float2(-m0, -m1);
        const float2 d0 = __fadd2_rn(make_float2(sc[u][0], sc[u][1]), nm);
        const float2 d1 = __fadd2_rn(make_float2(sc[u][2], sc[u][3]), nm);
        const float p00 = c0ok ? ex2(d0.x) : 0.f, p01 = c1ok ? ex2(d0.y) : 0.f;
        const float p10 = c0ok ? ex2(d1.x) : 0.f, p11 = c1ok ? ex2(d1.y) : 0.f;
        const float2 ls = __fadd2_rn(make_float2(l0, l1), __fadd2_rn(make_float2(p00, p01), make_float2(p10, p11)));
        l0 = ls.x;
        l1 = ls.y;
        // P^T per value group (the group's norm rides in P): transpose the two 8x8 halves
        uint32_t bg[2][2];
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          const float n0 = gg ? vn1[u][0] : vn0[u][0], n1 = gg ? vn1[u][1] : vn0[u][1];
          const float2 pt = __fmul2_rn(make_float2(p00, p01), make_float2(n0, n0));
          const float2 pb = __fmul2_rn(make_float2(p10, p11), make_float2(n1, n1));
          uint32_t th, tl, bh2, bl2;
          split_pair(pt.x, pt.y, th, tl);
          split_pair(pb.x, pb.y, bh2, bl2);
          bg[gg][0] = movmatrix_t(plo ? tl : th);
          bg[gg][1] = movmatrix_t(plo ? bl2 : bh2);
        }
        // ---- values, group 0 (3 bits): M-tile i rows g, g + 8 = run dims 2i, 2i + 1 ----
#pragma unroll
        for (int i = 0; i < KS0; ++i) {
          uint32_t a[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int dl = 2 * i + (r & 1);                 // run dim of the row
            const int pr = r >> 1;                          // token pair (kv 0,1) or (kv 2,3)
            a[r] = tab_ld((v3lo | ((f0[u][2 * pr] >> (3 * dl)) & 0x700u)) | ((f0[u][2 * pr + 1] >> (3 * dl)) & 0x3800u));
          }
          mma16816(o[i], a[0], a[1], a[2], a[3], bg[0][0], bg[0][1]);
        }
        // ---- values, group 1 (2 bits): codes of two tokens interleaved, one byte per
        // (dim 4m + par, dim 4m + 2 + par) row pair ----
        uint32_t ze[2], zo[2];
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
          const uint32_t fa = f1[u][2 * pr], fb = f1[u][2 * pr + 1];
          ze[pr] = (fa & 0x33333333u) | ((fb & 0x33333333u) << 2);
          zo[pr] = ((fa >> 2) & 0x33333333u) | (fb & 0xCCCCCCCCu);
        }
#pragma unroll
        for (int j = 0; j < KS1; ++j) {
          const int mm = j >> 1;
          const uint32_t sel = 0x7604u | (static_cast<uint32_t>(mm) << 4);
          uint32_t a0, a1, a2, a3;
          lds64(__byte_perm((j & 1) ? zo[0] : ze[0], v2lo, sel), a0, a1);
          lds64(__byte_perm((j & 1) ? zo[1] : ze[1], v2lo, sel), a2, a3);
          mma16816(o[KS0 + j], a0, a1, a2, a3, bg[1][0], bg[1][1]);
        }
      }
    }

    // ---- merge this item across the consumer warps ----
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) o[i][j] += __shfl_xor_sync(0xffffffffu, o[i][j], 2);
    // each warp publishes its row maxima, scales its own partial by 2^(m_w - M) in registers
    // and writes it; the item's partial is then a plain sum over the warps in a fixed order
    // (maxima in a buffer per item parity: a warp may publish the next item's while a slower
    // one still reads these)
    float* mb = mxb + ipar * (NC * kSmRows);        // [warp][4 rows]
    if (t < 2 && g == 0) {
      mb[warp * kSmRows + 2 * t] = m0;
      mb[warp * kSmRows + 2 * t + 1] = m1;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
    // one exit decision for every consumer warp, sampled between the two barriers
    if (tid == 0) *consumers_stop = *abort_flag;
    float* wm = mrg + warp * kSmRows * (D + 2);      // [row][-, l, o'[D]]
    if (t < 2) {
      float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
      for (int w = 0; w < NC; ++w) {
        M0 = fmaxf(M0, mb[w * kSmRows + 2 * t]);
        M1 = fmaxf(M1, mb[w * kSmRows + 2 * t + 1]);
      }
      const float2 f = make_float2(m0 == -INFINITY ? 0.f : ex2(m0 - M0), m1 == -INFINITY ? 0.f : ex2(m1 - M1));
      if (g == 0) {
        wm[(2 * t) * (D + 2) + 1] = l0 * f.x;
        wm[(2 * t + 1) * (D + 2) + 1] = l1 * f.y;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int da, db;                                  // rotated dims of rows g and g + 8
        if (i < KS0) {
          da = L0 * g + 2 * i;
          db = da + 1;
        } else {
          const int j = i - KS0, mm = j >> 1, par = j & 1;
          da = D0 + L1 * g + 4 * mm + par;
          db = da + 2;
        }
        const float2 x = __fmul2_rn(make_float2(o[i][0], o[i][1]), f);
        const float2 y = __fmul2_rn(make_float2(o[i][2], o[i][3]), f);
        wm[(2 * t) * (D + 2) + 2 + da] = x.x;
        wm[(2 * t + 1) * (D + 2) + 2 + da] = x.y;
        wm[(2 * t) * (D + 2) + 2 + db] = y.x;
        wm[(2 * t + 1) * (D + 2) + 2 + db] = y.y;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
    for (int idx = tid; idx < nh * D; idx += CONSUMERS) {
      const int r = idx / D, j = idx - r * D;
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int w = 0; w < NC; w += 2) {
        s0 += mrg[(w * kSmRows + r) * (D + 2) + 2 + j];
        if (w + 1 < NC) s1 += mrg[((w + 1) * kSmRows + r) * (D + 2) + 2 + j];
      }
      const int64_t pi = (qbase + r) * p.n_chunks + chunk;
      if (j == 0) {
        float M = -INFINITY, L = 0.f;
#pragma unroll
        for (int w = 0; w < NC; ++w) {
          M = fmaxf(M, mb[w * kSmRows + r]);
          L += mrg[(w * kSmRows + r) * (D + 2) + 1];
        }
        p.part_ml[pi * 2] = M;
        p.part_ml[pi * 2 + 1] = L;
      }
      p.part_o[pi * D + j] = (s0 + s1) * (j < D0 ? p.vscale[0] : p.vscale[1]);
    }
    // the next writes of mrg come after the next item's first barrier, which every thread
    // reaches only after this loop
    if (*consumers_stop) break;
  }
}

}  // namespace tq
