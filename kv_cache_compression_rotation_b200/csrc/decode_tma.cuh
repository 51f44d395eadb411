// Decode attention with bulk-copy (TMA engine) staging of the packed cache, d = 128.
//
// Same computation as decode_attn_kernel (decode.cuh) for MSE or PROD keys and MSE
// values; the difference is how the records reach the SM.  One producer warp streams
// each chunk of the context in stages of 112 tokens with cp.async.bulk (key codes,
// value codes, norms; prod adds sign words and residual norms), four stages deep, into
// shared memory; seven consumer warps each take 16 tokens of a stage, read their
// record slices with vector shared loads, release the stage, and run the lookup-table
// dequantization, the two mma.sync products and the online softmax from registers.
// Keeping ~70 KB of copies in flight per SM is what lets the stream run near HBM rate.
//
// Within a 16-token unit the score tile's columns are permuted (column n of n-tile nt
// is token 8 nt + n/2 + 4 (n mod 2)) so that the value-slice loads of a warp touch both
// halves of the banks evenly; the P.V operand uses the same permutation.
// All waits are bounded (TQ_ERR_TIMEOUT on expiry); a CTA that times out drains the
// copies it issued before it exits.
#pragma once

#include "decode.cuh"

namespace tq {

constexpr int kTmaConsumerWarps = 7;
constexpr int kTmaThreads = (kTmaConsumerWarps + 1) * 32;
constexpr int kTmaStageTokens = kTmaConsumerWarps * 16;
constexpr int kTmaStages = 4;

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

struct TmaStageLayout {
  uint32_t kcodes, vcodes, knorm, vnorm, ksign, krn, bytes;
};

// Byte offsets of the arrays of one stage (all 16-byte aligned).
__host__ __device__ inline TmaStageLayout tma_stage_layout(int kw, int vw, int kf, int ksw) {
  TmaStageLayout L{};
  uint32_t o = 0;
  L.kcodes = o; o += kTmaStageTokens * kw * 4;
  L.vcodes = o; o += kTmaStageTokens * vw * 4;
  L.knorm = o; o += (kTmaStageTokens + 4) * 4;
  L.vnorm = o; o += (kTmaStageTokens + 4) * 4;
  L.ksign = o; o += (kf == KFMT_PROD) ? kTmaStageTokens * ksw * 4 : 0;
  L.krn = o; o += (kf == KFMT_PROD) ? (kTmaStageTokens + 4) * 4 : 0;
  L.bytes = o;
  return L;
}

inline size_t decode_tma_smem_bytes(int kb, int vb, int kf, int ksw, bool g8) {
  const size_t tables = (static_cast<size_t>(1u << (2 * kb)) + (1u << (2 * vb)) + 4) * 32 * 4;
  const TmaStageLayout L = tma_stage_layout(128 * kb / 32, 128 * vb / 32, kf, ksw);
  const size_t merge = static_cast<size_t>(kTmaConsumerWarps) * (g8 ? 8 : 16) * (128 + 2) * 4;
  return tables + static_cast<size_t>(kTmaStages) * L.bytes + merge + 2 * kTmaStages * 8 + 64 + 16;
}

// G8: the GQA group has at most 8 query heads, so mma rows 8..15 are known to be zero.
// Persistent: CTA c processes work items c, c + gridDim.x, ... where item = (batch *
// kv-head, chunk); the lookup tables are built once per CTA and the stage ring runs on
// across items.  The consumer warps merge each item's partial with a named barrier of
// their own, so the producer keeps streaming the next item meanwhile.
template <int KF, int KB, int VB, bool G8>
__global__ void __launch_bounds__(kTmaThreads, 1)
decode_tma_kernel(const DecodeParams p, int* status, long long wait_lim) {
  constexpr int D = 128;
  constexpr int KST = D / 16;
  constexpr int TDK = D / 4;
  constexpr int NWK = (TDK * KB + 31) / 32;
  constexpr int TDV = D / 8;
  constexpr int NWV = (TDV * VB + 31) / 32;
  constexpr int NT = D / 8;
  constexpr int KLUT = 1 << (2 * KB), VLUT = 1 << (2 * VB);
  constexpr int KW = D * KB / 32, VW = D * VB / 32;     // record words
  constexpr int KSW = 4;                                // prod sign words (m = 128)
  constexpr int MROWS = G8 ? 8 : 16;
  constexpr int CONSUMERS = kTmaConsumerWarps * 32;
  extern __shared__ __align__(128) uint32_t tsm_[];
  uint32_t* lutk = tsm_;
  uint32_t* lutv = lutk + KLUT * 32;
  uint32_t* luts = lutv + VLUT * 32;
  unsigned char* stage0 = reinterpret_cast<unsigned char*>(luts + 4 * 32);
  const TmaStageLayout SL = tma_stage_layout(KW, VW, KF, KSW);
  float* mrg = reinterpret_cast<float*>(stage0 + static_cast<size_t>(kTmaStages) * SL.bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(mrg + kTmaConsumerWarps * MROWS * (D + 2));
  int* nb_count = reinterpret_cast<int*>(bars + 2 * kTmaStages);   // [kTmaStages] tokens with staged norms
  int* nb_off = nb_count + kTmaStages;                                 // [kTmaStages] their offset in the stage
  volatile int* abort_flag = nb_off + kTmaStages;
  volatile int* consumers_stop = abort_flag + 1;   // uniform exit decision of the consumer warps
  const uint32_t bar0 = tma_smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kTmaStages + s); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int n_items = p.B * p.Hkv * p.n_chunks;
  const int64_t total_recs = static_cast<int64_t>(p.B) * p.Hkv * p.Nmax;
  auto item_range = [&](int item, int& bh, int& chunk, int& k0, int& k1) {
    bh = item / p.n_chunks;
    chunk = item - bh * p.n_chunks;
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
  for (int i = tid; i < KLUT * 32; i += kTmaThreads) {
    const int e = i >> 5;
    lutk[i] = pack_half2(__ldg(p.kc + (e & ((1 << KB) - 1))) / p.k_scale, __ldg(p.kc + (e >> KB)) / p.k_scale);
  }
  for (int i = tid; i < VLUT * 32; i += kTmaThreads) {
    const int e = i >> 5;
    lutv[i] = pack_half2(__ldg(p.vc + (e & ((1 << VB) - 1))) / p.v_scale, __ldg(p.vc + (e >> VB)) / p.v_scale);
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
        int bh, chunk, k0, k1;
        item_range(item, bh, chunk, k0, k1);
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
  const int G = p.G;
  const int row0 = g, row1 = g + 8;
  const bool r0ok = row0 < G, r1ok = !G8 && row1 < G;
  const int kA = (g >> 1) + 4 * (g & 1);        // score n-tile 0 column g; n-tile 1 adds 8
  const int kc[4] = {t, t + 4, 8 + t, 12 + t};  // columns 2t, 2t+1 of n-tiles 0 and 1
  int gs = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    int bh, chunk, k0, k1;
    item_range(item, bh, chunk, k0, k1);
    const int bb = bh / p.Hkv, hk = bh - bb * p.Hkv;
    const int64_t rec0 = static_cast<int64_t>(bh) * p.Nmax;
    const int64_t qrow0 = static_cast<int64_t>(bb) * p.Hq + hk * G + row0;
    const int64_t qrow1 = static_cast<int64_t>(bb) * p.Hq + hk * G + row1;
    uint32_t qa[KST][4], ql[KST][4];
#pragma unroll
    for (int s = 0; s < KST; ++s) {
      const int dm = t * TDK + 4 * s;
      float a[4] = {0.f, 0.f, 0.f, 0.f}, b[4] = {0.f, 0.f, 0.f, 0.f};
      if (r0ok) for (int i = 0; i < 4; ++i) a[i] = p.qa[qrow0 * D + dm + i];
      if (r1ok) for (int i = 0; i < 4; ++i) b[i] = p.qa[qrow1 * D + dm + i];
      split_pair(a[0], a[1], qa[s][0], ql[s][0]);
      split_pair(a[2], a[3], qa[s][2], ql[s][2]);
      if constexpr (G8) {
        qa[s][1] = ql[s][1] = qa[s][3] = ql[s][3] = 0u;
      } else {
        split_pair(b[0], b[1], qa[s][1], ql[s][1]);
        split_pair(b[2], b[3], qa[s][3], ql[s][3]);
      }
    }
    // QJL operand: one half-precision pass suffices, since its term is the residual part
    // of the score (a 2^-12 relative error on it is ~1e-5 of the score)
    uint32_t qb[KST][4];
    if constexpr (KF == KFMT_PROD) {
#pragma unroll
      for (int s = 0; s < KST; ++s) {
        const int dm = t * TDK + 4 * s;
        float a[4] = {0.f, 0.f, 0.f, 0.f}, c[4] = {0.f, 0.f, 0.f, 0.f};
        if (r0ok) for (int i = 0; i < 4; ++i) a[i] = p.qb[qrow0 * p.qb_stride + dm + i];
        if (r1ok) for (int i = 0; i < 4; ++i) c[i] = p.qb[qrow1 * p.qb_stride + dm + i];
        qb[s][0] = pack_half2(a[0], a[1]);
        qb[s][1] = G8 ? 0u : pack_half2(c[0], c[1]);
        qb[s][2] = pack_half2(a[2], a[3]);
        qb[s][3] = G8 ? 0u : pack_half2(c[2], c[3]);
      }
    }
    const float sa0 = r0ok ? p.qs[qrow0 * 2] * p.k_scale : 0.f, sa1 = r1ok ? p.qs[qrow1 * 2] * p.k_scale : 0.f;
    const float sb0 = r0ok ? p.qs[qrow0 * 2 + 1] : 0.f, sb1 = r1ok ? p.qs[qrow1 * 2 + 1] : 0.f;

    float o[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int t0 = k0; t0 < k1; t0 += kTmaStageTokens, ++gs) {
      const int s = gs % kTmaStages;
      if (!tma_mbar_wait(full_bar(s), (gs / kTmaStages) & 1, wait_lim, status, abort_flag)) break;
      const unsigned char* sb = stage0 + static_cast<size_t>(s) * SL.bytes;
      const uint32_t* skc = reinterpret_cast<const uint32_t*>(sb + SL.kcodes);
      const uint32_t* svc = reinterpret_cast<const uint32_t*>(sb + SL.vcodes);
      const float* skn = reinterpret_cast<const float*>(sb + SL.knorm);
      const float* svn = reinterpret_cast<const float*>(sb + SL.vnorm);
      const int cnt = min(kTmaStageTokens, k1 - t0);
      const int nn = nb_count[s], noff = nb_off[s];
      const int u0 = warp * 16;                      // first token of this warp's unit (stage-local)
      // ---- pull this warp's slices out of the stage ----
      uint32_t ks0[NWK], ks1[NWK];
      load_slice<NWK, false>(skc + (u0 + kA) * KW, KW, t * TDK * KB, u0 + kA < cnt, ks0);
      load_slice<NWK, false>(skc + (u0 + 8 + kA) * KW, KW, t * TDK * KB, u0 + 8 + kA < cnt, ks1);
      uint32_t vs[4][NWV];
      float kn[4], vn[4], gm[4];
      uint32_t sw[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int lk = u0 + kc[i];
        const bool ok = lk < cnt;
        load_slice<NWV, false>(svc + lk * VW, VW, g * TDV * VB, ok, vs[i]);
        const int64_t gi = rec0 + t0 + lk;
        kn[i] = ok ? (lk < nn ? skn[noff + lk] : __ldg(p.knorms + gi)) : 0.f;
        vn[i] = ok ? (lk < nn ? svn[noff + lk] : __ldg(p.vnorms + gi)) : 0.f;
        if constexpr (KF == KFMT_PROD) {
          const float* srn = reinterpret_cast<const float*>(sb + SL.krn);
          gm[i] = ok ? (lk < nn ? srn[noff + lk] : __ldg(p.krnorms + gi)) : 0.f;
        } else {
          gm[i] = 0.f;
        }
      }
      if constexpr (KF == KFMT_PROD) {
        const uint32_t* ssg = reinterpret_cast<const uint32_t*>(sb + SL.ksign);
        sw[0] = (u0 + kA < cnt) ? ssg[(u0 + kA) * KSW + t] : 0u;
        sw[1] = (u0 + 8 + kA < cnt) ? ssg[(u0 + 8 + kA) * KSW + t] : 0u;
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty_bar(s)) : "memory");
      if (u0 >= cnt) continue;

      // ---- scores ----
      float sc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        // hi and lo query halves accumulate separately: two independent MMA chains
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, accl[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t(&ks)[NWK] = nt ? ks1 : ks0;
#pragma unroll
        for (int s2 = 0; s2 < KST; ++s2) {
          uint32_t b0, b1;
          if constexpr (KB == 4) {
            // the pair of dims (4 s2, 4 s2 + 1) is byte 2 (s2 % 2) of word s2 / 2
            const uint32_t w = ks[s2 >> 1];
            b0 = lutk[(__byte_perm(w, 0u, 0x4440u + 2 * (s2 & 1)) << 5) + lane];
            b1 = lutk[(__byte_perm(w, 0u, 0x4441u + 2 * (s2 & 1)) << 5) + lane];
          } else {
            b0 = lutk[(pair_at<KB, NWK>(ks, 4 * s2 * KB) << 5) + lane];
            b1 = lutk[(pair_at<KB, NWK>(ks, (4 * s2 + 2) * KB) << 5) + lane];
          }
          mma16816(acc, qa[s2][0], qa[s2][1], qa[s2][2], qa[s2][3], b0, b1);
          mma16816(accl, ql[s2][0], ql[s2][1], ql[s2][2], ql[s2][3], b0, b1);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += accl[i];
        float acc2[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (KF == KFMT_PROD) {
          const uint32_t w = sw[nt];
#pragma unroll
          for (int s2 = 0; s2 < KST; ++s2) {
            const uint32_t b0 = luts[(((w >> (4 * s2)) & 3u) << 5) + lane];
            const uint32_t b1 = luts[(((w >> (4 * s2 + 2)) & 3u) << 5) + lane];
            mma16816(acc2, qb[s2][0], qb[s2][1], qb[s2][2], qb[s2][3], b0, b1);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int ci = nt * 2 + (i & 1);
          const float sa = (i < 2) ? sa0 : sa1, sbv = (i < 2) ? sb0 : sb1;
          float v;
          if constexpr (KF == KFMT_PROD) v = kn[ci] * (sa * acc[i] + p.qjl_coef * gm[ci] * sbv * acc2[i]);
          else v = kn[ci] * sa * acc[i];
          sc[nt][i] = (u0 + kc[ci] < cnt) ? v : -INFINITY;
        }
      }
      // ---- online softmax (log2 domain) ----
      float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      const float mn0 = fmaxf(m0, mx0);
      if (mn0 > m0) {
        const float f = exp2f(m0 - mn0);
        l0 *= f;
#pragma unroll
        for (int i = 0; i < NT; ++i) { o[i][0] *= f; o[i][1] *= f; }
        m0 = mn0;
      }
      if constexpr (!G8) {
        float mx1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn1 = fmaxf(m1, mx1);
        if (G > 8 && mn1 > m1) {
          const float f = exp2f(m1 - mn1);
          l1 *= f;
#pragma unroll
          for (int i = 0; i < NT; ++i) { o[i][2] *= f; o[i][3] *= f; }
          m1 = mn1;
        }
      }
      float pr[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        pr[nt][0] = r0ok ? exp2f(sc[nt][0] - m0) : 0.f;
        pr[nt][1] = r0ok ? exp2f(sc[nt][1] - m0) : 0.f;
        pr[nt][2] = r1ok ? exp2f(sc[nt][2] - m1) : 0.f;
        pr[nt][3] = r1ok ? exp2f(sc[nt][3] - m1) : 0.f;
        l0 += pr[nt][0] + pr[nt][1];
        l1 += pr[nt][2] + pr[nt][3];
      }
      uint32_t pa0, pa1, pa2, pa3, pl0, pl1, pl2, pl3;
      split_pair(pr[0][0] * vn[0], pr[0][1] * vn[1], pa0, pl0);
      split_pair(pr[1][0] * vn[2], pr[1][1] * vn[3], pa2, pl2);
      if constexpr (G8) {
        pa1 = pl1 = pa3 = pl3 = 0u;
      } else {
        split_pair(pr[0][2] * vn[0], pr[0][3] * vn[1], pa1, pl1);
        split_pair(pr[1][2] * vn[2], pr[1][3] * vn[3], pa3, pl3);
      }
      // ---- P.V in the rotated domain ----
      if constexpr (VB == 4) {
        // byte j of lo (hi) holds the codes of keys (t, t + 4) for dim 2j (2j + 1) of a word
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const uint32_t a0 = vs[0][w], a1 = vs[1][w], c0 = vs[2][w], c1 = vs[3][w];
          const uint32_t lo01 = (a0 & 0x0F0F0F0Fu) | ((a1 << 4) & 0xF0F0F0F0u);
          const uint32_t hi01 = ((a0 >> 4) & 0x0F0F0F0Fu) | (a1 & 0xF0F0F0F0u);
          const uint32_t lo23 = (c0 & 0x0F0F0F0Fu) | ((c1 << 4) & 0xF0F0F0F0u);
          const uint32_t hi23 = ((c0 >> 4) & 0x0F0F0F0Fu) | (c1 & 0xF0F0F0F0u);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int i = 8 * w + j;                  // n-tile = dim within this thread's 16
            const uint32_t x01 = (j & 1) ? hi01 : lo01, x23 = (j & 1) ? hi23 : lo23;
            const uint32_t b0 = lutv[(__byte_perm(x01, 0u, 0x4440u + (j >> 1)) << 5) + lane];
            const uint32_t b1 = lutv[(__byte_perm(x23, 0u, 0x4440u + (j >> 1)) << 5) + lane];
            mma16816(o[i], pa0, pa1, pa2, pa3, b0, b1);
            mma16816(o[i], pl0, pl1, pl2, pl3, b0, b1);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < NT; ++i) {
          const uint32_t e01 = field_at<VB, NWV>(vs[0], i * VB) | (field_at<VB, NWV>(vs[1], i * VB) << VB);
          const uint32_t e23 = field_at<VB, NWV>(vs[2], i * VB) | (field_at<VB, NWV>(vs[3], i * VB) << VB);
          const uint32_t b0 = lutv[(e01 << 5) + lane], b1 = lutv[(e23 << 5) + lane];
          mma16816(o[i], pa0, pa1, pa2, pa3, b0, b1);
          mma16816(o[i], pl0, pl1, pl2, pl3, b0, b1);
        }
      }
    }

    // ---- merge this item across the consumer warps (named barrier 1) ----
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    float* wm = mrg + warp * MROWS * (D + 2);
    if (t == 0) {
      wm[row0 * (D + 2)] = m0; wm[row0 * (D + 2) + 1] = l0;
      if constexpr (!G8) { wm[row1 * (D + 2)] = m1; wm[row1 * (D + 2) + 1] = l1; }
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      wm[row0 * (D + 2) + 2 + (2 * t) * TDV + i] = o[i][0];
      wm[row0 * (D + 2) + 2 + (2 * t + 1) * TDV + i] = o[i][1];
      if constexpr (!G8) {
        wm[row1 * (D + 2) + 2 + (2 * t) * TDV + i] = o[i][2];
        wm[row1 * (D + 2) + 2 + (2 * t + 1) * TDV + i] = o[i][3];
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(CONSUMERS) : "memory");
    for (int idx = tid; idx < G * D; idx += CONSUMERS) {
      const int r = idx / D, j = idx - r * D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kTmaConsumerWarps; ++w) M = fmaxf(M, mrg[(w * MROWS + r) * (D + 2)]);
      float a = 0.f, L = 0.f;
#pragma unroll
      for (int w = 0; w < kTmaConsumerWarps; ++w) {
        const float* row = mrg + (w * MROWS + r) * (D + 2);
        const float f = (row[0] == -INFINITY) ? 0.f : exp2f(row[0] - M);
        L += f * row[1];
        a += f * row[2 + j];
      }
      const int64_t qi = static_cast<int64_t>(bb) * p.Hq + hk * G + r;
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
