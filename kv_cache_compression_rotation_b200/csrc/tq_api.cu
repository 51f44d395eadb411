// C ABI of libtq: argument validation, workspace planning and kernel launches.
// The declarations and their contracts are in include/tq.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "decode.cuh"
#include "decode_aux.cuh"
#include "decode_split.cuh"
#include "decode_split_mma.cuh"
#include "decode_tma.cuh"
#include "gemm_umma.cuh"
#include "device_common.cuh"
#include "launchers.h"
#include "quantize_simt.cuh"
#include "quantize_umma.cuh"
#include "score.cuh"
#include "tq_internal.h"

namespace tq {

__device__ int g_tq_status = 0;

namespace {
thread_local char g_msg[512] = "ok";
std::atomic<long long> g_wait_limit{0};
constexpr long long kDefaultWaitLimit = 1ll << 24;
}  // namespace

tq_status fail(tq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

int* device_status_ptr() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_tq_status) != cudaSuccess) return nullptr;
  return static_cast<int*>(ptr);
}

long long wait_limit() {
  const long long v = g_wait_limit.load();
  return v != 0 ? v : kDefaultWaitLimit;
}

namespace {

tq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(TQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  const void* p;
  size_t bytes;
};

bool overlaps(Range a, Range b) {
  if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
  return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

size_t dtype_size(int dtype) { return dtype == TQ_F32 ? 4 : 2; }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int spectral_head_bits(const tq_quantizer* q) {
  int s = 0;
  for (int j = 0; j < q->k_top; ++j) s += q->top_bits[j];
  return s + (q->qjl ? q->k_top : 0);
}

tq_status check_quantizer(const tq_quantizer* q) {
  if (!q) return fail(TQ_ERR_INVALID_ARG, "quantizer is NULL");
  if (q->d < 2 || q->d > 4096) return fail(TQ_ERR_INVALID_ARG, "d must be in 2..4096 (got %d)", q->d);
  if (!q->rot) return fail(TQ_ERR_INVALID_ARG, "rot is NULL");
  if (!aligned16(q->rot)) return fail(TQ_ERR_ALIGNMENT, "rot is not 16-byte aligned");
  switch (q->kind) {
    case TQ_KIND_MSE:
      if (q->bits < 1 || q->bits > 8) return fail(TQ_ERR_INVALID_ARG, "MSE bits must be 1..8");
      if (!q->centroids || !q->boundaries) return fail(TQ_ERR_INVALID_ARG, "codebook is NULL");
      break;
    case TQ_KIND_PROD:
      if (q->bits < 1 || q->bits > 9) return fail(TQ_ERR_INVALID_ARG, "PROD bits must be 1..9");
      if (q->m < 32 || q->m > 4096 || (q->m & 31)) return fail(TQ_ERR_INVALID_ARG, "PROD m must be a multiple of 32 in 32..4096");
      if (!q->S) return fail(TQ_ERR_INVALID_ARG, "S is NULL");
      if (q->bits > 1 && (!q->centroids || !q->boundaries)) return fail(TQ_ERR_INVALID_ARG, "codebook is NULL");
      break;
    case TQ_KIND_SPECTRAL: {
      if (q->k_top < 1 || q->k_top > TQ_MAX_TOP || q->k_top > q->d)
        return fail(TQ_ERR_INVALID_ARG, "k_top must be 1..%d and <= d", TQ_MAX_TOP);
      for (int j = 0; j < q->k_top; ++j)
        if (q->top_bits[j] < 0 || q->top_bits[j] > 8) return fail(TQ_ERR_INVALID_ARG, "top_bits must be 0..8");
      if (q->tail_bits < 1 || q->tail_bits > 4) return fail(TQ_ERR_INVALID_ARG, "tail_bits must be 1..4");
      if (spectral_head_bits(q) > 96) return fail(TQ_ERR_INVALID_ARG, "spectral head exceeds 96 bits");
      if (!q->dim_sigma || !q->unit_centroids || !q->unit_boundaries)
        return fail(TQ_ERR_INVALID_ARG, "spectral codebook arrays are NULL");
      if (q->qjl && !q->S) return fail(TQ_ERR_INVALID_ARG, "S is NULL (qjl)");
      break;
    }
    default:
      return fail(TQ_ERR_INVALID_ARG, "unknown quantizer kind %d", q->kind);
  }
  if (q->S && !aligned16(q->S)) return fail(TQ_ERR_ALIGNMENT, "S is not 16-byte aligned");
  return TQ_OK;
}

tq_layout layout_of(const tq_quantizer* q) {
  tq_layout L{};
  if (q->kind == TQ_KIND_MSE) {
    L.code_words = words_for(q->d, q->bits);
    L.has_norms = 1;
  } else if (q->kind == TQ_KIND_PROD) {
    L.code_words = q->bits > 1 ? words_for(q->d, q->bits - 1) : 0;
    L.sign_words = q->m / 32;
    L.has_norms = 1;
    L.has_rnorms = 1;
  } else {
    L.code_words = (spectral_head_bits(q) + 31) / 32 + words_for(q->d, q->tail_bits);
    L.has_rnorms = q->qjl ? 1 : 0;
  }
  return L;
}

tq_status check_packed(const tq_packed& pk, const tq_layout& L, bool need_codes = true) {
  if (need_codes && L.code_words > 0 && !pk.codes) return fail(TQ_ERR_INVALID_ARG, "codes is NULL");
  if (L.sign_words > 0 && !pk.signs) return fail(TQ_ERR_INVALID_ARG, "signs is NULL");
  if (L.has_norms && !pk.norms) return fail(TQ_ERR_INVALID_ARG, "norms is NULL");
  if (L.has_rnorms && !pk.rnorms) return fail(TQ_ERR_INVALID_ARG, "rnorms is NULL");
  const void* ps[4] = {pk.codes, pk.signs, pk.norms, pk.rnorms};
  for (const void* p : ps)
    if (p && !aligned16(p)) return fail(TQ_ERR_ALIGNMENT, "packed array is not 16-byte aligned");
  return TQ_OK;
}

void packed_ranges(const tq_packed& pk, const tq_layout& L, int64_t n, Range out[4]) {
  out[0] = {pk.codes, static_cast<size_t>(n) * L.code_words * 4};
  out[1] = {pk.signs, static_cast<size_t>(n) * L.sign_words * 4};
  out[2] = {L.has_norms ? pk.norms : nullptr, static_cast<size_t>(n) * 4};
  out[3] = {L.has_rnorms ? pk.rnorms : nullptr, static_cast<size_t>(n) * 4};
}

tq_status check_no_alias(const Range* outs, int nout, const Range* ins, int nin) {
  for (int i = 0; i < nout; ++i) {
    for (int j = 0; j < nin; ++j)
      if (overlaps(outs[i], ins[j])) return fail(TQ_ERR_ALIAS, "an output overlaps an input");
    for (int j = i + 1; j < nout; ++j)
      if (overlaps(outs[i], outs[j])) return fail(TQ_ERR_ALIAS, "two outputs overlap");
  }
  return TQ_OK;
}

// ---- tensor map for the tensor-core quantize ----
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// spectral records the tensor-core kernel writes: 1-bit tail, top dims of <= 6 bits in one
// head word, 4 tail words
bool umma_spectral(const tq_quantizer* q) {
  if (q->kind != TQ_KIND_SPECTRAL || q->tail_bits != 1 || q->k_top < 1 || q->k_top > TQ_MAX_TOP) return false;
  int hb = q->qjl ? q->k_top : 0;
  for (int j = 0; j < q->k_top; ++j) {
    if (q->top_bits[j] < 1 || q->top_bits[j] > kSpecMaxTopBits) return false;
    hb += q->top_bits[j];
  }
  return hb <= 32 && (!q->qjl || q->S);
}

// prod records the tensor-core kernel writes: m = d = 128, 1..4 MSE bits plus the QJL signs
bool umma_prod(const tq_quantizer* q) {
  return q->kind == TQ_KIND_PROD && q->m == 128 && q->bits >= 2 && q->bits <= 5 && q->S && q->centroids &&
         q->boundaries;
}

bool umma_supported(const tq_quantizer* q, int dtype, int64_t n) {
  if (q->d != 128) return false;
  if (q->kind == TQ_KIND_MSE ? q->bits > 4 : (q->kind == TQ_KIND_PROD ? !umma_prod(q) : !umma_spectral(q)))
    return false;
  if (dtype != TQ_BF16 && dtype != TQ_F16) return false;
  if (n < 1 || n >= (1ll << 31) - 256) return false;
  if (std::getenv("TQ_FORCE_SIMT")) return false;
  int dev = 0, major = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10 && get_encode() != nullptr;
}

// ld / cols: element j of row v is x[v * ld + (cols ? cols[j] : j)] (cols: device; the
// split's channel gather); a gather always takes the CUDA-core kernel.
// Paged output of an append: vector v = b * Hkv + h goes to the record of token
// seq[b] - 1 of (b, h) in the pool (see tq_pages).
struct PagedOut {
  const tq_pages* pages;
  const int32_t* seq;
  int Hkv;
};

tq_status quantize_common(const tq_quantizer* q, const void* x, int dtype, int64_t n, tq_packed out,
                          cudaStream_t stream, int want_kind, int64_t ld, const int32_t* cols,
                          const Range* extra_outs = nullptr, int n_extra = 0, const PagedOut* pgo = nullptr) {
  tq_status s = check_quantizer(q);
  if (s != TQ_OK) return s;
  if (q->kind != want_kind) return fail(TQ_ERR_INVALID_ARG, "quantizer kind does not match this entry point");
  if (dtype < TQ_F32 || dtype > TQ_F16) return fail(TQ_ERR_INVALID_ARG, "unknown dtype");
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, "n < 0");
  if (n == 0) return TQ_OK;
  if (!x) return fail(TQ_ERR_INVALID_ARG, "x is NULL");
  if (!aligned16(x)) return fail(TQ_ERR_ALIGNMENT, "x is not 16-byte aligned");
  if (q->d > 2048) return fail(TQ_ERR_UNSUPPORTED, "quantize supports d <= 2048");
  const tq_layout L = layout_of(q);
  if ((s = check_packed(out, L)) != TQ_OK) return s;
  Range outs[4];
  packed_ranges(out, L, pgo ? pgo->pages->num_pages * pgo->Hkv * pgo->pages->page_size : n, outs);
  // inputs: x, and the other groups' outputs of a split call (disjoint from this group's)
  Range ins[1 + 4 * TQ_MAX_GROUPS];
  ins[0] = {x, static_cast<size_t>(n) * static_cast<size_t>(ld) * dtype_size(dtype)};
  for (int i = 0; i < n_extra; ++i) ins[1 + i] = extra_outs[i];
  if ((s = check_no_alias(outs, 4, ins, 1 + n_extra)) != TQ_OK) return s;
  int* status = device_status_ptr();

  if (!cols && !pgo && umma_supported(q, dtype, n)) {
    auto encode = get_encode();
    CUtensorMap map;
    const cuuint64_t gdim[2] = {128, static_cast<cuuint64_t>(n)};
    const cuuint64_t gstride[1] = {256};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(&map, dtype == TQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                              2, const_cast<void*>(x), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    UmmaQuantParams p{};
    p.rot = q->rot;
    p.boundaries = q->boundaries;
    p.n = n;
    p.is_f16 = dtype == TQ_F16;
    p.codes = out.codes;
    p.norms = out.norms;
    p.status = status;
    p.wait_limit = wait_limit();
    p.pm1 = q->kind == TQ_KIND_MSE && q->rot_pm1 != 0;
    p.pm1_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(q->d)));
    if (q->kind == TQ_KIND_SPECTRAL) {
      p.k_top = q->k_top; p.qjl = q->qjl;
      for (int j = 0; j < TQ_MAX_TOP; ++j) p.top_bits[j] = q->top_bits[j];
      p.dim_sigma = q->dim_sigma; p.unit_c = q->unit_centroids; p.unit_t = q->unit_boundaries;
      p.S = q->S; p.rnorms = q->qjl ? out.rnorms : nullptr;
    }
    if (q->kind == TQ_KIND_PROD) {
      p.S = q->S; p.centroids = q->centroids; p.signs = out.signs; p.rnorms = out.rnorms;
    }
    const int64_t tiles = (n + 127) / 128;
    const int grid = static_cast<int>(std::min<int64_t>(tiles, sm_count()));
    const cudaError_t e = q->kind == TQ_KIND_PROD
                              ? launch_umma_quantize_prod(map, p, q->bits - 1, grid, stream)
                              : launch_umma_quantize(map, p, q->kind == TQ_KIND_SPECTRAL ? 0 : q->bits, grid, stream);
    return e == cudaSuccess ? TQ_OK : cuda_fail(e, "umma quantize launch");
  }

  SimtQuantParams p{};
  p.x = x; p.dtype = dtype; p.n = n; p.d = q->d; p.kind = q->kind;
  p.rot = q->rot; p.S = q->S;
  p.m = q->kind == TQ_KIND_PROD ? q->m : (q->kind == TQ_KIND_SPECTRAL && q->qjl ? q->k_top : 0);
  p.centroids = q->centroids; p.boundaries = q->boundaries;
  p.bmse = q->kind == TQ_KIND_MSE ? q->bits : (q->kind == TQ_KIND_PROD ? q->bits - 1 : 0);
  p.k_top = q->k_top; p.tail_bits = q->tail_bits; p.qjl = q->qjl;
  for (int j = 0; j < TQ_MAX_TOP; ++j) p.top_bits[j] = q->top_bits[j];
  p.dim_sigma = q->dim_sigma; p.unit_c = q->unit_centroids; p.unit_t = q->unit_boundaries;
  p.codes = out.codes; p.code_words = L.code_words;
  p.signs = out.signs; p.sign_words = L.sign_words;
  p.norms = L.has_norms ? out.norms : nullptr;
  p.rnorms = L.has_rnorms ? out.rnorms : nullptr;
  p.ld = ld;
  p.cols = cols;
  p.status = status;
  if (pgo) {
    p.pg_table = pgo->pages->block_table; p.pg_seq = pgo->seq; p.pg_size = pgo->pages->page_size;
    p.pg_max = pgo->pages->max_pages; p.pg_hkv = pgo->Hkv; p.pg_num = pgo->pages->num_pages;
  }
  const int d = q->d;
  // vectors per CTA: a multiple of 8 (the tiled product's row groups), at most 32, within
  // 200 KB of shared memory
  const int dp = (d + 31) & ~31, yp = (std::max(d, p.m) + 31) & ~31;
  auto smem_for = [&](int tvv) {
    return static_cast<size_t>(tvv) * (dp + yp) * 4 + 32 * 132 * 4 + static_cast<size_t>(tvv) * 12 +
           static_cast<size_t>(tvv) * d + 16;
  };
  // a few vectors (a decode step's append) spread over more CTAs
  int tv = n <= 16 * 148 ? 8 : 32;
  while (tv > 8 && smem_for(tv) > 200 * 1024) tv -= 8;
  if (smem_for(tv) > 220 * 1024) return fail(TQ_ERR_UNSUPPORTED, "d = %d too large for the general quantize kernel", d);
  p.tv = tv;
  const size_t smem = smem_for(tv);
  cudaError_t e = cudaFuncSetAttribute(simt_quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "simt quantize attribute");
  const int64_t blocks = (n + tv - 1) / tv;
  if (blocks > 0x7fffffff) return fail(TQ_ERR_INVALID_ARG, "n too large");
  simt_quantize_kernel<<<static_cast<unsigned>(blocks), kSimtThreads, smem, stream>>>(p);
  e = cudaGetLastError();
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "simt quantize launch");
}

// ---- decode planning ----
struct DecodePlan {
  int chunk_len, n_chunks, qb_stride;
  size_t off_qa, off_qb, off_qs, off_ml, off_o, bytes;
};

// Spectral records the bulk-copy staged decode kernel reads: 1-bit tails and one head word.
bool spectral_tma(const tq_quantizer* q) {
  return q->kind == TQ_KIND_SPECTRAL && q->tail_bits == 1 && q->k_top <= TQ_MAX_TOP &&
         spectral_head_bits(q) <= 32;
}

DecodePlan plan_decode(const tq_quantizer* kq, int B, int Hq, int Hkv, int64_t Nmax, bool causal = false) {
  DecodePlan P{};
  const int D = kq->d;
  const int64_t units = static_cast<int64_t>(B) * Hkv;
  const int64_t sms = sm_count();
  int64_t nch, cl;
  if (kq->kind != TQ_KIND_SPECTRAL || spectral_tma(kq)) {
    // persistent bulk-copy kernel: chunks of whole stages and (when the shape allows) an
    // item count that is a multiple of the SMs; a work item covers one GQA group of up to
    // 4 heads (packed columns) or one block of up to 8 heads
    const int kf = kq->kind == TQ_KIND_PROD ? KFMT_PROD : (kq->kind == TQ_KIND_SPECTRAL ? KFMT_SPEC : KFMT_MSE);
    const int64_t stage = tma_stage_tokens(kf, Hq / Hkv <= 4 && !causal);
    const int64_t wu = units * tma_head_blocks(Hq / Hkv);
    // at most ~16 items per SM, and items of at least ~4 stages when the context is short
    // (each item ends in a cross-warp merge and writes one partial per head)
    const int64_t stages_total = wu * ((Nmax + stage - 1) / stage);
    const int64_t want = std::max<int64_t>(sms, std::min<int64_t>(16 * sms, stages_total / 4));
    int64_t n0 = std::max<int64_t>(1, (want + wu - 1) / wu);
    for (int64_t cand = n0; cand < n0 + 8 && cand <= Nmax; ++cand)
      if ((wu * cand) % sms == 0) { n0 = cand; break; }
    cl = (Nmax + n0 - 1) / n0;
    cl = std::max<int64_t>(stage, (cl + stage - 1) / stage * stage);
    nch = (Nmax + cl - 1) / cl;
  } else {
    const int64_t target = sms * 6;
    nch = std::max<int64_t>(1, (target + units - 1) / units);
    cl = (Nmax + nch - 1) / nch;
    cl = std::max<int64_t>(256, (cl + 63) / 64 * 64);
    nch = (Nmax + cl - 1) / cl;
  }
  P.chunk_len = static_cast<int>(cl);
  P.n_chunks = static_cast<int>(nch);
  P.qb_stride = kq->kind == TQ_KIND_PROD ? kq->m : 16;
  const size_t rows = static_cast<size_t>(B) * Hq;
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t off = 0;
  P.off_qa = off; off = al(off + rows * D * 4);
  P.off_qb = off; off = al(off + rows * P.qb_stride * 4);
  P.off_qs = off; off = al(off + rows * 2 * 4);
  P.off_ml = off; off = al(off + rows * nch * 2 * 4);
  P.off_o = off; off = al(off + rows * nch * D * 4);
  P.bytes = off;
  return P;
}

tq_status check_decode_shape(const tq_quantizer* kq, const tq_quantizer* vq, int B, int Hq, int Hkv, int64_t Nmax,
                             int max_group = 16) {
  tq_status s = check_quantizer(kq);
  if (s != TQ_OK) return s;
  if ((s = check_quantizer(vq)) != TQ_OK) return s;
  if (B < 1 || Hkv < 1 || Hq < 1 || Nmax < 1) return fail(TQ_ERR_INVALID_ARG, "B, Hq, Hkv, Nmax must be >= 1");
  if (Hq % Hkv) return fail(TQ_ERR_INVALID_ARG, "Hq must be a multiple of Hkv");
  if (kq->d != vq->d) return fail(TQ_ERR_INVALID_ARG, "key and value d differ");
  if (Nmax > (1ll << 30)) return fail(TQ_ERR_INVALID_ARG, "Nmax too large");
  if (static_cast<int64_t>(B) * Hkv > 65535) return fail(TQ_ERR_UNSUPPORTED, "B*Hkv > 65535");
  if (kq->d != 128) return fail(TQ_ERR_UNSUPPORTED, "decode attention runs d = 128 only");
  if (Hq / Hkv > max_group) return fail(TQ_ERR_UNSUPPORTED, "Hq/Hkv > %d", max_group);
  if (vq->kind == TQ_KIND_PROD && (vq->m != 128 || vq->bits < 2 || vq->bits > 5 || !vq->S))
    return fail(TQ_ERR_UNSUPPORTED, "PROD values need m = d and 2..5 bits");
  if (vq->kind == TQ_KIND_SPECTRAL && vq->qjl) return fail(TQ_ERR_UNSUPPORTED, "spectral values with qjl");
  if ((kq->kind == TQ_KIND_SPECTRAL) != (vq->kind == TQ_KIND_SPECTRAL))
    return fail(TQ_ERR_UNSUPPORTED, "spectral keys need spectral values (and the reverse)");
  if (kq->kind == TQ_KIND_PROD && (kq->m != 128 || kq->bits < 2 || kq->bits > 5))
    return fail(TQ_ERR_UNSUPPORTED, "PROD keys need m = d and 2..5 bits");
  if (kq->kind == TQ_KIND_MSE && kq->bits > 4) return fail(TQ_ERR_UNSUPPORTED, "key bits > 4");
  if (vq->kind == TQ_KIND_MSE && vq->bits > 4) return fail(TQ_ERR_UNSUPPORTED, "value bits > 4");
  if (kq->kind == TQ_KIND_SPECTRAL && (kq->tail_bits > 2 || kq->tail_bits != vq->tail_bits))
    return fail(TQ_ERR_UNSUPPORTED, "spectral tail bits must be equal and <= 2");
  return TQ_OK;
}

// ---- wide vectors on the tensor cores (split-precision products, workspace) ----

// fp32 input, d a multiple of 128 (<= 4096): MSE with 1..4 bits, or PROD with 2..5 bits and m = d.
bool wide_supported(const tq_quantizer* q, int dtype) {
  if (dtype != TQ_F32 || q->d < 128 || q->d % 128 || q->d > 4096) return false;
  if (q->kind == TQ_KIND_MSE) return q->bits >= 1 && q->bits <= 4;
  if (q->kind == TQ_KIND_PROD) return q->bits >= 2 && q->bits <= 5 && q->m == q->d && q->S;
  return false;
}

constexpr int64_t kWideBatch = 32768;     // vectors per pass of the workspace

struct WidePlan {
  size_t pi, s, xh, xl, rh, rl, nx, r2, bytes;
  int64_t nb;
};

WidePlan plan_wide(const tq_quantizer* q, int64_t n) {
  WidePlan P{};
  const int64_t d = q->d, m = q->kind == TQ_KIND_PROD ? q->m : 0;
  P.nb = std::max<int64_t>(1, std::min<int64_t>(n, kWideBatch));
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t off = 0;
  P.pi = off; off = al(off + 2 * d * d * 2);
  P.s = off; off = al(off + 2 * m * d * 2);
  P.xh = off; off = al(off + P.nb * d * 2);
  P.xl = off; off = al(off + P.nb * d * 2);
  P.rh = off; off = al(off + (m ? P.nb * d * 2 : 0));
  P.rl = off; off = al(off + (m ? P.nb * d * 2 : 0));
  P.nx = off; off = al(off + P.nb * 4);
  P.r2 = off; off = al(off + P.nb * (d / gemm_tile_n(static_cast<int>(d))) * 4);
  P.bytes = off;
  return P;
}

// 2D bf16 tensor map of a row-major [rows][cols] array with a 64-column x box_rows box.
tq_status bf16_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int box_rows) {
  auto encode = get_encode();
  if (!encode) return fail(TQ_ERR_UNSUPPORTED, "tensor maps unavailable");
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(cols * 2)};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TQ_OK : fail(TQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
}

tq_status quantize_wide(const tq_quantizer* q, const float* x, int64_t n, tq_packed out, char* ws,
                        cudaStream_t stream) {
  const WidePlan P = plan_wide(q, n);
  const int d = q->d;
  const bool prod = q->kind == TQ_KIND_PROD;
  const int m = prod ? q->m : 0;
  const int bmse = prod ? q->bits - 1 : q->bits;
  const tq_layout L = layout_of(q);
  auto u16 = [&](size_t off) { return reinterpret_cast<uint16_t*>(ws + off); };
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  // rotation (and S) split once per call
  cudaError_t e = launch_split_rows(q->rot, d, d, u16(P.pi), u16(P.pi) + static_cast<size_t>(d) * d, nullptr, stream);
  if (e == cudaSuccess && prod)
    e = launch_split_rows(q->S, m, d, u16(P.s), u16(P.s) + static_cast<size_t>(m) * d, nullptr, stream);
  if (e != cudaSuccess) return cuda_fail(e, "split launch");
  CUtensorMap pimaps[2], smaps[2];
  tq_status s;
  // B operands: one box is one column tile of the product (the kernel's B stage)
  if ((s = bf16_map(&pimaps[0], u16(P.pi), d, d, gemm_tile_n(d))) != TQ_OK) return s;
  if ((s = bf16_map(&pimaps[1], u16(P.pi) + static_cast<size_t>(d) * d, d, d, gemm_tile_n(d))) != TQ_OK) return s;
  if (prod) {
    if ((s = bf16_map(&smaps[0], u16(P.s), m, d, gemm_tile_n(m))) != TQ_OK) return s;
    if ((s = bf16_map(&smaps[1], u16(P.s) + static_cast<size_t>(m) * d, m, d, gemm_tile_n(m))) != TQ_OK) return s;
  }
  int* status = device_status_ptr();
  for (int64_t v0 = 0; v0 < n; v0 += P.nb) {
    const int64_t nb = std::min<int64_t>(P.nb, n - v0);
    e = launch_split_rows(x + v0 * d, nb, d, u16(P.xh), u16(P.xl), f32(P.nx), stream);
    if (e != cudaSuccess) return cuda_fail(e, "split launch");
    CUtensorMap maps[4];
    if ((s = bf16_map(&maps[0], u16(P.xh), nb, d, 128)) != TQ_OK) return s;
    if ((s = bf16_map(&maps[1], u16(P.xl), nb, d, 128)) != TQ_OK) return s;
    maps[2] = pimaps[0];
    maps[3] = pimaps[1];
    SplitGemmParams g{};
    g.M = nb; g.N = d; g.K = d; g.status = status; g.wait_limit = wait_limit();
    g.rnorm_x = f32(P.nx); g.boundaries = q->boundaries; g.centroids = q->centroids;
    g.codes = out.codes + v0 * L.code_words; g.code_words = L.code_words;
    g.norms = out.norms + v0;
    if (prod) { g.r_hi = u16(P.rh); g.r_lo = u16(P.rl); g.r2_part = f32(P.r2); }
    const int64_t work = (nb + 127) / 128 * (d / gemm_tile_n(d));
    const int grid = static_cast<int>(std::min<int64_t>(work, sm_count()));
    e = launch_split_gemm(maps, g, GEMM_EPI_QUANT, bmse, grid, stream);
    if (e != cudaSuccess) return cuda_fail(e, "wide rotation launch");
    if (!prod) continue;
    if ((s = bf16_map(&maps[0], u16(P.rh), nb, d, 128)) != TQ_OK) return s;
    if ((s = bf16_map(&maps[1], u16(P.rl), nb, d, 128)) != TQ_OK) return s;
    maps[2] = smaps[0];
    maps[3] = smaps[1];
    SplitGemmParams z{};
    z.M = nb; z.N = m; z.K = d; z.status = status; z.wait_limit = wait_limit();
    z.signs = out.signs + v0 * L.sign_words; z.rnorms = out.rnorms + v0;
    z.r2_in = f32(P.r2); z.r2_chunks = d / gemm_tile_n(d);
    const int64_t zwork = (nb + 127) / 128 * (m / gemm_tile_n(m));
    e = launch_split_gemm(maps, z, GEMM_EPI_SIGNS, 1, static_cast<int>(std::min<int64_t>(zwork, sm_count())), stream);
    if (e != cudaSuccess) return cuda_fail(e, "wide projection launch");
  }
  return TQ_OK;
}

// One attention step over the packed cache, shared by the decode entry points and the
// causal prefill (whose query rows are the (head, position) pairs of a block: Hq counts
// rows per sequence, T the positions per head).
struct DecodeCall {
  const tq_quantizer* kq;
  const tq_quantizer* vq;
  const void* q;
  int dtype, B, Hq, Hkv;
  int64_t Nmax;
  const int32_t* seq_lens;
  tq_packed kc, vc;
  float scale;
  float* out;
  void* ws;
  size_t ws_bytes;
  cudaStream_t stream;
  const tq_pages* pages;     // paged pool, or nullptr
  const void* k_new;         // paged append (decode), or nullptr
  const void* v_new;
  const int32_t* q_pos;      // causal rows (prefill), or nullptr
  int T;
};

tq_status check_pages(const tq_pages* pg) {
  if (!pg || !pg->block_table) return fail(TQ_ERR_INVALID_ARG, "pages or block_table is NULL");
  if (!aligned16(pg->block_table)) return fail(TQ_ERR_ALIGNMENT, "block_table not 16-byte aligned");
  if (pg->page_size < 16 || pg->page_size % 16) return fail(TQ_ERR_INVALID_ARG, "page_size must be a multiple of 16");
  if (pg->max_pages < 1 || pg->num_pages < 1) return fail(TQ_ERR_INVALID_ARG, "max_pages and num_pages must be >= 1");
  if (static_cast<int64_t>(pg->max_pages) * pg->page_size > (1ll << 30))
    return fail(TQ_ERR_INVALID_ARG, "max_pages * page_size too large");
  if (pg->num_pages > (1ll << 31) - 1) return fail(TQ_ERR_INVALID_ARG, "num_pages too large");
  return TQ_OK;
}

tq_status decode_run(const DecodeCall& c) {
  const tq_quantizer* kq = c.kq;
  const tq_quantizer* vq = c.vq;
  const void* q = c.q;
  const int dtype = c.dtype, B = c.B, Hq = c.Hq, Hkv = c.Hkv;
  const int64_t Nmax = c.Nmax;
  const int32_t* seq_lens = c.seq_lens;
  const tq_packed kc = c.kc, vc = c.vc;
  const float scale = c.scale;
  float* out = c.out;
  void* workspace = c.ws;
  const size_t ws_bytes = c.ws_bytes;
  cudaStream_t stream = c.stream;
  const bool causal = c.q_pos != nullptr;
  tq_status s = check_decode_shape(kq, vq, B, Hq, Hkv, Nmax, causal ? (1 << 30) : 16);
  if (s != TQ_OK) return s;
  if ((c.pages || causal) && (kq->kind == TQ_KIND_SPECTRAL || vq->kind == TQ_KIND_SPECTRAL))
    return fail(TQ_ERR_UNSUPPORTED, "paged and causal attention take MSE or PROD keys and MSE or PROD values");
  if (causal && vq->kind == TQ_KIND_PROD) return fail(TQ_ERR_UNSUPPORTED, "causal attention takes MSE values");
  if (causal && c.q_pos && !aligned16(c.q_pos)) return fail(TQ_ERR_ALIGNMENT, "q_pos alignment");
  if (dtype < TQ_F32 || dtype > TQ_F16) return fail(TQ_ERR_INVALID_ARG, "unknown dtype");
  if (!q || !seq_lens || !out) return fail(TQ_ERR_INVALID_ARG, "NULL q, seq_lens or out");
  if (!aligned16(q) || !aligned16(seq_lens) || !aligned16(out)) return fail(TQ_ERR_ALIGNMENT, "q/seq_lens/out alignment");
  if (!std::isfinite(scale)) return fail(TQ_ERR_INVALID_ARG, "scale must be finite");
  if (!(kq->lut_scale >= 0.f) || !(vq->lut_scale >= 0.f) || !std::isfinite(kq->lut_scale) || !std::isfinite(vq->lut_scale))
    return fail(TQ_ERR_INVALID_ARG, "lut_scale must be finite and >= 0");
  const tq_layout LK = layout_of(kq), LV = layout_of(vq);
  if ((s = check_packed(kc, LK)) != TQ_OK) return s;
  if ((s = check_packed(vc, LV)) != TQ_OK) return s;
  const DecodePlan P = plan_decode(kq, B, Hq, Hkv, Nmax, causal);
  if (!workspace || ws_bytes < P.bytes) return fail(TQ_ERR_WORKSPACE, "workspace needs %zu bytes", P.bytes);
  if (!aligned16(workspace)) return fail(TQ_ERR_ALIGNMENT, "workspace not 16-byte aligned");
  const int64_t recs = c.pages ? c.pages->num_pages * Hkv * c.pages->page_size : static_cast<int64_t>(B) * Hkv * Nmax;
  Range ins[14];
  packed_ranges(kc, LK, recs, ins);
  packed_ranges(vc, LV, recs, ins + 4);
  ins[8] = {q, static_cast<size_t>(B) * Hq * kq->d * dtype_size(dtype)};
  ins[9] = {seq_lens, static_cast<size_t>(B) * 4};
  ins[10] = {workspace, ws_bytes};
  int n_ins = 11;
  if (c.pages) ins[n_ins++] = {c.pages->block_table, static_cast<size_t>(B) * c.pages->max_pages * 4};
  if (causal) ins[n_ins++] = {c.q_pos, static_cast<size_t>(B) * c.T * 4};
  const Range outs[1] = {{out, static_cast<size_t>(B) * Hq * kq->d * 4}};
  if ((s = check_no_alias(outs, 1, ins, n_ins)) != TQ_OK) return s;

  if (c.k_new) {
    // the step's own token: quantized into its slot of the pool before the attention reads it
    const PagedOut po{c.pages, seq_lens, Hkv};
    const Range news[2] = {{c.k_new, static_cast<size_t>(B) * Hkv * kq->d * dtype_size(dtype)},
                           {c.v_new, static_cast<size_t>(B) * Hkv * kq->d * dtype_size(dtype)}};
    if ((s = check_no_alias(outs, 1, news, 2)) != TQ_OK) return s;
    Range vouts[4];
    packed_ranges(vc, LV, recs, vouts);
    s = quantize_common(kq, c.k_new, dtype, static_cast<int64_t>(B) * Hkv, kc, stream, kq->kind, kq->d, nullptr,
                        vouts, 4, &po);
    if (s != TQ_OK) return s;
    Range kouts[4];
    packed_ranges(kc, LK, recs, kouts);
    s = quantize_common(vq, c.v_new, dtype, static_cast<int64_t>(B) * Hkv, vc, stream, vq->kind, vq->d, nullptr,
                        kouts, 4, &po);
    if (s != TQ_OK) return s;
  }

  const int D = kq->d, G = Hq / Hkv, rows = B * Hq;
  char* ws = static_cast<char*>(workspace);
  float* qa = reinterpret_cast<float*>(ws + P.off_qa);
  float* qb = reinterpret_cast<float*>(ws + P.off_qb);
  float* qs = reinterpret_cast<float*>(ws + P.off_qs);
  float* pml = reinterpret_cast<float*>(ws + P.off_ml);
  float* po = reinterpret_cast<float*>(ws + P.off_o);

  QPrepParams qp{};
  qp.q = q; qp.dtype = dtype; qp.rows = rows; qp.D = D; qp.kind = kq->kind;
  qp.scale = scale * kLog2e;
  qp.rot = kq->rot; qp.S = kq->S; qp.m = kq->m;
  qp.dim_sigma = kq->dim_sigma; qp.k_top = kq->k_top; qp.qjl = kq->qjl;
  qp.spec_coef = static_cast<float>(std::sqrt(M_PI / 2.0) / std::max(1, kq->k_top));
  qp.qa = qa; qp.qb = qb; qp.qs = qs; qp.qb_stride = P.qb_stride;
  const size_t qsm = static_cast<size_t>(2 * D + std::max(D, P.qb_stride)) * 4;
  if (D == 128 && (kq->kind != TQ_KIND_SPECTRAL || kq->k_top <= 8))
    qprep128_kernel<<<(rows + 7) / 8, 256, 0, stream>>>(qp);
  else
    qprep_kernel<<<rows, 128, qsm, stream>>>(qp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "qprep launch");

  DecodeParams dp{};
  dp.B = B; dp.Hq = Hq; dp.Hkv = Hkv; dp.G = G; dp.Nmax = Nmax;
  dp.chunk_len = P.chunk_len; dp.n_chunks = P.n_chunks; dp.seq_lens = seq_lens;
  dp.kcodes = kc.codes; dp.k_words = LK.code_words; dp.ksigns = kc.signs; dp.k_sign_words = LK.sign_words;
  dp.knorms = kc.norms; dp.krnorms = kc.rnorms;
  dp.vcodes = vc.codes; dp.v_words = LV.code_words; dp.vnorms = vc.norms;
  dp.unit_c = kq->kind == TQ_KIND_SPECTRAL ? kq->unit_centroids : nullptr;
  int kfmt, kb, vfmt, vb;
  if (kq->kind == TQ_KIND_SPECTRAL) {
    kfmt = KFMT_SPEC; kb = kq->tail_bits;
    dp.k_code_off = (spectral_head_bits(kq) + 31) / 32;
    dp.kc = kq->unit_centroids + unit_c_off(kb);
    dp.k_top_k = kq->k_top; dp.k_qjl = kq->qjl;
    for (int j = 0; j < TQ_MAX_TOP; ++j) dp.k_top_bits[j] = kq->top_bits[j];
  } else {
    kfmt = kq->kind == TQ_KIND_PROD ? KFMT_PROD : KFMT_MSE;
    kb = kq->kind == TQ_KIND_PROD ? kq->bits - 1 : kq->bits;
    dp.k_code_off = 0;
    dp.kc = kq->centroids;
  }
  if (vq->kind == TQ_KIND_SPECTRAL) {
    vfmt = VFMT_SPEC; vb = vq->tail_bits;
    dp.v_code_off = (spectral_head_bits(vq) + 31) / 32;
    dp.vc = vq->unit_centroids + unit_c_off(vb);
    dp.v_top = vq->k_top;
    for (int j = 0; j < TQ_MAX_TOP; ++j) dp.v_top_bits[j] = vq->top_bits[j];
    if (!dp.unit_c) dp.unit_c = vq->unit_centroids;
  } else if (vq->kind == TQ_KIND_PROD) {
    vfmt = VFMT_PROD; vb = vq->bits - 1;
    dp.v_code_off = 0;
    dp.vc = vq->centroids;
    dp.vsigns = vc.signs; dp.vrnorms = vc.rnorms; dp.vS = vq->S;
    dp.v_coef = static_cast<float>(std::sqrt(M_PI / 2.0) / vq->m);
  } else {
    vfmt = VFMT_MSE; vb = vq->bits;
    dp.v_code_off = 0;
    dp.vc = vq->centroids;
  }
  dp.qa = qa; dp.qb = qb; dp.qs = qs; dp.qb_stride = P.qb_stride;
  dp.qjl_coef = kq->kind == TQ_KIND_PROD ? static_cast<float>(std::sqrt(M_PI / 2.0) / kq->m) : 0.f;
  dp.k_scale = kq->lut_scale > 0.f ? kq->lut_scale : 1.f;
  dp.v_scale = vq->lut_scale > 0.f ? vq->lut_scale : 1.f;
  dp.part_ml = pml; dp.part_o = po;
  const int64_t items = static_cast<int64_t>(B) * Hkv * tma_head_blocks(G) * P.n_chunks;
  const bool spec_tma = kfmt == KFMT_SPEC && spectral_tma(kq);   // the plan follows the keys
  if (spec_tma && !spectral_tma(vq))
    return fail(TQ_ERR_UNSUPPORTED, "spectral values need a head of at most 32 bits with 1-bit-tail keys");
  const dim3 grid = (kfmt == KFMT_SPEC && !spec_tma)
                        ? dim3(static_cast<unsigned>(P.n_chunks), static_cast<unsigned>(B * Hkv))
                        : dim3(static_cast<unsigned>(std::min<int64_t>(items, sm_count())));
  const size_t smem = decode_smem_bytes(D, kb, vb);
  if (c.pages) {
    dp.block_table = c.pages->block_table; dp.page = c.pages->page_size; dp.max_pages = c.pages->max_pages;
    dp.num_pages = c.pages->num_pages;
  }
  if (causal) { dp.q_pos = c.q_pos; dp.T = c.T; }
  if (spec_tma)
    e = launch_decode_spec_tma(dp, grid, stream, device_status_ptr(), wait_limit());
  else if (causal)
    e = launch_decode_causal(dp, kfmt, kb, vb, grid, stream, device_status_ptr(), wait_limit());
  else
    e = launch_decode(dp, kfmt, kb, vfmt, vb, grid, smem, stream, device_status_ptr(), wait_limit());
  if (e == cudaErrorNotSupported) return fail(TQ_ERR_UNSUPPORTED, "decode variant not built (kbits %d, vbits %d)", kb, vb);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");

  CombineParams cp{};
  cp.rows = rows; cp.D = D; cp.n_chunks = P.n_chunks;
  cp.part_ml = pml; cp.part_o = po; cp.rot_v = vq->rot;
  cp.v_sigma = vq->kind == TQ_KIND_SPECTRAL ? vq->dim_sigma : nullptr;
  cp.out = out;
  // combine128: weights of 2 rows, then rot_V (64 KB); both combines wait on the decode
  // kernel inside (programmatic launch: their launch overlaps its tail)
  const size_t csm = static_cast<size_t>((2 * P.n_chunks + 3) & ~3) * 4 + 128 * 128 * 4;
  if (D == 128 && csm <= 200 * 1024) {
    e = cudaFuncSetAttribute(combine128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(csm));
    if (e != cudaSuccess) return cuda_fail(e, "combine attribute");
    e = launch_pdl(combine128_kernel, dim3(static_cast<unsigned>((rows + 1) / 2)), dim3(256), csm, stream, cp);
  } else {
    e = launch_pdl(combine_kernel, dim3(static_cast<unsigned>(rows)), dim3(128), static_cast<size_t>(D) * 4, stream, cp);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "combine launch");
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" {

const char* tq_version(void) { return "libtq 0.1 (sm_100a)"; }

const char* tq_last_error(void) { return g_msg; }

tq_status tq_codebook_build(int32_t d, int32_t bits, int32_t dist, double sigma, double* centroids,
                            double* boundaries, int32_t* iterations) {
  int it = 0;
  const tq_status s = codebook_build(d, bits, dist, sigma, centroids, boundaries, &it);
  if (iterations) *iterations = it;
  return s;
}

tq_status tq_waterfill(const double* lambda, int32_t k, int32_t budget_bits, int32_t max_bits, int32_t* bits_out) {
  return waterfill(lambda, k, budget_bits, max_bits, bits_out);
}

tq_status tq_spectral_calibrate(const float* X, int64_t n, int32_t d, double* eigvecs_out, double* eigvals_out) {
  return spectral_calibrate(X, n, d, eigvecs_out, eigvals_out);
}

tq_status tq_spectral_unit_codebooks(double* centroids_out, double* boundaries_out) {
  return spectral_unit_codebooks(centroids_out, boundaries_out);
}

tq_status tq_lut_scale(const double* values, int32_t count, float* scale_out) {
  return lut_scale(values, count, scale_out);
}

tq_status tq_spectral_descriptor(const double* eigvecs, const double* eigvals, int32_t d, int32_t k_top,
                                 int32_t budget_bits, int32_t tail_bits, int32_t max_bits, float* rot_out,
                                 float* dim_sigma_out, float* unit_centroids_out, float* unit_boundaries_out,
                                 int32_t* top_bits_out, float* lut_scale_out) {
  return spectral_descriptor(eigvecs, eigvals, d, k_top, budget_bits, tail_bits, max_bits, rot_out, dim_sigma_out,
                             unit_centroids_out, unit_boundaries_out, top_bits_out, lut_scale_out);
}

tq_status tq_spectral_prepare(const float* X, int64_t n, int32_t d, int32_t k_top, int32_t budget_bits,
                              int32_t tail_bits, int32_t max_bits, float* rot_out, float* dim_sigma_out,
                              float* unit_centroids_out, float* unit_boundaries_out, int32_t* top_bits_out,
                              float* lut_scale_out, double* eigvals_out) {
  if (d < 2 || d > 1024) return fail(TQ_ERR_INVALID_ARG, "spectral prepare: d out of range");
  std::vector<double> vecs(static_cast<size_t>(d) * d), vals(d);
  tq_status s = spectral_calibrate(X, n, d, vecs.data(), vals.data());
  if (s != TQ_OK) return s;
  if (eigvals_out)
    for (int j = 0; j < d; ++j) eigvals_out[j] = vals[j];
  return spectral_descriptor(vecs.data(), vals.data(), d, k_top, budget_bits, tail_bits, max_bits, rot_out,
                             dim_sigma_out, unit_centroids_out, unit_boundaries_out, top_bits_out, lut_scale_out);
}

tq_status tq_record_layout(const tq_quantizer* q, tq_layout* out) {
  const tq_status s = check_quantizer(q);
  if (s != TQ_OK) return s;
  if (!out) return fail(TQ_ERR_INVALID_ARG, "layout output is NULL");
  *out = layout_of(q);
  return TQ_OK;
}

tq_status tq_quantize_mse(const tq_quantizer* q, const void* x, int32_t dtype, int64_t n, tq_packed out,
                          tq_stream stream) {
  return quantize_common(q, x, dtype, n, out, reinterpret_cast<cudaStream_t>(stream), TQ_KIND_MSE,
                         q ? q->d : 0, nullptr);
}

tq_status tq_quantize_prod(const tq_quantizer* q, const void* x, int32_t dtype, int64_t n, tq_packed out,
                           tq_stream stream) {
  return quantize_common(q, x, dtype, n, out, reinterpret_cast<cudaStream_t>(stream), TQ_KIND_PROD,
                         q ? q->d : 0, nullptr);
}

tq_status tq_quantize_spectral(const tq_quantizer* q, const void* x, int32_t dtype, int64_t n, tq_packed out,
                               tq_stream stream) {
  return quantize_common(q, x, dtype, n, out, reinterpret_cast<cudaStream_t>(stream), TQ_KIND_SPECTRAL,
                         q ? q->d : 0, nullptr);
}

tq_status tq_quantize_workspace(const tq_quantizer* q, int32_t dtype, int64_t n, size_t* bytes) {
  tq_status s = check_quantizer(q);
  if (s != TQ_OK) return s;
  if (!bytes || n < 0) return fail(TQ_ERR_INVALID_ARG, "bad workspace query");
  *bytes = wide_supported(q, dtype) && n > 0 ? plan_wide(q, n).bytes : 0;
  return TQ_OK;
}

tq_status tq_quantize_ws(const tq_quantizer* q, const void* x, int32_t dtype, int64_t n, tq_packed out,
                         void* workspace, size_t ws_bytes, tq_stream stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  tq_status s = check_quantizer(q);
  if (s != TQ_OK) return s;
  if (q->kind == TQ_KIND_SPECTRAL || n <= 0 || !wide_supported(q, dtype))
    return quantize_common(q, x, dtype, n, out, stream, q->kind, q->d, nullptr);
  if (q->kind == TQ_KIND_PROD && q->bits > 1 && (!q->centroids || !q->boundaries))
    return fail(TQ_ERR_INVALID_ARG, "codebook is NULL");
  if (!x) return fail(TQ_ERR_INVALID_ARG, "x is NULL");
  if (!aligned16(x)) return fail(TQ_ERR_ALIGNMENT, "x is not 16-byte aligned");
  const tq_layout L = layout_of(q);
  if ((s = check_packed(out, L)) != TQ_OK) return s;
  const WidePlan P = plan_wide(q, n);
  if (!workspace || ws_bytes < P.bytes) return fail(TQ_ERR_WORKSPACE, "workspace needs %zu bytes", P.bytes);
  if (!aligned16(workspace)) return fail(TQ_ERR_ALIGNMENT, "workspace not 16-byte aligned");
  Range outs[4];
  packed_ranges(out, L, n, outs);
  const Range ins[2] = {{x, static_cast<size_t>(n) * q->d * 4}, {workspace, ws_bytes}};
  if ((s = check_no_alias(outs, 4, ins, 2)) != TQ_OK) return s;
  return quantize_wide(q, static_cast<const float*>(x), n, out, static_cast<char*>(workspace), stream);
}

tq_status tq_dequantize(const tq_quantizer* q, tq_packed in, int64_t n, float* out, tq_stream stream) {
  tq_status s = check_quantizer(q);
  if (s != TQ_OK) return s;
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, "n < 0");
  if (n == 0) return TQ_OK;
  if (n > 0x7fffffff) return fail(TQ_ERR_INVALID_ARG, "n too large");
  if (!out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
  if (!aligned16(out)) return fail(TQ_ERR_ALIGNMENT, "out is not 16-byte aligned");
  const tq_layout L = layout_of(q);
  if ((s = check_packed(in, L)) != TQ_OK) return s;
  Range ins[4];
  packed_ranges(in, L, n, ins);
  const Range outs[1] = {{out, static_cast<size_t>(n) * q->d * 4}};
  if ((s = check_no_alias(outs, 1, ins, 4)) != TQ_OK) return s;
  DequantParams p{};
  p.kind = q->kind; p.d = q->d; p.m = q->m;
  p.bmse = q->kind == TQ_KIND_MSE ? q->bits : (q->kind == TQ_KIND_PROD ? q->bits - 1 : 0);
  p.rot = q->rot; p.S = q->S; p.centroids = q->centroids;
  p.codes = in.codes; p.code_words = L.code_words;
  p.signs = in.signs; p.sign_words = L.sign_words;
  p.norms = in.norms; p.rnorms = in.rnorms;
  p.k_top = q->k_top; p.tail_bits = q->tail_bits; p.qjl = q->qjl;
  for (int j = 0; j < TQ_MAX_TOP; ++j) p.top_bits[j] = q->top_bits[j];
  p.dim_sigma = q->dim_sigma; p.unit_c = q->unit_centroids;
  p.out = out; p.n = n;
  const size_t smem = static_cast<size_t>(q->d) * 4;
  dequant_kernel<<<static_cast<unsigned>(n), kSimtThreads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "dequantize launch");
}

static int64_t score_block(int64_t nq, int64_t n) {
  int64_t qb = (1ll << 28) / (4 * std::max<int64_t>(n, 1));
  qb = std::max<int64_t>(8, std::min<int64_t>(1024, qb)) / 8 * 8;
  return std::min<int64_t>(qb, (nq + 7) / 8 * 8);
}

static int score_qu_stride(const tq_quantizer* q) {
  if (q->kind == TQ_KIND_PROD) return q->m;
  if (q->kind == TQ_KIND_SPECTRAL && q->qjl) return q->k_top;
  return 0;
}

// Estimates on the tensor cores: MSE (1..4 bits) or PROD (2..5 bits, m = d) records with d a
// multiple of 128, against at least 4096 records.  Queries [q' | S q'] and decoded records
// [c[code] | sqrt(pi/2)/m gamma (2s - 1)] become split-precision operands of one product;
// the column scale is the record norm.
static bool score_wide(const tq_quantizer* q, int64_t n) {
  if (q->d < 128 || q->d % 128 || q->d > 4096 || n < 4096 || std::getenv("TQ_FORCE_SIMT")) return false;
  if (q->kind == TQ_KIND_MSE) return q->bits >= 1 && q->bits <= 4;
  if (q->kind == TQ_KIND_PROD) return q->bits >= 2 && q->bits <= 5 && q->m == q->d;
  return false;
}

struct ScoreWidePlan {
  size_t qr, qu, ah, al, bh, bl, dense, cand, sym, bytes;
  int64_t qb;
  int K;
  int seg_n;                    // top-k segments per dense row
};

// Top-k over a dense row runs in segments of ~16k estimates (one CTA each), then over the
// segments' candidates.
static int topk_segments(int64_t n) {
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(64, (n + 16383) / 16384)));
}

static ScoreWidePlan plan_score_wide(const tq_quantizer* q, int64_t nq, int64_t n, int topk) {
  ScoreWidePlan P{};
  const int64_t d = q->d, m = q->kind == TQ_KIND_PROD ? q->m : 0;
  P.K = static_cast<int>(d + m);
  int64_t qb = (1ll << 28) / std::max<int64_t>(n, 1) / 128 * 128;
  qb = std::max<int64_t>(128, std::min<int64_t>(1024, qb));
  P.qb = std::min<int64_t>(qb, (nq + 127) / 128 * 128);
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t off = 0;
  P.qr = off; off = al(off + nq * d * 4);
  P.qu = off; off = al(off + nq * std::max<int64_t>(m, 1) * 4);
  P.ah = off; off = al(off + P.qb * P.K * 2);
  P.al = off; off = al(off + P.qb * P.K * 2);
  P.bh = off; off = al(off + n * P.K * 2);
  P.bl = off; off = al(off + n * P.K * 2);
  P.dense = off; off = al(off + (topk > 0 ? P.qb * n * 4 : 0));
  P.seg_n = topk_segments(n);
  P.cand = off; off = al(off + (topk > 0 ? P.qb * P.seg_n * 32 * 8 : 0));   // scores, then ids
  P.sym = off; off = al(off + 4);                  // records expanded as +-1 (int flag)
  P.bytes = off;
  return P;
}

// Estimator parameters of one quantizer's records (the rotated queries and the output are
// filled in per launch).
static ScoreParams score_params(const tq_quantizer* q, const tq_layout& L, const tq_packed& keys, int64_t n) {
  const int qus = score_qu_stride(q);
  ScoreParams p{};
  p.kind = q->kind; p.d = q->d; p.m = qus;
  p.bmse = q->kind == TQ_KIND_MSE ? q->bits : (q->kind == TQ_KIND_PROD ? q->bits - 1 : 0);
  p.codes = keys.codes; p.code_words = L.code_words;
  p.signs = keys.signs; p.sign_words = L.sign_words;
  p.norms = keys.norms; p.rnorms = keys.rnorms;
  p.centroids = q->centroids;
  p.k_top = q->k_top; p.tail_bits = q->tail_bits; p.qjl = q->qjl;
  for (int j = 0; j < TQ_MAX_TOP; ++j) p.top_bits[j] = q->top_bits[j];
  p.head_words = q->kind == TQ_KIND_SPECTRAL ? (spectral_head_bits(q) + 31) / 32 : 0;
  p.dim_sigma = q->dim_sigma; p.unit_c = q->unit_centroids;
  p.coef = q->kind == TQ_KIND_PROD ? static_cast<float>(std::sqrt(M_PI / 2.0) / q->m)
                                   : static_cast<float>(std::sqrt(M_PI / 2.0) / std::max(1, q->k_top));
  p.qu_stride = std::max(qus, 1);
  p.n = n;
  p.accumulate = 0;
  return p;
}

static size_t score_smem(const ScoreParams& p) {
  return static_cast<size_t>(kScoreQT) * (p.d + p.qu_stride) * 4 + 256 * 4;
}

tq_status tq_score_workspace(const tq_quantizer* q, int64_t nq, int64_t n, int32_t topk, size_t* bytes) {
  tq_status s = check_quantizer(q);
  if (s != TQ_OK) return s;
  if (!bytes || nq < 0 || n < 0) return fail(TQ_ERR_INVALID_ARG, "bad workspace query");
  if (score_wide(q, n) && nq > 0) {
    *bytes = plan_score_wide(q, nq, n, topk).bytes;
    return TQ_OK;
  }
  size_t b = static_cast<size_t>(nq) * q->d * 4 + 256;
  b += static_cast<size_t>(nq) * score_qu_stride(q) * 4 + 256;
  if (topk > 0) b += static_cast<size_t>(score_block(nq, n)) * static_cast<size_t>(n) * 4 + 256;
  *bytes = b;
  return TQ_OK;
}

tq_status tq_score(const tq_quantizer* q, const void* qv, int32_t dtype, int64_t nq, tq_packed keys, int64_t n,
                   int32_t topk, float* scores, int32_t* ids, void* workspace, size_t ws_bytes, tq_stream stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  tq_status s = check_quantizer(q);
  if (s != TQ_OK) return s;
  if (dtype < TQ_F32 || dtype > TQ_F16) return fail(TQ_ERR_INVALID_ARG, "unknown dtype");
  if (nq < 0 || n < 0) return fail(TQ_ERR_INVALID_ARG, "nq, n must be >= 0");
  if (topk < 0 || topk > 32) return fail(TQ_ERR_UNSUPPORTED, "topk must be 0..32");
  if (topk > 0 && topk > n) return fail(TQ_ERR_INVALID_ARG, "topk > n");
  if (n > 0x7fffffff || nq > 0x7fffffff) return fail(TQ_ERR_INVALID_ARG, "sizes too large");
  if (nq == 0 || n == 0) return TQ_OK;
  if (!qv || !scores || (topk > 0 && !ids)) return fail(TQ_ERR_INVALID_ARG, "NULL query or output");
  if (!aligned16(qv) || !aligned16(scores) || (ids && !aligned16(ids)))
    return fail(TQ_ERR_ALIGNMENT, "query/output not 16-byte aligned");
  if (q->d > 2048) return fail(TQ_ERR_UNSUPPORTED, "score supports d <= 2048");
  const tq_layout L = layout_of(q);
  if ((s = check_packed(keys, L)) != TQ_OK) return s;
  size_t need = 0;
  tq_score_workspace(q, nq, n, topk, &need);
  if (!workspace || ws_bytes < need) return fail(TQ_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  if (!aligned16(workspace)) return fail(TQ_ERR_ALIGNMENT, "workspace not 16-byte aligned");
  Range ins[6];
  packed_ranges(keys, L, n, ins);
  ins[4] = {qv, static_cast<size_t>(nq) * q->d * dtype_size(dtype)};
  ins[5] = {workspace, ws_bytes};
  Range outs[2] = {{scores, topk > 0 ? static_cast<size_t>(nq) * topk * 4 : static_cast<size_t>(nq) * n * 4},
                   {topk > 0 ? ids : nullptr, static_cast<size_t>(nq) * topk * 4}};
  if ((s = check_no_alias(outs, 2, ins, 6)) != TQ_OK) return s;

  const int d = q->d;
  const int qus = score_qu_stride(q);
  char* ws = static_cast<char*>(workspace);
  if (score_wide(q, n)) {
    const ScoreWidePlan P = plan_score_wide(q, nq, n, topk);
    float* qr = reinterpret_cast<float*>(ws + P.qr);
    float* qu = reinterpret_cast<float*>(ws + P.qu);
    const int m = q->kind == TQ_KIND_PROD ? q->m : 0;
    auto u16 = [&](size_t off) { return reinterpret_cast<uint16_t*>(ws + off); };
    // q' = Pi q and S q' (PROD), fp32
    const size_t mv_smem = static_cast<size_t>(kMvQ) * d * 4;
    cudaError_t e = cudaFuncSetAttribute(rows_matvec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(mv_smem));
    if (e != cudaSuccess) return cuda_fail(e, "query rotation attribute");
    // queries along x (up to 2^31 - 1 blocks), row blocks along y (d <= 4096: at most 128)
    const dim3 mv_grid(static_cast<unsigned>((nq + kMvQ - 1) / kMvQ), static_cast<unsigned>((d + kMvRows - 1) / kMvRows));
    rows_matvec_kernel<<<mv_grid, 128, mv_smem, stream>>>(q->rot, d, d, qv, dtype, nq, d, qr, d);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "query rotation launch");
    if (m) {
      const dim3 sg(mv_grid.x, static_cast<unsigned>((m + kMvRows - 1) / kMvRows));
      rows_matvec_kernel<<<sg, 128, mv_smem, stream>>>(q->S, m, d, qr, TQ_F32, nq, d, qu, qus);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "query projection launch");
    }
    const int bm = q->kind == TQ_KIND_PROD ? q->bits - 1 : q->bits;
    const float coef = m ? static_cast<float>(std::sqrt(M_PI / 2.0) / m) : 0.f;
    int* sym = reinterpret_cast<int*>(ws + P.sym);
    e = launch_expand_records(keys.codes, L.code_words, keys.signs, L.sign_words, keys.rnorms, q->centroids, coef, n,
                              d, m, bm, u16(P.bh), u16(P.bl), sym, stream);
    if (e != cudaSuccess) return cuda_fail(e, "record expansion launch");
    CUtensorMap maps[4];
    const int tn = gemm_tile_n(static_cast<int>(n));      // B box = one column tile
    if ((s = bf16_map(&maps[2], u16(P.bh), n, P.K, tn)) != TQ_OK) return s;
    if ((s = bf16_map(&maps[3], u16(P.bl), n, P.K, tn)) != TQ_OK) return s;
    float* dense = reinterpret_cast<float*>(ws + P.dense);
    for (int64_t q0 = 0; q0 < nq; q0 += P.qb) {
      const int64_t nb = std::min(P.qb, nq - q0);
      e = launch_split_cat(qr + q0 * d, d, qu + q0 * m, m, nb, u16(P.ah), u16(P.al), stream, sym, q->centroids);
      if (e != cudaSuccess) return cuda_fail(e, "query split launch");
      if ((s = bf16_map(&maps[0], u16(P.ah), nb, P.K, 128)) != TQ_OK) return s;
      if ((s = bf16_map(&maps[1], u16(P.al), nb, P.K, 128)) != TQ_OK) return s;
      SplitGemmParams g{};
      g.M = nb; g.N = static_cast<int>(n); g.K = P.K; g.status = device_status_ptr(); g.wait_limit = wait_limit();
      g.out = topk > 0 ? dense : scores + q0 * n; g.ldo = n; g.col_scale = keys.norms;
      g.lo_skip_flag = sym; g.lo_skip_k = d;
      const int64_t work = (nb + 127) / 128 * ((n + tn - 1) / tn);
      e = launch_split_gemm(maps, g, GEMM_EPI_SCORE, 1, static_cast<int>(std::min<int64_t>(work, sm_count())), stream);
      if (e != cudaSuccess) return cuda_fail(e, "estimate launch");
      if (topk > 0) {
        // the segments' best K (pass 1), then the top-k of those candidates (pass 2)
        const int S = P.seg_n;
        const int64_t seg = (n + S - 1) / S;
        float* cs = reinterpret_cast<float*>(ws + P.cand);
        int32_t* ci = reinterpret_cast<int32_t*>(ws + P.cand + static_cast<size_t>(P.qb) * S * 32 * 4);
        const dim3 g1(static_cast<unsigned>(S), static_cast<unsigned>(nb)), g2(1, static_cast<unsigned>(nb));
        if (topk <= 16) {
          topk_seg_kernel<16><<<g1, 128, 0, stream>>>(dense, nullptr, n, seg, 16, cs, ci, 0);
          topk_seg_kernel<16><<<g2, 128, 0, stream>>>(cs, ci, static_cast<int64_t>(S) * 16, static_cast<int64_t>(S) * 16,
                                                      topk, scores, ids, q0);
        } else {
          topk_seg_kernel<32><<<g1, 128, 0, stream>>>(dense, nullptr, n, seg, 32, cs, ci, 0);
          topk_seg_kernel<32><<<g2, 128, 0, stream>>>(cs, ci, static_cast<int64_t>(S) * 32, static_cast<int64_t>(S) * 32,
                                                      topk, scores, ids, q0);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "topk launch");
      }
    }
    return TQ_OK;
  }
  float* qr = reinterpret_cast<float*>(ws);
  float* qu = qus ? reinterpret_cast<float*>(ws + (static_cast<size_t>(nq) * d * 4 + 255) / 256 * 256) : nullptr;
  float* dense = reinterpret_cast<float*>(
      ws + (static_cast<size_t>(nq) * d * 4 + 255) / 256 * 256 + (static_cast<size_t>(nq) * qus * 4 + 255) / 256 * 256);
  score_qprep_kernel<<<static_cast<unsigned>(nq), 128, 2 * d * 4, stream>>>(
      qv, dtype, d, q->kind, q->rot, q->S, q->m, q->k_top, qr, qu, qus, d, nullptr, device_status_ptr());
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "score qprep launch");
  ScoreParams p = score_params(q, L, keys, n);
  const size_t smem = score_smem(p);
  e = cudaFuncSetAttribute(score_dense_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "score attribute");
  const int64_t qb = topk > 0 ? score_block(nq, n) : nq;
  for (int64_t q0 = 0; q0 < nq; q0 += qb) {
    const int64_t nb = std::min(qb, nq - q0);
    p.qr = qr + q0 * d;
    p.qu = qu ? qu + q0 * qus : nullptr;
    p.nq = nb;
    p.out = topk > 0 ? dense : scores + q0 * n;
    const dim3 grid(static_cast<unsigned>((n + kScoreThreads - 1) / kScoreThreads),
                    static_cast<unsigned>((nb + kScoreQT - 1) / kScoreQT));
    if (grid.y > 65535) return fail(TQ_ERR_UNSUPPORTED, "too many queries per block");
    score_dense_kernel<<<grid, kScoreThreads, smem, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "score launch");
    if (topk > 0) {
      if (topk <= 16) topk_kernel<16><<<static_cast<unsigned>(nb), 128, 0, stream>>>(dense, n, topk, q0, scores, ids);
      else topk_kernel<32><<<static_cast<unsigned>(nb), 128, 0, stream>>>(dense, n, topk, q0, scores, ids);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "topk launch");
    }
  }
  return TQ_OK;
}

// ---- outlier-channel split ----
static tq_status check_split(const tq_split* sp) {
  if (!sp) return fail(TQ_ERR_INVALID_ARG, "split descriptor is NULL");
  if (sp->n_groups < 1 || sp->n_groups > TQ_MAX_GROUPS)
    return fail(TQ_ERR_INVALID_ARG, "n_groups must be 1..%d", TQ_MAX_GROUPS);
  int64_t total = 0;
  for (int g = 0; g < sp->n_groups; ++g) {
    const tq_quantizer* q = sp->groups[g];
    const tq_status s = check_quantizer(q);
    if (s != TQ_OK) return s;
    if (q->kind != TQ_KIND_MSE && q->kind != TQ_KIND_PROD)
      return fail(TQ_ERR_UNSUPPORTED, "split groups are MSE or PROD instances");
    if (!sp->cols[g]) return fail(TQ_ERR_INVALID_ARG, "cols[%d] is NULL", g);
    if (reinterpret_cast<uintptr_t>(sp->cols[g]) & 3u) return fail(TQ_ERR_ALIGNMENT, "cols[%d] not 4-byte aligned", g);
    total += q->d;
  }
  if (total != sp->d) return fail(TQ_ERR_INVALID_ARG, "the groups' widths add up to %lld, not d = %d",
                                  static_cast<long long>(total), sp->d);
  return TQ_OK;
}

// The outlier split of the KV experiments on the tensor cores: two MSE groups, 32 channels
// at 3 bits + 96 at 2 (or 4 + 3), 16-bit rows of 128 channels.
static bool umma_split(const tq_split* sp, int dtype, int64_t n) {
  if (sp->d != 128 || sp->n_groups != 2) return false;
  const tq_quantizer* a = sp->groups[0];
  const tq_quantizer* b = sp->groups[1];
  if (a->kind != TQ_KIND_MSE || b->kind != TQ_KIND_MSE || a->d != 32 || b->d != 96) return false;
  if (!((a->bits == 3 && b->bits == 2) || (a->bits == 4 && b->bits == 3))) return false;
  tq_quantizer probe = *a;                        // the hardware and size checks of the d = 128 path
  probe.d = 128;
  probe.bits = 2;
  return umma_supported(&probe, dtype, n);
}

static tq_status quantize_split_umma(const tq_split* sp, const void* x, int dtype, int64_t n, const tq_packed* out,
                                     cudaStream_t stream) {
  tq_status s;
  const tq_layout L0 = layout_of(sp->groups[0]), L1 = layout_of(sp->groups[1]);
  if ((s = check_packed(out[0], L0)) != TQ_OK) return s;
  if ((s = check_packed(out[1], L1)) != TQ_OK) return s;
  if (!x) return fail(TQ_ERR_INVALID_ARG, "x is NULL");
  if (!aligned16(x)) return fail(TQ_ERR_ALIGNMENT, "x is not 16-byte aligned");
  Range outs[8];
  packed_ranges(out[0], L0, n, outs);
  packed_ranges(out[1], L1, n, outs + 4);
  const Range ins[1] = {{x, static_cast<size_t>(n) * 128 * dtype_size(dtype)}};
  if ((s = check_no_alias(outs, 8, ins, 1)) != TQ_OK) return s;     // and the groups' outputs pairwise
  auto encode = get_encode();
  CUtensorMap map;
  const cuuint64_t gdim[2] = {128, static_cast<cuuint64_t>(n)};
  const cuuint64_t gstride[1] = {256};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(&map, dtype == TQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                            2, const_cast<void*>(x), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  UmmaQuantParams p{};
  p.rot = sp->groups[0]->rot; p.rot1 = sp->groups[1]->rot;
  p.cols0 = sp->cols[0]; p.cols1 = sp->cols[1];
  p.boundaries = sp->groups[0]->boundaries; p.boundaries1 = sp->groups[1]->boundaries;
  p.n = n;
  p.is_f16 = dtype == TQ_F16;
  p.codes = out[0].codes; p.norms = out[0].norms;
  p.codes1 = out[1].codes; p.norms1 = out[1].norms;
  p.status = device_status_ptr();
  p.wait_limit = wait_limit();
  const int64_t tiles = (n + 127) / 128;
  const int grid = static_cast<int>(std::min<int64_t>(tiles, sm_count()));
  const cudaError_t e = launch_umma_quantize_split(map, p, sp->groups[0]->bits, sp->groups[1]->bits, grid, stream);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "split quantize launch");
}

tq_status tq_quantize_split(const tq_split* sp, const void* x, int32_t dtype, int64_t n, const tq_packed* out,
                            tq_stream stream) {
  tq_status s = check_split(sp);
  if (s != TQ_OK) return s;
  if (!out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, "n < 0");
  if (n == 0) return TQ_OK;
  if (dtype < TQ_F32 || dtype > TQ_F16) return fail(TQ_ERR_INVALID_ARG, "unknown dtype");
  if (umma_split(sp, dtype, n)) return quantize_split_umma(sp, x, dtype, n, out, reinterpret_cast<cudaStream_t>(stream));
  // every group's outputs must be disjoint from the other groups' (checked as inputs)
  Range others[4 * TQ_MAX_GROUPS];
  for (int g = 0; g < sp->n_groups; ++g) {
    int k = 0;
    for (int h = 0; h < sp->n_groups; ++h) {
      if (h == g) continue;
      if ((s = check_packed(out[h], layout_of(sp->groups[h]))) != TQ_OK) return s;
      packed_ranges(out[h], layout_of(sp->groups[h]), n, others + k);
      k += 4;
    }
    s = quantize_common(sp->groups[g], x, dtype, n, out[g], reinterpret_cast<cudaStream_t>(stream),
                        sp->groups[g]->kind, sp->d, sp->cols[g], others, k);
    if (s != TQ_OK) return s;
  }
  return TQ_OK;
}

// Workspace of tq_score_split: per group the gathered rotated queries (and S q' for PROD),
// then, for top-k, one block of summed dense scores.
// The summed estimates on the tensor cores (score_split_tc.cu): MSE (1..4 bits) or PROD
// (2..5 bits, m = d) groups whose widths d_g + m_g add up to a multiple of 64 (at most 4096),
// against at least 4096 records.
static bool split_score_tc(const tq_split* sp, int64_t n, int* K) {
  if (n < 4096 || std::getenv("TQ_FORCE_SIMT")) return false;
  int k = 0;
  for (int g = 0; g < sp->n_groups; ++g) {
    const tq_quantizer* q = sp->groups[g];
    if (q->kind == TQ_KIND_MSE) {
      if (q->bits < 1 || q->bits > 4) return false;
      k += q->d;
    } else if (q->kind == TQ_KIND_PROD) {
      if (q->bits < 2 || q->bits > 5 || q->m != q->d) return false;
      k += 2 * q->d;
    } else {
      return false;
    }
  }
  if (k % 64 || k > 4096) return false;
  if (K) *K = k;
  return true;
}

// Workspace of tq_score_split: per group the gathered, rotated queries (and S q' for PROD);
// then either the tensor-core operands (query block and records as bf16 hi + lo, a column
// of ones) or the CUDA-core estimator's block of dense scores; top-k keeps one block of
// summed dense scores.
struct SplitScorePlan {
  size_t qr[TQ_MAX_GROUPS], qu[TQ_MAX_GROUPS], ah, al, bh, bl, ones, dense, bytes;
  bool tc;
  int K;
  int64_t qb;                // queries per pass
};

static SplitScorePlan plan_split_score(const tq_split* sp, int64_t nq, int64_t n, int32_t topk) {
  SplitScorePlan P{};
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t b = 0;
  for (int g = 0; g < sp->n_groups; ++g) {
    P.qr[g] = b;
    b = al(b + static_cast<size_t>(nq) * sp->groups[g]->d * 4);
    P.qu[g] = b;
    b = al(b + static_cast<size_t>(nq) * score_qu_stride(sp->groups[g]) * 4);
  }
  P.tc = split_score_tc(sp, n, &P.K);
  if (P.tc) {
    int64_t qb = (1ll << 28) / std::max<int64_t>(n, 1) / 128 * 128;
    qb = std::max<int64_t>(128, std::min<int64_t>(1024, qb));
    P.qb = std::min<int64_t>(qb, (nq + 127) / 128 * 128);
    P.ah = b; b = al(b + P.qb * P.K * 2);
    P.al = b; b = al(b + P.qb * P.K * 2);
    P.bh = b; b = al(b + static_cast<size_t>(n) * P.K * 2);
    P.bl = b; b = al(b + static_cast<size_t>(n) * P.K * 2);
    P.ones = b; b = al(b + static_cast<size_t>(n) * 4);
    P.dense = b;
    if (topk > 0) b = al(b + static_cast<size_t>(P.qb) * n * 4);
  } else {
    P.qb = topk > 0 ? score_block(nq, n) : nq;
    P.dense = b;
    if (topk > 0) b += static_cast<size_t>(P.qb) * static_cast<size_t>(n) * 4 + 256;
  }
  P.bytes = b + 256;
  return P;
}

tq_status tq_score_split_workspace(const tq_split* sp, int64_t nq, int64_t n, int32_t topk, size_t* bytes) {
  tq_status s = check_split(sp);
  if (s != TQ_OK) return s;
  if (!bytes || nq < 0 || n < 0 || topk < 0) return fail(TQ_ERR_INVALID_ARG, "bad workspace query");
  *bytes = plan_split_score(sp, nq, n, topk).bytes;
  return TQ_OK;
}

tq_status tq_score_split(const tq_split* sp, const void* qv, int32_t dtype, int64_t nq, const tq_packed* keys,
                         int64_t n, int32_t topk, float* scores, int32_t* ids, void* workspace, size_t ws_bytes,
                         tq_stream stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  tq_status s = check_split(sp);
  if (s != TQ_OK) return s;
  if (!keys) return fail(TQ_ERR_INVALID_ARG, "keys is NULL");
  if (dtype < TQ_F32 || dtype > TQ_F16) return fail(TQ_ERR_INVALID_ARG, "unknown dtype");
  if (nq < 0 || n < 0) return fail(TQ_ERR_INVALID_ARG, "nq, n must be >= 0");
  if (topk < 0 || topk > 32) return fail(TQ_ERR_UNSUPPORTED, "topk must be 0..32");
  if (topk > 0 && topk > n) return fail(TQ_ERR_INVALID_ARG, "topk > n");
  if (n > 0x7fffffff || nq > 0x7fffffff) return fail(TQ_ERR_INVALID_ARG, "sizes too large");
  if (nq == 0 || n == 0) return TQ_OK;
  if (!qv || !scores || (topk > 0 && !ids)) return fail(TQ_ERR_INVALID_ARG, "NULL query or output");
  if (!aligned16(qv) || !aligned16(scores) || (ids && !aligned16(ids)))
    return fail(TQ_ERR_ALIGNMENT, "query/output not 16-byte aligned");
  const SplitScorePlan PL = plan_split_score(sp, nq, n, topk);
  const size_t need = PL.bytes;
  if (!workspace || ws_bytes < need) return fail(TQ_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  if (!aligned16(workspace)) return fail(TQ_ERR_ALIGNMENT, "workspace not 16-byte aligned");
  Range ins[4 * TQ_MAX_GROUPS + 2];
  int nin = 0;
  for (int g = 0; g < sp->n_groups; ++g) {
    const tq_layout L = layout_of(sp->groups[g]);
    if ((s = check_packed(keys[g], L)) != TQ_OK) return s;
    packed_ranges(keys[g], L, n, ins + nin);
    nin += 4;
  }
  ins[nin++] = {qv, static_cast<size_t>(nq) * sp->d * dtype_size(dtype)};
  ins[nin++] = {workspace, ws_bytes};
  const Range outs[2] = {{scores, topk > 0 ? static_cast<size_t>(nq) * topk * 4 : static_cast<size_t>(nq) * n * 4},
                         {topk > 0 ? ids : nullptr, static_cast<size_t>(nq) * topk * 4}};
  if ((s = check_no_alias(outs, 2, ins, nin)) != TQ_OK) return s;

  char* ws = static_cast<char*>(workspace);
  int* status = device_status_ptr();
  ScoreParams P[TQ_MAX_GROUPS];
  size_t smem = 0;
  cudaError_t e;
  for (int g = 0; g < sp->n_groups; ++g) {
    const tq_quantizer* q = sp->groups[g];
    const int qus = score_qu_stride(q);
    float* qr = reinterpret_cast<float*>(ws + PL.qr[g]);
    float* qu = qus ? reinterpret_cast<float*>(ws + PL.qu[g]) : nullptr;
    score_qprep_kernel<<<static_cast<unsigned>(nq), 128, 2 * q->d * 4, stream>>>(
        qv, dtype, q->d, q->kind, q->rot, q->S, q->m, q->k_top, qr, qu, qus, sp->d, sp->cols[g], status);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "score qprep launch");
    P[g] = score_params(q, layout_of(q), keys[g], n);
    P[g].qr = qr;
    P[g].qu = qu;
    P[g].accumulate = g > 0;
    smem = std::max(smem, score_smem(P[g]));
  }
  float* dense = reinterpret_cast<float*>(ws + PL.dense);
  if (PL.tc) {
    // one split-precision product of [queries of every group] x [decoded records of every group]
    auto u16 = [&](size_t off) { return reinterpret_cast<uint16_t*>(ws + off); };
    float* ones = reinterpret_cast<float*>(ws + PL.ones);
    SplitScoreGroups G{};
    G.n = sp->n_groups;
    for (int g = 0; g < sp->n_groups; ++g) {
      const tq_quantizer* q = sp->groups[g];
      const tq_layout L = layout_of(q);
      const bool prod = q->kind == TQ_KIND_PROD;
      G.d[g] = q->d; G.m[g] = prod ? q->m : 0;
      G.bits[g] = prod ? q->bits - 1 : q->bits;
      G.code_words[g] = L.code_words; G.sign_words[g] = L.sign_words;
      G.codes[g] = keys[g].codes; G.signs[g] = keys[g].signs;
      G.norms[g] = keys[g].norms; G.rnorms[g] = keys[g].rnorms;
      G.centroids[g] = q->centroids;
      G.coef[g] = prod ? static_cast<float>(std::sqrt(M_PI / 2.0) / q->m) : 0.f;
    }
    e = launch_split_score_records(G, n, PL.K, u16(PL.bh), u16(PL.bl), ones, stream);
    if (e != cudaSuccess) return cuda_fail(e, "split record expansion launch");
    CUtensorMap maps[4];
    const int tn = gemm_tile_n(static_cast<int>(n));       // B box = one column tile
    if ((s = bf16_map(&maps[2], u16(PL.bh), n, PL.K, tn)) != TQ_OK) return s;
    if ((s = bf16_map(&maps[3], u16(PL.bl), n, PL.K, tn)) != TQ_OK) return s;
    for (int64_t q0 = 0; q0 < nq; q0 += PL.qb) {
      const int64_t nb = std::min(PL.qb, nq - q0);
      for (int g = 0; g < sp->n_groups; ++g) {
        G.qr[g] = P[g].qr + q0 * G.d[g];
        G.qu[g] = P[g].qu ? P[g].qu + q0 * G.m[g] : nullptr;
      }
      e = launch_split_score_queries(G, nb, PL.K, u16(PL.ah), u16(PL.al), stream);
      if (e != cudaSuccess) return cuda_fail(e, "split query operand launch");
      if ((s = bf16_map(&maps[0], u16(PL.ah), nb, PL.K, 128)) != TQ_OK) return s;
      if ((s = bf16_map(&maps[1], u16(PL.al), nb, PL.K, 128)) != TQ_OK) return s;
      SplitGemmParams gp{};
      gp.M = nb; gp.N = static_cast<int>(n); gp.K = PL.K; gp.status = status; gp.wait_limit = wait_limit();
      gp.out = topk > 0 ? dense : scores + q0 * n; gp.ldo = n; gp.col_scale = ones;
      const int64_t work = (nb + 127) / 128 * ((n + tn - 1) / tn);
      e = launch_split_gemm(maps, gp, GEMM_EPI_SCORE, 1, static_cast<int>(std::min<int64_t>(work, sm_count())), stream);
      if (e != cudaSuccess) return cuda_fail(e, "split estimate launch");
      if (topk > 0) {
        if (topk <= 16) topk_kernel<16><<<static_cast<unsigned>(nb), 128, 0, stream>>>(dense, n, topk, q0, scores, ids);
        else topk_kernel<32><<<static_cast<unsigned>(nb), 128, 0, stream>>>(dense, n, topk, q0, scores, ids);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "topk launch");
      }
    }
    return TQ_OK;
  }
  e = cudaFuncSetAttribute(score_dense_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "score attribute");
  const int64_t qb = PL.qb;
  for (int64_t q0 = 0; q0 < nq; q0 += qb) {
    const int64_t nb = std::min(qb, nq - q0);
    const dim3 grid(static_cast<unsigned>((n + kScoreThreads - 1) / kScoreThreads),
                    static_cast<unsigned>((nb + kScoreQT - 1) / kScoreQT));
    if (grid.y > 65535) return fail(TQ_ERR_UNSUPPORTED, "too many queries per block");
    for (int g = 0; g < sp->n_groups; ++g) {
      ScoreParams p = P[g];
      const int d = sp->groups[g]->d;
      p.qr = P[g].qr + q0 * d;
      p.qu = P[g].qu ? P[g].qu + q0 * score_qu_stride(sp->groups[g]) : nullptr;
      p.nq = nb;
      p.out = topk > 0 ? dense : scores + q0 * n;
      score_dense_kernel<<<grid, kScoreThreads, score_smem(p), stream>>>(p);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "score launch");
    }
    if (topk > 0) {
      if (topk <= 16) topk_kernel<16><<<static_cast<unsigned>(nb), 128, 0, stream>>>(dense, n, topk, q0, scores, ids);
      else topk_kernel<32><<<static_cast<unsigned>(nb), 128, 0, stream>>>(dense, n, topk, q0, scores, ids);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "topk launch");
    }
  }
  return TQ_OK;
}

// ---- decode attention over a split cache ----
struct SplitDecodePlan {
  bool fast;                 // the tensor-core kernel (decode_split_mma.cuh)
  int chunk_len, n_chunks;
  size_t off_qr[TQ_MAX_GROUPS], off_qu[TQ_MAX_GROUPS], off_ml, off_o, bytes;
  int mu;                    // sum of the PROD key groups' m
};

// The tensor-core split decode takes the 2.5-bit outlier split of the KV experiments: two
// MSE groups, 32 rotated dims at 3 bits then 96 at 2 bits, for keys and values alike;
// GQA groups of at most 4 heads; rows of a multiple of 4 records (16-byte aligned copies).
static bool split_mma_ok(const tq_split* ks, const tq_split* vs, int G, int64_t Nmax) {
  auto shape = [](const tq_split* s) {
    return s->d == 128 && s->n_groups == 2 && s->groups[0]->kind == TQ_KIND_MSE &&
           s->groups[1]->kind == TQ_KIND_MSE && s->groups[0]->d == 32 && s->groups[0]->bits == 3 &&
           s->groups[1]->d == 96 && s->groups[1]->bits == 2;
  };
  return shape(ks) && shape(vs) && G <= 4 && Nmax % 4 == 0;
}

static SplitDecodePlan plan_split_decode(const tq_split* ks, const tq_split* vs, int B, int Hq, int Hkv,
                                         int64_t Nmax) {
  SplitDecodePlan P{};
  P.fast = split_mma_ok(ks, vs, Hq / Hkv, Nmax);
  int64_t cl;
  if (P.fast) {
    // persistent kernel: chunks of whole 256-token stages, ~16 items per SM at most and
    // items of at least ~4 stages, an item count that is a multiple of the SMs when the
    // shape allows (as the packed-cache decode plans its work)
    const int64_t stage = kSmStage, sms = sm_count(), wu = static_cast<int64_t>(B) * Hkv;
    const int64_t stages_total = wu * ((Nmax + stage - 1) / stage);
    const int64_t want = std::max<int64_t>(sms, std::min<int64_t>(16 * sms, stages_total / 4));
    int64_t n0 = std::max<int64_t>(1, (want + wu - 1) / wu);
    for (int64_t cand = n0; cand < n0 + 8 && cand <= Nmax; ++cand)
      if ((wu * cand) % sms == 0) { n0 = cand; break; }
    cl = (Nmax + n0 - 1) / n0;
    cl = std::max<int64_t>(stage, (cl + stage - 1) / stage * stage);
  } else {
    // at most 64 chunks per row: the partials stay small and the combine's weights fit in
    // shared memory; chunks of at least 256 tokens
    cl = (Nmax + 63) / 64;
    cl = std::max<int64_t>(256, (cl + 31) / 32 * 32);
  }
  P.chunk_len = static_cast<int>(std::min<int64_t>(cl, 1 << 30));
  P.n_chunks = static_cast<int>((Nmax + P.chunk_len - 1) / P.chunk_len);
  const size_t rows = static_cast<size_t>(B) * Hq;
  size_t b = 0;
  for (int g = 0; g < ks->n_groups; ++g) {
    P.off_qr[g] = b;
    b += (rows * ks->groups[g]->d * 4 + 255) / 256 * 256;
    const int m = ks->groups[g]->kind == TQ_KIND_PROD ? ks->groups[g]->m : 0;
    P.off_qu[g] = b;
    b += (rows * m * 4 + 255) / 256 * 256;
    P.mu += m;
  }
  P.off_ml = b;
  b += (rows * P.n_chunks * 2 * 4 + 255) / 256 * 256;
  P.off_o = b;
  b += (rows * P.n_chunks * static_cast<size_t>(ks->d) * 4 + 255) / 256 * 256;
  P.bytes = b + 256;
  return P;
}

static tq_status check_split_decode(const tq_split* ks, const tq_split* vs, int B, int Hq, int Hkv, int64_t Nmax) {
  tq_status s = check_split(ks);
  if (s != TQ_OK) return s;
  if ((s = check_split(vs)) != TQ_OK) return s;
  if (ks->d != vs->d) return fail(TQ_ERR_INVALID_ARG, "key and value splits have different widths");
  if (ks->d > kSplitMaxD) return fail(TQ_ERR_UNSUPPORTED, "split decode runs d <= %d", kSplitMaxD);
  for (int g = 0; g < ks->n_groups; ++g)
    if (ks->groups[g]->kind != TQ_KIND_MSE && ks->groups[g]->kind != TQ_KIND_PROD)
      return fail(TQ_ERR_UNSUPPORTED, "split decode runs MSE or PROD key groups");
  for (int g = 0; g < vs->n_groups; ++g)
    if (vs->groups[g]->kind != TQ_KIND_MSE) return fail(TQ_ERR_UNSUPPORTED, "split decode runs MSE value groups");
  if (B < 1 || Hq < 1 || Hkv < 1 || Nmax < 1) return fail(TQ_ERR_INVALID_ARG, "B, Hq, Hkv, Nmax must be >= 1");
  if (Hq % Hkv) return fail(TQ_ERR_INVALID_ARG, "Hq must be a multiple of Hkv");
  if (Hq / Hkv > kSplitMaxG) return fail(TQ_ERR_UNSUPPORTED, "Hq/Hkv > %d", kSplitMaxG);
  if (static_cast<int64_t>(B) * Hkv > 65535) return fail(TQ_ERR_UNSUPPORTED, "B*Hkv > 65535");
  if (Nmax > (1ll << 30)) return fail(TQ_ERR_INVALID_ARG, "Nmax too large");
  return TQ_OK;
}

tq_status tq_decode_attn_split_workspace(const tq_split* ks, const tq_split* vs, int32_t B, int32_t Hq, int32_t Hkv,
                                         int64_t Nmax, size_t* bytes) {
  tq_status s = check_split_decode(ks, vs, B, Hq, Hkv, Nmax);
  if (s != TQ_OK) return s;
  if (!bytes) return fail(TQ_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = plan_split_decode(ks, vs, B, Hq, Hkv, Nmax).bytes;
  return TQ_OK;
}

tq_status tq_decode_attn_split(const tq_split* ks, const tq_split* vs, const void* q, int32_t dtype, int32_t B,
                               int32_t Hq, int32_t Hkv, int64_t Nmax, const int32_t* seq_lens,
                               const tq_packed* kcache, const tq_packed* vcache, float scale, float* out,
                               void* workspace, size_t ws_bytes, tq_stream stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  tq_status s = check_split_decode(ks, vs, B, Hq, Hkv, Nmax);
  if (s != TQ_OK) return s;
  if (dtype < TQ_F32 || dtype > TQ_F16) return fail(TQ_ERR_INVALID_ARG, "unknown dtype");
  if (!q || !seq_lens || !out || !kcache || !vcache) return fail(TQ_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(q) || !aligned16(seq_lens) || !aligned16(out)) return fail(TQ_ERR_ALIGNMENT, "q/seq_lens/out alignment");
  if (!std::isfinite(scale)) return fail(TQ_ERR_INVALID_ARG, "scale must be finite");
  const SplitDecodePlan P = plan_split_decode(ks, vs, B, Hq, Hkv, Nmax);
  if (!workspace || ws_bytes < P.bytes) return fail(TQ_ERR_WORKSPACE, "workspace needs %zu bytes", P.bytes);
  if (!aligned16(workspace)) return fail(TQ_ERR_ALIGNMENT, "workspace not 16-byte aligned");
  const int64_t recs = static_cast<int64_t>(B) * Hkv * Nmax;
  const int d = ks->d, G = Hq / Hkv, rows = B * Hq;
  Range ins[8 * TQ_MAX_GROUPS + 3];
  int nin = 0;
  for (int g = 0; g < ks->n_groups; ++g) {
    const tq_layout L = layout_of(ks->groups[g]);
    if ((s = check_packed(kcache[g], L)) != TQ_OK) return s;
    packed_ranges(kcache[g], L, recs, ins + nin);
    nin += 4;
  }
  for (int g = 0; g < vs->n_groups; ++g) {
    const tq_layout L = layout_of(vs->groups[g]);
    if ((s = check_packed(vcache[g], L)) != TQ_OK) return s;
    packed_ranges(vcache[g], L, recs, ins + nin);
    nin += 4;
  }
  ins[nin++] = {q, static_cast<size_t>(rows) * d * dtype_size(dtype)};
  ins[nin++] = {seq_lens, static_cast<size_t>(B) * 4};
  ins[nin++] = {workspace, ws_bytes};
  const Range outs[1] = {{out, static_cast<size_t>(rows) * d * 4}};
  if ((s = check_no_alias(outs, 1, ins, nin)) != TQ_OK) return s;

  char* ws = static_cast<char*>(workspace);
  int* status = device_status_ptr();
  SplitDecodeParams dp{};
  dp.B = B; dp.Hq = Hq; dp.Hkv = Hkv; dp.G = G; dp.d = d; dp.Nmax = Nmax;
  dp.chunk_len = P.chunk_len; dp.n_chunks = P.n_chunks; dp.seq_lens = seq_lens;
  dp.nkg = ks->n_groups; dp.nvg = vs->n_groups;
  cudaError_t e;
  int off = 0, uoff = 0;
  for (int g = 0; g < ks->n_groups; ++g) {
    const tq_quantizer* kq = ks->groups[g];
    const bool prod = kq->kind == TQ_KIND_PROD;
    float* qr = reinterpret_cast<float*>(ws + P.off_qr[g]);
    float* qu = prod ? reinterpret_cast<float*>(ws + P.off_qu[g]) : nullptr;
    score_qprep_kernel<<<static_cast<unsigned>(rows), 128, 2 * kq->d * 4, stream>>>(
        q, dtype, kq->d, kq->kind, kq->rot, prod ? kq->S : nullptr, prod ? kq->m : 0, 0, qr, qu, prod ? kq->m : 0, d,
        ks->cols[g], status);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "split qprep launch");
    const tq_layout L = layout_of(kq);
    dp.kd[g] = kq->d; dp.kbits[g] = prod ? kq->bits - 1 : kq->bits; dp.kwords[g] = L.code_words; dp.koff[g] = off;
    dp.kcodes[g] = kcache[g].codes; dp.knorms[g] = kcache[g].norms; dp.kcent[g] = kq->centroids;
    dp.qr[g] = qr;
    if (prod) {
      dp.km[g] = kq->m; dp.ksw[g] = L.sign_words; dp.kuoff[g] = uoff;
      dp.ksigns[g] = kcache[g].signs; dp.krnorms[g] = kcache[g].rnorms; dp.qu[g] = qu;
      dp.kcoef[g] = static_cast<float>(std::sqrt(M_PI / 2.0) / kq->m);
      uoff += kq->m;
    }
    off += kq->d;
  }
  dp.mu = P.mu;
  off = 0;
  for (int g = 0; g < vs->n_groups; ++g) {
    const tq_quantizer* vq = vs->groups[g];
    const tq_layout L = layout_of(vq);
    dp.vd[g] = vq->d; dp.vbits[g] = vq->bits; dp.vwords[g] = L.code_words; dp.voff[g] = off;
    dp.vcodes[g] = vcache[g].codes; dp.vnorms[g] = vcache[g].norms; dp.vcent[g] = vq->centroids;
    off += vq->d;
  }
  dp.logit_scale = static_cast<float>(scale * kLog2e);
  dp.part_ml = reinterpret_cast<float*>(ws + P.off_ml);
  dp.part_o = reinterpret_cast<float*>(ws + P.off_o);
  if (P.fast) {
    SplitMmaParams mp{};
    mp.B = B; mp.Hq = Hq; mp.Hkv = Hkv; mp.G = G; mp.Nmax = Nmax;
    mp.chunk_len = P.chunk_len; mp.n_chunks = P.n_chunks; mp.seq_lens = seq_lens;
    for (int g = 0; g < 2; ++g) {
      mp.kc[g] = kcache[g].codes; mp.kn[g] = kcache[g].norms;
      mp.vc[g] = vcache[g].codes; mp.vn[g] = vcache[g].norms;
      mp.kcent[g] = ks->groups[g]->centroids; mp.vcent[g] = vs->groups[g]->centroids;
      mp.kscale[g] = ks->groups[g]->lut_scale > 0.f ? ks->groups[g]->lut_scale : 1.f;
      mp.vscale[g] = vs->groups[g]->lut_scale > 0.f ? vs->groups[g]->lut_scale : 1.f;
      mp.qr[g] = dp.qr[g];
    }
    mp.logit_scale = dp.logit_scale;
    mp.part_ml = dp.part_ml;
    mp.part_o = dp.part_o;
    const int64_t items = static_cast<int64_t>(B) * Hkv * P.n_chunks;
    const int grid = static_cast<int>(std::min<int64_t>(items, sm_count()));
    e = launch_decode_split_mma(mp, grid, stream, status, wait_limit());
    if (e != cudaSuccess) return cuda_fail(e, "split decode launch");
  } else {
    const size_t smem = split_decode_smem(G, d, P.mu);
    if (smem > 227 * 1024) return fail(TQ_ERR_UNSUPPORTED, "split decode: shared memory for Hq/Hkv and widths too large");
    e = cudaFuncSetAttribute(split_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e, "split decode attribute");
    split_decode_kernel<<<dim3(static_cast<unsigned>(P.n_chunks), static_cast<unsigned>(B * Hkv)), kSplitDecThreads,
                          smem, stream>>>(dp);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "split decode launch");
  }

  SplitCombineParams cp{};
  cp.rows = rows; cp.d = d; cp.n_chunks = P.n_chunks; cp.nvg = vs->n_groups;
  off = 0;
  for (int g = 0; g < vs->n_groups; ++g) {
    cp.vd[g] = vs->groups[g]->d; cp.voff[g] = off; cp.vrot[g] = vs->groups[g]->rot; cp.vcols[g] = vs->cols[g];
    off += vs->groups[g]->d;
  }
  cp.status = status;
  cp.part_ml = dp.part_ml; cp.part_o = dp.part_o; cp.out = out;
  split_combine_kernel<<<static_cast<unsigned>(rows), 128, static_cast<size_t>(P.n_chunks + d) * 4, stream>>>(cp);
  e = cudaGetLastError();
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "split combine launch");
}

tq_status tq_decode_attn_workspace(const tq_quantizer* kq, int32_t B, int32_t Hq, int32_t Hkv, int64_t Nmax,
                                   size_t* bytes) {
  tq_status s = check_quantizer(kq);
  if (s != TQ_OK) return s;
  if (!bytes || B < 1 || Hq < 1 || Hkv < 1 || Nmax < 1) return fail(TQ_ERR_INVALID_ARG, "bad workspace query");
  *bytes = plan_decode(kq, B, Hq, Hkv, Nmax).bytes;
  return TQ_OK;
}

tq_status tq_decode_attn(const tq_quantizer* kq, const tq_quantizer* vq, const void* q, int32_t dtype, int32_t B,
                         int32_t Hq, int32_t Hkv, int64_t Nmax, const int32_t* seq_lens, tq_packed kc,
                         tq_packed vc, float scale, float* out, void* workspace, size_t ws_bytes,
                         tq_stream stream_) {
  DecodeCall c{};
  c.kq = kq; c.vq = vq; c.q = q; c.dtype = dtype; c.B = B; c.Hq = Hq; c.Hkv = Hkv; c.Nmax = Nmax;
  c.seq_lens = seq_lens; c.kc = kc; c.vc = vc; c.scale = scale; c.out = out; c.ws = workspace;
  c.ws_bytes = ws_bytes; c.stream = reinterpret_cast<cudaStream_t>(stream_);
  return decode_run(c);
}

tq_status tq_decode_attn_paged(const tq_quantizer* kq, const tq_quantizer* vq, const void* q, const void* k_new,
                               const void* v_new, int32_t dtype, int32_t B, int32_t Hq, int32_t Hkv,
                               const int32_t* seq_lens, const tq_pages* pages, tq_packed kpool, tq_packed vpool,
                               float scale, float* out, void* workspace, size_t ws_bytes, tq_stream stream_) {
  tq_status s = check_pages(pages);
  if (s != TQ_OK) return s;
  if ((k_new == nullptr) != (v_new == nullptr)) return fail(TQ_ERR_INVALID_ARG, "k_new and v_new go together");
  if (!seq_lens || !aligned16(seq_lens)) return fail(TQ_ERR_ALIGNMENT, "seq_lens NULL or not 16-byte aligned");
  DecodeCall c{};
  c.kq = kq; c.vq = vq; c.q = q; c.dtype = dtype; c.B = B; c.Hq = Hq; c.Hkv = Hkv;
  c.Nmax = static_cast<int64_t>(pages->max_pages) * pages->page_size;
  c.seq_lens = seq_lens; c.kc = kpool; c.vc = vpool; c.scale = scale; c.out = out; c.ws = workspace;
  c.ws_bytes = ws_bytes; c.stream = reinterpret_cast<cudaStream_t>(stream_); c.pages = pages;
  c.k_new = k_new; c.v_new = v_new;
  return decode_run(c);
}

tq_status tq_prefill_attn_workspace(const tq_quantizer* kq, int32_t B, int32_t Hq, int32_t Hkv, int32_t T,
                                    int64_t Nmax, size_t* bytes) {
  tq_status s = check_quantizer(kq);
  if (s != TQ_OK) return s;
  if (!bytes || B < 1 || Hq < 1 || Hkv < 1 || T < 1 || Nmax < 1 || static_cast<int64_t>(Hq) * T > (1 << 24))
    return fail(TQ_ERR_INVALID_ARG, "bad workspace query");
  *bytes = plan_decode(kq, B, Hq * T, Hkv, Nmax, true).bytes;
  return TQ_OK;
}

tq_status tq_prefill_attn(const tq_quantizer* kq, const tq_quantizer* vq, const void* q, int32_t dtype, int32_t B,
                          int32_t Hq, int32_t Hkv, int32_t T, const int32_t* q_pos, const int32_t* kv_lens,
                          const tq_pages* pages, int64_t Nmax, tq_packed kcache, tq_packed vcache, float scale,
                          float* out, void* workspace, size_t ws_bytes, tq_stream stream_) {
  if (T < 1 || Hq < 1 || static_cast<int64_t>(Hq) * T > (1 << 24)) return fail(TQ_ERR_INVALID_ARG, "T out of range");
  if (!q_pos || !aligned16(q_pos)) return fail(TQ_ERR_ALIGNMENT, "q_pos NULL or not 16-byte aligned");
  if (pages) {
    tq_status s = check_pages(pages);
    if (s != TQ_OK) return s;
    Nmax = static_cast<int64_t>(pages->max_pages) * pages->page_size;
  }
  DecodeCall c{};
  c.kq = kq; c.vq = vq; c.q = q; c.dtype = dtype; c.B = B; c.Hq = Hq * T; c.Hkv = Hkv; c.Nmax = Nmax;
  c.seq_lens = kv_lens; c.kc = kcache; c.vc = vcache; c.scale = scale; c.out = out; c.ws = workspace;
  c.ws_bytes = ws_bytes; c.stream = reinterpret_cast<cudaStream_t>(stream_); c.pages = pages;
  c.q_pos = q_pos; c.T = T;
  return decode_run(c);
}

tq_status tq_get_status(tq_stream stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_tq_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_tq_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "status clear");
  if (v == TQ_ERR_TIMEOUT) return fail(TQ_ERR_TIMEOUT, "a device-side bounded wait timed out");
  return v == 0 ? TQ_OK : fail(static_cast<tq_status>(v), "device reported status %d", v);
}

tq_status tq_set_wait_limit(int64_t polls) {
  if (polls < -1) return fail(TQ_ERR_INVALID_ARG, "polls < -1");
  g_wait_limit.store(polls);
  return TQ_OK;
}

}  // extern "C"

namespace tq {
tq_status decode_shape_ok(const tq_quantizer* kq, const tq_quantizer* vq, int B, int Hq, int Hkv, int64_t Nmax) {
  return check_decode_shape(kq, vq, B, Hq, Hkv, Nmax);
}

cudaError_t launch_decode(const DecodeParams& p, int kfmt, int kb, int vfmt, int vb, dim3 grid, size_t smem,
                          cudaStream_t stream, int* status, long long lim) {
  if (vfmt == VFMT_PROD) return launch_decode_vprod(p, kfmt, kb, vb, grid, stream, status, lim);
  if (kfmt == KFMT_MSE && vfmt == VFMT_MSE) return launch_decode_mse(p, kb, vb, grid, smem, stream, status, lim);
  if (kfmt == KFMT_PROD && vfmt == VFMT_MSE) return launch_decode_prod(p, kb, vb, grid, smem, stream, status, lim);
  if (kfmt == KFMT_SPEC && vfmt == VFMT_SPEC) return launch_decode_spec(p, kb, vb, grid, smem, stream);
  return cudaErrorNotSupported;
}
}  // namespace tq
