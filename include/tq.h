/*
 * tq.h -- C ABI of libtq, a B200 (sm_100a) implementation of the TurboQuant hot path.
 *
 * The method (TurboQuant: Online Vector Quantization with Near-optimal Distortion Rate,
 * paper review, section "Method"): rotate each vector by a random orthogonal matrix Pi,
 * quantize every rotated coordinate with a Lloyd-Max scalar codebook precomputed for the
 * post-rotation coordinate law, and bit-pack the codes ("TurboQuant-mse").  The inner-
 * product variant ("TurboQuant-prod") spends b-1 bits on that stage and one bit per
 * projection on a Quantized-JL sketch of the residual, which makes inner products
 * unbiased.  Attention reads the cache only through query-key inner products (review,
 * "Problem"), so decode attention runs directly on the packed records.
 * A SpectralQuant-style variant (SpectralQuant thread by @ashwingop, posts 4-6) replaces
 * Pi by calibrated covariance eigenvectors, water-fills bits over the top signal dims and
 * applies the QJL correction to those dims only.
 *
 * Conventions shared by every entry point:
 *   - Every function returns a tq_status; nothing throws across the ABI.  On a non-OK
 *     status tq_last_error() returns a thread-local message.
 *   - Ownership: the caller owns every buffer.  The library never allocates, frees or
 *     retains caller memory beyond the call (device work is stream-ordered).
 *   - "device" pointers are CUDA device memory of the current device; "host" pointers
 *     are ordinary host memory.  Device entry points are asynchronous on `stream`
 *     (NULL = legacy default stream); arguments are validated on the host before any
 *     launch and a failed validation launches nothing.
 *   - Alignment: device pointers must be 16-byte aligned, else TQ_ERR_ALIGNMENT.
 *   - Aliasing: an output that overlaps an input gives TQ_ERR_ALIAS.
 *   - Device-side failures (a bounded wait that ran out) are recorded in a device status
 *     word; tq_get_status() synchronizes the stream and returns it.  No kernel traps.
 *   - Non-finite inputs give unspecified codes (never out-of-bounds accesses).
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle as cudaStream_t / CUstream. */
typedef struct CUstream_st* tq_stream;

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,   /* null pointer, size out of range, inconsistent descriptor */
  TQ_ERR_UNSUPPORTED = 2,   /* valid request outside what libtq implements */
  TQ_ERR_ALIGNMENT = 3,     /* device pointer not 16-byte aligned */
  TQ_ERR_ALIAS = 4,         /* an output overlaps an input */
  TQ_ERR_CUDA = 5,          /* CUDA runtime error (message has the CUDA error string) */
  TQ_ERR_TIMEOUT = 6,       /* a device-side bounded wait ran out (see tq_get_status) */
  TQ_ERR_NOT_CONVERGED = 7, /* host iteration did not reach its tolerance */
  TQ_ERR_WORKSPACE = 8      /* workspace pointer null or smaller than required */
} tq_status;

/* Coordinate law the codebook is solved for (review, Method: "known Beta distribution,
 * converging to N(0, 1/d)"). */
typedef enum { TQ_DIST_BETA_SPHERE = 0, TQ_DIST_GAUSSIAN = 1 } tq_dist;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 } tq_dtype;

typedef enum { TQ_KIND_MSE = 0, TQ_KIND_PROD = 1, TQ_KIND_SPECTRAL = 2 } tq_kind;

#define TQ_MAX_TOP 8

/*
 * Quantizer descriptor.  Plain data; all pointers are DEVICE pointers owned by the caller
 * and read (never written) by the library.
 *
 *  MSE       bits = b (1..8).  centroids [2^b] ascending, boundaries [2^b-1] with
 *            t_k = (c_k + c_{k+1})/2 (from tq_codebook_build).
 *  PROD      bits = b total (1..9): b-1 MSE bits (centroids/boundaries of the (b-1)-bit
 *            codebook; ignored when b = 1) plus m QJL sign bits; S [m*d] row-major,
 *            i.i.d. N(0,1).  m must be a multiple of 32.
 *  SPECTRAL  rot = calibrated eigenvectors (row j = eigenvector j, descending eigenvalue);
 *            dims j < k_top use top_bits[j] bits (0..8), the rest tail_bits (1..4);
 *            dim j's codebook is dim_sigma[j] * (standard-normal Lloyd-Max codebook);
 *            unit_centroids / unit_boundaries hold those codebooks for 1..8 bits
 *            concatenated (see tq_spectral_unit_codebooks).  qjl != 0 adds k_top sign bits
 *            of S [k_top*k_top] applied to the top-k residual.
 *  rot       [d*d] row-major fp32; the rotated vector is y = rot @ x.
 */
typedef struct {
  int32_t kind;                 /* tq_kind */
  int32_t d;                    /* vector dimension (2..4096) */
  int32_t bits;                 /* MSE: bits; PROD: total bits; SPECTRAL: unused (0) */
  int32_t m;                    /* PROD: QJL rows (multiple of 32); SPECTRAL: unused */
  const float* rot;             /* [d*d] */
  const float* S;               /* PROD [m*d]; SPECTRAL+qjl [k_top*k_top]; else NULL */
  const float* centroids;       /* MSE/PROD */
  const float* boundaries;      /* MSE/PROD */
  int32_t k_top;                /* SPECTRAL: number of signal dims (1..TQ_MAX_TOP) */
  int32_t tail_bits;            /* SPECTRAL: bits of dims >= k_top (1..4) */
  int32_t qjl;                  /* SPECTRAL: 1 = QJL on the top-k residual */
  int32_t top_bits[TQ_MAX_TOP]; /* SPECTRAL: bits of dims 0..k_top-1 */
  const float* dim_sigma;       /* SPECTRAL: [d] sqrt(eigenvalue) per dim */
  const float* unit_centroids;  /* SPECTRAL: [510] codebook of b bits at offset 2^b - 2 */
  const float* unit_boundaries; /* SPECTRAL: [502] boundaries of b bits at offset 2^b - b - 1 */
  float lut_scale;              /* decode/score: shared scale s of the half-precision codebook
                                   table (entries c_k / s); 0 means 1.  tq_lut_scale picks one
                                   that keeps every entry within ~1e-4 of c_k. */
  int32_t rot_pm1;              /* non-zero: every entry of rot is +1/sqrt(d) or -1/sqrt(d) in
                                   fp32 (a randomized Hadamard rotation H diag(s) / sqrt(d), the
                                   launch kit's O(d log d) rotation mode).  The tensor-core
                                   quantize then multiplies by the exact +-1 matrix in one pass and
                                   rescales; an entry of another magnitude makes it report
                                   TQ_ERR_INVALID_ARG through tq_get_status. */
} tq_quantizer;

/*
 * Packed records, structure-of-arrays (each array indexed by record).  Record v owns
 * codes[v*code_words .. +code_words), signs[v*sign_words ..), norms[v], rnorms[v]
 * (word counts from tq_record_layout).  Code stream: code j occupies bits
 * [j*b, j*b+b) of the record's little-endian uint32 stream, LSB first; unused bits 0.
 * Signs: bit i%32 of word i/32 is 1 iff (S r)_i >= 0.  norms = ||x|| (fp32),
 * rnorms = ||r|| of the QJL residual (fp32).  Spectral records: a head of
 * ceil((sum top_bits + qjl*k_top)/32) words with the top-k codes LSB-first then the
 * k_top sign bits, followed by ceil(d*tail_bits/32) words with dim j's code at bits
 * [j*tail_bits, ...) (dims < k_top hold 0).  Unused arrays may be NULL.
 * A KV cache is the same arrays laid out [B][Hkv][Nmax] records.
 */
typedef struct {
  uint32_t* codes;
  uint32_t* signs;
  float* norms;
  float* rnorms;
} tq_packed;

typedef struct {
  int32_t code_words;   /* uint32 words of codes per record */
  int32_t sign_words;   /* uint32 words of QJL signs per record (PROD) */
  int32_t has_norms;    /* 1 if norms[] is written (MSE, PROD) */
  int32_t has_rnorms;   /* 1 if rnorms[] is written (PROD, SPECTRAL with qjl) */
} tq_layout;

/* Library version string (static storage). */
const char* tq_version(void);

/* Thread-local message for the last non-OK status returned on this thread. */
const char* tq_last_error(void);

/*
 * HOST.  Lloyd-Max codebook with 2^bits levels for one coordinate (review, Method:
 * "solved once as a continuous 1-D k-means").  dist = TQ_DIST_BETA_SPHERE uses the
 * exact marginal of a uniform point on S^{d-1} (d >= 2, sigma ignored);
 * TQ_DIST_GAUSSIAN uses N(0, sigma^2) (sigma > 0, d ignored).  Iterates
 * t_k = (c_k + c_{k+1})/2, c_k = E[t | cell k] until the largest move < 1e-13 * scale.
 * Outputs (host, caller-allocated): centroids [2^bits] ascending, boundaries [2^bits-1];
 * iterations may be NULL.  bits 1..8.  TQ_ERR_NOT_CONVERGED after 10^7 iterations.
 */
tq_status tq_codebook_build(int32_t d, int32_t bits, int32_t dist, double sigma,
                            double* centroids, double* boundaries, int32_t* iterations);

/*
 * HOST.  Integer reverse water-filling (SpectralQuant thread, post 6: "[3,3,3,3] ->
 * [5,3,2,2]"): starting from zero, each of budget_bits bits goes to
 * argmax_j lambda_j * 4^(-b_j) (ties to the lowest j; dims capped at max_bits).
 * lambda [k] host, bits_out [k] host.
 */
tq_status tq_waterfill(const double* lambda, int32_t k, int32_t budget_bits, int32_t max_bits,
                       int32_t* bits_out);

/*
 * HOST.  SpectralQuant calibration (thread, post 4): eigen-decomposition of the second
 * moment M = X^T X / n of n calibration rows X [n*d] (host, row-major fp32) by cyclic
 * Jacobi rotations.  eigvecs_out [d*d] (row j = eigenvector j, sign fixed so its largest-
 * magnitude entry is positive), eigvals_out [d] descending.  d <= 1024.
 */
tq_status tq_spectral_calibrate(const float* X, int64_t n, int32_t d,
                                double* eigvecs_out, double* eigvals_out);

/* HOST.  Standard-normal codebooks for 1..8 bits in the concatenated layout the
 * SPECTRAL descriptor expects: centroids_out [510], boundaries_out [502]. */
tq_status tq_spectral_unit_codebooks(double* centroids_out, double* boundaries_out);

/*
 * HOST.  Shared scale s in [1, 2) for representing `values` [count] (host) in half
 * precision as s * half(v / s): searches s on a uniform grid of 2^22 points for the
 * smallest worst-case relative rounding error over the distinct magnitudes.  Decode
 * attention multiplies products back by s in fp32; the result is written to *scale_out.
 * This is an encoding detail of the half-precision MMA operands, not part of the method.
 */
tq_status tq_lut_scale(const double* values, int32_t count, float* scale_out);

/*
 * HOST.  Everything a SPECTRAL descriptor points at, from an eigen-decomposition
 * (SpectralQuant thread, posts 4-6): eigvecs [d*d] (row j = eigenvector j, descending
 * eigenvalue, as tq_spectral_calibrate writes them) and eigvals [d], host float64.
 *   top_bits_out [k_top]       reverse water-filling of budget_bits over eigvals[0..k_top)
 *                              (as tq_waterfill, negative eigenvalues taken as 0,
 *                              dims capped at max_bits);
 *   dim_sigma_out [d]          sqrt(max(eigvals_j, 0)), the scale of dim j's codebook;
 *   rot_out [d*d]              the eigenvectors in fp32;
 *   unit_centroids_out [510],
 *   unit_boundaries_out [502]  the unit-normal codebooks of tq_spectral_unit_codebooks in fp32;
 *   *lut_scale_out             tq_lut_scale of the tail_bits unit codebook.
 * All outputs are host memory the caller allocated; copied to the device they are the
 * descriptor's rot, dim_sigma, unit_centroids, unit_boundaries, top_bits and lut_scale.
 * d 2..1024, k_top 1..TQ_MAX_TOP, tail_bits 1..4, max_bits 1..8; TQ_ERR_UNSUPPORTED when
 * the top bits plus k_top sign bits exceed 32.
 */
tq_status tq_spectral_descriptor(const double* eigvecs, const double* eigvals, int32_t d, int32_t k_top,
                                 int32_t budget_bits, int32_t tail_bits, int32_t max_bits, float* rot_out,
                                 float* dim_sigma_out, float* unit_centroids_out, float* unit_boundaries_out,
                                 int32_t* top_bits_out, float* lut_scale_out);

/*
 * HOST.  Calibration and descriptor in one call: tq_spectral_calibrate of the n host rows
 * X [n*d] (fp32), then tq_spectral_descriptor of the result.  eigvals_out [d] (host,
 * may be NULL) receives the eigenvalues.
 */
tq_status tq_spectral_prepare(const float* X, int64_t n, int32_t d, int32_t k_top, int32_t budget_bits,
                              int32_t tail_bits, int32_t max_bits, float* rot_out, float* dim_sigma_out,
                              float* unit_centroids_out, float* unit_boundaries_out, int32_t* top_bits_out,
                              float* lut_scale_out, double* eigvals_out);

/* HOST.  Words per record and which norm arrays a quantizer writes. */
tq_status tq_record_layout(const tq_quantizer* q, tq_layout* out);

/*
 * DEVICE.  TurboQuant-mse quantize of n rows x [n*d] (dtype TQ_F32 / TQ_BF16 / TQ_F16,
 * row-major): norms[v] = ||x_v||; y = rot @ (x_v/||x_v||); code_j = #{k : t_k < y_j};
 * codes packed as described at tq_packed.  q->kind must be TQ_KIND_MSE.
 * Appending a decode-time token is this call with `out` pointing at its cache slot.
 */
tq_status tq_quantize_mse(const tq_quantizer* q, const void* x, int32_t dtype, int64_t n,
                          tq_packed out, tq_stream stream);

/*
 * DEVICE.  TurboQuant-prod quantize (review, Method): the (bits-1)-bit MSE stage as above,
 * residual r = y - c[code] in the rotated unit-scale domain, rnorms[v] = ||r||,
 * sign_i = [(S r)_i >= 0].  q->kind must be TQ_KIND_PROD.
 */
tq_status tq_quantize_prod(const tq_quantizer* q, const void* x, int32_t dtype, int64_t n,
                           tq_packed out, tq_stream stream);

/*
 * DEVICE.  SpectralQuant-style quantize: z = rot @ x (no normalization), dim j coded with
 * dim_sigma[j] * unit codebook of its bits; with qjl, r = z_top - c_hat_top,
 * rnorms[v] = ||r||, sign_i = [(S r)_i >= 0] for i < k_top.  q->kind TQ_KIND_SPECTRAL.
 */
tq_status tq_quantize_spectral(const tq_quantizer* q, const void* x, int32_t dtype, int64_t n,
                               tq_packed out, tq_stream stream);

/*
 * Workspace bytes that tq_quantize_ws needs for n vectors of this quantizer and dtype; 0
 * when the call takes the same kernels as tq_quantize_mse / _prod / _spectral.
 */
tq_status tq_quantize_workspace(const tq_quantizer* q, int32_t dtype, int64_t n, size_t* bytes);

/*
 * DEVICE.  Quantize with caller-provided device scratch: the records are exactly those of
 * tq_quantize_mse / tq_quantize_prod / tq_quantize_spectral (by q->kind).  For fp32 input
 * with d a multiple of 128 (up to 4096; the review's d = 1536 vector-search embeddings),
 * MSE with 1..4 bits or PROD with 2..5 bits and m = d, the rotation and the QJL projection
 * run on the tensor cores as split-precision products (x, Pi, S and the residual split
 * into bf16 hi + lo parts in the workspace, three products per pair, fp32 accumulation),
 * in passes of up to 32768 vectors; the workspace holds the split operands of one pass.
 * Other shapes ignore the workspace.  workspace: device, >= tq_quantize_workspace bytes.
 */
tq_status tq_quantize_ws(const tq_quantizer* q, const void* x, int32_t dtype, int64_t n, tq_packed out,
                         void* workspace, size_t ws_bytes, tq_stream stream);

/*
 * Outlier-channel split (TurboQuant review, Method: for the KV-cache experiments the
 * channels are split into an outlier group and the rest, each quantized by its own
 * TurboQuant instance; the setting it calls 2.5-bit is 32 outlier channels at 3 bits plus
 * 96 channels at 2 bits).  Group g reads channels cols[g][0 .. groups[g]->d) of every
 * d-wide vector and is an independent MSE or PROD instance of dimension groups[g]->d,
 * with its own rotation, codebook, norm and packed records.  The descriptor and the
 * quantizers are host memory; cols[g] are DEVICE int32 arrays owned by the caller.
 * Channel indices must lie in 0..d-1; an index outside that range is read as channel 0
 * and sets the device status to TQ_ERR_INVALID_ARG (see tq_get_status).  For the
 * estimates below to be those of the split, the groups must be disjoint and cover every
 * channel; the library does not check this on the host (it would need a device read).
 */
#define TQ_MAX_GROUPS 4

typedef struct {
  int32_t n_groups;                           /* 1..TQ_MAX_GROUPS */
  int32_t d;                                  /* width of the full vectors */
  const tq_quantizer* groups[TQ_MAX_GROUPS];  /* kind TQ_KIND_MSE or TQ_KIND_PROD */
  const int32_t* cols[TQ_MAX_GROUPS];         /* DEVICE, groups[g]->d channel indices */
} tq_split;

/*
 * DEVICE.  Quantize n rows x [n*d] (dtype, row-major) group by group: out[g] receives
 * the records of group g (layout from tq_record_layout(groups[g])), the quantization by
 * groups[g] of the gathered rows (x_v[cols[g][0]], ..., x_v[cols[g][d_g - 1]]): what
 * tq_quantize_mse / tq_quantize_prod write for those rows, up to the code of a coordinate
 * within rounding of a boundary when the two calls run different kernels.  16-bit rows
 * of the outlier split of the KV experiments (d = 128, two MSE groups: 32 channels at 3
 * bits then 96 at 2, or 4 then 3) take one tensor-core pass over whole rows; other splits
 * gather their channels on the loads of the CUDA-core kernel.  out is a host array of
 * n_groups packed descriptors.  Validation as for tq_quantize_mse, per group.
 */
tq_status tq_quantize_split(const tq_split* sp, const void* x, int32_t dtype, int64_t n,
                            const tq_packed* out, tq_stream stream);

/* Workspace bytes needed by tq_score_split. */
tq_status tq_score_split_workspace(const tq_split* sp, int64_t nq, int64_t n, int32_t topk,
                                   size_t* bytes);

/*
 * DEVICE.  Split inner-product estimates: est(q, x_i) = sum over the groups of the
 * group's tq_score estimate for the gathered query q[cols[g]] against keys[g] (record i
 * of every group belongs to vector i).  Output as tq_score: topk == 0 gives scores
 * [nq*n] dense; topk in 1..32 gives the topk records of the summed estimate per query
 * (descending, ties to the lower id).  keys is a host array of n_groups packed
 * descriptors; workspace: device, >= tq_score_split_workspace bytes.  From 4096 records
 * (MSE groups of 1..4 bits or PROD groups of 2..5 bits with m = d, total width of the
 * groups' parts a multiple of 64) the estimates are one split-precision tensor-core
 * product; otherwise the CUDA-core estimator adds the groups.
 */
tq_status tq_score_split(const tq_split* sp, const void* qv, int32_t dtype, int64_t nq,
                         const tq_packed* keys, int64_t n, int32_t topk, float* scores,
                         int32_t* ids, void* workspace, size_t ws_bytes, tq_stream stream);

/* Workspace bytes needed by tq_decode_attn_split for this shape. */
tq_status tq_decode_attn_split_workspace(const tq_split* ks, const tq_split* vs, int32_t B,
                                         int32_t Hq, int32_t Hkv, int64_t Nmax, size_t* bytes);

/*
 * DEVICE.  One decode-attention step over split caches (keys split by ks, values by vs;
 * the splits may differ but have the same width d):
 *   logit_i = scale * sum_g est_g(q[cols_g], k_i,g),  p = softmax(logit),
 *   out[cols_g] = rot_g^T sum_i p_i ||v_i,g|| c_g[code_i,g]   for every value group g,
 * where est_g is the group's estimate: ||k|| <rot_g q', c_g[code]> for an MSE group, plus
 * ||k|| sqrt(pi/2)/m ||r|| <S_g rot_g q', 2s - 1> for a PROD group (TurboQuant review,
 * Method: the outlier and non-outlier channels are independent instances),
 * over the first seq_lens[b] records of each (b, kv-head) row; query head h reads KV head
 * h / (Hq/Hkv).  q [B*Hq*d] (dtype), seq_lens [B] device int32 (1..Nmax), kcache/vcache
 * host arrays of one packed descriptor per group, each group's records laid out
 * [B][Hkv][Nmax]; out [B*Hq*d] fp32.  libtq runs MSE or PROD key groups, MSE value
 * groups, d <= 256 and Hq/Hkv <= 8 (TQ_ERR_UNSUPPORTED otherwise).  The outlier split
 * of the KV experiments for keys and values (d = 128, two MSE groups: 32 rotated dims at
 * 3 bits then 96 at 2) with Hq/Hkv <= 4 and Nmax a multiple of 4 runs on the tensor
 * cores; other shapes on CUDA cores.  A value channel index out of
 * range sets TQ_ERR_INVALID_ARG on the device and its output is not written.
 */
tq_status tq_decode_attn_split(const tq_split* ks, const tq_split* vs, const void* q,
                               int32_t dtype, int32_t B, int32_t Hq, int32_t Hkv, int64_t Nmax,
                               const int32_t* seq_lens, const tq_packed* kcache,
                               const tq_packed* vcache, float scale, float* out, void* workspace,
                               size_t ws_bytes, tq_stream stream);

/*
 * DEVICE.  Reconstruction out [n*d] fp32: MSE x_hat = ||x|| rot^T c[code];
 * PROD adds ||x|| rot^T (sqrt(pi/2)/m ||r|| S^T (2s-1)) (unbiased);
 * SPECTRAL x_hat = rot^T c_hat (the QJL bits are not used).
 */
tq_status tq_dequantize(const tq_quantizer* q, tq_packed in, int64_t n, float* out,
                        tq_stream stream);

/*
 * Workspace bytes needed by tq_score for nq queries against n records with topk (0 = dense).
 */
tq_status tq_score_workspace(const tq_quantizer* q, int64_t nq, int64_t n, int32_t topk,
                             size_t* bytes);

/*
 * DEVICE.  Inner-product estimates of queries qv [nq*d] (dtype) against n packed records:
 *   MSE       ||x|| <rot q, c[code]>
 *   PROD      ||x|| (<rot q, c_hat> + sqrt(pi/2)/m ||r|| <S rot q, 2s-1>)   (unbiased)
 *   SPECTRAL  sum_j (rot q)_j c_hat_j + sqrt(pi/2)/k ||r|| <S (rot q)_top, 2s-1>
 * topk == 0: scores [nq*n] fp32 dense, ids unused.  topk in 1..32: for each query the
 * topk records by descending estimate, ties to the lower id: ids [nq*topk] int32,
 * scores [nq*topk].  workspace: device, >= tq_score_workspace bytes.
 * From 4096 records with d a multiple of 128 (MSE 1..4 bits, PROD 2..5 bits with m = d) the
 * estimates are one split-precision tensor-core product; its top-k keeps the best of
 * segments of ~16k estimates and then of their candidates (the one-pass result).
 */
tq_status tq_score(const tq_quantizer* q, const void* qv, int32_t dtype, int64_t nq,
                   tq_packed keys, int64_t n, int32_t topk, float* scores, int32_t* ids,
                   void* workspace, size_t ws_bytes, tq_stream stream);

/* Workspace bytes needed by tq_decode_attn for this shape. */
tq_status tq_decode_attn_workspace(const tq_quantizer* kq, int32_t B, int32_t Hq, int32_t Hkv,
                                   int64_t Nmax, size_t* bytes);

/*
 * DEVICE.  One decode-attention step straight from the packed cache:
 *   for query head h (KV head h / (Hq/Hkv)), logit_i = scale * est(q_h, k_i) over the
 *   first seq_lens[b] records, p = softmax(logit), out = sum_i p_i v_hat_i.
 * q [B*Hq*d] (dtype), seq_lens [B] device int32 (1..Nmax), caches laid out
 * [B][Hkv][Nmax] records, out [B*Hq*d] fp32.  Keys: MSE, PROD or SPECTRAL; values: MSE,
 * PROD or SPECTRAL (without qjl).  Values as PROD use their unbiased reconstruction
 * ||v|| rot^T (c[code] + sqrt(pi/2)/m ||r|| S^T (2s-1)) (review, Method; the sign part is
 * accumulated in the sketch domain and mapped back once per row).  libtq runs d = 128,
 * code bits <= 4, PROD m = d, Hq/Hkv in 1..16; other shapes give TQ_ERR_UNSUPPORTED.  Value norms must stay below
 * 6.0e4 (the probability-weighted norm is a half-precision MMA operand).  The call
 * enqueues three kernels (query preparation, decode, chunk combine); the last two use
 * programmatic dependent launch, so each may start while the one before it drains, and
 * every read of a predecessor's output waits for that kernel to complete.
 */
tq_status tq_decode_attn(const tq_quantizer* kq, const tq_quantizer* vq, const void* q,
                         int32_t dtype, int32_t B, int32_t Hq, int32_t Hkv, int64_t Nmax,
                         const int32_t* seq_lens, tq_packed kcache, tq_packed vcache,
                         float scale, float* out, void* workspace, size_t ws_bytes,
                         tq_stream stream);

/*
 * Paged record pool (TurboQuant review, "Comparison": serving engines keep the cache in
 * pages and quantize the tokens generated during decoding into it).  Every record array of
 * a pool (codes, signs, norms, rnorms) holds num_pages pages; page p holds page_size
 * consecutive records for each KV head, so token t of sequence b and KV head h is record
 *     (block_table[b * max_pages + t / page_size] * Hkv + h) * page_size + t % page_size.
 * block_table is a DEVICE int32 array [B][max_pages] owned by the caller; page ids must
 * lie in 0..num_pages-1 (a page id out of range is read as page 0 and sets the device
 * status to TQ_ERR_INVALID_ARG).  page_size is a multiple of 16.
 */
typedef struct {
  const int32_t* block_table;
  int32_t page_size;
  int32_t max_pages;
  int64_t num_pages;
} tq_pages;

/*
 * DEVICE.  One decode step over a paged cache, appending the step's token first (review,
 * "Comparison": decode-time tokens are quantized too).  For every (b, kv-head h):
 *   1. k_new / v_new row b * Hkv + h ([B*Hkv*d], dtype) is quantized with kq / vq into
 *      the record of token seq_lens[b] - 1 (its slot from the block table);
 *   2. attention as tq_decode_attn over tokens 0..seq_lens[b]-1 of the pool.
 * k_new and v_new may both be NULL (no append).  seq_lens [B] device int32 counts the
 * tokens including the appended one (1..max_pages*page_size).  Workspace: the bytes
 * tq_decode_attn_workspace gives for Nmax = max_pages * page_size.  Keys MSE or PROD,
 * values MSE (spectral records are not paged: TQ_ERR_UNSUPPORTED).  The append runs as
 * one extra kernel per array before the attention kernels, in stream order.
 */
tq_status tq_decode_attn_paged(const tq_quantizer* kq, const tq_quantizer* vq, const void* q,
                               const void* k_new, const void* v_new, int32_t dtype, int32_t B, int32_t Hq,
                               int32_t Hkv, const int32_t* seq_lens, const tq_pages* pages,
                               tq_packed kpool, tq_packed vpool, float scale, float* out, void* workspace,
                               size_t ws_bytes, tq_stream stream);

/* Workspace bytes needed by tq_prefill_attn for this shape. */
tq_status tq_prefill_attn_workspace(const tq_quantizer* kq, int32_t B, int32_t Hq, int32_t Hkv, int32_t T,
                                    int64_t Nmax, size_t* bytes);

/*
 * DEVICE.  Causal prefill attention over the packed cache (TurboQuant launch kit, X thread
 * and Show HN post: prefill at long context runs over the compressed cache).  For a block
 * of T queries per sequence, q [B][Hq][T][d] (dtype), query (b, h, i) sits at absolute
 * position q_pos[b * T + i] (DEVICE int32 [B][T], 0-based) and attends, with the decode
 * step's scale and GQA map, to the cached tokens 0..q_pos[b*T+i] of its KV head:
 *   out[b][h][i] = sum_{t <= pos} softmax_t(scale * est(q, k_t)) v_hat_t.
 * kv_lens [B] (device int32) is the number of cached tokens of each sequence; every
 * position must be below it.  The cache is the packed [B][Hkv][Nmax] layout (pages NULL)
 * or a paged pool (pages non-NULL, Nmax ignored and taken as max_pages * page_size).
 * out [B][Hq][T][d] fp32.  Keys MSE or PROD, values MSE, d = 128.  The cache must already
 * hold the block's own tokens (quantize them first, as for decode).
 */
tq_status tq_prefill_attn(const tq_quantizer* kq, const tq_quantizer* vq, const void* q, int32_t dtype,
                          int32_t B, int32_t Hq, int32_t Hkv, int32_t T, const int32_t* q_pos,
                          const int32_t* kv_lens, const tq_pages* pages, int64_t Nmax, tq_packed kcache,
                          tq_packed vcache, float scale, float* out, void* workspace, size_t ws_bytes,
                          tq_stream stream);

/* Size of the fixed device scratch array behind tq_decode_attn_fixed_ws (8 MiB per device). */
#define TQ_DECODE_FIXED_WS_BYTES (8u << 20)

/*
 * DEVICE.  The same step as tq_decode_attn, with the same arguments, results and errors,
 * but it allocates nothing and takes no workspace: its scratch is one file-scope device
 * array of TQ_DECODE_FIXED_WS_BYTES in this library (one per device).  The pages have no
 * counterpart of this call; it serves callers that cannot hand over device scratch.
 *   - A shape whose tq_decode_attn_workspace exceeds TQ_DECODE_FIXED_WS_BYTES returns
 *     TQ_ERR_WORKSPACE before any launch (the 128k-token workload with B = 8, Hq = 32
 *     needs about 4.9 MB).
 *   - The first call on a device, with that device current, looks up the array address
 *     (cudaGetSymbolAddress); make it before any latency-critical loop.  A failed lookup
 *     returns TQ_ERR_CUDA.  The address is kept per device and belongs to the device's
 *     primary context: calls under another driver context, or after cudaDeviceReset,
 *     are not supported.
 *   - Shape and descriptor errors are those of tq_decode_attn and are checked first;
 *     TQ_ERR_WORKSPACE means a valid shape whose scratch exceeds the array.
 *   - All calls on one device share the array: calls that can overlap in time (other
 *     streams, unordered host threads) race on it; calls in order on one stream do not.
 *     Nothing in it has to start at zero.
 */
tq_status tq_decode_attn_fixed_ws(const tq_quantizer* kq, const tq_quantizer* vq, const void* q,
                                  int32_t dtype, int32_t B, int32_t Hq, int32_t Hkv, int64_t Nmax,
                                  const int32_t* seq_lens, tq_packed kcache, tq_packed vcache,
                                  float scale, float* out, tq_stream stream);

/*
 * Synchronizes `stream`, then returns and clears the device status word of the current
 * device: TQ_OK, or TQ_ERR_TIMEOUT if a bounded device wait ran out since the last call.
 */
tq_status tq_get_status(tq_stream stream);

/*
 * Test hook: iteration limit of every device-side bounded wait launched after this call
 * (0 = default, about 2^24 polls).  Lowering it makes waits that are not immediately
 * satisfied time out; TQ_WAIT_EXPIRE_AT_ONCE (-1) makes every bounded wait give up before
 * its first poll, so a kernel with such a wait reports TQ_ERR_TIMEOUT on every launch.
 * Either way the kernel drains the copies it issued, frees its tensor memory and exits;
 * nothing hangs and the context stays usable.  Other negative values: TQ_ERR_INVALID_ARG.
 */
#define TQ_WAIT_EXPIRE_AT_ONCE (-1)
tq_status tq_set_wait_limit(int64_t polls);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
