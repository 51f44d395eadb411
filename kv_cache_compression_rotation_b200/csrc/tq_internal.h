// Internal declarations shared by the libtq translation units (host side).
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/tq.h"

namespace tq {

// Records a thread-local message and returns the status (for `return fail(...)`).
tq_status fail(tq_status s, const char* fmt, ...);

// Host math (host_math.cpp).
tq_status codebook_build(int d, int bits, int dist, double sigma, double* c_out, double* t_out,
                         int* iters_out);
tq_status waterfill(const double* lambda, int k, int budget, int max_bits, int32_t* out);
tq_status spectral_calibrate(const float* X, int64_t n, int d, double* vecs, double* vals);
tq_status spectral_unit_codebooks(double* c_out, double* t_out);
tq_status lut_scale(const double* values, int count, float* scale_out);
tq_status spectral_descriptor(const double* vecs, const double* vals, int d, int k_top, int budget, int tail_bits,
                              int max_bits, float* rot_out, float* sigma_out, float* unit_c_out, float* unit_t_out,
                              int32_t* top_bits_out, float* lut_scale_out);

// The shape and descriptor checks tq_decode_attn runs before anything else (tq_api.cu).
tq_status decode_shape_ok(const tq_quantizer* kq, const tq_quantizer* vq, int B, int Hq, int Hkv, int64_t Nmax);

// Device-side status word and wait limit (tq_api.cu).
int* device_status_ptr();      // address of the current device's status word
long long wait_limit();        // polls per bounded wait

}  // namespace tq
