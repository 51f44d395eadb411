// Device helpers shared by the libtq kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "../../include/tq.h"

namespace tq {

// Status codes written to the device status word (first writer wins).
constexpr int kDevOk = 0;
constexpr int kDevTimeout = TQ_ERR_TIMEOUT;

__device__ __forceinline__ void report_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Programmatic dependent launch.  A kernel launched with the programmatic-serialization
// attribute may begin while the kernel before it in the stream is still running:
// pdl_wait() returns once that kernel has completed and its writes are visible, and
// pdl_trigger() lets the kernel after this one begin launching.  Both are no-ops for a
// kernel launched the ordinary way.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float load_elem(const void* base, int dtype, int64_t i) {
  if (dtype == TQ_F32) return __ldg(reinterpret_cast<const float*>(base) + i);
  if (dtype == TQ_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return __half2float(reinterpret_cast<const __half*>(base)[i]);
}

// Number of boundaries strictly below y (nearest centroid, ties to the lower cell).
__device__ __forceinline__ int count_below(const float* t, int nb, float y) {
  int lo = 0, hi = nb;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (t[mid] < y) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Extract `nbits` (<= 32) starting at bit `pos` of a little-endian word stream.
__device__ __forceinline__ uint32_t stream_bits(const uint32_t* w, int pos, int nbits) {
  const int wi = pos >> 5, sh = pos & 31;
  uint64_t v = w[wi];
  if (sh + nbits > 32) v |= static_cast<uint64_t>(w[wi + 1]) << 32;
  v >>= sh;
  return static_cast<uint32_t>(v & ((nbits >= 32) ? 0xffffffffull : ((1ull << nbits) - 1ull)));
}

__host__ __device__ __forceinline__ int words_for(int count, int bits) {
  return (count * bits + 31) >> 5;
}

// Offsets of the b-bit standard-normal codebook inside the concatenated 1..8-bit tables.
__host__ __device__ __forceinline__ int unit_c_off(int b) { return (1 << b) - 2; }
__host__ __device__ __forceinline__ int unit_t_off(int b) { return (1 << b) - b - 1; }

}  // namespace tq
