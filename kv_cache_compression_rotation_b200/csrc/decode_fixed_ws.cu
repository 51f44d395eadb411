// tq_decode_attn_fixed_ws: the decode-attention step with its scratch in a fixed
// device array of this library instead of a caller-supplied workspace.
//
// Some callers have no way to hand over device scratch: a C host that links only this
// library and owns no device allocator, or a serving loop whose device memory is all
// reserved up front by its own cache pool and which must not call cudaMalloc between
// steps (cudaMalloc and cudaFree take driver locks and can synchronize the device).
// For them the scratch lives in one file-scope __device__ array, sized for modest
// shapes; a shape that needs more is refused with TQ_ERR_WORKSPACE.
//
// The first call on a device (with that device current) looks up the array's address
// with cudaGetSymbolAddress; that call should come before any latency-critical loop.
// Every later call on the device reuses the address, which belongs to the device's
// primary context (the one the CUDA runtime uses): calls made under another driver
// context, or after cudaDeviceReset of the device, are not supported.  All calls on one device share the
// array, so two calls that can overlap in time (different streams, or different host
// threads without ordering between them) race on it; calls issued in order on one
// stream do not.  Nothing in the array needs to start at zero: each call writes every
// scratch byte it later reads.

#include <cuda_runtime.h>

#include <mutex>

#include "tq_internal.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_fixed_ws[TQ_DECODE_FIXED_WS_BYTES];

std::mutex g_fixed_mu;
void* g_fixed_ptr[kMaxDevices] = {};

}  // namespace

extern "C" tq_status tq_decode_attn_fixed_ws(const tq_quantizer* kq, const tq_quantizer* vq, const void* q,
                                             int32_t dtype, int32_t B, int32_t Hq, int32_t Hkv, int64_t Nmax,
                                             const int32_t* seq_lens, tq_packed kcache, tq_packed vcache,
                                             float scale, float* out, tq_stream stream) {
  // the shape checks of tq_decode_attn come first, so a bad shape gets the same status
  // from both entry points whatever its scratch size
  tq_status s = tq::decode_shape_ok(kq, vq, B, Hq, Hkv, Nmax);
  if (s != TQ_OK) return s;
  size_t need = 0;
  s = tq_decode_attn_workspace(kq, B, Hq, Hkv, Nmax, &need);
  if (s != TQ_OK) return s;
  if (need > static_cast<size_t>(TQ_DECODE_FIXED_WS_BYTES))
    return tq::fail(TQ_ERR_WORKSPACE, "shape needs %zu scratch bytes; the fixed array holds %zu", need,
                    static_cast<size_t>(TQ_DECODE_FIXED_WS_BYTES));
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tq::fail(TQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return tq::fail(TQ_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_fixed_mu);
    if (!g_fixed_ptr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_fixed_ws);
      if (e != cudaSuccess)
        return tq::fail(TQ_ERR_CUDA, "cudaGetSymbolAddress of the fixed decode scratch: %s", cudaGetErrorString(e));
      if (!p) return tq::fail(TQ_ERR_CUDA, "fixed decode scratch has no device address");
      g_fixed_ptr[dev] = p;
    }
    ws = g_fixed_ptr[dev];
  }
  return tq_decode_attn(kq, vq, q, dtype, B, Hq, Hkv, Nmax, seq_lens, kcache, vcache, scale, out, ws,
                        static_cast<size_t>(TQ_DECODE_FIXED_WS_BYTES), stream);
}
