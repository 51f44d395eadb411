// Instantiations of decode_attn_kernel with keys in the spec format (D = 128).
#include "decode.cuh"
#include "launchers.h"

namespace tq {
namespace {

template <int KB, int VB>
cudaError_t go(const DecodeParams& p, dim3 grid, size_t smem, cudaStream_t s) {
  auto k = decode_attn_kernel<128, KFMT_SPEC, KB, VFMT_SPEC, VB>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  k<<<grid, kDecThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_spec(const DecodeParams& p, int kb, int vb, dim3 grid, size_t smem, cudaStream_t s) {
  switch (kb * 10 + vb) {
    case 11: return go<1, 1>(p, grid, smem, s);
    case 22: return go<2, 2>(p, grid, smem, s);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace tq
