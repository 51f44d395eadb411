// Instantiations of decode_attn_kernel with keys in the mse format (D = 128).
#include "decode.cuh"
#include "launchers.h"

namespace tq {
namespace {

template <int KB, int VB>
cudaError_t go(const DecodeParams& p, dim3 grid, size_t smem, cudaStream_t s) {
  auto k = decode_attn_kernel<128, KFMT_MSE, KB, VFMT_MSE, VB>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  k<<<grid, kDecThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_mse(const DecodeParams& p, int kb, int vb, dim3 grid, size_t smem, cudaStream_t s) {
  switch (kb * 10 + vb) {
    case 11: return go<1, 1>(p, grid, smem, s);
    case 12: return go<1, 2>(p, grid, smem, s);
    case 13: return go<1, 3>(p, grid, smem, s);
    case 14: return go<1, 4>(p, grid, smem, s);
    case 21: return go<2, 1>(p, grid, smem, s);
    case 22: return go<2, 2>(p, grid, smem, s);
    case 23: return go<2, 3>(p, grid, smem, s);
    case 24: return go<2, 4>(p, grid, smem, s);
    case 31: return go<3, 1>(p, grid, smem, s);
    case 32: return go<3, 2>(p, grid, smem, s);
    case 33: return go<3, 3>(p, grid, smem, s);
    case 34: return go<3, 4>(p, grid, smem, s);
    case 41: return go<4, 1>(p, grid, smem, s);
    case 42: return go<4, 2>(p, grid, smem, s);
    case 43: return go<4, 3>(p, grid, smem, s);
    case 44: return go<4, 4>(p, grid, smem, s);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace tq
