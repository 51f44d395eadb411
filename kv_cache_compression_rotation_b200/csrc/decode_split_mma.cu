// Instantiation of the tensor-core split-cache decode (32 rotated dims at 3 bits, then 96
// at 2 bits: the 2.5-bit outlier split).
#include "decode_split_mma.cuh"
#include "launchers.h"

namespace tq {

cudaError_t launch_decode_split_mma(const SplitMmaParams& p, int grid, cudaStream_t s, int* status, long long lim) {
  auto k = decode_split_mma_kernel<32, 3, 2>;
  const size_t smem = decode_split_mma_smem(32, 3, 2);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  k<<<grid, kSmThreads, smem, s>>>(p, status, lim);
  return cudaGetLastError();
}

}  // namespace tq
