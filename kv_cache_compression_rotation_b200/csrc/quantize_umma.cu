// Instantiations of the tensor-core quantize kernel.
#include "launchers.h"
#include "quantize_umma.cuh"

namespace tq {
namespace {

template <int B, bool SPEC = false, bool PRODK = false, int B1 = 0>
cudaError_t go(const CUtensorMap& map, const UmmaQuantParams& p, int grid, cudaStream_t s) {
  auto k = umma_quantize_kernel<B, SPEC, PRODK, B1>;
  const uint32_t smem = PRODK ? kUmmaProdSmemBytes : kUmmaSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  k<<<grid, kUmmaThreads, smem, s>>>(map, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_umma_quantize(const CUtensorMap& map, const UmmaQuantParams& p, int bits, int grid,
                                 cudaStream_t s) {
  if (bits == 0) return go<1, true>(map, p, grid, s);       // spectral records
  switch (bits) {
    case 1: return go<1>(map, p, grid, s);
    case 2: return go<2>(map, p, grid, s);
    case 3: return go<3>(map, p, grid, s);
    case 4: return go<4>(map, p, grid, s);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t launch_umma_quantize_prod(const CUtensorMap& map, const UmmaQuantParams& p, int mse_bits, int grid,
                                      cudaStream_t s) {
  switch (mse_bits) {
    case 1: return go<1, false, true>(map, p, grid, s);
    case 2: return go<2, false, true>(map, p, grid, s);
    case 3: return go<3, false, true>(map, p, grid, s);
    case 4: return go<4, false, true>(map, p, grid, s);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t launch_umma_quantize_split(const CUtensorMap& map, const UmmaQuantParams& p, int b0, int b1, int grid,
                                       cudaStream_t s) {
  if (b0 == 3 && b1 == 2) return go<3, false, false, 2>(map, p, grid, s);
  if (b0 == 4 && b1 == 3) return go<4, false, false, 3>(map, p, grid, s);
  return cudaErrorNotSupported;
}

}  // namespace tq
