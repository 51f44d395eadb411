// Instantiations of the decode kernels for spectral keys and values (D = 128): the
// bulk-copy staged kernel for 1-bit tails with one head word, the 4-warp kernel otherwise.
#include "decode.cuh"
#include "decode_tma.cuh"
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

template <bool PK>
cudaError_t go_tma(const DecodeParams& p, dim3 grid, cudaStream_t s, int* status, long long lim) {
  auto k = decode_tma_kernel<KFMT_SPEC, 1, 1, PK>;
  const size_t smem = decode_tma_smem_bytes(1, 1, KFMT_SPEC, PK);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // the query preparation kernel runs just before: the prologue and the first copies overlap it
  return launch_pdl(k, grid, dim3((tma_consumers(KFMT_SPEC, PK) + 1) * 32), smem, s, p, status, lim);
}

}  // namespace

cudaError_t launch_decode_spec_tma(const DecodeParams& p, dim3 grid, cudaStream_t s, int* status, long long lim) {
  return p.G <= 4 ? go_tma<true>(p, grid, s, status, lim) : go_tma<false>(p, grid, s, status, lim);
}

cudaError_t launch_decode_spec(const DecodeParams& p, int kb, int vb, dim3 grid, size_t smem, cudaStream_t s) {
  switch (kb * 10 + vb) {
    case 11: return go<1, 1>(p, grid, smem, s);
    case 22: return go<2, 2>(p, grid, smem, s);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace tq
