// Instantiations of the bulk-copy staged decode kernel with prod keys and MSE values (d = 128).
#include "decode_tma.cuh"
#include "launchers.h"

namespace tq {
namespace {

template <int KB, int VB, bool PK>
cudaError_t go_pk(const DecodeParams& p, dim3 grid, size_t smem, cudaStream_t s, int* status, long long lim) {
  auto k = decode_tma_kernel<KFMT_PROD, KB, VB, PK>;
  smem = decode_tma_smem_bytes(KB, VB, KFMT_PROD, PK);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // the query preparation kernel runs just before: the prologue and the first copies overlap it
  return launch_pdl(k, grid, dim3((tma_consumers(KFMT_PROD, PK) + 1) * 32), smem, s, p, status, lim);
}

// GQA groups of at most 4 heads take the packed-column variant
template <int KB, int VB>
cudaError_t go(const DecodeParams& p, dim3 grid, size_t smem, cudaStream_t s, int* status, long long lim) {
  return p.G <= 4 ? go_pk<KB, VB, true>(p, grid, smem, s, status, lim)
                  : go_pk<KB, VB, false>(p, grid, smem, s, status, lim);
}

}  // namespace

cudaError_t launch_decode_prod(const DecodeParams& p, int kb, int vb, dim3 grid, size_t, cudaStream_t s,
                              int* status, long long lim) {
  size_t smem = 0;
  switch (kb * 10 + vb) {
    case 11: return go<1, 1>(p, grid, smem, s, status, lim);
    case 12: return go<1, 2>(p, grid, smem, s, status, lim);
    case 13: return go<1, 3>(p, grid, smem, s, status, lim);
    case 14: return go<1, 4>(p, grid, smem, s, status, lim);
    case 21: return go<2, 1>(p, grid, smem, s, status, lim);
    case 22: return go<2, 2>(p, grid, smem, s, status, lim);
    case 23: return go<2, 3>(p, grid, smem, s, status, lim);
    case 24: return go<2, 4>(p, grid, smem, s, status, lim);
    case 31: return go<3, 1>(p, grid, smem, s, status, lim);
    case 32: return go<3, 2>(p, grid, smem, s, status, lim);
    case 33: return go<3, 3>(p, grid, smem, s, status, lim);
    case 34: return go<3, 4>(p, grid, smem, s, status, lim);
    case 41: return go<4, 1>(p, grid, smem, s, status, lim);
    case 42: return go<4, 2>(p, grid, smem, s, status, lim);
    case 43: return go<4, 3>(p, grid, smem, s, status, lim);
    case 44: return go<4, 4>(p, grid, smem, s, status, lim);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace tq
