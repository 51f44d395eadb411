// Instantiations of the bulk-copy staged decode kernel with values quantized as
// TurboQuant-prod (MSE stage of 1..4 bits plus 128 QJL signs and gamma per value), keys MSE
// or PROD, d = 128.
#include "decode_tma.cuh"
#include "launchers.h"

namespace tq {
namespace {

template <int KF, int KB, int VB, bool PK>
cudaError_t go_pk(const DecodeParams& p, dim3 grid, cudaStream_t s, int* status, long long lim) {
  auto k = decode_tma_kernel<KF, KB, VB, PK, false, true>;
  const size_t smem = decode_tma_smem_bytes(KB, VB, KF, PK, true);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(k, grid, dim3((tma_consumers(KF, PK) + 1) * 32), smem, s, p, status, lim);
}

template <int KF, int KB, int VB>
cudaError_t go(const DecodeParams& p, dim3 grid, cudaStream_t s, int* status, long long lim) {
  return p.G <= 4 ? go_pk<KF, KB, VB, true>(p, grid, s, status, lim) : go_pk<KF, KB, VB, false>(p, grid, s, status, lim);
}

template <int KF>
cudaError_t pick(const DecodeParams& p, int kb, int vb, dim3 grid, cudaStream_t s, int* status, long long lim) {
  switch (kb * 10 + vb) {
    case 11: return go<KF, 1, 1>(p, grid, s, status, lim);
    case 12: return go<KF, 1, 2>(p, grid, s, status, lim);
    case 13: return go<KF, 1, 3>(p, grid, s, status, lim);
    case 14: return go<KF, 1, 4>(p, grid, s, status, lim);
    case 21: return go<KF, 2, 1>(p, grid, s, status, lim);
    case 22: return go<KF, 2, 2>(p, grid, s, status, lim);
    case 23: return go<KF, 2, 3>(p, grid, s, status, lim);
    case 24: return go<KF, 2, 4>(p, grid, s, status, lim);
    case 31: return go<KF, 3, 1>(p, grid, s, status, lim);
    case 32: return go<KF, 3, 2>(p, grid, s, status, lim);
    case 33: return go<KF, 3, 3>(p, grid, s, status, lim);
    case 34: return go<KF, 3, 4>(p, grid, s, status, lim);
    case 41: return go<KF, 4, 1>(p, grid, s, status, lim);
    case 42: return go<KF, 4, 2>(p, grid, s, status, lim);
    case 43: return go<KF, 4, 3>(p, grid, s, status, lim);
    case 44: return go<KF, 4, 4>(p, grid, s, status, lim);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_decode_vprod(const DecodeParams& p, int kfmt, int kb, int vb, dim3 grid, cudaStream_t s,
                                int* status, long long lim) {
  if (kfmt == KFMT_MSE) return pick<KFMT_MSE>(p, kb, vb, grid, s, status, lim);
  if (kfmt == KFMT_PROD) return pick<KFMT_PROD>(p, kb, vb, grid, s, status, lim);
  return cudaErrorNotSupported;
}

}  // namespace tq
