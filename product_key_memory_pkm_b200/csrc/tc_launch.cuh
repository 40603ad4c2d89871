// Host launcher of the tcgen05 GEMM engine for one problem type.
#pragma once

#include <mutex>

#include "tc_gemm.cuh"

namespace pkm {
namespace tc {

template <class Prob>
cudaError_t launch_tc(const CUtensorMap& A0, const CUtensorMap& A1, const CUtensorMap& B,
                      const typename Prob::Params& P, int nunits, int sm_count, cudaStream_t st,
                      const CUtensorMap* B1 = nullptr, const CUtensorMap* O0 = nullptr,
                      const CUtensorMap* O1 = nullptr) {
  constexpr size_t smem = smem_bytes<Prob>();
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, []() {
    attr_err = cudaFuncSetAttribute(tc_gemm_kernel<Prob>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int grid = nunits < sm_count ? nunits : sm_count;
  if (grid <= 0) return cudaSuccess;
  tc_gemm_kernel<Prob><<<grid, threads_of<Prob>(), smem, st>>>(A0, A1, B, B1 ? *B1 : B,
                                                               O0 ? *O0 : B, O1 ? *O1 : B, P);
  PKM_COUNT(1);
  return cudaGetLastError();
}

}  // namespace tc
}  // namespace pkm
