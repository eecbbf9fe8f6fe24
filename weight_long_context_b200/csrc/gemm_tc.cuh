// tcgen05 GEMM engine (placeholder: routes to the CUDA-core engine).
#pragma once
#include "gemm_simt.cuh"
namespace ttt { namespace tc {
constexpr int HEAD_BN = simt::BN;
template <int NACC, class Epi>
cudaError_t launch_gemm_tc(const GemmShape& s, const Operand& A, const Operand& A2, const Operand& B,
                           const Epi& epi, cudaStream_t st, int*) {
  return launch_gemm_simt<__nv_bfloat16, NACC, Epi>(s, A, A2, B, epi, st);
}
}}
