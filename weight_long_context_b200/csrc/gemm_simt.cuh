// CUDA-core GEMM engine: D[z](m, n) = sum_k A[z](m, k) * B[z](n, k) with
// float32 accumulation, for the fp32 mode (tolerance 1e-4 on the final state
// rules out tf32 tensor-core arithmetic).  Operands may be K-major or
// MN-major; the epilogue receives each row in 32-column spans.
#pragma once

#include "common.cuh"
#include "gemm_types.cuh"

namespace ttt {

namespace simt {
constexpr int BM = 64;
constexpr int BN = 64;
constexpr int BK = 16;
constexpr int THREADS = 256;
}  // namespace simt

template <typename T>
__device__ __forceinline__ float simt_load(const Operand& op, int z, int mn, int k, int MN, int K) {
  if (mn >= MN || k >= K) return 0.f;
  const T* p = static_cast<const T*>(op.ptr) + (int64_t)z * op.batch_stride;
  int64_t off = op.kmajor ? (int64_t)mn * op.ld + k : (int64_t)k * op.ld + mn;
  return to_f<T>(p[off]);
}

// NACC == 2: dualb = 0 -> acc_j = A_j B^T (A2 is a second A operand);
// dualb = 1 -> acc_j = A B_j^T (A2 carries the second B operand, staged in the
// otherwise unused second A tile).
template <typename T, int NACC, class Epi>
__global__ void __launch_bounds__(simt::THREADS)
gemm_simt_kernel(GemmShape s, Operand A, Operand A2, Operand B, Epi epi, int dualb) {
  using namespace simt;
  __shared__ float As[NACC][BK][BM + 1];
  __shared__ float Bs[BK][BN + 1];
  __shared__ float Cs[NACC][BM][BN + 1];

  const int z = blockIdx.z;
  const int m0 = blockIdx.y * BM;
  const int n0 = blockIdx.x * BN;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;

  float acc[NACC][4][4];
#pragma unroll
  for (int a = 0; a < NACC; ++a)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[a][i][j] = 0.f;

  // The next k-tile's operands are loaded into registers while the current
  // tile is multiplied (one global-load latency per tile is hidden).
  constexpr int PER = (BM * BK) / THREADS;
  float ra[2][PER], rb[PER];
  auto load_tile = [&](int k0) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int idx = tid + i * THREADS;
      int mm, kk, nn;
      if (A.kmajor) { mm = idx / BK; kk = idx % BK; } else { kk = idx / BM; mm = idx % BM; }
      ra[0][i] = simt_load<T>(A, z, m0 + mm, k0 + kk, s.M, s.K);
      if (NACC == 2 && !dualb) ra[1][i] = simt_load<T>(A2, z, m0 + mm, k0 + kk, s.M, s.K);
      if (B.kmajor) { nn = idx / BK; kk = idx % BK; } else { kk = idx / BN; nn = idx % BN; }
      rb[i] = simt_load<T>(B, z, n0 + nn, k0 + kk, s.N, s.K);
      if (NACC == 2 && dualb) ra[1][i] = simt_load<T>(A2, z, n0 + nn, k0 + kk, s.N, s.K);
    }
  };
  auto store_tile = [&]() {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int idx = tid + i * THREADS;
      int mm, kk, nn;
      if (A.kmajor) { mm = idx / BK; kk = idx % BK; } else { kk = idx / BM; mm = idx % BM; }
      As[0][kk][mm] = ra[0][i];
      if (NACC == 2 && !dualb) As[NACC - 1][kk][mm] = ra[1][i];
      if (B.kmajor) { nn = idx / BK; kk = idx % BK; } else { kk = idx / BN; nn = idx % BN; }
      Bs[kk][nn] = rb[i];
      if (NACC == 2 && dualb) As[NACC - 1][kk][nn] = ra[1][i];
    }
  };
  if (s.K > 0) load_tile(0);
  for (int k0 = 0; k0 < s.K; k0 += BK) {
    store_tile();
    __syncthreads();
    if (k0 + BK < s.K) load_tile(k0 + BK);
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float b[NACC][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b[0][j] = Bs[kk][tx * 4 + j];
        if (NACC == 2) b[NACC - 1][j] = dualb ? As[NACC - 1][kk][tx * 4 + j] : b[0][j];
      }
#pragma unroll
      for (int a = 0; a < NACC; ++a) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float av = As[(NACC == 2 && dualb) ? 0 : a][kk][ty * 4 + i];
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[a][i][j] = fmaf(av, b[a][j], acc[a][i][j]);
        }
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int a = 0; a < NACC; ++a)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) Cs[a][ty * 4 + i][tx * 4 + j] = acc[a][i][j];
  __syncthreads();

  if (tid < BM) {
    int r = m0 + tid;
    if (r < s.M) {
      typename Epi::RowState st;
      epi.row_begin(st, z, r);
#pragma unroll 1
      for (int sp = 0; sp < BN / 32; ++sp) {
        int c0 = n0 + sp * 32;
        if (c0 >= s.N) break;
        int nv = min(32, s.N - c0);
        float v[32], v2[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] = Cs[0][tid][sp * 32 + j];
          v2[j] = Cs[NACC - 1][tid][sp * 32 + j];
        }
        if constexpr (Epi::kPreload) epi.preload(st, z, r, c0, nv);
        epi.span(st, z, r, c0, v, v2, nv);
      }
      epi.row_end(st, z, r, blockIdx.x);
    }
  }
}

template <typename T, int NACC, class Epi>
cudaError_t launch_gemm_simt(const GemmShape& s, const Operand& A, const Operand& A2,
                             const Operand& B, const Epi& epi, cudaStream_t st, int dualb = 0) {
  if (s.M <= 0 || s.N <= 0 || s.batch <= 0) return cudaSuccess;
  dim3 grid((s.N + simt::BN - 1) / simt::BN, (s.M + simt::BM - 1) / simt::BM, s.batch);
  gemm_simt_kernel<T, NACC, Epi><<<grid, simt::THREADS, 0, st>>>(s, A, A2, B, epi, dualb);
  return cudaGetLastError();
}

}  // namespace ttt
