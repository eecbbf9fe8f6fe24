// K1: the scalar kernels of Proposition 3.1 for every chunk in one launch
// ("Rethinking Expressivity and Efficiency in Test-Time Training",
// 定义高效后缀乘积与比例和 and 命题3.1).
//
// For a chunk of C tokens (0-based k = t - 1):
//   bt[k] = prod_{i>k} beta_i        (suffix product, bt[C-1] = 1)
//   gt[k] = prod_{i>k} gamma_i       (gt[C-1] = 1)
//   S[k]  = gt[k] + beta_{k+1} S[k+1],  S[C-1] = 1       (= btilde_t R_t)
//   K_M[k] = eta_k bt[k],  K_W[k] = eta_k S[k]
//   consts = (gtilde_0 = gamma_0 gt[0], btilde_0 = beta_0 bt[0],
//             btilde_0 R_1 = beta_0 S[0], 0)
// S is the division-free form of btilde_t R_t = sum_{i>=t} gtilde_i
// btilde_t / btilde_i: it stays finite where a beta is 0 and where prod beta
// underflows.  All three recurrences run right to left; each is an affine map
// x_k = a_k x_{k+1} + c_k, so one warp scans a chunk: every lane folds a
// contiguous segment, a shuffle scan composes the lanes' maps, and a second
// pass writes the outputs.  Arithmetic in float64 (negligible cost: the
// kernel touches 5 floats per token once per call).
#pragma once

#include "common.cuh"

namespace ttt {

__global__ void scalar_scan_kernel(const float* __restrict__ eta, const float* __restrict__ beta,
                                   const float* __restrict__ gamma, int T, int b, int nchunks,
                                   float* __restrict__ KW, float* __restrict__ KM,
                                   float* __restrict__ consts) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t job = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5);
  const int64_t jobs = (int64_t)gridDim.y * nchunks;  // gridDim.y = batch
  (void)jobs;
  const int s = blockIdx.y;
  if (job >= nchunks) return;
  const int c = (int)job;
  const int64_t base = (int64_t)s * T + (int64_t)c * b;
  const float* be = beta + base;
  const float* ga = gamma + base;
  const float* et = eta + base;
  const int per = (b + 31) / 32;
  const int k0 = min(b, lane * per), k1 = min(b, k0 + per);

  // Pass 1: segment products of beta and gamma over (k0 .. k1-1) shifted by
  // one: the carry into token k-1 multiplies by beta_k.
  double pb = 1.0, pg = 1.0;
  for (int k = k0; k < k1; ++k) { pb *= (double)be[k]; pg *= (double)ga[k]; }
  // Exclusive suffix products over lanes to the right: Qb_j = prod_{lanes > j}.
  double qb = pb, qg = pg;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    double ob = __shfl_down_sync(0xffffffffu, qb, off);
    double og = __shfl_down_sync(0xffffffffu, qg, off);
    if (lane + off < 32) { qb *= ob; qg *= og; }
  }
  // qb is now the inclusive suffix product from this lane; exclusive = next lane's.
  double eb = __shfl_down_sync(0xffffffffu, qb, 1);
  double eg = __shfl_down_sync(0xffffffffu, qg, 1);
  if (lane == 31) { eb = 1.0; eg = 1.0; }

  // Pass 2 (right to left): bt[k], gt[k]; K_M; and the segment's affine map
  // for S: S[k0] = A * S[k1] + Bc.
  double rb = eb, rg = eg;       // bt[k1-1] = prod_{i >= k1} beta_i = eb
  double A = 1.0, Bc = 0.0;
  for (int k = k1 - 1; k >= k0; --k) {
    // rb = bt[k], rg = gt[k]
    double a = (k + 1 < b) ? (double)be[k + 1] : 0.0;
    A = a * A;
    Bc = rg + a * Bc;
    KM[base + k] = (float)((double)et[k] * rb);
    rb *= (double)be[k];
    rg *= (double)ga[k];
  }
  // Compose maps to the right: F_j = f_j o f_{j+1} o ... ; S at k1_j = F_{j+1}(0).
  double FA = A, FB = Bc;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    double oA = __shfl_down_sync(0xffffffffu, FA, off);
    double oB = __shfl_down_sync(0xffffffffu, FB, off);
    if (lane + off < 32) { FB = FA * oB + FB; FA = FA * oA; }
  }
  double sin = __shfl_down_sync(0xffffffffu, FB, 1);
  if (lane == 31) sin = 0.0;

  // Pass 3: S[k] right to left from S[k1] = sin, then K_W.
  double S = sin;
  rg = eg;
  double S0 = 0.0;
  for (int k = k1 - 1; k >= k0; --k) {
    double a = (k + 1 < b) ? (double)be[k + 1] : 0.0;
    S = rg + a * S;
    KW[base + k] = (float)((double)et[k] * S);
    if (k == 0) S0 = S;
    rg *= (double)ga[k];
  }
  if (lane == 0 && b > 0) {
    // consts: gtilde_0 = gamma_0 * gt[0], btilde_0 = beta_0 * bt[0], cM = beta_0 * S[0]
    double bt0 = eb, gt0 = eg;
    for (int k = k1 - 1; k >= 1; --k) { bt0 *= (double)be[k]; gt0 *= (double)ga[k]; }
    float* o = consts + ((int64_t)s * nchunks + c) * 4;
    o[0] = (float)((double)ga[0] * gt0);
    o[1] = (float)((double)be[0] * bt0);
    o[2] = (float)((double)be[0] * S0);
    o[3] = 0.f;
  }
}

// LaCT's chunk-wise rule as "Rethinking Expressivity and Efficiency in
// Test-Time Training" states it (高效的逐块（Chunk-wise）更新机制): one direction
// G = sum_t eta_t G_t, M_C = (mean_t beta_t) M_0 + G, W_C = W_0 + M_C.  In the
// update GEMM's terms K_W = K_M = eta and consts = (1, bbar, bbar, 0).  One warp
// per chunk; the mean of beta is summed in float64 in a fixed order.
__global__ void lact_scan_kernel(const float* __restrict__ eta, const float* __restrict__ beta, int T, int b,
                                 int nchunks, float* __restrict__ KW, float* __restrict__ KM,
                                 float* __restrict__ consts) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t job = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5);
  const int s = blockIdx.y;
  if (job >= nchunks) return;
  const int c = (int)job;
  const int64_t base = (int64_t)s * T + (int64_t)c * b;
  double sum = 0.0;
  for (int k = lane; k < b; k += 32) {
    const float e = eta[base + k];
    KW[base + k] = e;
    KM[base + k] = e;
    sum += (double)beta[base + k];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane == 0) {
    const float bbar = (float)(sum / (double)b);
    float* o = consts + ((int64_t)s * nchunks + c) * 4;
    o[0] = 1.f;
    o[1] = bbar;
    o[2] = bbar;
    o[3] = 0.f;
  }
}

inline cudaError_t launch_scalar_scan(int rule, const float* eta, const float* beta, const float* gamma,
                                      int batch, int T, int b, float* KW, float* KM,
                                      float* consts, cudaStream_t st) {
  if (batch <= 0 || T <= 0) return cudaSuccess;
  int nchunks = T / b;
  const int warps = 4;
  dim3 grid((nchunks + warps - 1) / warps, batch);
  if (rule == TTT_RULE_LACT)
    lact_scan_kernel<<<grid, warps * 32, 0, st>>>(eta, beta, T, b, nchunks, KW, KM, consts);
  else
    scalar_scan_kernel<<<grid, warps * 32, 0, st>>>(eta, beta, gamma, T, b, nchunks, KW, KM, consts);
  return cudaGetLastError();
}

}  // namespace ttt
