// Frozen sliding-window attention in front of each updated block
// ("TTT-E2E：端到端测试时训练的长上下文语言建模": the sketch's TTTE2EBlock,
// TTTSelfAttention and RotaryEmbedding; 滑动窗口注意力, 关键设计参数).
//
// Epilogues and row kernels around the attention GEMMs (which run on the same
// engines as the MLP GEMMs, batched over heads).  The scores never reach HBM:
// a first score pass leaves masked online-softmax partials, a second one
// recomputes the scores and writes the probabilities, and the dP GEMM forms
// dS in its epilogue.  Row kernels: LayerNorm with frozen gain and bias, the
// rotary embedding and the split of the fused q|k|v projection into
// head-major operands, the rows' log-sum-exp and D = dO . O, the rotary
// backward that packs dq|dk|dv for the input projection's backward, and the
// split of the residual-stream gradient into the two weighted cotangent
// streams the chunk update needs once attention mixes the rows.
//
// Layouts (T = operand type):
//   q of the chunk       [B][H][b][dh]  T, rotated
//   key/value history    [L][B][H][T][dh] T per block; keys rotated, at their
//                        absolute positions, written when their chunk runs
//   score partials       [H][b][ntn][2] fp32 for one sequence; lse, D [H][b]
//   P, dS                [H][b][ldS] T, zero outside the window, ldS % 8 == 0
//   o, dq, dk, dv        [rows][d] fp32, token-major (head h at columns h*dh)
//   rotary table         [T][dh/2] (cos, sin) fp32, angles in fp64
#pragma once

#include "common.cuh"
#include "epilogue.cuh"
#include "rows.cuh"

namespace ttt {

// GEMM output [rows, H*dh] stored head-major per sequence:
// out[((s*H + h)*b + i)*dh + e] for row r = s*b + i and column c = h*dh + e.
template <typename T>
struct EpiStoreHeads {
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = true;
  using RowState = NoRowState;
  using SpanRegs = NoSpanRegs;
  T* out;
  int b;
  int H;
  int dh;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  // Row-walking form (tcgen05 engine): the lane's 4 columns lie in one head
  // (dh % 16 == 0).
  __device__ void load_span(SpanRegs&, int, int, int, int, int, int, int) const {}
  __device__ void finish_span(const SpanRegs&, int half, int, int row0, int c0, const float* sv, int nv, int nrows,
                              int lane) const {
    const int cj = rw_col(lane);
    if (cj >= nv) return;
    const int c = c0 + cj, hh = c / dh, e = c - hh * dh;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = rw_row(half, k, lane);
      if (i >= nrows) continue;
      const int r = row0 + i, s = r / b, ii = r - s * b;
      float a[4];
      rw_read4(sv, i, cj, a);
      T* o = out + (((int64_t)s * H + hh) * b + ii) * dh + e;
      if (cj + 4 <= nv) store_x4(o, a);
      else for (int j = 0; j < nv - cj; ++j) o[j] = from_f<T>(a[j]);
    }
  }
  __device__ void span(RowState&, int, int r, int c0, const float* v, const float*, int nv) const {
    const int s = r / b, i = r - s * b;
    const int h0 = c0 / dh, e0 = c0 - h0 * dh;
    if (nv == 32 && e0 + 32 <= dh && (e0 & 7) == 0 && (dh & 7) == 0) {
      vst<32>(out + (((int64_t)s * H + h0) * b + i) * dh + e0, v);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j < nv) {
        const int c = c0 + j, h = c / dh, e = c - h * dh;
        out[(((int64_t)s * H + h) * b + i) * dh + e] = from_f<T>(v[j]);
      }
    }
  }
};

// Scores pass A: per (head, query) row and column part of the tile, the
// online-softmax partial (max, sum exp) of scale * s over the keys inside the
// window (empty parts give (-inf, 0)).  The scores never reach HBM.  The
// exponential is exp_op<T>: with bf16 operands the hardware approximation.
template <typename T>
struct EpiScorePartial {
  static constexpr bool kFixedHeadTile = true;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = false;
  struct RowState { float m, s; };
  float* part;     // [H][b][ntn][2]
  int b;
  int ntn;
  int64_t q0, j0;  // positions of query row 0 and key column 0
  int window;
  float scale;
  __device__ void row_begin(RowState& st, int, int) const { st.m = -INFINITY; st.s = 0.f; }
  __device__ void span(RowState& st, int, int r, int c0, const float* v, const float*, int nv) const {
    // query position minus the span's first key position (|.| < 2^31)
    const int base = (int)(q0 + r - (j0 + c0));
    float x[32];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const bool in = j < nv && (unsigned)(base - j) < (unsigned)window;
      x[j] = in ? v[j] * scale : -INFINITY;
      mx = fmaxf(mx, x[j]);
    }
    if (mx == -INFINITY) return;
    if (mx > st.m) { st.s *= exp_op<T>(st.m - mx); st.m = mx; }
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) acc += exp_op<T>(x[j] - st.m);
    st.s += acc;
  }
  __device__ void row_end(RowState& st, int z, int r, int part_index) const {
    float* p = part + (((int64_t)z * b + r) * ntn + part_index) * 2;
    *reinterpret_cast<float2*>(p) = make_float2(st.m, st.s);
  }
};

// Scores pass B: the probabilities from the recomputed scores and each row's
// log-sum-exp, P = exp(scale * s - lse) inside the window, 0 outside; stored
// in the operand type for P V and the backward.
template <typename T>
struct EpiScoreP {
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = false;
  using RowState = NoRowState;
  T* P;                // [H][b][ldS]
  const float* lse;    // [H][b]
  int b;
  int ldS;
  int64_t q0, j0;
  int window;
  float scale;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState&, int z, int r, int c0, const float* v, const float*, int nv) const {
    const int64_t row = (int64_t)z * b + r;
    const float l = lse[row];
    const int base = (int)(q0 + r - (j0 + c0));   // as in EpiScorePartial
    float x[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = (unsigned)(base - j) < (unsigned)window ? exp_op<T>(v[j] * scale - l) : 0.f;
    T* o = P + row * ldS + c0;
    if (nv == 32 && (ldS & 7) == 0 && (c0 & 7) == 0) {
      vst<32>(o, x);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j < nv) o[j] = from_f<T>(x[j]);
    }
  }
};

// dP epilogue: dS = P (dP - D) * scale from the kept probabilities and each
// row's D = sum_e dO O, stored in the operand type; dP never reaches HBM.
template <typename T>
struct EpiDScore {
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = false;
  using RowState = NoRowState;
  T* dS;               // [H][b][ldS]
  const T* P;          // [H][b][ldS]
  const float* D;      // [H][b]
  int b;
  int ldS;
  float scale;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState&, int z, int r, int c0, const float* v, const float*, int nv) const {
    const int64_t row = (int64_t)z * b + r;
    const float dd = D[row];
    const T* pr = P + row * ldS + c0;
    T* o = dS + row * ldS + c0;
    float x[32];
    if (nv == 32 && (ldS & 7) == 0 && (c0 & 7) == 0) {
      float p[32];
      vld<32>(pr, p);
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] = p[j] * (v[j] - dd) * scale;
      vst<32>(o, x);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j < nv) o[j] = from_f<T>(to_f<T>(pr[j]) * (v[j] - dd) * scale);
    }
  }
};

// Log-sum-exp of each (head, query) row from its pass-A partials.
__global__ void attn_lse_kernel(const float* __restrict__ part, int ntn, int64_t rows, float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float2* p = reinterpret_cast<const float2*>(part + row * ntn * 2);
  float m = -INFINITY;
  for (int t = lane; t < ntn; t += 32) m = fmaxf(m, p[t].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sum = 0.f;
  for (int t = lane; t < ntn; t += 32) { const float2 q = p[t]; if (q.y > 0.f) sum += q.y * expf(q.x - m); }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) lse[row] = m + logf(sum);
}

// D = sum_e dO[e] O[e] over each head's columns, one warp per (head, query) of
// one sequence.
template <typename T>
__global__ void attn_rowdot_kernel(const T* __restrict__ dO, const float* __restrict__ O, int rows, int b, int d,
                                   int dh, float* __restrict__ D) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int h = (int)(row / b), i = (int)(row % b);
  float acc = 0.f;
  for (int e = lane; e < dh; e += 32) acc += to_f<T>(dO[row * dh + e]) * O[(int64_t)i * d + h * dh + e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) D[row] = acc;
}

// LayerNorm with frozen gain and bias, one warp per row (two passes over the
// row: mean, then the centred variance).  Keeps x_hat and 1/sigma for the
// backward.  d % 4 == 0.
template <typename T>
__global__ void ln_affine_fwd_kernel(const float* __restrict__ x, const float* __restrict__ gain,
                                     const float* __restrict__ bias, float eps, int64_t n, int d,
                                     T* __restrict__ a, float* __restrict__ xhat, float* __restrict__ rstd) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n) return;
  const float4* xr = reinterpret_cast<const float4*>(x + row * d);
  float s = 0.f;
  for (int c = lane; c < (d >> 2); c += 32) { float4 v = xr[c]; s += v.x + v.y + v.z + v.w; }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mu = s / (float)d;
  float ss = 0.f;
  for (int c = lane; c < (d >> 2); c += 32) {
    float4 v = xr[c];
    float a0 = v.x - mu, a1 = v.y - mu, a2 = v.z - mu, a3 = v.w - mu;
    ss += a0 * a0 + a1 * a1 + a2 * a2 + a3 * a3;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / (float)d + eps);
  if (lane == 0) rstd[row] = r;
  const float4* gr = reinterpret_cast<const float4*>(gain);
  const float4* br = reinterpret_cast<const float4*>(bias);
  for (int c = lane; c < (d >> 2); c += 32) {
    float4 v = xr[c], g = gr[c], bb = br[c];
    float4 xh = make_float4((v.x - mu) * r, (v.y - mu) * r, (v.z - mu) * r, (v.w - mu) * r);
    reinterpret_cast<float4*>(xhat + row * d)[c] = xh;
    store4<T>(a + row * d + 4 * c, make_float4(xh.x * g.x + bb.x, xh.y * g.y + bb.y, xh.z * g.z + bb.z,
                                               xh.w * g.w + bb.w));
  }
}

// LayerNorm backward (gain and bias frozen): dx = r (g*da - mean(g*da) -
// x_hat mean(g*da * x_hat)); dout += dx and its operand copy.
template <typename T>
__global__ void ln_affine_bwd_kernel(const float* __restrict__ da, const float* __restrict__ xhat,
                                     const float* __restrict__ rstd, const float* __restrict__ gain, int64_t n,
                                     int d, float* __restrict__ dout, T* __restrict__ dout_t) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n) return;
  const float4* dr = reinterpret_cast<const float4*>(da + row * d);
  const float4* xr = reinterpret_cast<const float4*>(xhat + row * d);
  const float4* gr = reinterpret_cast<const float4*>(gain);
  float m1 = 0.f, m2 = 0.f;
  for (int c = lane; c < (d >> 2); c += 32) {
    float4 g = dr[c], w = gr[c], x = xr[c];
    float g0 = g.x * w.x, g1 = g.y * w.y, g2 = g.z * w.z, g3 = g.w * w.w;
    m1 += g0 + g1 + g2 + g3;
    m2 += g0 * x.x + g1 * x.y + g2 * x.z + g3 * x.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m1 += __shfl_xor_sync(0xffffffffu, m1, o);
    m2 += __shfl_xor_sync(0xffffffffu, m2, o);
  }
  m1 /= (float)d;
  m2 /= (float)d;
  const float r = rstd[row];
  for (int c = lane; c < (d >> 2); c += 32) {
    float4 g = dr[c], w = gr[c], x = xr[c];
    float4 o = reinterpret_cast<float4*>(dout + row * d)[c];
    o.x += r * (g.x * w.x - m1 - x.x * m2);
    o.y += r * (g.y * w.y - m1 - x.y * m2);
    o.z += r * (g.z * w.z - m1 - x.z * m2);
    o.w += r * (g.w * w.w - m1 - x.w * m2);
    reinterpret_cast<float4*>(dout + row * d)[c] = o;
    store4<T>(dout_t + row * d + 4 * c, o);
  }
}

// Rotary table: (cos, sin) of pos * base^(-2i/dh) for pos < T, i < dh/2.  The
// angle and its sine and cosine are taken in fp64 (positions reach 2^17 and
// more, where an fp32 angle is off by 1e-2 rad), then rounded to fp32.
__global__ void rope_table_kernel(int64_t T_, int half, double base, float2* __restrict__ table) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < T_ * half;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = e / half;
    const int i = (int)(e - t * half);
    const double ang = (double)t * pow(base, -2.0 * (double)i / (double)(2 * half));
    double s, c;
    sincos(ang, &s, &c);
    table[e] = make_float2((float)c, (float)s);
  }
}

// Split of the fused projection qkv [n][3d] (fp32) for chunk c: rotate q and
// k (rotate-half form: (x1, x2) -> (x1 c - x2 s, x1 s + x2 c) per frequency i),
// write q head-major for the chunk and k, v into the block's history at the
// tokens' absolute positions.  One thread per (row, head, frequency).
template <typename T>
__global__ void rope_split_kernel(const float* __restrict__ qkv, const float2* __restrict__ table, int64_t n,
                                  int b, int d, int H, int64_t T_, int chunk, T* __restrict__ q,
                                  T* __restrict__ kh, T* __restrict__ vh) {
  const int dh = d / H, half = dh >> 1;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * H * half;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / (H * half);
    const int rem = (int)(e - r * H * half);
    const int h = rem / half, i = rem - h * half;
    const int64_t s = r / b, ii = r - s * b;
    const int64_t pos = (int64_t)chunk * b + ii;
    const float2 cs = table[pos * half + i];
    const float* src = qkv + r * 3 * d + h * dh;
    const float q1 = src[i], q2 = src[half + i];
    const float k1 = src[d + i], k2 = src[d + half + i];
    T* qo = q + ((s * H + h) * b + ii) * dh;
    qo[i] = from_f<T>(q1 * cs.x - q2 * cs.y);
    qo[half + i] = from_f<T>(q1 * cs.y + q2 * cs.x);
    const int64_t hist = ((s * H + h) * T_ + pos) * dh;
    kh[hist + i] = from_f<T>(k1 * cs.x - k2 * cs.y);
    kh[hist + half + i] = from_f<T>(k1 * cs.y + k2 * cs.x);
    vh[hist + i] = from_f<T>(src[2 * d + i]);
    vh[hist + half + i] = from_f<T>(src[2 * d + half + i]);
  }
}

// Rotary backward of dq and dk (the transpose rotation) and the pack of
// dq|dk|dv into [rows][3d] for the input projection's backward; rows of one
// sequence, chunk c.  One thread per (row, head, frequency).
template <typename T>
__global__ void rope_bwd_pack_kernel(const float* __restrict__ dq, const float* __restrict__ dk,
                                     const float* __restrict__ dv, const float2* __restrict__ table, int b, int d,
                                     int H, int chunk, T* __restrict__ dqkv) {
  const int dh = d / H, half = dh >> 1;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < (int64_t)b * H * half;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / (H * half);
    const int rem = (int)(e - i * H * half);
    const int h = rem / half, f = rem - h * half;
    const float2 cs = table[((int64_t)chunk * b + i) * half + f];
    const int64_t src = i * d + h * dh;
    T* o = dqkv + i * 3 * d + h * dh;
    const float g1 = dq[src + f], g2 = dq[src + half + f];
    o[f] = from_f<T>(g1 * cs.x + g2 * cs.y);
    o[half + f] = from_f<T>(-g1 * cs.y + g2 * cs.x);
    const float k1 = dk[src + f], k2 = dk[src + half + f];
    o[d + f] = from_f<T>(k1 * cs.x + k2 * cs.y);
    o[d + half + f] = from_f<T>(-k1 * cs.y + k2 * cs.x);
    o[2 * d + f] = from_f<T>(dv[src + f]);
    o[2 * d + half + f] = from_f<T>(dv[src + half + f]);
  }
}

// The two weighted cotangent streams of the chunk update: rows of the
// residual-stream gradient scaled by -kscale K_W[t] and -kscale K_M[t]
// (the gradients of sum_t K_t l_t, valid above the first attention layer
// where every path is row-local), fp32 and operand copies.
template <typename T>
__global__ void stream_split_kernel(const float* __restrict__ dout, const float* __restrict__ KW,
                                    const float* __restrict__ KM, float kscale, TokenMap tm, int64_t n, int d,
                                    float* __restrict__ sW, float* __restrict__ sM, T* __restrict__ tW,
                                    T* __restrict__ tM) {
  const int64_t q = d >> 2;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * q;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / q;
    const int64_t ti = tm.index((int)r);
    const float kw = -KW[ti] * kscale, km = -KM[ti] * kscale;
    const float4 x = reinterpret_cast<const float4*>(dout)[e];
    const float4 w = make_float4(kw * x.x, kw * x.y, kw * x.z, kw * x.w);
    const float4 m = make_float4(km * x.x, km * x.y, km * x.z, km * x.w);
    reinterpret_cast<float4*>(sW)[e] = w;
    reinterpret_cast<float4*>(sM)[e] = m;
    store4<T>(tW + 4 * e, w);
    store4<T>(tM + 4 * e, m);
  }
}

}  // namespace ttt
