// GEMM epilogues of the inner loop.  Both GEMM engines (the fp32 CUDA-core
// engine and the tcgen05 engine) hand every output row to the epilogue in
// spans of 32 consecutive columns (c0 % 32 == 0), after row_begin() and
// before row_end().  A span carries the fp32 accumulator values v[0..31]
// (and v2[] for the dual-accumulator update GEMM); only the first `nv`
// columns are inside the matrix.
//
// The arithmetic here is the elementwise part of the chunk step:
//   forward MLP activations ("Rethinking Expressivity and Efficiency in
//   Test-Time Training", 快速权重网络实例化), residual adds, the online-softmax
//   pieces of the next-token cross-entropy, the backward factors, and the
//   Proposition 3.1 state update (same page, 命题3.1 and Algorithm 1 lines 6-7).
#pragma once

#include "common.cuh"

namespace ttt {

// Row r of batch z of a token GEMM is token (s, t) with
// grow = z * rows_per_z + r, s = grow / b, t = chunk * b + grow % b.
struct TokenMap {
  int b;
  int T;
  int chunk;
  __device__ __forceinline__ int64_t index(int grow) const {
    int s = grow / b;
    return (int64_t)s * T + (int64_t)chunk * b + (grow - s * b);
  }
};

struct NoRowState {};

__device__ __forceinline__ float gelu_f(float u) { return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad_f(float u) {
  float cdf = 0.5f * (1.0f + erff(u * 0.70710678118654752f));
  float pdf = 0.39894228040143268f * expf(-0.5f * u * u);
  return cdf + u * pdf;
}
__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + expf(-x)); }

// ---------------------------------------------------------------------------
// F1: U = a W1^T (GELU: [n,h]; SwiGLU: [n,2h] in the interleaved layout).
// Writes the activation A (input of the second matrix) and the factors the
// backward needs: GELU'(U), or for SwiGLU dA/dgate = up * SiLU'(gate) and
// dA/dup = SiLU(gate) at the gate / up positions.
// ---------------------------------------------------------------------------
template <typename T, bool SWIGLU>
struct EpiF1 {
  using RowState = NoRowState;
  T* act;        // [rows, h]
  T* fac;        // [rows, H2] or nullptr when no backward passes through
  int h;
  int rows_per_z;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState&, int z, int r, int c0, const float* v, const float*, int nv) const {
    int64_t grow = (int64_t)z * rows_per_z + r;
    if (!SWIGLU) {
      T* a = act + grow * h + c0;
      T* f = fac ? fac + grow * h + c0 : nullptr;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j < nv) {
          float u = v[j];
          a[j] = from_f<T>(gelu_f(u));
          if (f) f[j] = from_f<T>(gelu_grad_f(u));
        }
      }
    } else {
      int g = c0 >> 5;            // full 32-wide group (2h % 32 == 0)
      T* a = act + grow * h + (g << 4);
      T* f = fac ? fac + grow * (2 * (int64_t)h) + c0 : nullptr;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float gv = v[k], uv = v[16 + k];
        float sg = sigmoid_f(gv);
        float silu = gv * sg;
        a[k] = from_f<T>(silu * uv);
        if (f) {
          f[k] = from_f<T>(uv * sg * (1.0f + gv * (1.0f - sg)));
          f[16 + k] = from_f<T>(silu);
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// F2: residual add.  resid += A W2^T; optional operand copy of the new stream.
// ---------------------------------------------------------------------------
template <typename T>
struct EpiResid {
  using RowState = NoRowState;
  float* resid;   // [rows, d]
  T* act_next;    // [rows, d] or nullptr
  int d;
  int rows_per_z;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState&, int z, int r, int c0, const float* v, const float*, int nv) const {
    int64_t grow = (int64_t)z * rows_per_z + r;
    float* p = resid + grow * d + c0;
    T* q = act_next ? act_next + grow * d + c0 : nullptr;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j < nv) {
        float x = p[j] + v[j];
        p[j] = x;
        if (q) q[j] = from_f<T>(x);
      }
    }
  }
};

// ---------------------------------------------------------------------------
// B1: dA = dOut W2 ([n,h]); dU = dA * factor at the U positions; for a
// dynamic MLP also the K-scaled negated copies -K_W dU and -K_M dU that are
// the A operands of the aggregation (so the aggregation GEMM yields
// sum_t K_t G_t directly, G_t being the negative gradient).
// ---------------------------------------------------------------------------
template <typename T, bool SWIGLU>
struct EpiB1 {
  using RowState = NoRowState;
  const T* fac;   // [rows, H2]
  T* dU;          // [rows, H2] or nullptr
  T* dUW;         // [rows, H2] or nullptr (static MLP)
  T* dUM;
  const float* KW;
  const float* KM;
  float kscale;   // 1/b (mean reduction) or 1 (sum)
  TokenMap tm;
  int h;
  int rows_per_z;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState&, int z, int r, int c0, const float* v, const float*, int nv) const {
    int64_t grow = (int64_t)z * rows_per_z + r;
    const int64_t H2 = SWIGLU ? 2 * (int64_t)h : h;
    float kw = 0.f, km = 0.f;
    if (dUW) {
      int64_t ti = tm.index((int)grow);
      kw = -KW[ti] * kscale;
      km = -KM[ti] * kscale;
    }
    const T* f = fac + grow * H2;
    int64_t ob = grow * H2;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j < nv) {
        int c = c0 + j;
        float da = v[j];
        if (!SWIGLU) {
          float du = da * to_f<T>(f[c]);
          if (dU) dU[ob + c] = from_f<T>(du);
          if (dUW) { dUW[ob + c] = from_f<T>(kw * du); dUM[ob + c] = from_f<T>(km * du); }
        } else {
          int pg = swiglu_pos_gate(c), pu = pg + 16;
          float dg = da * to_f<T>(f[pg]);
          float du = da * to_f<T>(f[pu]);
          if (dU) { dU[ob + pg] = from_f<T>(dg); dU[ob + pu] = from_f<T>(du); }
          if (dUW) {
            dUW[ob + pg] = from_f<T>(kw * dg); dUW[ob + pu] = from_f<T>(kw * du);
            dUM[ob + pg] = from_f<T>(km * dg); dUM[ob + pu] = from_f<T>(km * du);
          }
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// B2: dX through the MLP branch plus the residual: dout += dU W1; operand copy
// and, when the MLP below is dynamic, its K-scaled negated copies.
// ---------------------------------------------------------------------------
template <typename T>
struct EpiB2 {
  using RowState = NoRowState;
  float* dout;    // [rows, d]
  T* dout_a;      // [rows, d]
  T* doutW;       // [rows, d] or nullptr
  T* doutM;
  const float* KW;
  const float* KM;
  float kscale;
  TokenMap tm;
  int d;
  int rows_per_z;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState&, int z, int r, int c0, const float* v, const float*, int nv) const {
    int64_t grow = (int64_t)z * rows_per_z + r;
    float kw = 0.f, km = 0.f;
    if (doutW) {
      int64_t ti = tm.index((int)grow);
      kw = -KW[ti] * kscale;
      km = -KM[ti] * kscale;
    }
    int64_t o = grow * d + c0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j < nv) {
        float x = dout[o + j] + v[j];
        dout[o + j] = x;
        dout_a[o + j] = from_f<T>(x);
        if (doutW) { doutW[o + j] = from_f<T>(kw * x); doutM[o + j] = from_f<T>(km * x); }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Cross-entropy, pass A: per (row, N-tile) running max and sum of exp of the
// logits (online softmax), and the target logit.  The logits stay on chip.
// ---------------------------------------------------------------------------
struct EpiCEPartial {
  struct RowState { float m, s; int y; };
  float* part;        // [rows, ntn, 2]
  float* tgt;         // [rows]
  const int* tokens;  // [B, T]
  TokenMap tm;
  int ntn;
  __device__ void row_begin(RowState& st, int, int r) const {
    st.m = -INFINITY;
    st.s = 0.f;
    st.y = tokens[tm.index(r)];
  }
  __device__ void span(RowState& st, int, int r, int c0, const float* v, const float*, int nv) const {
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j) if (j < nv) mx = fmaxf(mx, v[j]);
    if (mx > st.m) { st.s *= expf(st.m - mx); st.m = mx; }
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) if (j < nv) acc += expf(v[j] - st.m);
    st.s += acc;
    int k = st.y - c0;
    if (k >= 0 && k < nv) {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j == k) tgt[r] = v[j];
    }
  }
  __device__ void row_end(RowState& st, int, int r, int tile_n) const {
    float* p = part + ((int64_t)r * ntn + tile_n) * 2;
    p[0] = st.m;
    p[1] = st.s;
  }
};

// ---------------------------------------------------------------------------
// Cross-entropy, pass B over one vocabulary slab: dl/dlogit = softmax - onehot,
// written as an operand for dz = P E_slab.
// ---------------------------------------------------------------------------
template <typename T>
struct EpiCEGrad {
  using RowState = int;  // the row's label
  T* P;               // [rows, Vs]
  const float* lse;   // [rows]
  const int* tokens;
  TokenMap tm;
  int Vs;
  int slab0;
  __device__ void row_begin(RowState& y, int, int r) const { y = tokens[tm.index(r)]; }
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState& y, int, int r, int c0, const float* v, const float*, int nv) const {
    float l = lse[r];
    T* o = P + (int64_t)r * Vs + c0;
    int k = y - slab0 - c0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j < nv) {
        float p = expf(v[j] - l);
        if (j == k) p -= 1.0f;
        o[j] = from_f<T>(p);
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Plain fp32 store (dz over the vocabulary slabs: first slab stores, the next
// ones accumulate).
// ---------------------------------------------------------------------------
struct EpiStoreF32 {
  using RowState = NoRowState;
  float* out;
  int ld;
  int accumulate;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState&, int, int r, int c0, const float* v, const float*, int nv) const {
    float* o = out + (int64_t)r * ld + c0;
#pragma unroll
    for (int j = 0; j < 32; ++j) if (j < nv) o[j] = accumulate ? o[j] + v[j] : v[j];
  }
};

// ---------------------------------------------------------------------------
// Aggregation + in-place update (Algorithm 1 lines 4-7): v = sum_t K_W_t G_t,
// v2 = sum_t K_M_t G_t for this element;
//   W <- gtilde_0 W + btilde_0 R_1 M + v,   M <- btilde_0 M + v2,
// and the operand shadow of the new W.  Batch z = sequence.
// ---------------------------------------------------------------------------
template <typename T>
struct EpiUpdate {
  using RowState = NoRowState;
  float* W;            // this matrix, sequence 0 (rows of the packed layout)
  float* M;
  T* Wsh;              // shadow of this matrix, sequence 0 (library row order)
  int64_t seq_stride;  // floats between sequences in W / M
  int64_t sh_stride;   // elements between sequences in the shadow
  const float* consts; // [B, nchunks, 4]
  int chunk;
  int nchunks;
  int cols;
  int h;               // > 0: rows are SwiGLU [gate; up] positions to remap
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState&, int z, int r, int c0, const float* v, const float* v2, int nv) const {
    const float* cs = consts + ((int64_t)z * nchunks + chunk) * 4;
    float g0 = cs[0], b0 = cs[1], cM = cs[2];
    int fr = h > 0 ? swiglu_row_of_pos(r, h) : r;
    float* wp = W + z * seq_stride + (int64_t)fr * cols + c0;
    float* mp = M + z * seq_stride + (int64_t)fr * cols + c0;
    T* sp = Wsh + z * sh_stride + (int64_t)r * cols + c0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j < nv) {
        float w = wp[j], m = mp[j];
        float wn = fmaf(g0, w, fmaf(cM, m, v[j]));
        float mn = fmaf(b0, m, v2[j]);
        wp[j] = wn;
        mp[j] = mn;
        sp[j] = from_f<T>(wn);
      }
    }
  }
};

}  // namespace ttt
