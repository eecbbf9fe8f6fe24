// GEMM epilogues of the inner loop.  Both GEMM engines (the fp32 CUDA-core
// engine and the tcgen05 engine) hand every output row to the epilogue in
// spans of 32 consecutive columns (c0 % 32 == 0), after row_begin() and
// before row_end().  A span carries the fp32 accumulator values v[0..31]
// (and v2[] for the dual-accumulator update GEMM); only the first `nv`
// columns are inside the matrix.  One thread owns a row, so every span is a
// contiguous run in memory: full spans use 16-byte vector accesses (all row
// pitches are multiples of 16 elements), the ragged tail goes element-wise.
//
// The arithmetic here is the elementwise part of the chunk step:
//   forward MLP activations ("Rethinking Expressivity and Efficiency in
//   Test-Time Training", 快速权重网络实例化), residual adds, the online-softmax
//   pieces of the next-token cross-entropy, the backward factors, and the
//   Proposition 3.1 state update (same page, 命题3.1 and Algorithm 1).
#pragma once

#include <type_traits>

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

// Every epilogue declares kFixedHeadTile: true when its output layout depends
// on the N tile of the tcgen05 engine (the engine then always uses its head
// tile width), false when any N tile will do.

__device__ __forceinline__ float gelu_f(float u) { return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad_f(float u) {
  float cdf = 0.5f * (1.0f + erff(u * 0.70710678118654752f));
  float pdf = 0.39894228040143268f * expf(-0.5f * u * u);
  return cdf + u * pdf;
}
__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + expf(-x)); }
// The exponential and the logistic function inside the GEMM epilogues: the
// accurate library forms with fp32 operands; with bf16 operands, whose
// results are rounded to 8 significant bits or only feed the chunk loss, the
// hardware approximations __expf and __frcp_rn (relative error about 1e-6
// over the arguments met here), which keep the epilogue of the cross-entropy
// and SwiGLU tiles off the critical path of the next tile's MMAs.
template <typename T> __device__ __forceinline__ float exp_op(float x) { return expf(x); }
template <> __device__ __forceinline__ float exp_op<__nv_bfloat16>(float x) { return __expf(x); }
template <typename T> __device__ __forceinline__ float sigmoid_op(float x) { return sigmoid_f(x); }
template <> __device__ __forceinline__ float sigmoid_op<__nv_bfloat16>(float x) { return __frcp_rn(1.0f + __expf(-x)); }

// ---------------------------------------------------------------------------
// Vector access helpers: N contiguous elements, 16-byte aligned.  Where the
// address is 32-byte aligned they move 32 bytes per instruction: measured on
// B200 in the one-row-per-thread epilogues, where every warp instruction
// touches 32 rows, 32-byte stores cost about half the time of 16-byte ones
// (a 5632-column dA tile's fp32 store: 7 us -> 2.5 us over the bare GEMM).
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31) == 0; }
__device__ __forceinline__ void st256(void* p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4,
                                      uint32_t a5, uint32_t a6, uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a0), "r"(a1), "r"(a2),
               "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}
__device__ __forceinline__ void ld256(const void* p, uint32_t* a) {
  asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7])
               : "l"(p)
               : "memory");
}
template <int N>
__device__ __forceinline__ void vld(const float* p, float* v) {
  if (N % 8 == 0 && aligned32(p)) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
      uint32_t a[8];
      ld256(p + 8 * i, a);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[8 * i + j] = __uint_as_float(a[j]);
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < N / 4; ++i) {
    float4 x = reinterpret_cast<const float4*>(p)[i];
    v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
  }
}
template <int N>
__device__ __forceinline__ void vst(float* p, const float* v) {
  if (N % 8 == 0 && aligned32(p)) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
      const float* w = v + 8 * i;
      st256(p + 8 * i, __float_as_uint(w[0]), __float_as_uint(w[1]), __float_as_uint(w[2]), __float_as_uint(w[3]),
            __float_as_uint(w[4]), __float_as_uint(w[5]), __float_as_uint(w[6]), __float_as_uint(w[7]));
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < N / 4; ++i)
    reinterpret_cast<float4*>(p)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(h);
}
// 16 bf16 from 8 packed words
__device__ __forceinline__ void unpack_bf16x16(const uint32_t* a, float* v) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 x = unpack_bf16x2(a[j]);
    v[2 * j] = x.x; v[2 * j + 1] = x.y;
  }
}
template <int N>
__device__ __forceinline__ void vld(const __nv_bfloat16* p, float* v) {
  if (N % 16 == 0 && aligned32(p)) {
#pragma unroll
    for (int i = 0; i < N / 16; ++i) {
      uint32_t a[8];
      ld256(p + 16 * i, a);
      unpack_bf16x16(a, v + 16 * i);
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < N / 8; ++i) {
    uint4 x = reinterpret_cast<const uint4*>(p)[i];
    float2 a = unpack_bf16x2(x.x), b = unpack_bf16x2(x.y), c = unpack_bf16x2(x.z), d = unpack_bf16x2(x.w);
    v[8 * i] = a.x; v[8 * i + 1] = a.y; v[8 * i + 2] = b.x; v[8 * i + 3] = b.y;
    v[8 * i + 4] = c.x; v[8 * i + 5] = c.y; v[8 * i + 6] = d.x; v[8 * i + 7] = d.y;
  }
}
template <int N>
__device__ __forceinline__ void vst(__nv_bfloat16* p, const float* v) {
  if (N % 16 == 0 && aligned32(p)) {
#pragma unroll
    for (int i = 0; i < N / 16; ++i) {
      const float* w = v + 16 * i;
      st256(p + 16 * i, pack_bf16x2(w[0], w[1]), pack_bf16x2(w[2], w[3]), pack_bf16x2(w[4], w[5]),
            pack_bf16x2(w[6], w[7]), pack_bf16x2(w[8], w[9]), pack_bf16x2(w[10], w[11]), pack_bf16x2(w[12], w[13]),
            pack_bf16x2(w[14], w[15]));
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < N / 8; ++i)
    reinterpret_cast<uint4*>(p)[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                                pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
}
// Scaled store: p[j] = T(s * v[j]).
template <int N, typename T>
__device__ __forceinline__ void vst_scaled(T* p, const float* v, float s) {
  float t[N];
#pragma unroll
  for (int j = 0; j < N; ++j) t[j] = s * v[j];
  vst<N>(p, t);
}

// Four consecutive elements from float values (8 bytes for bf16, 16 for fp32).
__device__ __forceinline__ void store_x4(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store_x4(__nv_bfloat16* p, const float* v) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}
// ---------------------------------------------------------------------------
// Row-walking form (kWarpRows), used by the tcgen05 engine for the plain
// stores and the state update.  The engine stages a 32 x 32 span of the
// accumulators in shared memory (element (row i, column j) at
// sv[i * 32 + ((j + i) & 31)]) and calls load_span() / finish_span() for each
// half of it (rows [16 half, 16 half + 16)).  Lane l covers columns
// [4 (l % 8), 4 (l % 8) + 4) of the rows 16 half + 4 k + l / 8, k < 4, so a
// warp instruction touches 4 rows x 32 contiguous columns.  row0 is the
// span's first row inside batch entry z, c0 its first column; only rows
// < nrows and columns < nv of the span are inside the matrix.  Measured on
// B200, this form pays for stores only: epilogues that read per-row scalars
// or per-element operands (the MLP and cross-entropy epilogues) keep the
// one-row-per-thread form, where each thread loads its row once per tile and
// a whole span's operands are in flight at once.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int rw_row(int half, int k, int lane) { return 16 * half + 4 * k + (lane >> 3); }
__device__ __forceinline__ int rw_col(int lane) { return (lane & 7) * 4; }
// Four consecutive staged values of span row i starting at span column c.
__device__ __forceinline__ void rw_read4(const float* sv, int i, int c, float* a) {
#pragma unroll
  for (int j = 0; j < 4; ++j) a[j] = sv[i * 32 + ((c + j + i) & 31)];
}
struct NoSpanRegs {};

// ---------------------------------------------------------------------------
// F1: U = a W1^T (GELU: [n,h]; SwiGLU: [n,2h] in the interleaved layout).
// Writes the activation A (input of the second matrix) and the factors the
// backward needs: GELU'(U), or for SwiGLU dA/dgate = up * SiLU'(gate) and
// dA/dup = SiLU(gate) at the gate / up positions.
// ---------------------------------------------------------------------------
template <typename T, bool SWIGLU>
struct EpiF1 {
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = false;
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
      float av[32], fv[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        av[j] = gelu_f(v[j]);
        fv[j] = f ? gelu_grad_f(v[j]) : 0.f;
      }
      if (nv == 32) {
        vst<32>(a, av);
        if (f) vst<32>(f, fv);
      } else {
  #pragma unroll
      for (int j = 0; j < 32; ++j) if (j < nv) {
          a[j] = from_f<T>(av[j]);
          if (f) f[j] = from_f<T>(fv[j]);
        }
      }
    } else {
      // a full 32-wide group (2h % 32 == 0): gate in v[0..15], up in v[16..31]
      const int g = c0 >> 5;
      float av[16], fv[32];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float gv = v[k], uv = v[16 + k];
        float sg = sigmoid_op<T>(gv);
        float silu = gv * sg;
        av[k] = silu * uv;
        fv[k] = uv * sg * (1.0f + gv * (1.0f - sg));
        fv[16 + k] = silu;
      }
      vst<16>(act + grow * h + (g << 4), av);
      if (fac) vst<32>(fac + grow * (2 * (int64_t)h) + c0, fv);
    }
  }
};

// ---------------------------------------------------------------------------
// F2: residual add.  resid += A W2^T; optional operand copy of the new stream
// and, when the next MLP is dynamic, its K-scaled negated copies
// -kscale K_W x and -kscale K_M x: the B operands of that MLP's first-matrix
// aggregation (sum_t dU_t (x) (-K_t x_t) = sum_t K_t G_t).
// ---------------------------------------------------------------------------
template <typename T>
struct EpiResid {
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = false;
  using RowState = NoRowState;
  float* resid;   // [rows, d]
  T* act_next;    // [rows, d] or nullptr
  T* aw_next;     // [rows, d] or nullptr
  T* am_next;
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
    if (aw_next) {
      int64_t ti = tm.index((int)grow);
      kw = -KW[ti] * kscale;
      km = -KM[ti] * kscale;
    }
    float* p = resid + grow * d + c0;
    const int64_t o = grow * d + c0;
    if (nv == 32) {
      float x[32];
      vld<32>(p, x);
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] += v[j];
      vst<32>(p, x);
      if (act_next) vst<32>(act_next + o, x);
      if (aw_next) { vst_scaled<32>(aw_next + o, x, kw); vst_scaled<32>(am_next + o, x, km); }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j < nv) {
        float x = p[j] + v[j];
        p[j] = x;
        if (act_next) act_next[o + j] = from_f<T>(x);
        if (aw_next) { aw_next[o + j] = from_f<T>(kw * x); am_next[o + j] = from_f<T>(km * x); }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// B1: dA = dOut W2 ([n,h]); dU = dA * factor at the U positions.  dU feeds
// the dX GEMM and, for a dynamic MLP, is the shared A operand of its
// first-matrix aggregation.
// SwiGLU: the 32 dA columns [c0, c0+32) own the 64 contiguous interleaved
// positions [2 c0, 2 c0 + 64) (gate/up groups of 16).
// ---------------------------------------------------------------------------
template <typename T, bool SWIGLU>
struct EpiB1 {
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = false;
  using RowState = NoRowState;
  const T* fac;   // [rows, H2]
  T* dU;          // [rows, H2]
  int h;
  int rows_per_z;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState&, int z, int r, int c0, const float* v, const float*, int nv) const {
    int64_t grow = (int64_t)z * rows_per_z + r;
    const int64_t H2 = SWIGLU ? 2 * (int64_t)h : h;
    const int64_t ob = grow * H2;
    if (!SWIGLU) {
      if (nv == 32) {
        float f[32], du[32];
        vld<32>(fac + ob + c0, f);
#pragma unroll
        for (int j = 0; j < 32; ++j) du[j] = v[j] * f[j];
        vst<32>(dU + ob + c0, du);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) if (j < nv) {
          int c = c0 + j;
          dU[ob + c] = from_f<T>(v[j] * to_f<T>(fac[ob + c]));
        }
      }
    } else {
      // h % 16 == 0 and c0 % 32 == 0: nv is 16 or 32, whole groups of 16.
      // dA columns c0 + 16 g + k own positions 2 c0 + 32 g + k (gate) and + 16 (up).
      // bf16: both groups' factors are loaded (packed) before either dU
      // group is stored, so their latencies overlap.
      const int ng = nv > 16 ? 2 : 1;
      const int64_t p0 = ob + 2 * (int64_t)c0;
      if constexpr (!std::is_same<T, __nv_bfloat16>::value) {
        for (int g = 0; g < ng; ++g) {
          float f[32], du[32];
          vld<32>(fac + p0 + 32 * g, f);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            du[k] = v[16 * g + k] * f[k];
            du[16 + k] = v[16 * g + k] * f[16 + k];
          }
          vst<32>(dU + p0 + 32 * g, du);
        }
        return;
      }
      // 32-byte loads where the row is 32-byte aligned (h % 16 == 0 and an
      // aligned buffer: every row), else 16-byte ones
      uint32_t fr[2][16];
      const bool a32 = aligned32(fac + p0);
#pragma unroll
      for (int g = 0; g < 2; ++g)
        if (g < ng) {
          if (a32) {
            ld256(fac + p0 + 32 * g, fr[g]);
            ld256(fac + p0 + 32 * g + 16, fr[g] + 8);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 x = reinterpret_cast<const uint4*>(fac + p0 + 32 * g)[i];
              fr[g][4 * i] = x.x; fr[g][4 * i + 1] = x.y; fr[g][4 * i + 2] = x.z; fr[g][4 * i + 3] = x.w;
            }
          }
        }
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        if (g >= ng) break;
        float f[32], du[32];
        unpack_bf16x16(fr[g], f);
        unpack_bf16x16(fr[g] + 8, f + 16);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          du[k] = v[16 * g + k] * f[k];
          du[16 + k] = v[16 * g + k] * f[16 + k];
        }
        vst<32>(dU + p0 + 32 * g, du);
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
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = false;
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
    if (nv == 32) {
      float x[32];
      vld<32>(dout + o, x);
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] += v[j];
      vst<32>(dout + o, x);
      vst<32>(dout_a + o, x);
      if (doutW) { vst_scaled<32>(doutW + o, x, kw); vst_scaled<32>(doutM + o, x, km); }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j < nv) {
        float x = dout[o + j] + v[j];
        dout[o + j] = x;
        dout_a[o + j] = from_f<T>(x);
        if (doutW) { doutW[o + j] = from_f<T>(kw * x); doutM[o + j] = from_f<T>(km * x); }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Cross-entropy, pass A: per (row, column part) running max and sum of exp of
// the logits (online softmax), and the target logit.  The logits stay on chip.
// `part_index` (from the engine) numbers the column parts of a row.
// ---------------------------------------------------------------------------
template <typename T>
struct EpiCEPartial {
  static constexpr bool kFixedHeadTile = true;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = false;
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
    if (mx > st.m) { st.s *= exp_op<T>(st.m - mx); st.m = mx; }
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) if (j < nv) acc += exp_op<T>(v[j] - st.m);
    st.s += acc;
    int k = st.y - c0;
    if (k >= 0 && k < nv) {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j == k) tgt[r] = v[j];
    }
  }
  __device__ void row_end(RowState& st, int, int r, int part_index) const {
    float* p = part + ((int64_t)r * ntn + part_index) * 2;
    *reinterpret_cast<float2*>(p) = make_float2(st.m, st.s);
  }
};

// ---------------------------------------------------------------------------
// Cross-entropy, pass B over one vocabulary slab: dl/dlogit = softmax - onehot,
// written as an operand for dz = P E_slab.
// ---------------------------------------------------------------------------
template <typename T>
struct EpiCEGrad {
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = false;
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
    const float l = lse[r];
    T* o = P + (int64_t)r * Vs + c0;
    const int k = y - slab0 - c0;
    float p[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) p[j] = exp_op<T>(v[j] - l) - (j == k ? 1.0f : 0.0f);
    if (nv == 32) vst<32>(o, p);
    else {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j < nv) o[j] = from_f<T>(p[j]);
    }
  }
};

// ---------------------------------------------------------------------------
// Plain fp32 store (dz over the vocabulary slabs: first slab stores, the next
// ones accumulate).
// ---------------------------------------------------------------------------
struct EpiStoreF32 {
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = false;
  using RowState = NoRowState;
  float* out;
  int ld;
  int accumulate;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void span(RowState&, int, int r, int c0, const float* v, const float*, int nv) const {
    float* o = out + (int64_t)r * ld + c0;
    if (nv == 32) {
      float x[32];
      if (accumulate) {
        vld<32>(o, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] += v[j];
        vst<32>(o, x);
      } else {
        vst<32>(o, v);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j < nv) o[j] = accumulate ? o[j] + v[j] : v[j];
    }
  }
};

// Batched fp32 store: out[z](r, c) at out + z * zstride + r * ld + c.
struct EpiStoreBatched {
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = false;
  static constexpr bool kWarpRows = true;
  using RowState = NoRowState;
  using SpanRegs = NoSpanRegs;
  float* out;
  int64_t ld;
  int64_t zstride;
  __device__ void row_begin(RowState&, int, int) const {}
  __device__ void row_end(RowState&, int, int, int) const {}
  __device__ void load_span(SpanRegs&, int, int, int, int, int, int, int) const {}
  __device__ void finish_span(const SpanRegs&, int half, int z, int row0, int c0, const float* sv, int nv,
                              int nrows, int lane) const {
    const int cj = rw_col(lane);
    if (cj >= nv) return;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = rw_row(half, k, lane);
      if (i >= nrows) continue;
      float a[4];
      rw_read4(sv, i, cj, a);
      float* o = out + (int64_t)z * zstride + (int64_t)(row0 + i) * ld + c0 + cj;
      if (cj + 4 <= nv && (reinterpret_cast<uintptr_t>(o) & 15) == 0) store_x4(o, a);
      else for (int j = 0; j < 4 && j < nv - cj; ++j) o[j] = a[j];
    }
  }
  __device__ void span(RowState&, int z, int r, int c0, const float* v, const float*, int nv) const {
    float* o = out + (int64_t)z * zstride + (int64_t)r * ld + c0;
    if (nv == 32 && ((reinterpret_cast<uintptr_t>(o) & 15) == 0)) {
      vst<32>(o, v);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j < nv) o[j] = v[j];
    }
  }
};

// ---------------------------------------------------------------------------
// Aggregation + in-place update (Algorithm 1, update step): v = sum_t K_W_t G_t,
// v2 = sum_t K_M_t G_t for this element;
//   W <- gtilde_0 W + btilde_0 R_1 M + v,   M <- btilde_0 M + v2,
// and the operand shadow of the new W.  Batch z = sequence.
// ---------------------------------------------------------------------------
template <typename T>
struct EpiUpdate {
  static constexpr bool kFixedHeadTile = false;
  static constexpr bool kPreload = true;
  // The tcgen05 engine stages each warp's 32 x 32 accumulator span through
  // shared memory and calls span_warp(): the warp then walks the span row by
  // row, 8 lanes x 4 columns per row, so every W / M / shadow access of an
  // instruction covers whole 128-byte rows (the CUDA-core engine uses span()).
  static constexpr bool kWarpRows = true;
  // The span's W and M values, loaded by preload() before the engine reads
  // the accumulators from TMEM, so the state reads overlap the TMEM reads.
  struct RowState { float w[32], m[32]; };
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
  // Row-walking epilogue (used by the tcgen05 engine): a warp updates a span
  // of 32 rows x 32 columns, half a span (16 rows) per call, 8 lanes x 4
  // columns per row, so every W / M / shadow access of an instruction covers
  // whole 128-byte rows.  load_span() issues the half's W and M loads into
  // registers; finish_span() combines them with the two accumulators staged
  // in shared memory (sv: the half's row r of the first accumulator at
  // buffer row r, of the second at buffer row 16 + r; element (buffer row i,
  // column j) at [i * 32 + ((j + i) & 31)], rotated so both the staging
  // writes and these reads are conflict-free) and stores the results.
  struct SpanRegs { float4 w[4], m[4]; };
  // half: rows [16 half, 16 half + 16) of the span (8 lanes x 4 rows per step).
  __device__ void load_span(SpanRegs& R, int half, int z, int row0, int c0, int nv, int nrows, int lane) const {
    const int sub = lane >> 3, cj = (lane & 7) * 4;
    if (cj + 4 > nv) return;
    const float* Wz = W + z * seq_stride + c0 + cj;
    const float* Mz = M + z * seq_stride + c0 + cj;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = 16 * half + 4 * k + sub;
      if (i < nrows) {
        const int r = row0 + i;
        const int64_t off = (int64_t)(h > 0 ? swiglu_row_of_pos(r, h) : r) * cols;
        R.w[k] = *reinterpret_cast<const float4*>(Wz + off);
        R.m[k] = *reinterpret_cast<const float4*>(Mz + off);
      }
    }
  }
  __device__ void finish_span(const SpanRegs& R, int half, int z, int row0, int c0, const float* sv, int nv,
                              int nrows, int lane) const {
    const float4 cs = *reinterpret_cast<const float4*>(consts + ((int64_t)z * nchunks + chunk) * 4);
    const float g0 = cs.x, b0 = cs.y, cM = cs.z;
    const int sub = lane >> 3, cj = (lane & 7) * 4;
    const bool vec = cj + 4 <= nv;
    float* const Wz = W + z * seq_stride + c0 + cj;
    float* const Mz = M + z * seq_stride + c0 + cj;
    T* const Sz = Wsh + z * sh_stride + c0 + cj;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = 16 * half + 4 * k + sub;
      if (i >= nrows || cj >= nv) continue;
      const int r = row0 + i;
      const int64_t off = (int64_t)(h > 0 ? swiglu_row_of_pos(r, h) : r) * cols;
      const int b = 4 * k + sub;   // the row inside this half
      float a[4], a2[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        a[j] = sv[b * 32 + ((cj + j + b) & 31)];
        a2[j] = sv[(16 + b) * 32 + ((cj + j + 16 + b) & 31)];
      }
      T* sp = Sz + (int64_t)r * cols;
      if (vec) {
        float wn[4] = {R.w[k].x, R.w[k].y, R.w[k].z, R.w[k].w};
        float mn[4] = {R.m[k].x, R.m[k].y, R.m[k].z, R.m[k].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float wv = fmaf(g0, wn[j], fmaf(cM, mn[j], a[j]));
          mn[j] = fmaf(b0, mn[j], a2[j]);
          wn[j] = wv;
        }
        *reinterpret_cast<float4*>(Wz + off) = make_float4(wn[0], wn[1], wn[2], wn[3]);
        *reinterpret_cast<float4*>(Mz + off) = make_float4(mn[0], mn[1], mn[2], mn[3]);
        store_x4(sp, wn);
      } else {
        float* wq = Wz + off;
        float* mq = Mz + off;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (cj + j < nv) {
            const float wv = fmaf(g0, wq[j], fmaf(cM, mq[j], a[j]));
            mq[j] = fmaf(b0, mq[j], a2[j]);
            wq[j] = wv;
            sp[j] = from_f<T>(wv);
          }
        }
      }
    }
  }
  __device__ void preload(RowState& st, int z, int r, int c0, int nv) const {
    if (nv != 32) return;
    int fr = h > 0 ? swiglu_row_of_pos(r, h) : r;
    vld<32>(W + z * seq_stride + (int64_t)fr * cols + c0, st.w);
    vld<32>(M + z * seq_stride + (int64_t)fr * cols + c0, st.m);
  }
  __device__ void span(RowState& st, int z, int r, int c0, const float* v, const float* v2, int nv) const {
    const float4 cs = *reinterpret_cast<const float4*>(consts + ((int64_t)z * nchunks + chunk) * 4);
    const float g0 = cs.x, b0 = cs.y, cM = cs.z;
    int fr = h > 0 ? swiglu_row_of_pos(r, h) : r;
    float* wp = W + z * seq_stride + (int64_t)fr * cols + c0;
    float* mp = M + z * seq_stride + (int64_t)fr * cols + c0;
    T* sp = Wsh + z * sh_stride + (int64_t)r * cols + c0;
    if (nv == 32) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float wn = fmaf(g0, st.w[j], fmaf(cM, st.m[j], v[j]));
        st.m[j] = fmaf(b0, st.m[j], v2[j]);
        st.w[j] = wn;
      }
      vst<32>(wp, st.w);
      vst<32>(mp, st.m);
      vst<32>(sp, st.w);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) if (j < nv) {
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
