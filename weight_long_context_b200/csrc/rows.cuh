// Row-wise kernels of the chunk step: gather of the chunk's hidden rows,
// RMSNorm forward/backward, the cross-entropy reduction, operand casts, and
// the bounded-wait primitive.  All are bandwidth-bound, one warp per row with
// 16-byte accesses where the layout allows.
#pragma once

#include "common.cuh"
#include "epilogue.cuh"

namespace ttt {

template <typename T>
__device__ __forceinline__ void store4(T* p, float4 x);
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 x) { *reinterpret_cast<float4*>(p) = x; }
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 x) {
  __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y), b = __floats2bfloat162_rn(x.z, x.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// ---------------------------------------------------------------------------
// Gather chunk c of every sequence: resid[s*b + i] = hidden[s, c*b + i] and
// its operand copy.
// ---------------------------------------------------------------------------
// When the first MLP is dynamic, also its K-scaled negated input copies
// (B operands of its first-matrix aggregation).
template <typename T>
__global__ void gather_chunk_kernel(const float* __restrict__ hidden, int T_, int b, int chunk, int d,
                                    int64_t n, float* __restrict__ resid, T* __restrict__ act,
                                    T* __restrict__ aw, T* __restrict__ am, const float* __restrict__ KW,
                                    const float* __restrict__ KM, float kscale) {
  const int64_t q = d >> 2;  // float4 per row (d % 16 == 0)
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * q;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t r = e / q, c4 = e - r * q;
    int64_t s = r / b, i = r - s * b;
    const int64_t ti = s * T_ + (int64_t)chunk * b + i;
    const float4 x = reinterpret_cast<const float4*>(hidden + ti * d)[c4];
    reinterpret_cast<float4*>(resid + r * d)[c4] = x;
    store4<T>(act + r * d + c4 * 4, x);
    if (aw) {
      const float kw = -KW[ti] * kscale, km = -KM[ti] * kscale;
      store4<T>(aw + r * d + c4 * 4, make_float4(kw * x.x, kw * x.y, kw * x.z, kw * x.w));
      store4<T>(am + r * d + c4 * 4, make_float4(km * x.x, km * x.y, km * x.z, km * x.w));
    }
  }
}

// ---------------------------------------------------------------------------
// RMSNorm forward: z = g * h / sqrt(mean(h^2) + eps); keeps 1/rms for backward.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void rmsnorm_fwd_kernel(const float* __restrict__ h, const float* __restrict__ g, float eps,
                                   int64_t n, int d, T* __restrict__ z, float* __restrict__ rstd) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n) return;
  const float4* hr = reinterpret_cast<const float4*>(h + row * d);
  float ss = 0.f;
  for (int c = lane; c < (d >> 2); c += 32) {
    float4 x = hr[c];
    ss += x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / (float)d + eps);
  if (lane == 0) rstd[row] = r;
  T* zr = z + row * d;
  const float4* gr = reinterpret_cast<const float4*>(g);
  for (int c = lane; c < (d >> 2); c += 32) {
    float4 x = hr[c], gg = gr[c];
    store4<T>(zr + 4 * c, make_float4(x.x * r * gg.x, x.y * r * gg.y, x.z * r * gg.z, x.w * r * gg.w));
  }
}

// ---------------------------------------------------------------------------
// RMSNorm backward: dh = r * (g*dz) - h * r^3 * <g*dz, h> / d.
// Writes the gradient of the residual stream (fp32), its operand copy, and,
// when the top MLP is dynamic, the K-scaled negated copies.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void rmsnorm_bwd_kernel(const float* __restrict__ dz, const float* __restrict__ h,
                                   const float* __restrict__ rstd, const float* __restrict__ g,
                                   int64_t n, int d, float* __restrict__ dout, T* __restrict__ dout_a,
                                   T* __restrict__ doutW, T* __restrict__ doutM,
                                   const float* __restrict__ KW, const float* __restrict__ KM, float kscale,
                                   TokenMap tm) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n) return;
  const float4* dzr = reinterpret_cast<const float4*>(dz + row * d);
  const float4* hr = reinterpret_cast<const float4*>(h + row * d);
  const float4* gr = reinterpret_cast<const float4*>(g);
  float dot = 0.f;
  for (int c = lane; c < (d >> 2); c += 32) {
    float4 a = dzr[c], x = hr[c], gg = gr[c];
    dot += a.x * gg.x * x.x + a.y * gg.y * x.y + a.z * gg.z * x.z + a.w * gg.w * x.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  const float r = rstd[row];
  const float coef = r * r * r * dot / (float)d;
  float kw = 0.f, km = 0.f;
  if (doutW) {
    int64_t ti = tm.index((int)row);
    kw = -KW[ti] * kscale;
    km = -KM[ti] * kscale;
  }
  for (int c = lane; c < (d >> 2); c += 32) {
    float4 a = dzr[c], x = hr[c], gg = gr[c];
    float o4[4] = {r * a.x * gg.x - x.x * coef, r * a.y * gg.y - x.y * coef,
                   r * a.z * gg.z - x.z * coef, r * a.w * gg.w - x.w * coef};
    reinterpret_cast<float4*>(dout + row * d)[c] = make_float4(o4[0], o4[1], o4[2], o4[3]);
    const int64_t idx = row * d + 4 * c;
    store4<T>(dout_a + idx, make_float4(o4[0], o4[1], o4[2], o4[3]));
    if (doutW) {
      store4<T>(doutW + idx, make_float4(kw * o4[0], kw * o4[1], kw * o4[2], kw * o4[3]));
      store4<T>(doutM + idx, make_float4(km * o4[0], km * o4[1], km * o4[2], km * o4[3]));
    }
  }
}

// ---------------------------------------------------------------------------
// Cross-entropy reduction, one warp per row: combine the row's online-softmax
// partials (max, sum exp) into lse and form l_t = lse - logit[y_t]; with
// tok_out also store l_t at the token's [B, T] position.
// ---------------------------------------------------------------------------
__global__ void ce_rows_kernel(const float* __restrict__ part, const float* __restrict__ tgt, int ntn,
                               const int* __restrict__ tokens, TokenMap tm, int V, int64_t n,
                               float* __restrict__ lse, float* __restrict__ ltok, int* status,
                               float* __restrict__ tok_out = nullptr) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= n) return;
  const float2* p = reinterpret_cast<const float2*>(part + r * ntn * 2);
  float m = -INFINITY;
  for (int t = lane; t < ntn; t += 32) m = fmaxf(m, p[t].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sum = 0.f;
  for (int t = lane; t < ntn; t += 32) { float2 q = p[t]; sum += q.y * expf(q.x - m); }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) {
    float l = m + logf(sum);
    lse[r] = l;
    int y = tokens[tm.index((int)r)];
    const float lt = (y < 0 || y >= V) ? 0.f : l - tgt[r];
    if (y < 0 || y >= V) record_error(status, TTT_ERR_TOKEN_RANGE);
    ltok[r] = lt;
    if (tok_out) tok_out[tm.index((int)r)] = lt;
  }
}

// E2-TTT's own layer ("Rethinking Expressivity and Efficiency in Test-Time
// Training": TTT modelling background, 快速权重网络实例化, Algorithm 1), one warp
// per chunk row r (token ti):
//   keys:    f = k + LN(y_k), L_t = mean_j (f - v)_j^2, g_f = 2 (f - v) / d,
//            g_y = rs (g_f - mean(g_f) - LN(y_k) mean(g_f LN(y_k)))
//            -> dout_a = g_y (operand of dA = g_y W_down) and the K_W / K_M
//            scaled, negated copies (operands of the output matrix's update);
//   queries: o = q + LN(y_q), written to the caller's O at token ti.
// LN is the parameter-free LayerNorm (epsilon eps); statistics in two passes
// over the row (mean, then centred sum of squares), float32.
template <typename T>
__global__ void recon_rows_kernel(const float* __restrict__ yk, const float* __restrict__ kres,
                                  const float* __restrict__ Vt, const float* __restrict__ yq,
                                  const float* __restrict__ qres, TokenMap tm, int64_t n, int d, float eps,
                                  const float* __restrict__ KW, const float* __restrict__ KM, float kscale,
                                  float* __restrict__ ltok, T* __restrict__ dout_a, T* __restrict__ doutW,
                                  T* __restrict__ doutM, float* __restrict__ O) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= n) return;
  const int64_t ti = tm.index((int)r);
  const int q4 = d >> 2;
  const float invd = 1.f / (float)d;
  auto wsum = [](float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
  };
  // LayerNorm statistics of one row
  auto stats = [&](const float4* y, float& mu, float& rs) {
    float s1 = 0.f;
    for (int c = lane; c < q4; c += 32) { const float4 a = y[c]; s1 += (a.x + a.y) + (a.z + a.w); }
    mu = wsum(s1) * invd;
    float s2 = 0.f;
    for (int c = lane; c < q4; c += 32) {
      const float4 a = y[c];
      const float e0 = a.x - mu, e1 = a.y - mu, e2 = a.z - mu, e3 = a.w - mu;
      s2 += (e0 * e0 + e1 * e1) + (e2 * e2 + e3 * e3);
    }
    rs = rsqrtf(wsum(s2) * invd + eps);
  };
  // ---- keys: loss and the gradient at the MLP output
  const float4* yr = reinterpret_cast<const float4*>(yk + r * d);
  const float4* kr = reinterpret_cast<const float4*>(kres + r * d);
  const float4* vr = reinterpret_cast<const float4*>(Vt + ti * d);
  float mu, rs;
  stats(yr, mu, rs);
  float sl = 0.f, sg = 0.f, sgl = 0.f;
  for (int c = lane; c < q4; c += 32) {
    const float4 y = yr[c], k = kr[c], v = vr[c];
    const float yy[4] = {y.x, y.y, y.z, y.w}, kk[4] = {k.x, k.y, k.z, k.w}, vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float ln = (yy[j] - mu) * rs;
      const float e = kk[j] + ln - vv[j];
      const float g = 2.f * e * invd;
      sl += e * e;
      sg += g;
      sgl += g * ln;
    }
  }
  sl = wsum(sl);
  const float mg = wsum(sg) * invd, mgl = wsum(sgl) * invd;
  if (lane == 0) ltok[r] = sl * invd;
  const float kw = -KW[ti] * kscale, km = -KM[ti] * kscale;
  for (int c = lane; c < q4; c += 32) {
    const float4 y = yr[c], k = kr[c], v = vr[c];
    const float yy[4] = {y.x, y.y, y.z, y.w}, kk[4] = {k.x, k.y, k.z, k.w}, vv[4] = {v.x, v.y, v.z, v.w};
    float gy[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float ln = (yy[j] - mu) * rs;
      const float g = 2.f * (kk[j] + ln - vv[j]) * invd;
      gy[j] = rs * (g - mg - ln * mgl);
    }
    const int64_t o = r * d + 4 * c;
    store4<T>(dout_a + o, make_float4(gy[0], gy[1], gy[2], gy[3]));
    store4<T>(doutW + o, make_float4(kw * gy[0], kw * gy[1], kw * gy[2], kw * gy[3]));
    store4<T>(doutM + o, make_float4(km * gy[0], km * gy[1], km * gy[2], km * gy[3]));
  }
  // ---- queries: the outputs at the chunk-start weights
  const float4* zr = reinterpret_cast<const float4*>(yq + r * d);
  const float4* qr = reinterpret_cast<const float4*>(qres + r * d);
  stats(zr, mu, rs);
  float4* orow = reinterpret_cast<float4*>(O + ti * d);
  for (int c = lane; c < q4; c += 32) {
    const float4 y = zr[c], q = qr[c];
    orow[c] = make_float4(q.x + (y.x - mu) * rs, q.y + (y.y - mu) * rs, q.z + (y.z - mu) * rs, q.w + (y.w - mu) * rs);
  }
}

// Input-dependent update scalars ("Rethinking Expressivity and Efficiency in
// Test-Time Training", 依赖于输入的动态参数化), one warp per token row x_t:
//   eta_t   = eta_base sigmoid(w_eta . x_t + b_eta)
//   beta_t  = sigmoid(w_beta . x_t + b_beta)^(1/tau)
//   gamma_t = 1 - eta_t alpha_base sigmoid(w_alpha . x_t + b_alpha)
// heads [3, d] = (w_eta, w_beta, w_alpha).  The three dot products are summed
// in float32 in a fixed order (lane-strided float4, then a shuffle tree), so
// the result does not depend on scheduling.  d % 4 == 0.
__global__ void scalar_heads_kernel(const float* __restrict__ x, int64_t rows, int d, const float* __restrict__ heads,
                                    float b_eta, float b_beta, float b_alpha, float eta_base, float alpha_base,
                                    float inv_tau, float* __restrict__ eta, float* __restrict__ beta,
                                    float* __restrict__ gamma) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const float4* xr = reinterpret_cast<const float4*>(x + r * d);
  const float4* h0 = reinterpret_cast<const float4*>(heads);
  const float4* h1 = reinterpret_cast<const float4*>(heads + d);
  const float4* h2 = reinterpret_cast<const float4*>(heads + 2 * (int64_t)d);
  float z0 = 0.f, z1 = 0.f, z2 = 0.f;
  for (int i = lane; i < d / 4; i += 32) {
    const float4 v = xr[i], a = h0[i], b = h1[i], c = h2[i];
    z0 += v.x * a.x + v.y * a.y + v.z * a.z + v.w * a.w;
    z1 += v.x * b.x + v.y * b.y + v.z * b.z + v.w * b.w;
    z2 += v.x * c.x + v.y * c.y + v.z * c.z + v.w * c.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    z0 += __shfl_xor_sync(0xffffffffu, z0, o);
    z1 += __shfl_xor_sync(0xffffffffu, z1, o);
    z2 += __shfl_xor_sync(0xffffffffu, z2, o);
  }
  if (lane == 0) {
    const float se = 1.f / (1.f + expf(-(z0 + b_eta)));
    const float sb = 1.f / (1.f + expf(-(z1 + b_beta)));
    const float sa = 1.f / (1.f + expf(-(z2 + b_alpha)));
    const float e = eta_base * se;
    eta[r] = e;
    beta[r] = powf(sb, inv_tau);
    gamma[r] = 1.f - e * (alpha_base * sa);
  }
}

// Chunk mean of the token losses, one block per sequence, fixed reduction
// order (the result does not depend on scheduling).
__global__ void ce_mean_kernel(const float* __restrict__ ltok, int b, float* __restrict__ chunk_loss, int chunk,
                               int nchunks, int* status) {
  __shared__ float red[32];
  const int s = blockIdx.x;
  float acc = 0.f;
  for (int i = threadIdx.x; i < b; i += blockDim.x) acc += ltok[(int64_t)s * b + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    int nw = blockDim.x >> 5;
    float v = threadIdx.x < nw ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) {
      float mean = v / (float)b;
      chunk_loss[(int64_t)s * nchunks + chunk] = mean;
      if (!isfinite(mean)) record_error(status, TTT_ERR_NONFINITE);
    }
  }
}

// ---------------------------------------------------------------------------
// Operand shadow of packed fast weights (or static weights): a cast to the
// operand type, with the SwiGLU [W1; W2] rows placed in the interleaved
// library order.  count = number of blocks (sequences x n_blocks).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void build_shadow_kernel(const float* __restrict__ W, T* __restrict__ sh, int64_t count,
                                    int h, int d, int swiglu) {
  const int64_t blk = (swiglu ? 3 : 2) * (int64_t)h * d;
  const int64_t total4 = count * blk / 4;   // d % 16 == 0: a group of 4 never crosses a row
  for (int64_t e4 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e4 < total4;
       e4 += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = 4 * e4;
    const int64_t o = e % blk, base = e - o;
    int64_t src = e;
    if (swiglu && o < 2 * (int64_t)h * d) {
      const int p = (int)(o / d);
      const int64_t c = o - (int64_t)p * d;
      src = base + (int64_t)swiglu_row_of_pos(p, h) * d + c;
    }
    store4<T>(sh + e, *reinterpret_cast<const float4*>(W + src));
  }
}

template <typename T>
__global__ void cast_kernel(const float* __restrict__ x, T* __restrict__ y, int64_t n) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    y[e] = from_f<T>(x[e]);
}

// ---------------------------------------------------------------------------
// Bounded wait: poll a device flag at most `limit` times.  Returns true if
// the flag became nonzero; otherwise records TTT_ERR_TIMEOUT and returns
// false.  Every spin loop in the library has such a limit.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool bounded_wait_flag(const volatile int* flag, uint32_t limit, int* status) {
  for (uint32_t i = 0; i < limit; ++i) {
    if (*flag != 0) return true;
    __nanosleep(64);
  }
  record_error(status, TTT_ERR_TIMEOUT);
  return false;
}

__global__ void selftest_wait_kernel(const int* flag, uint32_t limit, int* status) {
  if (threadIdx.x == 0) bounded_wait_flag(flag, limit, status);
}

}  // namespace ttt
