// Shared host/device helpers for libttt (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <cstdlib>
#include <utility>

#include "../../include/ttt.h"

namespace ttt {

// ----------------------------------------------------------------------------
// Element types of the GEMM operands: float (fp32 mode) or bfloat16 (bf16 mode)
// ----------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// ----------------------------------------------------------------------------
// Device status word: first error wins (TTT_OK = 0 means none yet).
// ----------------------------------------------------------------------------
__device__ __forceinline__ void record_error(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ----------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched with the programmatic
// stream-serialisation attribute (launch_dependent below) may be scheduled
// while the previous kernel of its stream still runs, once every CTA of that
// kernel has called grid_launch_dependents() or exited.  It may set up shared
// memory, barriers and TMEM, but must not read or write global memory before
// grid_dependency_wait() returns: that waits for the previous kernel to
// complete with its writes visible (to TMA loads too).  Both are no-ops in a
// kernel launched the ordinary way.  Because every kernel so launched waits
// before it completes, completion stays ordered along the whole stream.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// 1: kernels are launched as programmatic dependents of the previous kernel
// in their stream, so their launch and set-up overlap its tail (env
// TTT_PDL=0 launches them the ordinary way, for A/B timing).
inline int pdl_mode() {
  static int m = -1;
  if (m < 0) {
    const char* e = getenv("TTT_PDL");
    m = (e && e[0] == '0') ? 0 : 1;
  }
  return m;
}

// Launch `kernel` with the programmatic stream-serialisation attribute (see
// grid_dependency_wait); the kernel must wait before its first global access.
template <class... KArgs, class... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_mode() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// SwiGLU layout of the fused [gate; up] dimension inside the library:
// 32-wide groups, gate columns j in [16g, 16g+16) at positions [32g, 32g+16),
// up columns at [32g+16, 32g+32).  h must be a multiple of 16.
__host__ __device__ __forceinline__ int swiglu_pos_gate(int j) { return ((j >> 4) << 5) + (j & 15); }
__host__ __device__ __forceinline__ int swiglu_pos_up(int j) { return ((j >> 4) << 5) + 16 + (j & 15); }
// Inverse: position p in [0, 2h) -> row of the packed [W1; W2] (W1 rows 0..h-1, W2 rows h..2h-1).
__host__ __device__ __forceinline__ int swiglu_row_of_pos(int p, int h) {
  int g = p >> 5, k = p & 31;
  return k < 16 ? (g << 4) + k : h + (g << 4) + (k - 16);
}

}  // namespace ttt

#define TTT_CUDA_TRY(expr)                                             \
  do {                                                                 \
    cudaError_t _e = (expr);                                           \
    if (_e != cudaSuccess) {                                           \
      ::ttt::set_last_error(#expr, cudaGetErrorString(_e), __FILE__, __LINE__); \
      return TTT_ERR_CUDA;                                             \
    }                                                                  \
  } while (0)

namespace ttt {
void set_last_error(const char* what, const char* why, const char* file, int line);
void set_last_error_msg(const char* msg);
}  // namespace ttt
