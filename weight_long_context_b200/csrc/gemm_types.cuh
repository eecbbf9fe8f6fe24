// Shapes and operand descriptions shared by the two GEMM engines.
#pragma once

#include <stdint.h>

namespace ttt {

// D[z](m, n) = sum_{k < K} A[z](m, k) * B[z](n, k), z < batch.
struct GemmShape {
  int M, N, K, batch;
};

// One operand.  K-major: element (mn, k) at ptr + z*batch_stride + mn*ld + k.
// MN-major:              element (mn, k) at ptr + z*batch_stride + k*ld + mn.
// Strides in elements.  batch_stride == 0 shares the operand across z.
struct Operand {
  const void* ptr;
  int64_t ld;
  int64_t batch_stride;
  int kmajor;
  // Rows (K-major: mn extent; MN-major: k extent) that exist per batch entry
  // in memory; loads beyond them read zero.  Used by the TMA engine to stop a
  // per-sequence tile from reading the next sequence's rows.
  int64_t rows_per_batch;
};

// Scratch for split-K partial tiles of the CTA-pair GEMM (both may be null:
// no split-K).  counters must be zero before the first GEMM that uses them;
// every GEMM leaves them zero.
struct SplitScratch {
  float* partial = nullptr;
  size_t partial_bytes = 0;
  int* counters = nullptr;
  size_t counter_count = 0;
};

}  // namespace ttt
