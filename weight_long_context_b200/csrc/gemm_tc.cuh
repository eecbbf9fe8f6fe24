// tcgen05 GEMM engine for sm_100a: D[z](m, n) = sum_k A[z](m, k) B[z](n, k),
// bf16 operands, fp32 accumulation in tensor memory (TMEM).
//
// Structure (one persistent CTA per SM, 320 threads):
//   warp 0      TMA producer: one lane streams 128x64 A tiles (and a second A
//               for the dual-accumulator aggregation) and BNx64 B tiles into a
//               ring of shared-memory stages, 128-byte swizzled, arriving on
//               the stage's "full" mbarrier with the transaction byte count;
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (M=128, N=BN,
//               K=16 per instruction) and frees each stage with tcgen05.commit;
//   warps 2..9  epilogue: wait for a finished accumulator, tcgen05.ld 32
//               columns at a time and hand the row spans to the epilogue
//               functor.  A warp may only read the TMEM lane quarter
//               (warp % 4); two warps share each quarter and split the tile's
//               columns in halves, one row per thread.
// Accumulators are double-buffered in TMEM so the epilogue of tile i overlaps
// the MMAs of tile i+1.  Operands may be K-major or MN-major (the matrix
// descriptors and the instruction descriptor carry the layout), so the
// backward and aggregation GEMMs read the forward buffers without transposes.
// No TMA multicast is used anywhere.
//
// Every mbarrier wait is bounded by the global timer; on expiry the kernel
// records TTT_ERR_TIMEOUT, raises a CTA-wide abort flag, waits (bounded) for
// its own TMA copies and MMAs in flight, frees its TMEM and returns.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstdlib>
#include <utility>

#include "common.cuh"
#include "gemm_types.cuh"

namespace ttt {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;             // 64 bf16 = 128 bytes: one swizzle row
constexpr int HEAD_BN = 256;       // N tile of the single-accumulator GEMMs
constexpr int EPI_WARPS = 8;
constexpr int EPI_PARTS = EPI_WARPS / 4;   // column parts per tile row
// Epilogue warps of the two-accumulator state update (which streams 18 bytes
// of fp32 W / M state per parameter).  Measured on B200 at the 128K stack's
// shapes: 16 warps (four per TMEM lane quarter) run no faster than 8.
constexpr int AGG_EPI_WARPS = 8;
__host__ __device__ constexpr int epi_warps(int nacc, bool warprows) {
  return (nacc == 2 && warprows) ? AGG_EPI_WARPS : EPI_WARPS;
}
constexpr uint64_t WAIT_NS = 4000000000ull;   // 4 s per wait before giving up

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait.  Returns false on abort (flag raised elsewhere) or timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (abort_flag && *abort_flag) return false;
      if (global_ns() - t0 > WAIT_NS) {
        record_error(status, TTT_ERR_TIMEOUT);
        if (abort_flag) *abort_flag = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
// Bring a kernel-parameter tensor map into the TMA unit's descriptor cache
// ahead of the first copy that uses it.
__device__ __forceinline__ void tmap_prefetch(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// 32 lanes x 32 columns of 32-bit: thread i of the warp gets row (lane base + i),
// columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// 32 lanes x 16 columns of 32-bit (same lane mapping as tmem_ld32).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: version 1
// at bit 46, layout type 2 at bits 61-63).  Addresses and offsets in bytes.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, M=128, N=n.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Kernel configuration per (accumulators, N tile)
// ---------------------------------------------------------------------------
template <int NACC, int BN, bool WARPROWS = false>
struct Cfg {
  // Epilogue warps: two (four for the state update) per TMEM lane quarter,
  // splitting the tile's columns.
  static constexpr int EW = epi_warps(NACC, WARPROWS);
  static constexpr int PARTS = EW / 4;
  static constexpr int NTHREADS = 64 + 32 * EW;
  static constexpr int A_BYTES = BM * BK * 2;            // 16 KiB
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = NACC * A_BYTES + B_BYTES;
  // Epilogues that walk rows stage each warp's 32x32 span in shared memory:
  // 4 KiB per epilogue warp (the state update stages its two accumulators in turn).
  static constexpr int ROWSTAGE_BYTES = WARPROWS ? EW * 32 * 32 * 4 : 0;
  // as many operand stages as the 227 KiB per CTA leave beside the staging,
  // the 1 KiB alignment slack and the barriers
  static constexpr int STAGES = (232448 - 1280 - ROWSTAGE_BYTES) / STAGE_BYTES;
  static constexpr int TMEM_COLS = 2 * NACC * BN;         // two accumulator buffers
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + ROWSTAGE_BYTES + 1024 /*align slack*/ + 256 /*barriers*/;
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of two");
  static_assert(STAGES >= 2 && STAGES <= 16, "two to sixteen stages (the barriers take 256 bytes)");
  static_assert(SMEM_BYTES <= 232448, "shared memory above the 227 KiB per-CTA limit");
};

struct TcParams {
  GemmShape s;
  int a_mn, b_mn;       // 1 = MN-major operand
  // Dual accumulators (NACC = 2, BN = 128, 1-SM kernel): dualb = 0 shares B
  // (acc_j += A_j B^T, maps A, A2, B); dualb = 1 shares A (acc_j += A B_j^T,
  // maps A, B, and A2 holding B_2).  Both use three 16 KiB slots per stage.
  int dualb;
  int tiles_m, tiles_n, num_tiles, num_kb;
  int* status;
  // Split-K (pair kernel): unit u = tile * splits + ks covers k-blocks
  // [ks * kb_per_split, min(num_kb, (ks + 1) * kb_per_split)).
  int splits, kb_per_split;
  // pair_finish: tiles [0, full_tiles) run whole, the remaining tiles as two
  // halves of the k-blocks (units full_tiles + 2 i, + 1), all of them in the
  // last wave so both halves of a tile are resident at once; half 0 finishes
  // the rows of TMEM lane quarters 0-1, half 1 those of quarters 2-3, and a
  // warp parks only the partial its partner finishes, in
  // [tile - full_tiles][2 CTAs][128 rows][BN].
  int pair_finish, full_tiles, num_units;
  float* partial;   // [num_tiles][splits][2 CTAs][128 rows][BN] fp32 when splits > 1
  int* counters;    // [num_tiles][2 CTAs][EPI_WARPS], zero on entry, left zero on exit
};

// Work unit u of the pair kernel: tile t, k-blocks [kb0, kb1), split index ks.
struct Unit {
  int t, ks, kb0, kb1;
  bool split;
};
__device__ __forceinline__ Unit decode_unit(const TcParams& p, int u) {
  Unit x;
  if (p.pair_finish) {
    if (u < p.full_tiles) {
      x.t = u; x.ks = 0; x.kb0 = 0; x.kb1 = p.num_kb; x.split = false;
    } else {
      const int v = u - p.full_tiles;
      x.t = p.full_tiles + (v >> 1);
      x.ks = v & 1;
      x.kb0 = x.ks ? p.kb_per_split : 0;
      x.kb1 = x.ks ? p.num_kb : p.kb_per_split;
      x.split = true;
    }
  } else {
    x.t = u / p.splits;
    x.ks = u - x.t * p.splits;
    x.kb0 = x.ks * p.kb_per_split;
    x.kb1 = min(p.num_kb, x.kb0 + p.kb_per_split);
    x.split = p.splits > 1;
  }
  return x;
}

// Tile t -> (row tile tm, column tile tn, batch entry z).  Consecutive tiles
// run on consecutive CTAs (pairs) at the same time.  The GEMMs walk row tiles
// first (the tiles in flight share a column block of B); the two-accumulator
// state update walks column tiles first, so the state rows it streams at once
// are whole rows (measured on B200: 3 % faster than row tiles first).
template <int NACC>
__device__ __forceinline__ void decode_tile(const TcParams& p, int t, int& tm, int& tn, int& z) {
  if constexpr (NACC == 2) {
    tn = t % p.tiles_n;
    const int rest = t / p.tiles_n;
    tm = rest % p.tiles_m;
    z = rest / p.tiles_m;
  } else {
    tm = t % p.tiles_m;
    const int rest = t / p.tiles_m;
    tn = rest % p.tiles_n;
    z = rest / p.tiles_n;
  }
}

// Row-walking epilogues.  The accumulators arrive one row per thread (the
// TMEM lane layout); global rows are contiguous, so a thread writing its own
// row would touch 32 separate lines per warp instruction.  Instead each warp
// stages a 32 x 32 span in shared memory (element (row i, column j) at
// [i * 32 + ((j + i) & 31)], rotated so the staging writes and the row reads
// are both conflict-free) and the epilogue functor walks it row by row, half
// a span (16 rows) at a time: 8 lanes x 4 columns per row, 4 rows per step,
// so every global access of an instruction covers whole row segments.

// Stage this thread's row of a 32-column span.
__device__ __forceinline__ void stage_row32(float* sv, const float* v, int lane) {
#pragma unroll
  for (int j = 0; j < 32; ++j) sv[lane * 32 + ((j + lane) & 31)] = v[j];
}

// Walk a staged span: rows [row0, row0 + nrows) and columns [c0, c0 + nv) of
// batch entry z, both halves.
template <class Epi>
__device__ __forceinline__ void finish_rows(const Epi& epi, int z, int row0, int c0, int nv, int nrows,
                                            const float* sv, int lane) {
  if (nrows <= 0 || nv <= 0) return;
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    typename Epi::SpanRegs R;
    epi.load_span(R, half, z, row0, c0, nv, nrows, lane);
    epi.finish_span(R, half, z, row0, c0, sv, nv, nrows, lane);
  }
}

// One tile of a row-walking epilogue read straight from TMEM (tbase: this
// warp's lane quarter of the accumulator buffer).  The warp owns rows
// [row0, row0 + 32) and the PART_COLS columns of its part.  release() frees
// the accumulator buffer once every span of the tile is staged.
// Stage columns [c, c + 32) of the accumulator at tbase (this thread's row).
__device__ __forceinline__ void stage_tmem32(float* sv, uint32_t taddr, int lane) {
#pragma unroll
  for (int hc = 0; hc < 32; hc += 16) {
    float v[16];
    tmem_ld16(taddr + hc, v);
#pragma unroll
    for (int j = 0; j < 16; ++j) sv[lane * 32 + ((hc + j + lane) & 31)] = v[j];
  }
}

template <int NACC, int BN, int PART_COLS, class Epi, class Release>
__device__ __forceinline__ void rows_tile(const Epi& epi, const GemmShape& s, int z, int row0, int tn, uint32_t tbase,
                                          float* sv, int part, int lane, Release release) {
  constexpr int NSP = PART_COLS / 32;
  const int nrows = min(32, s.M - row0);
#pragma unroll 1
  for (int spi = 0; spi < NSP; ++spi) {
    const int c = part * PART_COLS + spi * 32;
    const int c0 = tn * BN + c;
    const int nv = min(32, s.N - c0);
    if constexpr (NACC == 1) {
      stage_tmem32(sv, tbase + c, lane);
      if (spi == NSP - 1) {  // every accumulator of this tile is staged: free the buffer
        tc_fence_before();
        release();
      }
      __syncwarp();
      finish_rows(epi, z, row0, c0, nv, nrows, sv, lane);
      __syncwarp();
    } else {
      // Two accumulators through one 32 x 32 staging buffer, half a span at a
      // time: rows [0, 16) of the buffer hold the half's rows of the first
      // accumulator, rows [16, 32) the same rows of the second.  The half's
      // global loads are issued before the TMEM reads.
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        typename Epi::SpanRegs R;
        const bool live = nrows > 0 && nv > 0;
        if (live) epi.load_span(R, half, z, row0, c0, nv, nrows, lane);
        const bool mine = (lane >> 4) == half;
        const int r = lane & 15;
#pragma unroll
        for (int a = 0; a < 2; ++a) {
#pragma unroll
          for (int hc = 0; hc < 32; hc += 16) {
            float v[16];
            tmem_ld16(tbase + a * BN + c + hc, v);
            if (mine) {
#pragma unroll
              for (int j = 0; j < 16; ++j) sv[(16 * a + r) * 32 + ((hc + j + 16 * a + r) & 31)] = v[j];
            }
          }
        }
        if (half == 1 && spi == NSP - 1) {  // every accumulator of this tile is read: free the buffer
          tc_fence_before();
          release();
        }
        __syncwarp();
        if (live) epi.finish_span(R, half, z, row0, c0, sv, nv, nrows, lane);
        __syncwarp();
      }
    }
  }
}

// Row-walking epilogue loop of the 1-SM kernel and of the pair kernel's
// two-accumulator aggregation (never split): the tiles this CTA processes
// are first, first + step, ...; tile rows start at tm * rows_per_tile + row_off.
template <int NACC, int BN, int PART_COLS, class Epi, class Release>
__device__ __forceinline__ void warp_rows_loop(const Epi& epi, const TcParams& p, int first, int step,
                                               int rows_per_tile, int row_off, uint32_t tmem_base,
                                               uint64_t* tfull, float* sv, int q, int part, int lane,
                                               volatile int* abort_flag, Release release) {
  uint32_t tcount = 0;
  for (int t = first; t < p.num_tiles; t += step, ++tcount) {
    const uint32_t buf = tcount & 1u;
    const uint32_t aph = (tcount >> 1) & 1u;
    const bool ready = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], aph, abort_flag, p.status));
    if (!ready) break;
    tc_fence_after();
    int tm, tn, z;
    decode_tile<NACC>(p, t, tm, tn, z);
    const int row0 = tm * rows_per_tile + row_off + q * 32;
    const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + buf * (NACC * BN);
    rows_tile<NACC, BN, PART_COLS>(epi, p.s, z, row0, tn, tbase, sv, part, lane, [&]() { release(buf); });
  }
}

template <int NACC, int BN, class Epi>
__global__ void __launch_bounds__(Cfg<NACC, BN, Epi::kWarpRows>::NTHREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapA2,
               const __grid_constant__ CUtensorMap mapB, const TcParams p, const Epi epi) {
  using C = Cfg<NACC, BN, Epi::kWarpRows>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* rowstage = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::ROWSTAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    tmap_prefetch(&mapA);
    tmap_prefetch(&mapA2);
    tmap_prefetch(&mapB);
    for (int i = 0; i < C::STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], 32 * C::EW); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Barriers and TMEM are set up: wait for the previous kernel of the stream
  // before the first global access, then let the next one be scheduled onto
  // SMs as they free up.
  grid_dependency_wait();
  grid_launch_dependents();

  const GemmShape& s = p.s;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int tm, tn, z;
        decode_tile<NACC>(p, t, tm, tn, z);
        const int m0 = tm * BM, n0 = tn * BN;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const int st = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
          uint8_t* sa = smem + st * C::STAGE_BYTES;
          uint8_t* sb = sa + NACC * C::A_BYTES;
          mbar_expect_tx(&full[st], C::STAGE_BYTES);
          const int k0 = kb * BK;
          if (NACC == 2 && p.dualb) {
            // slot 0: A, slot 1: B_1, slot 2: B_2 (BN == BM: all slots 16 KiB)
            if (!p.a_mn) {
              tma_load_3d(sa, &mapA, &full[st], k0, m0, z);
            } else {
#pragma unroll
              for (int j = 0; j < BM / 64; ++j) tma_load_3d(sa + j * 8192, &mapA, &full[st], m0 + 64 * j, k0, z);
            }
            uint8_t* sb1 = sa + C::A_BYTES;
            uint8_t* sb2 = sb1 + C::B_BYTES;
            if (!p.b_mn) {
              tma_load_3d(sb1, &mapB, &full[st], k0, n0, z);
              tma_load_3d(sb2, &mapA2, &full[st], k0, n0, z);
            } else {
#pragma unroll
              for (int j = 0; j < BN / 64; ++j) {
                tma_load_3d(sb1 + j * 8192, &mapB, &full[st], n0 + 64 * j, k0, z);
                tma_load_3d(sb2 + j * 8192, &mapA2, &full[st], n0 + 64 * j, k0, z);
              }
            }
          } else {
            if (!p.a_mn) {
              tma_load_3d(sa, &mapA, &full[st], k0, m0, z);
              if (NACC == 2) tma_load_3d(sa + C::A_BYTES, &mapA2, &full[st], k0, m0, z);
            } else {
#pragma unroll
              for (int j = 0; j < BM / 64; ++j) {
                tma_load_3d(sa + j * 8192, &mapA, &full[st], m0 + 64 * j, k0, z);
                if (NACC == 2) tma_load_3d(sa + C::A_BYTES + j * 8192, &mapA2, &full[st], m0 + 64 * j, k0, z);
              }
            }
            if (!p.b_mn) {
              tma_load_3d(sb, &mapB, &full[st], k0, n0, z);
            } else {
#pragma unroll
              for (int j = 0; j < BN / 64; ++j) tma_load_3d(sb + j * 8192, &mapB, &full[st], n0 + 64 * j, k0, z);
            }
          }
        }
      }
      // Drain: every copy issued above completes on its stage's full barrier.
      const uint32_t issued = it;
      const uint32_t first = issued > (uint32_t)C::STAGES ? issued - C::STAGES : 0;
      for (uint32_t j = first; j < issued; ++j)
        mbar_wait(&full[j % C::STAGES], (j / C::STAGES) & 1u, nullptr, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ----------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(BN, p.a_mn, p.b_mn);
      // Descriptors: a fixed high part (layout, strides) | the slot address in
      // 16-byte units; each k-step / accumulator slot adds a constant to the
      // address field (no carry: shared addresses stay below 256 KiB).
      const uint64_t a_hi = smem_desc_sw128(0, p.a_mn ? 8192 : 16, 1024);
      const uint64_t b_hi = smem_desc_sw128(0, p.b_mn ? 8192 : 16, 1024);
      const uint32_t a_ks = p.a_mn ? 2048 >> 4 : 32 >> 4;   // one k-step of 16
      const uint32_t b_ks = p.b_mn ? 2048 >> 4 : 32 >> 4;
      const bool db = NACC == 2 && p.dualb;
      const uint32_t a_slot = db ? 0u : (uint32_t)(C::A_BYTES >> 4);   // accumulator a's A slot step
      const uint32_t b_slot = db ? (uint32_t)(C::B_BYTES >> 4) : 0u;   // accumulator a's B slot step
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++tcount) {
        const uint32_t buf = tcount & 1u;
        const uint32_t aph = (tcount >> 1) & 1u;
        if (!mbar_wait(&tempty[buf], aph ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem_base + buf * (NACC * BN);
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const int st = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(&full[st], ph, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * C::STAGE_BYTES);
          const uint32_t sb = sa + (db ? C::A_BYTES : NACC * C::A_BYTES);
          const uint64_t ad = a_hi | (uint64_t)((sa >> 4) & 0x3FFFu);
          const uint64_t bd = b_hi | (uint64_t)((sb >> 4) & 0x3FFFu);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // K-major: advance 16 elements = 32 bytes inside the swizzled row.
            // MN-major: advance 16 K-rows = two 8-row groups of 1024 bytes.
#pragma unroll
            for (int a = 0; a < NACC; ++a)
              mma_bf16(d0 + a * BN, ad + (kk * a_ks + a * a_slot), bd + (kk * b_ks + a * b_slot), idesc,
                       (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[st]);   // frees the stage once these MMAs have read it
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);    // accumulator ready for the epilogue
      }
      // Drain: wait for every MMA this thread issued.
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.status);
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int part = (warp - 2) >> 2;       // which column part of the tile
    constexpr int PART_COLS = BN / C::PARTS;
    const int row_in_tile = q * 32 + lane;
    if constexpr (Epi::kWarpRows) {
      float* sv = rowstage + (warp - 2) * 1024;
      warp_rows_loop<NACC, BN, PART_COLS>(epi, p, blockIdx.x, gridDim.x, BM, 0, tmem_base, tfull, sv, q, part,
                                          lane, abort_flag,
                                          [&](uint32_t b) { mbar_arrive(&tempty[b]); });
    } else {
      uint32_t tcount = 0;
      for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++tcount) {
        int tm, tn, z;
        decode_tile<NACC>(p, t, tm, tn, z);
        const uint32_t buf = tcount & 1u;
        const uint32_t aph = (tcount >> 1) & 1u;
        // Warp-uniform decision: tcgen05.ld below is .sync.aligned.
        const bool ready = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], aph, abort_flag, p.status));
        if (!ready) break;
        tc_fence_after();
        const int r = tm * BM + row_in_tile;
        const bool row_ok = r < s.M;
        typename Epi::RowState rs;
        if (row_ok) epi.row_begin(rs, z, r);
        const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + buf * (NACC * BN);
#pragma unroll 1
        for (int c = part * PART_COLS; c < (part + 1) * PART_COLS; c += 32) {
          float v[32], v2[32];
          const int c0 = tn * BN + c;
          if constexpr (Epi::kPreload) {
            if (row_ok && c0 < s.N) epi.preload(rs, z, r, c0, min(32, s.N - c0));
          }
          tmem_ld32(tbase + c, v);
          if (NACC == 2) tmem_ld32(tbase + BN + c, v2);
          if (row_ok && c0 < s.N) epi.span(rs, z, r, c0, v, NACC == 2 ? v2 : v, min(32, s.N - c0));
        }
        if (row_ok) epi.row_end(rs, z, r, tn * C::PARTS + part);
        tc_fence_before();
        mbar_arrive(&tempty[buf]);
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// CTA-pair (2-SM) variant: tcgen05.mma.cta_group::2, M = 256 per pair.
//
// Each CTA of a cluster pair holds 128 rows of A and BN/2 columns of B per
// stage (no TMA multicast: each CTA loads its own halves); the leader CTA
// (rank 0) issues M=256 x N=BN MMAs that read both CTAs' shared memory and
// write each CTA's 128-row slice of the accumulator into that CTA's TMEM.
// Per SM this halves the B bytes per FLOP against the 1-SM kernel (a 256x256
// pair tile needs 64 B/clk of operand feed per SM instead of 96 B/clk).
// Barriers: both CTAs' TMA loads complete on the leader's "full" barrier
// (the leader arms it with both CTAs' bytes); the leader's tcgen05.commit
// multicasts "empty" and "accumulator full" to both CTAs; both epilogues
// release the leader's "accumulator empty" barrier (remote arrive).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load whose completion is signalled on a barrier that may live in the
// peer CTA of the pair (cluster address); no multicast.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at this shared offset in both CTAs of the pair once
// the leader's prior MMAs are complete.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar, uint16_t mask = 0x3) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}
__host__ __device__ constexpr uint32_t idesc_bf16_m256(int n, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

// DUALB (NACC = 2 only): the two accumulators share A and take two B
// operands; stage layout [A | B] where CTA 0's B slot holds the whole B1 tile
// and CTA 1's the whole B2 tile; otherwise [A1 | (A2) | B half].
template <int NACC, int BN, bool WARPROWS = false, bool DUALB = false>
struct Cfg2 {
  static constexpr int EW = epi_warps(NACC, WARPROWS);
  static constexpr int PARTS = EW / 4;
  static constexpr int NTHREADS = 64 + 32 * EW;
  static constexpr int A_BYTES = BM * BK * 2;            // this CTA's 128 rows
  static constexpr int B_BYTES = (BN / 2) * BK * 2;      // this CTA's BN/2 columns
  static constexpr int NA = DUALB ? 1 : NACC;            // A slots per stage
  static constexpr int NB = DUALB ? 2 : 1;               // B slots per stage
  static constexpr int STAGE_BYTES = NA * A_BYTES + NB * B_BYTES;
  static constexpr int ROWSTAGE_BYTES = WARPROWS ? EW * 32 * 32 * 4 : 0;
  static constexpr int STAGES = (232448 - 1280 - ROWSTAGE_BYTES) / STAGE_BYTES;
  static constexpr int TMEM_COLS = 2 * NACC * BN;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + ROWSTAGE_BYTES + 1024 + 256;
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of two");
  static_assert(BN % 128 == 0, "each CTA loads whole 64-column boxes of B");
  static_assert(!DUALB || NACC == 2, "dual B operands need two accumulators");
  static_assert(STAGES >= 2 && STAGES <= 16, "two to sixteen stages (the barriers take 256 bytes)");
  static_assert(SMEM_BYTES <= 232448, "shared memory above the 227 KiB per-CTA limit");
};

// mapA2: the second A operand, or with DUALB the second B operand.
template <int NACC, int BN, class Epi, bool DUALB = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg2<NACC, BN, Epi::kWarpRows, DUALB>::NTHREADS, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapA2,
                const __grid_constant__ CUtensorMap mapB, const TcParams p, const Epi epi) {
  using C = Cfg2<NACC, BN, Epi::kWarpRows, DUALB>;
  constexpr int HBN = BN / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* rowstage = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::ROWSTAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    tmap_prefetch(&mapA);
    tmap_prefetch(&mapA2);
    tmap_prefetch(&mapB);
    for (int i = 0; i < C::STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], 2 * 32 * C::EW); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Barriers and TMEM are set up: wait for the previous kernel of the stream
  // before the first global access, then let the next one be scheduled onto
  // SMs as they free up.
  grid_dependency_wait();
  grid_launch_dependents();
  const GemmShape& s = p.s;

  if (warp == 0) {
    // ------------------------------ producer (both CTAs) ------------------------------
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = pair; u < p.num_units && ok; u += npairs) {
        const Unit un = decode_unit(p, u);
        const int t = un.t;
        int tm, tn, z;
        decode_tile<NACC>(p, t, tm, tn, z);
        const int m0 = tm * 2 * BM + (int)rank * BM;     // this CTA's 128 rows
        const int n0 = tn * BN + (int)rank * HBN;        // this CTA's BN/2 columns
        for (int kb = un.kb0; kb < un.kb1; ++kb, ++it) {
          const int st = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
          uint8_t* sa = smem + st * C::STAGE_BYTES;
          uint8_t* sb = sa + C::NA * C::A_BYTES;
          if (leader) mbar_expect_tx(&full[st], 2 * C::STAGE_BYTES);
          const uint32_t fb = mapa_shared(smem_u32(&full[st]), 0);
          const int k0 = kb * BK;
          constexpr bool A2 = NACC == 2 && !DUALB;
          if (!p.a_mn) {
            tma_load_3d_pair(sa, &mapA, fb, k0, m0, z);
            if (A2) tma_load_3d_pair(sa + C::A_BYTES, &mapA2, fb, k0, m0, z);
          } else {
#pragma unroll
            for (int j = 0; j < BM / 64; ++j) {
              tma_load_3d_pair(sa + j * 8192, &mapA, fb, m0 + 64 * j, k0, z);
              if (A2) tma_load_3d_pair(sa + C::A_BYTES + j * 8192, &mapA2, fb, m0 + 64 * j, k0, z);
            }
          }
          if constexpr (DUALB) {
            // CTA 0 stages the whole B1 tile, CTA 1 the whole B2 tile: the
            // pair's N = 2 BN MMA then reads [B1 | B2] and fills both
            // accumulators (columns [0, BN) and [BN, 2 BN)) at once.
            const CUtensorMap* mb = rank == 0 ? &mapB : &mapA2;
            const int nb0 = tn * BN;
            if (!p.b_mn) {
              tma_load_3d_pair(sb, mb, fb, k0, nb0, z);
            } else {
#pragma unroll
              for (int j = 0; j < BN / 64; ++j) tma_load_3d_pair(sb + j * 8192, mb, fb, nb0 + 64 * j, k0, z);
            }
          } else if (!p.b_mn) {
            tma_load_3d_pair(sb, &mapB, fb, k0, n0, z);
          } else {
#pragma unroll
            for (int j = 0; j < HBN / 64; ++j) tma_load_3d_pair(sb + j * 8192, &mapB, fb, n0 + 64 * j, k0, z);
          }
        }
      }
      if (leader) {
        const uint32_t issued = it;
        const uint32_t first = issued > (uint32_t)C::STAGES ? issued - C::STAGES : 0;
        for (uint32_t j = first; j < issued; ++j)
          mbar_wait(&full[j % C::STAGES], (j / C::STAGES) & 1u, nullptr, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (leader) ------------------------------
    if (leader && lane == 0) {
      const uint32_t idesc = idesc_bf16_m256(DUALB ? 2 * BN : BN, p.a_mn, p.b_mn);
      // Descriptors as in the 1-SM kernel: fixed high part | slot address.
      const uint64_t a_hi = smem_desc_sw128(0, p.a_mn ? 8192 : 16, 1024);
      const uint64_t b_hi = smem_desc_sw128(0, p.b_mn ? 8192 : 16, 1024);
      const uint32_t a_ks = p.a_mn ? 2048 >> 4 : 32 >> 4;
      const uint32_t b_ks = p.b_mn ? 2048 >> 4 : 32 >> 4;
      constexpr uint32_t a_slot = (uint32_t)(C::A_BYTES >> 4);
      constexpr int NMMA = DUALB ? 1 : NACC;   // MMAs per k-step
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int u = pair; u < p.num_units && ok; u += npairs, ++tcount) {
        const Unit un = decode_unit(p, u);
        const int kb0 = un.kb0, kb1 = un.kb1;
        const uint32_t buf = tcount & 1u;
        const uint32_t aph = (tcount >> 1) & 1u;
        if (!mbar_wait(&tempty[buf], aph ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem_base + buf * (NACC * BN);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int st = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(&full[st], ph, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * C::STAGE_BYTES);
          const uint32_t sb = sa + C::NA * C::A_BYTES;
          const uint64_t ad = a_hi | (uint64_t)((sa >> 4) & 0x3FFFu);
          const uint64_t bd = b_hi | (uint64_t)((sb >> 4) & 0x3FFFu);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
#pragma unroll
            for (int a = 0; a < NMMA; ++a)
              mma_bf16_pair(d0 + a * BN, ad + (kk * a_ks + a * a_slot), bd + kk * b_ks, idesc,
                            (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[st]);
        }
        if (!ok) break;
        mma_commit_pair(&tfull[buf]);
      }
      mma_commit_pair(drain, 0x1);   // the leader's own barrier only
      mbar_wait(drain, 0, nullptr, p.status);
    }
  } else {
    // ------------------------------ epilogue (both CTAs) ------------------------------
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;
    constexpr int PART_COLS = BN / C::PARTS;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    float* sv = rowstage + (warp - 2) * 1024;   // row-walk staging (row-walking epilogues only)
    uint32_t tcount = 0;
    if constexpr (Epi::kWarpRows && NACC == 2) {   // the aggregation: never split
      warp_rows_loop<NACC, BN, PART_COLS>(epi, p, pair, npairs, 2 * BM, (int)rank * BM, tmem_base, tfull, sv, q,
                                          part, lane, abort_flag, [&](uint32_t b) {
                                            mbar_arrive_remote(b ? tempty_leader1 : tempty_leader0);
                                          });
    } else
    for (int u = pair; u < p.num_units; u += npairs, ++tcount) {
      const Unit un = decode_unit(p, u);
      const int t = un.t, ks = un.ks;
      int tm, tn, z;
      decode_tile<NACC>(p, t, tm, tn, z);
      const uint32_t buf = tcount & 1u;
      const uint32_t aph = (tcount >> 1) & 1u;
      const bool ready = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], aph, abort_flag, p.status));
      if (!ready) break;
      tc_fence_after();
      const int row0 = tm * 2 * BM + (int)rank * BM + q * 32;   // this warp's 32 rows
      const int nrows = min(32, s.M - row0);
      const int r = row0 + lane;                                 // this thread's row
      const bool row_ok = r < s.M;
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + buf * (NACC * BN);
      // The finished fp32 values of one 32-column span of this thread's row
      // go to the epilogue functor: staged and walked by rows, or per row.
      auto emit_span = [&](typename Epi::RowState& rs, int c0, const float* v) {
        if constexpr (Epi::kWarpRows) {
          stage_row32(sv, v, lane);
          __syncwarp();
          finish_rows(epi, z, row0, c0, min(32, s.N - c0), nrows, sv, lane);
          __syncwarp();
        } else {
          if constexpr (Epi::kPreload) {
            if (row_ok && c0 < s.N) epi.preload(rs, z, r, c0, min(32, s.N - c0));
          }
          if (row_ok && c0 < s.N) epi.span(rs, z, r, c0, v, v, min(32, s.N - c0));
        }
      };
      if (!un.split) {
        if constexpr (Epi::kWarpRows) {
          rows_tile<NACC, BN, PART_COLS>(epi, s, z, row0, tn, tbase, sv, part, lane, [&]() {
            mbar_arrive_remote(buf ? tempty_leader1 : tempty_leader0);
          });
        } else {
          typename Epi::RowState rs;
          if (row_ok) epi.row_begin(rs, z, r);
#pragma unroll 1
          for (int c = part * PART_COLS; c < (part + 1) * PART_COLS; c += 32) {
            float v[32], v2[32];
            const int c0 = tn * BN + c;
            if constexpr (Epi::kPreload) {
              if (row_ok && c0 < s.N) epi.preload(rs, z, r, c0, min(32, s.N - c0));
            }
            tmem_ld32(tbase + c, v);
            if (NACC == 2) tmem_ld32(tbase + BN + c, v2);
            if (row_ok && c0 < s.N) epi.span(rs, z, r, c0, v, NACC == 2 ? v2 : v, min(32, s.N - c0));
          }
          if (row_ok) epi.row_end(rs, z, r, tn * EPI_PARTS + part);
          tc_fence_before();
          mbar_arrive_remote(buf ? tempty_leader1 : tempty_leader0);
        }
      } else if (p.pair_finish) {
        // Two splits resident at once: each finishes half of the tile's rows.
        // The warp whose rows the partner finishes parks its fp32 partial and
        // raises a flag; the finishing warp waits for the flag (bounded), adds
        // its own accumulator and the partial (two terms: the same sum as
        // partial 0 + partial 1) and runs the epilogue on its 32 rows.
        const bool finisher = (ks == 0) == (q < 2);
        const size_t slab = (size_t)BM * BN;
        const int ew = warp - 2;
        float4* region = reinterpret_cast<float4*>(p.partial + ((size_t)(t - p.full_tiles) * 2 + rank) * slab) +
                         (size_t)ew * (PART_COLS / 4) * 32 + lane;
        int* flag = p.counters + ((size_t)t * 2 + rank) * EPI_WARPS + ew;
        if (!finisher) {
#pragma unroll 1
          for (int c = part * PART_COLS, sp = 0; c < (part + 1) * PART_COLS; c += 32, ++sp) {
            float v[32];
            tmem_ld32(tbase + c, v);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              region[(sp * 8 + i) * 32] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
          tc_fence_before();
          mbar_arrive_remote(buf ? tempty_leader1 : tempty_leader0);
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicExch(flag, 1);
        } else {
          int ok = 1;
          if (lane == 0) {
            const uint64_t t0 = global_ns();
            while (*reinterpret_cast<volatile int*>(flag) == 0) {
              if (global_ns() - t0 > WAIT_NS || *abort_flag) {
                record_error(p.status, TTT_ERR_TIMEOUT);
                *abort_flag = 1;
                ok = 0;
                break;
              }
              __nanosleep(100);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          __threadfence();
          if (ok) {
            typename Epi::RowState rs;
            if (!Epi::kWarpRows && row_ok) epi.row_begin(rs, z, r);
#pragma unroll 1
            for (int c = part * PART_COLS, sp = 0; c < (part + 1) * PART_COLS; c += 32, ++sp) {
              float v[32];
              tmem_ld32(tbase + c, v);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 x = __ldcg(region + (sp * 8 + i) * 32);
                v[4 * i] += x.x; v[4 * i + 1] += x.y; v[4 * i + 2] += x.z; v[4 * i + 3] += x.w;
              }
              emit_span(rs, tn * BN + c, v);
            }
            if (!Epi::kWarpRows && row_ok) epi.row_end(rs, z, r, tn * EPI_PARTS + part);
          }
          tc_fence_before();
          mbar_arrive_remote(buf ? tempty_leader1 : tempty_leader0);
          __syncwarp();
          if (lane == 0) *flag = 0;
        }
      } else {
        // Split-K: park this split's fp32 partial, free the accumulator, and
        // let the last split to arrive sum all partials in split order.
        // Partial layout is warp-major: [unit][cta][epi warp][span][8 float4][lane],
        // so each warp store / load instruction covers 512 contiguous bytes.
        const size_t slab = (size_t)BM * BN;                 // one CTA's partial tile
        const int ew = warp - 2;
        float4* mine = reinterpret_cast<float4*>(p.partial + ((size_t)(t * p.splits + ks) * 2 + rank) * slab) +
                       (size_t)ew * (PART_COLS / 4) * 32 + lane;
#pragma unroll 1
        for (int c = part * PART_COLS, sp = 0; c < (part + 1) * PART_COLS; c += 32, ++sp) {
          float v[32];
          tmem_ld32(tbase + c, v);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            mine[(sp * 8 + i) * 32] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
        tc_fence_before();
        mbar_arrive_remote(buf ? tempty_leader1 : tempty_leader0);
        // One arrival counter per epilogue-warp region (32 rows x PART_COLS):
        // no barrier across warps, so an aborting warp cannot strand others.
        int* ctr = p.counters + ((size_t)t * 2 + rank) * EPI_WARPS + (warp - 2);
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(ctr, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == p.splits - 1) {
          __threadfence();
          typename Epi::RowState rs;
          if (!Epi::kWarpRows && row_ok) epi.row_begin(rs, z, r);
          const float4* base = reinterpret_cast<const float4*>(p.partial + ((size_t)t * p.splits * 2 + rank) * slab) +
                               (size_t)ew * (PART_COLS / 4) * 32 + lane;
#pragma unroll 1
          for (int c = part * PART_COLS, sp = 0; c < (part + 1) * PART_COLS; c += 32, ++sp) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
            for (int k2 = 0; k2 < p.splits; ++k2) {
              const float4* src = base + (size_t)k2 * 2 * (slab / 4) + sp * 8 * 32;
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 x = __ldcg(src + i * 32);
                v[4 * i] += x.x; v[4 * i + 1] += x.y; v[4 * i + 2] += x.z; v[4 * i + 3] += x.w;
              }
            }
            emit_span(rs, tn * BN + c, v);
          }
          if (!Epi::kWarpRows && row_ok) epi.row_end(rs, z, r, tn * EPI_PARTS + part);
          __syncwarp();
          if (lane == 0) *ctr = 0;
        }
      }
    }
  }

  // On an abort, give copies issued by either CTA time to land before the
  // pair synchronises and releases its shared memory and TMEM.
  if (*abort_flag) {
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < 200000ull) {}
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps (via the driver entry point, no libcuda link) and launch
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

inline int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// 3-D map of a bf16 operand: dims (inner, outer, batch).  K-major: inner = K,
// outer = MN rows; MN-major: inner = MN, outer = K rows.  Box: 64 inner
// elements (128 bytes, 128-byte swizzle) by box_outer rows.
inline cudaError_t make_map(CUtensorMap* m, const Operand& op, int64_t inner, int64_t outer, int batch,
                            int box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)outer, (cuuint64_t)(batch > 0 ? batch : 1)};
  cuuint64_t bs = op.batch_stride > 0 ? (cuuint64_t)op.batch_stride * 2 : (cuuint64_t)op.ld * 2 * outer;
  if (bs % 16) bs = (bs + 15) / 16 * 16;
  cuuint64_t strides[2] = {(cuuint64_t)op.ld * 2, bs};
  cuuint32_t box[3] = {64u, (cuuint32_t)box_outer, 1u};
  cuuint32_t es[3] = {1u, 1u, 1u};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(op.ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Operand of the A side (rows = M) or B side (rows = N).  For a batched GEMM
// whose batch_stride is 0 the map has one batch entry and z is clamped.
inline cudaError_t make_operand_map(CUtensorMap* m, const Operand& op, int mn_extent, int k_extent, int batch,
                                    int box_mn) {
  const int nb = op.batch_stride > 0 ? batch : 1;
  if (op.kmajor) return make_map(m, op, k_extent, op.rows_per_batch, nb, box_mn);
  return make_map(m, op, mn_extent, op.rows_per_batch, nb, 64);
}

template <int NACC, int BN, class Epi>
cudaError_t launch_tc(const GemmShape& s, const Operand& A, const Operand& A2, const Operand& B, const Epi& epi,
                      cudaStream_t st, int* status, int dualb = 0) {
  static_assert(NACC == 1 || BN == BM, "dual accumulators use equal A and B slots");
  using C = Cfg<NACC, BN, Epi::kWarpRows>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<NACC, BN, Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  // Shared operands (batch_stride 0) always use batch coordinate 0.
  if ((A.batch_stride == 0 || B.batch_stride == 0) && s.batch > 1) return cudaErrorInvalidValue;
  CUtensorMap ma, ma2, mb;
  cudaError_t e;
  // For K-major operands rows_per_batch is the MN extent in memory; for
  // MN-major ones it is the K extent (rows of the buffer per batch entry).
  e = make_operand_map(&ma, A, s.M, s.K, s.batch, BM);
  if (e != cudaSuccess) return e;
  if (NACC == 2) {
    // dual-B: the second operand is a B (N extent, B major-ness)
    e = dualb ? make_operand_map(&ma2, A2, s.N, s.K, s.batch, BN) : make_operand_map(&ma2, A2, s.M, s.K, s.batch, BM);
    if (e != cudaSuccess) return e;
    if (dualb && A2.kmajor != B.kmajor) return cudaErrorInvalidValue;
  } else {
    ma2 = ma;
  }
  e = make_operand_map(&mb, B, s.N, s.K, s.batch, BN);
  if (e != cudaSuccess) return e;
  TcParams p;
  p.s = s;
  p.dualb = dualb;
  p.a_mn = A.kmajor ? 0 : 1;
  p.b_mn = B.kmajor ? 0 : 1;
  p.tiles_m = (s.M + BM - 1) / BM;
  p.tiles_n = (s.N + BN - 1) / BN;
  p.num_tiles = p.tiles_m * p.tiles_n * s.batch;
  p.num_kb = (s.K + BK - 1) / BK;
  p.status = status;
  p.splits = 1;
  p.kb_per_split = p.num_kb;
  p.pair_finish = 0;
  p.full_tiles = p.num_tiles;
  p.num_units = p.num_tiles;
  p.partial = nullptr;
  p.counters = nullptr;
  const int grid = p.num_tiles < num_sms() ? p.num_tiles : num_sms();
  return launch_dependent(gemm_tc_kernel<NACC, BN, Epi>, grid, C::NTHREADS, C::SMEM_BYTES, st, ma, ma2, mb, p, epi);
}

// Fraction of the machine a GEMM keeps busy with N tile `bn`: tiles over
// (waves x SMs), discounted for N=128 tiles, which need 4/3 more operand
// bytes per FLOP than N=256 (128x128: 128 B/clk of TMA feed at full MMA rate,
// 128x256: 96 B/clk); the 0.78 factor is the measured ratio on B200.
inline double tile_efficiency(const GemmShape& s, int bn) {
  const int sms = num_sms();
  const long tiles = (long)((s.M + BM - 1) / BM) * ((s.N + bn - 1) / bn) * s.batch;
  const long waves = (tiles + sms - 1) / sms;
  return (double)tiles / (double)(waves * sms) * (bn == 128 ? 0.78 : 1.0);
}

// 1: pair-kernel GEMMs may finish the tiles of their last wave as paired halves (env TTT_GEMM_PAIRFINISH=0
// keeps the last-arriver reduction, for A/B timing).
inline int pair_finish_mode() {
  static int m = -1;
  if (m < 0) {
    const char* e = getenv("TTT_GEMM_PAIRFINISH");
    m = (e && e[0] == '0') ? 0 : 1;
  }
  return m;
}

// Paired-finish schedule of a pair-kernel GEMM: the whole waves of tiles run
// whole, the tiles of the last partial wave as two halves of the k-blocks
// (2 x remainder <= pairs, so all halves are resident together and each pair
// runs at most one).  Cost in k-blocks of one pair: whole waves x num_kb +
// half a tile + PF_FIXUP_KB for parking and adding half a partial.  Returns
// the number of whole tiles, or -1 when the plain whole-tile schedule is cheaper
// or the scratch is missing.
constexpr int PF_FIXUP_KB = 4;
inline long paired_finish_plan(long tiles, int num_kb, const SplitScratch& ss, double* cost = nullptr) {
  const int pairs = num_sms() / 2;
  const long full = tiles / pairs * pairs;
  const long rem = tiles - full;
  const double whole = (double)((tiles + pairs - 1) / pairs) * num_kb;
  if (cost) *cost = whole;
  if (!pair_finish_mode() || rem == 0 || 2 * rem > pairs || num_kb < 2) return -1;
  if (!ss.partial || !ss.counters) return -1;
  if ((size_t)rem * 2 * BM * 256 * sizeof(float) > ss.partial_bytes) return -1;
  if ((size_t)tiles * 2 * EPI_WARPS > ss.counter_count) return -1;
  const double pf = (double)(full / pairs) * num_kb + (num_kb + 1) / 2 + PF_FIXUP_KB;
  if (pf >= whole) return -1;
  if (cost) *cost = pf;
  return full;
}

// Split count for a pair-kernel GEMM: minimise waves x (k-blocks per split +
// a fixed cost for parking and reducing a partial), with no empty split and
// within the partial-tile scratch.
inline int choose_splits(long tiles, int num_kb, const SplitScratch& ss, double* cost_out = nullptr) {
  static int forced = -1;
  if (forced < 0) {
    const char* e = getenv("TTT_GEMM_SPLITS");   // tuning knob: force a split count
    forced = e ? atoi(e) : 0;
  }
  if (forced > 0) {
    const int kbps = (num_kb + forced - 1) / forced;
    const int s_eff = (num_kb + kbps - 1) / kbps;
    const bool fits = forced == 1 || (ss.partial && ss.counters &&
                                      (size_t)tiles * s_eff * 2 * BM * 256 * sizeof(float) <= ss.partial_bytes &&
                                      (size_t)tiles * 2 * EPI_WARPS <= ss.counter_count);
    return fits ? s_eff : 1;
  }
  const int pairs = num_sms() / 2;
  // Measured on B200: splitting pays only when unsplit tiles leave most pairs
  // idle; with 1-2 waves of tiles the partial round trip costs more than the
  // quantisation it removes.
  if (tiles >= (long)(0.6 * pairs)) {
    if (cost_out) *cost_out = (double)((tiles + pairs - 1) / pairs) * num_kb;
    return 1;
  }
  int best = 1;
  double best_cost = 1e30;
  for (int S = 1; S <= 8 && S <= num_kb; ++S) {
    const int kbps = (num_kb + S - 1) / S;
    const int s_eff = (num_kb + kbps - 1) / kbps;
    if (s_eff != S) continue;
    if (S > 1) {
      if (!ss.partial || !ss.counters) break;
      if ((size_t)tiles * S * 2 * BM * 256 * sizeof(float) > ss.partial_bytes) break;
      if ((size_t)tiles * 2 * EPI_WARPS > ss.counter_count) break;
    }
    const long units = tiles * S;
    const long waves = (units + pairs - 1) / pairs;
    const double cost = (double)waves * (kbps + (S > 1 ? 4 : 0));
    if (cost < best_cost - 1e-9) { best_cost = cost; best = S; }
  }
  if (cost_out) *cost_out = best_cost;
  return best;
}

// DUALB: A2 is the second B operand (same layout as B).
template <int NACC, int BN, class Epi, bool DUALB = false>
cudaError_t launch_tc2(const GemmShape& s, const Operand& A, const Operand& A2, const Operand& B, const Epi& epi,
                       cudaStream_t st, int* status, const SplitScratch& ss = SplitScratch()) {
  using C = Cfg2<NACC, BN, Epi::kWarpRows, DUALB>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc2_kernel<NACC, BN, Epi, DUALB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if ((A.batch_stride == 0 || B.batch_stride == 0) && s.batch > 1) return cudaErrorInvalidValue;
  CUtensorMap ma, ma2, mb;
  cudaError_t e = make_operand_map(&ma, A, s.M, s.K, s.batch, BM);
  if (e != cudaSuccess) return e;
  if (NACC == 2) {
    if (DUALB && A2.kmajor != B.kmajor) return cudaErrorInvalidValue;
    e = DUALB ? make_operand_map(&ma2, A2, s.N, s.K, s.batch, BN) : make_operand_map(&ma2, A2, s.M, s.K, s.batch, BM);
    if (e != cudaSuccess) return e;
  } else {
    ma2 = ma;
  }
  e = make_operand_map(&mb, B, s.N, s.K, s.batch, DUALB ? BN : BN / 2);
  if (e != cudaSuccess) return e;
  TcParams p;
  p.s = s;
  p.dualb = DUALB ? 1 : 0;
  p.a_mn = A.kmajor ? 0 : 1;
  p.b_mn = B.kmajor ? 0 : 1;
  p.tiles_m = (s.M + 2 * BM - 1) / (2 * BM);
  p.tiles_n = (s.N + BN - 1) / BN;
  p.num_tiles = p.tiles_m * p.tiles_n * s.batch;
  p.num_kb = (s.K + BK - 1) / BK;
  p.status = status;
  const bool may_split = NACC == 1 && BN == 256;
  double pf_cost = 0.0, split_cost = 1e30;
  long full = may_split ? paired_finish_plan(p.num_tiles, p.num_kb, ss, &pf_cost) : -1;
  const int split_S = may_split ? choose_splits(p.num_tiles, p.num_kb, ss, &split_cost) : 1;
  if (full >= 0 && split_S > 1 && split_cost < pf_cost) full = -1;   // few tiles, long K: plain split-K
  if (full >= 0) {   // whole waves, then the last wave's tiles as paired halves
    p.pair_finish = 1;
    p.full_tiles = (int)full;
    p.splits = 2;
    p.kb_per_split = (p.num_kb + 1) / 2;
    p.num_units = (int)full + 2 * (p.num_tiles - (int)full);
  } else {
    p.pair_finish = 0;
    p.full_tiles = p.num_tiles;
    p.splits = split_S;
    p.kb_per_split = (p.num_kb + p.splits - 1) / p.splits;
    p.num_units = p.num_tiles * p.splits;
  }
  p.partial = ss.partial;
  p.counters = ss.counters;
  const int pairs = num_sms() / 2;
  const int units = p.num_units;
  const int grid = 2 * (units < pairs ? units : pairs);
  return launch_dependent(gemm_tc2_kernel<NACC, BN, Epi, DUALB>, grid, C::NTHREADS, C::SMEM_BYTES, st, ma, ma2, mb, p,
                          epi);
}

// 0: 1-SM kernel, 1: CTA-pair kernel (env TTT_GEMM_PAIR=0 forces 1-SM, for A/B timing).
inline int pair_mode() {
  static int m = -1;
  if (m < 0) {
    const char* e = getenv("TTT_GEMM_PAIR");
    m = (e && e[0] == '0') ? 0 : 1;
  }
  return m;
}

// Pair tiles (256 x 256): fraction of the pairs kept busy; the pair kernel
// needs 2/3 of the operand bytes per FLOP of the 1-SM 128x256 tile.
inline double tile_efficiency2(const GemmShape& s) {
  const int pairs = num_sms() / 2;
  const long tiles = (long)((s.M + 2 * BM - 1) / (2 * BM)) * ((s.N + 255) / 256) * s.batch;
  const long waves = (tiles + pairs - 1) / pairs;
  return (double)tiles / (double)(waves * pairs);
}

template <int NACC, class Epi>
cudaError_t launch_gemm_tc(const GemmShape& s, const Operand& A, const Operand& A2, const Operand& B,
                           const Epi& epi, cudaStream_t st, int* status, const SplitScratch& ss = SplitScratch()) {
  if (s.M <= 0 || s.N <= 0 || s.batch <= 0 || s.K <= 0) return cudaSuccess;
  if constexpr (NACC == 2) {
    // Pair tiles (M = 256) halve the B bytes per FLOP; both shapes quantise alike.
    if (pair_mode() && s.M > BM) return launch_tc2<2, 128, Epi>(s, A, A2, B, epi, st, status);
    return launch_tc<2, 128, Epi>(s, A, A2, B, epi, st, status);
  } else {
    // Expected throughput = fraction of the machine busy x relative rate of
    // the tile shape under the operand-feed limit (pair 256x256: 1.3,
    // 1-SM 128x256: 1.0, 1-SM 128x128: 0.78, already in tile_efficiency).
    // The pair kernel may split K, which lifts its occupancy.
    // A few row tiles and a long K (the cross-entropy dz of a short chunk:
    // M = b rows, K = the vocabulary): one SM per tile would walk the whole K
    // alone, so the pair kernel runs it split over K across many pairs
    // (its 256-row tile reads zeros past row M and stores only rows < M).
    if (pair_mode() && s.M <= BM && ss.partial && ss.counters) {
      const long ptiles = (long)((s.N + 255) / 256) * s.batch;
      const int num_kb = (s.K + BK - 1) / BK;
      // measured on B200: pays from K = 8192 (128 k-blocks: 49.6 -> 31 us for
      // the dz of a 64-row chunk), loses at K = 2048 (20.9 -> 29.4 us)
      if (ptiles * 4 <= num_sms() / 2 && num_kb >= 64) return launch_tc2<1, 256, Epi>(s, A, A2, B, epi, st, status, ss);
    }
    double s_pair = 0.0;
    if (pair_mode() && s.M > BM) {
      const long tiles = (long)((s.M + 2 * BM - 1) / (2 * BM)) * ((s.N + 255) / 256) * s.batch;
      const int num_kb = (s.K + BK - 1) / BK;
      const int pairs = num_sms() / 2;
      double cost = 0.0;
      if (paired_finish_plan(tiles, num_kb, ss, &cost) >= 0) {
        // useful k-blocks over issued k-block slots of the paired-finish schedule
        s_pair = 1.3 * (double)tiles * num_kb / ((double)pairs * cost);
      } else {
        const int S = choose_splits(tiles, num_kb, ss);
        const long units = tiles * S;
        const long waves = (units + pairs - 1) / pairs;
        const int kbps = (num_kb + S - 1) / S;
        // useful k-blocks over issued k-block slots (with the split overhead)
        s_pair = 1.3 * (double)tiles * num_kb / ((double)waves * pairs * (kbps + (S > 1 ? 4 : 0)));
      }
    }
    const double s256 = tile_efficiency(s, 256);
    const double s128 = Epi::kFixedHeadTile ? 0.0 : tile_efficiency(s, 128);
    if (s_pair >= s256 && s_pair >= s128) return launch_tc2<1, 256, Epi>(s, A, A2, B, epi, st, status, ss);
    if constexpr (!Epi::kFixedHeadTile) {
      if (s128 > s256) return launch_tc<1, 128, Epi>(s, A, A2, B, epi, st, status);
    }
    return launch_tc<1, HEAD_BN, Epi>(s, A, A2, B, epi, st, status);
  }
}

// Dual accumulators sharing A: acc_0 = A B1^T, acc_1 = A B2^T (B1, B2 same layout).
template <class Epi>
cudaError_t launch_gemm_tc_dualb(const GemmShape& s, const Operand& A, const Operand& B1, const Operand& B2,
                                 const Epi& epi, cudaStream_t st, int* status) {
  if (s.M <= 0 || s.N <= 0 || s.batch <= 0 || s.K <= 0) return cudaSuccess;
  if (pair_mode() && s.M > BM) return launch_tc2<2, 128, Epi, true>(s, A, B2, B1, epi, st, status);
  return launch_tc<2, 128, Epi>(s, A, B2, B1, epi, st, status, 1);
}

}  // namespace tc
}  // namespace ttt
