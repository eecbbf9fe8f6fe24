// libttt: C ABI, argument validation, workspace plan and the chunk-serial
// driver of the TTT inner loop ("Rethinking Expressivity and Efficiency in
// Test-Time Training", Algorithm 1, applied chunk after chunk as the
// "TTT-E2E：端到端测试时训练的长上下文语言建模" inner loop describes).
//
// One prefill call = K1 scan over all chunks, the operand shadow of W, then
// per chunk (strictly serial: chunk r's gradients need chunk r-1's state):
//   gather -> [static F1, F2] / dynamic F1, F2 per block -> RMSNorm ->
//   CE pass A (logit tiles -> online-softmax partials) -> CE reduce ->
//   per vocabulary slab: CE pass B (softmax - onehot) and dz += P E_slab ->
//   RMSNorm backward -> per MLP, top down: B1 (dA, dU), B2 (dX) when a
//   dynamic MLP lies below, and for dynamic MLPs the dual-accumulator
//   aggregation whose epilogue writes W, M and the operand shadow in place
//   (on a second stream, beside the backward of the MLPs below).
// The final prediction (ttt_predict) runs the same forward and CE pass A at
// fixed weights, with no backward.  The whole sequence of launches of a call
// is captured once into a CUDA graph on a private stream and replayed on the
// caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <iterator>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "epilogue.cuh"
#include "attention.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "rows.cuh"
#include "scan.cuh"

namespace ttt {

static thread_local std::string g_last_error;

void set_last_error(const char* what, const char* why, const char* file, int line) {
  char buf[512];
  snprintf(buf, sizeof(buf), "%s failed: %s (%s:%d)", what, why, file, line);
  g_last_error = buf;
}
void set_last_error_msg(const char* msg) { g_last_error = msg; }

static ttt_status fail(ttt_status s, const char* msg) {
  g_last_error = msg;
  return s;
}

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------------------
// Handle
// ---------------------------------------------------------------------------
// Pointers and sizes a captured graph was built for: a graph is replayed only
// for exactly the call it was captured from.
struct CallKey {
  int batch = 0, T = 0, b = 0;
  const void* ptr[16] = {};
  size_t ws_bytes = 0;
  bool operator==(const CallKey& o) const {
    if (batch != o.batch || T != o.T || b != o.b || ws_bytes != o.ws_bytes) return false;
    for (int i = 0; i < 16; ++i)
      if (ptr[i] != o.ptr[i]) return false;
    return true;
  }
};

// One cached graph per kind of call.
struct GraphSlot {
  cudaGraphExec_t exec = nullptr;
  CallKey key;
  bool have = false;
};
// SLOT_HOST0/1: the host-buffer prefill's segments in input slot 0 / 1;
// SLOT_HOST_LAST: its last segment when that one is shorter.
enum { SLOT_PREFILL, SLOT_RECON, SLOT_PREDICT, SLOT_HOST0, SLOT_HOST1, SLOT_HOST_LAST, N_SLOTS };

}  // namespace ttt

struct ttt_handle {
  ttt_config cfg;
  int device = 0;
  void* E = nullptr;        // [V, d] operand copy
  float* gain = nullptr;    // [d]
  void* S = nullptr;        // static shadow [n_blocks][m*h*d] or nullptr
  int* status = nullptr;    // device status word
  int* zero_flag = nullptr; // a device int that stays 0 (bounded-wait self-test)
  cudaStream_t cap = nullptr;
  // host-buffer prefill: copy stream and the two input slots' events
  cudaStream_t copy = nullptr;
  cudaEvent_t ev_copied[2] = {nullptr, nullptr};
  cudaEvent_t ev_consumed[2] = {nullptr, nullptr};
  // the plain prefill's aggregation stream: each dynamic MLP's two
  // aggregations run on it beside the next MLPs' backward GEMMs
  cudaStream_t agg = nullptr;
  bool agg_stream = true;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  cudaEvent_t ev_up[3] = {nullptr, nullptr, nullptr};    // dU buffer k read by its aggregation
  cudaEvent_t ev_out[3] = {nullptr, nullptr, nullptr};   // doutW/doutM buffer k read by its aggregation
  ttt::GraphSlot graph[ttt::N_SLOTS];
  bool use_graph = true;
  // Frozen sliding-window attention in front of every updated block
  // (ttt_set_attention); attn_heads == 0: none.
  int attn_heads = 0;
  int attn_window = 0;
  float attn_ln_eps = 1e-5f;
  void* Wqkv = nullptr;       // [n_blocks][3d][d] operand copy (rows q | k | v)
  void* Wo = nullptr;         // [n_blocks][d][d] operand copy
  float* ln_gain = nullptr;   // [n_blocks][d]
  float* ln_bias = nullptr;   // [n_blocks][d]
};

namespace ttt {

// ---------------------------------------------------------------------------
// Workspace plan
// ---------------------------------------------------------------------------
struct Plan {
  int B, T, b, nchunks, n, d, h, H2, V, L, m, nM, Vs, nslabs, ntn;
  float kscale;  // 1/b for the mean reduction, 1 for the sum
  bool swiglu, has_static;
  size_t esz;  // operand element size
  size_t KW, KM, consts, Wsh, resid, actin, aw, am, act, fac, z, rstd, part, tgt, lse, ltok, P, dz, dout, dout_a,
      doutW[3], doutM[3], dU, dUx[2], sk_partial, sk_counters, total;
  bool recon;           // reconstruction head: no LM-head buffers; yk, yq, qres below
  size_t yk, yq, qres;  // fp32 [n, d]: MLP outputs on the keys and queries, the query rows
  size_t sk_partial_bytes, sk_counter_count;
  // frozen sliding-window attention (attn_heads > 0)
  int H, dh, window, ldS;
  int ntnS;   // score partials per (head, query) row
  size_t rope_tab, xhat, lnr, qkv, qh, kh, vh, spart, slse, sD, Pa, Of, Oc, dOh, dSa, dq, dk, dv, dqkv, da, sdout[2],
      sdoutT[2][2], sdU[2];
};

static inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Online-softmax partials per row: one per N tile (fp32 engine) or per column
// part of an N tile (tcgen05 engine).
static int head_parts(int precision, int V) {
  if (precision == TTT_PREC_FP32) return (V + simt::BN - 1) / simt::BN;
  return (V + tc::HEAD_BN - 1) / tc::HEAD_BN * tc::EPI_PARTS;
}

static Plan make_plan(const ttt_handle* hd, int B, int T, int b) {
  const ttt_config& c = hd->cfg;
  Plan p{};
  p.B = B; p.T = T; p.b = b; p.nchunks = b > 0 ? T / b : 0; p.n = B * b;
  p.recon = c.head == TTT_HEAD_RECON;
  p.d = c.d; p.h = c.hidden; p.V = p.recon ? 0 : c.vocab; p.L = c.n_blocks;
  p.swiglu = c.mlp == TTT_MLP_SWIGLU; p.has_static = c.has_static != 0;
  p.m = p.swiglu ? 3 : 2; p.H2 = p.swiglu ? 2 * p.h : p.h;
  p.nM = p.L * (p.has_static ? 2 : 1);
  p.esz = c.precision == TTT_PREC_FP32 ? 4 : 2;
  p.kscale = (c.loss_reduction == TTT_REDUCE_MEAN && b > 0) ? 1.0f / (float)b : 1.0f;
  p.ntn = head_parts(c.precision, p.V);
  // vocabulary slab: CE pass B recomputes the logits of one slab of Vs
  // columns at a time and writes softmax - onehot for it as the operand of
  // dz += P_slab E_slab, so no [n, V] buffer exists.  A slab is at most 32 MiB
  // (it stays resident in L2 between the two GEMMs); the vocabulary is cut
  // into equal slabs of whole 256-column tiles.
  const size_t cap = 32ull << 20;
  int64_t vs = 0;
  if (p.n > 0 && p.V > 0) {
    const size_t full = (size_t)p.n * p.V * p.esz;
    const int64_t ns = (int64_t)((full + cap - 1) / cap);
    vs = ((p.V + ns - 1) / ns + 255) / 256 * 256;
    const int64_t vmax = std::max<int64_t>(256, (int64_t)(cap / ((size_t)p.n * p.esz)) / 256 * 256);
    if (vs > vmax) vs = vmax;
    if (vs >= p.V) vs = p.V;
  }
  p.Vs = (int)vs;
  p.nslabs = p.Vs > 0 ? (p.V + p.Vs - 1) / p.Vs : 0;

  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  const size_t n = p.n, d = p.d, h = p.h, H2 = p.H2, e = p.esz;
  p.KW = take(4ull * B * T);
  p.KM = take(4ull * B * T);
  p.consts = take(16ull * B * p.nchunks);
  p.Wsh = take(e * B * p.L * p.m * h * d);
  p.resid = take(4 * n * d);
  p.actin = take(e * p.nM * n * d);
  p.aw = take(e * p.nM * n * d);
  p.am = take(e * p.nM * n * d);
  p.act = take(e * (p.nM + (p.recon ? 1 : 0)) * n * h);   // reconstruction: key and query activations
  p.fac = take(e * p.nM * n * H2);
  p.z = take(e * n * d);
  p.rstd = take(4 * n);
  p.part = take(8 * n * p.ntn);
  p.tgt = take(4 * n);
  p.lse = take(4 * n);
  p.ltok = take(4 * n);
  p.P = take(e * n * p.Vs);
  p.dz = take(4 * n * d);
  p.dout = take(4 * n * d);
  p.dout_a = take(e * n * d);
  for (int i = 0; i < 3; ++i) { p.doutW[i] = take(e * n * d); p.doutM[i] = take(e * n * d); }
  p.dU = take(e * n * H2);
  for (int i = 0; i < 2; ++i) p.dUx[i] = take(e * n * H2);
  p.yk = take(p.recon ? 4 * n * d : 0);
  p.yq = take(p.recon ? 4 * n * d : 0);
  p.qres = take(p.recon ? 4 * n * d : 0);
  // split-K scratch of the CTA-pair GEMMs (bf16 path)
  p.sk_partial_bytes = c.precision == TTT_PREC_BF16 ? std::min<size_t>(64ull << 20, 64ull * 1024 * std::max<size_t>(n, 64)) : 0;
  p.sk_counter_count = p.sk_partial_bytes ? 65536 : 0;
  p.sk_partial = take(p.sk_partial_bytes);
  p.sk_counters = take(4 * p.sk_counter_count);
  // Attention: a query of chunk c sees keys from j0 = c*b - window + 1 rounded
  // down to a multiple of 8 (16-byte aligned operand rows) up to the chunk's
  // end, so at most b + window + 6 keys; the key/value history spans the
  // whole sequence.
  p.H = hd->attn_heads;
  if (p.H > 0) {
    p.window = hd->attn_window;
    p.dh = p.d / p.H;
    int64_t ks = std::min<int64_t>((int64_t)T, (int64_t)b + p.window + 6);
    p.ldS = (int)align_up((size_t)ks, 8);
    const size_t H = p.H, L = p.L, ldS = p.ldS;
    p.rope_tab = take(8ull * T * (p.dh / 2));
    p.xhat = take(4 * L * n * d);
    p.lnr = take(4 * L * n);
    p.qkv = take(4 * n * 3 * d);
    p.qh = take(e * L * n * d);
    p.kh = take(e * L * B * T * d);
    p.vh = take(e * L * B * T * d);
    p.ntnS = head_parts(c.precision, p.ldS);
    p.spart = take(8 * H * b * (size_t)p.ntnS);
    p.slse = take(4 * H * b);
    p.sD = take(4 * H * b);
    p.Pa = take(e * L * B * H * b * ldS);
    p.Of = take(4 * L * n * d);
    p.Oc = take(e * n * d);
    p.dOh = take(e * n * d);
    p.dSa = take(e * H * b * ldS);
    p.dq = take(4 * n * d);
    p.dk = take(4 * n * d);
    p.dv = take(4 * n * d);
    p.dqkv = take(e * n * 3 * d);
    p.da = take(4 * n * d);
    for (int i = 0; i < 2; ++i) {
      p.sdout[i] = take(4 * n * d);
      p.sdoutT[i][0] = take(e * n * d);
      p.sdoutT[i][1] = take(e * n * d);
      p.sdU[i] = take(e * n * H2);
    }
  }
  p.total = off;
  return p;
}

// ---------------------------------------------------------------------------
// GEMM dispatch by operand type: fp32 -> CUDA-core engine, bf16 -> tcgen05.
// ---------------------------------------------------------------------------
template <typename T, int NACC, class Epi>
static cudaError_t gemm(const GemmShape& s, const Operand& A, const Operand& A2, const Operand& B,
                        const Epi& epi, cudaStream_t st, int* status, const SplitScratch& ss = SplitScratch()) {
  if constexpr (std::is_same<T, float>::value) {
    (void)status;
    (void)ss;
    return launch_gemm_simt<T, NACC, Epi>(s, A, A2, B, epi, st);
  } else {
    return tc::launch_gemm_tc<NACC, Epi>(s, A, A2, B, epi, st, status, ss);
  }
}

// Dual accumulators sharing the A operand: acc_0 = A B1^T, acc_1 = A B2^T.
template <typename T, class Epi>
static cudaError_t gemm_dualb(const GemmShape& s, const Operand& A, const Operand& B1, const Operand& B2,
                              const Epi& epi, cudaStream_t st, int* status) {
  if constexpr (std::is_same<T, float>::value) {
    (void)status;
    return launch_gemm_simt<T, 2, Epi>(s, A, B2, B1, epi, st, 1);
  } else {
    return tc::launch_gemm_tc_dualb<Epi>(s, A, B1, B2, epi, st, status);
  }
}

static Operand opnd(const void* p, int64_t ld, int64_t bs, int kmajor, int64_t rows_per_batch) {
  Operand o;
  o.ptr = p; o.ld = ld; o.batch_stride = bs; o.kmajor = kmajor; o.rows_per_batch = rows_per_batch;
  return o;
}

// ---------------------------------------------------------------------------
// Launch recorder: counts launches always; with timing on (the profiled
// entry point, eager launches) brackets every launch with CUDA events and
// accumulates per-class time, executed MMA FLOPs and algorithmic bytes.
// ---------------------------------------------------------------------------
enum KernelClass {
  K_SCAN, K_SHADOW, K_GATHER, K_MLP_UP, K_MLP_DOWN, K_RMS_FWD, K_CE_LSE, K_CE_ROWS, K_CE_MEAN,
  K_CE_GRAD, K_CE_DZ, K_RMS_BWD, K_BWD_DA, K_BWD_DX, K_AGG_UPDATE, K_RECON_ROWS, K_ATTN_PROJ, K_ATTN_SCORE,
  K_ATTN_ROWS, K_NCLASS
};
static const char* kClassName[K_NCLASS] = {
    "scalar_scan", "w_shadow", "gather", "mlp_up", "mlp_down", "rmsnorm_fwd", "ce_logits_lse", "ce_rows",
    "ce_mean", "ce_logits_grad", "ce_dz", "rmsnorm_bwd", "mlp_bwd_dA", "mlp_bwd_dX", "agg_update", "recon_rows",
    "attn_proj", "attn_scores", "attn_rows"};

struct Prof {
  bool timing = false;
  int64_t launches = 0;
  struct Rec { int cls; cudaEvent_t a, b; double flops, bytes; };
  std::vector<Rec> recs;
  int cur = -1;
  void begin(int cls, cudaStream_t st) {
    ++launches;
    if (!timing) return;
    Rec r{cls, nullptr, nullptr, 0, 0};
    cudaEventCreate(&r.a);
    cudaEventCreate(&r.b);
    cudaEventRecord(r.a, st);
    recs.push_back(r);
  }
  void end(double flops, double bytes, cudaStream_t st) {
    if (!timing) return;
    Rec& r = recs.back();
    r.flops = flops;
    r.bytes = bytes;
    cudaEventRecord(r.b, st);
  }
  ~Prof() {
    for (auto& r : recs) { cudaEventDestroy(r.a); cudaEventDestroy(r.b); }
  }
};

// Launch helpers of the enqueue functions below: each has `err`, `prof` and
// `st` in scope.
#define TRY(x) do { err = (x); if (err != cudaSuccess) return err; } while (0)
#define LAUNCH(cls, flops, bytes, expr) do { prof.begin(cls, st); expr; TRY(cudaGetLastError()); prof.end(flops, bytes, st); } while (0)

// ---------------------------------------------------------------------------
// Forward of chunk c's rows at the operand shadow Wsh: gather, then per block
// [static MLP], dynamic MLP, each with its residual.  With `train` the
// launches also keep what the backward reads: the activation factors and the
// K-scaled copies of each dynamic MLP's input.
// ---------------------------------------------------------------------------
template <typename T>
static cudaError_t enqueue_forward(ttt_handle* hd, const Plan& p, const float* hidden, const T* Wsh, int c,
                                   bool train, const float* KW, const float* KM, char* ws,
                                   const SplitScratch& ss, cudaStream_t st, Prof& prof) {
  const int B = p.B, b = p.b, n = p.n, d = p.d, h = p.h, H2 = p.H2, L = p.L;
  float* resid = reinterpret_cast<float*>(ws + p.resid);
  T* actin = reinterpret_cast<T*>(ws + p.actin);
  T* aw = reinterpret_cast<T*>(ws + p.aw);
  T* am = reinterpret_cast<T*>(ws + p.am);
  T* act = reinterpret_cast<T*>(ws + p.act);
  T* fac = reinterpret_cast<T*>(ws + p.fac);
  const T* S = static_cast<const T*>(hd->S);
  int* status = hd->status;
  cudaError_t err;
  const double e = (double)p.esz;
  const TokenMap tm{b, p.T, c};
  const int64_t blk = (int64_t)p.m * h * d;          // params per block
  const int64_t seqW = (int64_t)L * blk;             // params per sequence
  const bool sw = p.swiglu;
  // Forward order: per block [static], dynamic.  Lowest MLP the backward reaches:
  const int per_blk = p.has_static ? 2 : 1;
  const int i_min = per_blk - 1;
  auto is_dyn = [&](int i) { return (i % per_blk) == per_blk - 1; };
  auto blk_of = [&](int i) { return i / per_blk; };
  {
    const bool first_dyn = train && is_dyn(0);
    LAUNCH(K_GATHER, 0, (8.0 + e * (first_dyn ? 3 : 1)) * n * d,
           (gather_chunk_kernel<T><<<592, 256, 0, st>>>(hidden, p.T, b, c, d, n, resid, actin,
                                                        first_dyn ? aw : nullptr, first_dyn ? am : nullptr,
                                                        KW, KM, p.kscale)));
  }
  for (int i = 0; i < p.nM; ++i) {
    const bool dyn = is_dyn(i);
    const int l = blk_of(i);
    const T* w1 = dyn ? Wsh + l * blk : S + l * blk;
    const T* w2 = w1 + (int64_t)H2 * d;
    const int64_t wstride = dyn ? seqW : 0;
    const int Bz = dyn ? B : 1, Mz = dyn ? b : n;
    T* ain = actin + (int64_t)i * n * d;
    T* aout = act + (int64_t)i * n * h;
    T* fi = fac + (int64_t)i * n * H2;
    {
      GemmShape s{Mz, H2, d, Bz};
      Operand A = opnd(ain, d, (int64_t)Mz * d, 1, Mz);
      Operand Bw = opnd(w1, d, wstride, 1, H2);
      T* fptr = (train && i >= i_min) ? fi : nullptr;
      const double fl = 2.0 * Mz * H2 * d * Bz;
      const double by = e * ((double)n * d + (double)H2 * d * Bz + (double)n * h + (fptr ? (double)n * H2 : 0.0));
      if (sw) LAUNCH(K_MLP_UP, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiF1<T, true>{aout, fptr, h, Mz}, st, status, ss))));
      else LAUNCH(K_MLP_UP, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiF1<T, false>{aout, fptr, h, Mz}, st, status, ss))));
    }
    {
      GemmShape s{Mz, d, h, Bz};
      Operand A = opnd(aout, h, (int64_t)Mz * h, 1, Mz);
      Operand Bw = opnd(w2, h, wstride, 1, d);
      T* next = (i + 1 < p.nM) ? actin + (int64_t)(i + 1) * n * d : nullptr;
      const bool next_dyn = train && i + 1 < p.nM && is_dyn(i + 1);
      T* nw = next_dyn ? aw + (int64_t)(i + 1) * n * d : nullptr;
      T* nmm = next_dyn ? am + (int64_t)(i + 1) * n * d : nullptr;
      LAUNCH(K_MLP_DOWN, 2.0 * Mz * d * h * Bz,
             e * ((double)n * h + (double)d * h * Bz + (next ? (double)n * d : 0.0) + (nw ? 2.0 * n * d : 0.0)) +
                 8.0 * n * d,
             TRY((gemm<T, 1>(s, A, A, Bw, EpiResid<T>{resid, next, nw, nmm, KW, KM, p.kscale, tm, d, Mz}, st,
                              status, ss))));
    }
  }
  return cudaSuccess;
}

// ---------------------------------------------------------------------------
// Head of chunk c: RMSNorm, CE pass A (logit tiles -> online-softmax
// partials), the per-token and chunk losses, CE pass B and dz per vocabulary
// slab, RMSNorm backward.  Leaves the residual-stream gradient in dout (fp32),
// its operand copy in dout_a and the K-scaled copies for the top MLP in
// doutW / doutM [top_buf].
// ---------------------------------------------------------------------------
template <typename T>
static cudaError_t enqueue_head(ttt_handle* hd, const Plan& p, const int* tokens, float* chunk_loss, int c,
                                const float* KW, const float* KM, char* ws, const SplitScratch& ss,
                                cudaStream_t st, Prof& prof, int top_buf) {
  const int B = p.B, b = p.b, n = p.n, d = p.d, V = p.V;
  float* resid = reinterpret_cast<float*>(ws + p.resid);
  T* z = reinterpret_cast<T*>(ws + p.z);
  float* rstd = reinterpret_cast<float*>(ws + p.rstd);
  float* part = reinterpret_cast<float*>(ws + p.part);
  float* tgt = reinterpret_cast<float*>(ws + p.tgt);
  float* lse = reinterpret_cast<float*>(ws + p.lse);
  float* ltok = reinterpret_cast<float*>(ws + p.ltok);
  T* P = reinterpret_cast<T*>(ws + p.P);
  float* dz = reinterpret_cast<float*>(ws + p.dz);
  float* dout = reinterpret_cast<float*>(ws + p.dout);
  T* dout_a = reinterpret_cast<T*>(ws + p.dout_a);
  T* doutW = reinterpret_cast<T*>(ws + p.doutW[top_buf]);
  T* doutM = reinterpret_cast<T*>(ws + p.doutM[top_buf]);
  const T* E = static_cast<const T*>(hd->E);
  int* status = hd->status;
  cudaError_t err;
  const double e = (double)p.esz;
  const TokenMap tm{b, p.T, c};
  LAUNCH(K_RMS_FWD, 0, (4.0 + e) * n * d,
         (rmsnorm_fwd_kernel<T><<<(n + 7) / 8, 256, 0, st>>>(resid, hd->gain, hd->cfg.rms_eps, n, d, z, rstd)));
  {
    GemmShape s{n, V, d, 1};
    Operand A = opnd(z, d, 0, 1, n);
    Operand Be = opnd(E, d, 0, 1, V);
    LAUNCH(K_CE_LSE, 2.0 * n * V * d, e * ((double)n * d + (double)V * d) + 8.0 * n * p.ntn,
           TRY((gemm<T, 1>(s, A, A, Be, EpiCEPartial<T>{part, tgt, tokens, tm, p.ntn}, st, status, ss))));
  }
  LAUNCH(K_CE_ROWS, 0, 8.0 * n * p.ntn + 16.0 * n,
         (ce_rows_kernel<<<(n + 7) / 8, 256, 0, st>>>(part, tgt, p.ntn, tokens, tm, V, n, lse, ltok, status)));
  LAUNCH(K_CE_MEAN, 0, 4.0 * n, (ce_mean_kernel<<<B, 256, 0, st>>>(ltok, b, chunk_loss, c, p.nchunks, status)));
  // ---- CE pass B and dz, one vocabulary slab at a time ----
  for (int sl = 0; sl < p.nslabs; ++sl) {
    const int v0 = sl * p.Vs;
    const int vs = V - v0 < p.Vs ? V - v0 : p.Vs;
    {   // recompute the slab's logits; the epilogue writes softmax - onehot
      GemmShape s{n, vs, d, 1};
      Operand A = opnd(z, d, 0, 1, n);
      Operand Be = opnd(E + (int64_t)v0 * d, d, 0, 1, vs);
      LAUNCH(K_CE_GRAD, 2.0 * n * vs * d, e * ((double)n * d + (double)vs * d + (double)n * vs),
             TRY((gemm<T, 1>(s, A, A, Be, EpiCEGrad<T>{P, lse, tokens, tm, p.Vs, v0}, st, status, ss))));
    }
    {
      GemmShape s{n, d, vs, 1};
      Operand A = opnd(P, p.Vs, 0, 1, n);
      Operand Be = opnd(E + (int64_t)v0 * d, d, 0, 0, vs);
      LAUNCH(K_CE_DZ, 2.0 * n * d * vs, e * ((double)n * vs + (double)vs * d) + (sl > 0 ? 8.0 : 4.0) * n * d,
             TRY((gemm<T, 1>(s, A, A, Be, EpiStoreF32{dz, d, sl > 0 ? 1 : 0}, st, status, ss))));
    }
  }
  LAUNCH(K_RMS_BWD, 0, (12.0 + 3.0 * e) * n * d,
         (rmsnorm_bwd_kernel<T><<<(n + 7) / 8, 256, 0, st>>>(dz, resid, rstd, hd->gain, n, d, dout, dout_a, doutW,
                                                             doutM, KW, KM, p.kscale, tm)));
  return cudaSuccess;
}

// ---------------------------------------------------------------------------
// Enqueue one prefill (all chunks) on `st`.
// ---------------------------------------------------------------------------
template <typename T>
static cudaError_t enqueue_prefill(ttt_handle* hd, const Plan& p, const float* hidden, const int* tokens,
                                   float* W, float* M, const float* eta, const float* beta,
                                   const float* gamma, float* chunk_loss, char* ws, cudaStream_t st,
                                   Prof& prof) {
  const int B = p.B, b = p.b, n = p.n, d = p.d, h = p.h, H2 = p.H2, L = p.L;
  float* KW = reinterpret_cast<float*>(ws + p.KW);
  float* KM = reinterpret_cast<float*>(ws + p.KM);
  float* consts = reinterpret_cast<float*>(ws + p.consts);
  T* Wsh = reinterpret_cast<T*>(ws + p.Wsh);
  T* aw = reinterpret_cast<T*>(ws + p.aw);
  T* am = reinterpret_cast<T*>(ws + p.am);
  T* act = reinterpret_cast<T*>(ws + p.act);
  T* fac = reinterpret_cast<T*>(ws + p.fac);
  float* dout = reinterpret_cast<float*>(ws + p.dout);
  T* dout_a = reinterpret_cast<T*>(ws + p.dout_a);
  // three rotating buffers each: an aggregation on the side stream may still
  // read the ones of the MLP two levels up while this level writes its own
  T* doutW[3];
  T* doutM[3];
  T* dUb[3];
  for (int k = 0; k < 3; ++k) {
    doutW[k] = reinterpret_cast<T*>(ws + p.doutW[k]);
    doutM[k] = reinterpret_cast<T*>(ws + p.doutM[k]);
    dUb[k] = reinterpret_cast<T*>(ws + (k == 0 ? p.dU : p.dUx[k - 1]));
  }
  const T* S = static_cast<const T*>(hd->S);
  int* status = hd->status;
  SplitScratch ss;
  ss.partial = reinterpret_cast<float*>(ws + p.sk_partial);
  ss.partial_bytes = p.sk_partial_bytes;
  ss.counters = reinterpret_cast<int*>(ws + p.sk_counters);
  ss.counter_count = p.sk_counter_count;
  if (!p.sk_partial_bytes) ss = SplitScratch();
  cudaError_t err;
  const double e = (double)p.esz;

  // K1 for all chunks (depends only on the scalars).
  // Split-K arrival counters start at zero (every GEMM leaves them zero).
  if (p.sk_counter_count) TRY(cudaMemsetAsync(ws + p.sk_counters, 0, 4 * p.sk_counter_count, st));
  LAUNCH(K_SCAN, 0, 5.0 * 4 * B * p.T,
         TRY(launch_scalar_scan(hd->cfg.update_rule, eta, beta, gamma, B, p.T, b, KW, KM, consts, st)));
  // Operand shadow of W_0.
  LAUNCH(K_SHADOW, 0, (4.0 + e) * B * L * p.m * h * d,
         (build_shadow_kernel<T><<<1184, 256, 0, st>>>(W, Wsh, (int64_t)B * L, h, d, p.swiglu ? 1 : 0)));

  const int64_t blk = (int64_t)p.m * h * d;          // params per block
  const int64_t seqW = (int64_t)L * blk;             // params per sequence
  const bool sw = p.swiglu;
  // Lowest dynamic MLP index (forward order: per block [static], dynamic).
  const int per_blk = p.has_static ? 2 : 1;
  const int i_min = per_blk - 1;
  auto is_dyn = [&](int i) { return (i % per_blk) == per_blk - 1; };
  auto blk_of = [&](int i) { return i / per_blk; };

  // Each dynamic MLP's two aggregations depend only on its own backward
  // (dU, the K-scaled copies) and write only its own weights, so they run on
  // the handle's aggregation stream beside the backward GEMMs of the MLPs
  // below, which fill each other's last waves.  The forward of the next chunk
  // waits for all of them.  Serial when the launches are timed one by one.
  const bool conc = hd->agg_stream && hd->agg && !prof.timing;
  const cudaStream_t ast = conc ? hd->agg : st;
  bool up_pend[3] = {false, false, false}, out_pend[3] = {false, false, false};

  auto chunks = [&]() -> cudaError_t {
    for (int c = 0; c < p.nchunks; ++c) {
      TokenMap tm{b, p.T, c};
      TRY(enqueue_forward<T>(hd, p, hidden, Wsh, c, true, KW, KM, ws, ss, st, prof));

      TRY(enqueue_head<T>(hd, p, tokens, chunk_loss, c, KW, KM, ws, ss, st, prof, (p.nM - 1) % 3));

      // ---- backward, top down ----
      for (int i = p.nM - 1; i >= i_min; --i) {
        const bool dyn = is_dyn(i);
        const int l = blk_of(i);
        const T* w1 = dyn ? Wsh + l * blk : S + l * blk;
        const T* w2 = w1 + (int64_t)H2 * d;
        const int64_t wstride = dyn ? seqW : 0;
        const int Bz = dyn ? B : 1, Mz = dyn ? b : n;
        const bool need_dx = i > i_min;
        T* fi = fac + (int64_t)i * n * H2;
        const int k = i % 3;
        T* dU = dUb[k];
        if (up_pend[k]) {   // the aggregation of MLP i + 3 still reads dU[k]
          TRY(cudaStreamWaitEvent(st, hd->ev_up[k], 0));
          up_pend[k] = false;
        }
        {  // B1: dA = dOut W2 -> dU
          GemmShape s{Mz, h, d, Bz};
          Operand A = opnd(dout_a, d, (int64_t)Mz * d, 1, Mz);
          Operand Bw = opnd(w2, h, wstride, 0, d);
          const double fl = 2.0 * Mz * h * d * Bz;
          const double by = e * ((double)n * d + (double)d * h * Bz + 2.0 * n * H2);
          if (sw) LAUNCH(K_BWD_DA, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiB1<T, true>{fi, dU, h, Mz}, st, status, ss))));
          else LAUNCH(K_BWD_DA, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiB1<T, false>{fi, dU, h, Mz}, st, status, ss))));
        }
        if (need_dx) {  // B2: dout += dU W1
          GemmShape s{Mz, d, H2, Bz};
          Operand A = opnd(dU, H2, (int64_t)Mz * H2, 1, Mz);
          Operand Bw = opnd(w1, d, wstride, 0, H2);
          const bool below_dyn = is_dyn(i - 1);
          const int ko = (i - 1) % 3;
          if (below_dyn && out_pend[ko]) {   // the aggregation of MLP i + 2 still reads doutW/doutM[ko]
            TRY(cudaStreamWaitEvent(st, hd->ev_out[ko], 0));
            out_pend[ko] = false;
          }
          T* ow = below_dyn ? doutW[ko] : nullptr;
          T* om = below_dyn ? doutM[ko] : nullptr;
          LAUNCH(K_BWD_DX, 2.0 * Mz * d * H2 * Bz,
                 e * ((double)n * H2 + (double)H2 * d * Bz + (double)n * d * (ow ? 3 : 1)) + 8.0 * n * d,
                 TRY((gemm<T, 1>(s, A, A, Bw, EpiB2<T>{dout, dout_a, ow, om, KW, KM, p.kscale, tm, d, Mz}, st, status, ss))));
        }
        if (dyn) {
          T* aout = act + (int64_t)i * n * h;
          float* Wl = W + l * blk;
          float* Ml = M + l * blk;
          T* Sl = Wsh + l * blk;
          // after this MLP's dA and dX, which read the shadow rows these update
          if (conc) {
            TRY(cudaEventRecord(hd->ev_fork, st));
            TRY(cudaStreamWaitEvent(ast, hd->ev_fork, 0));
          }
          const cudaStream_t st = ast;
          {  // rows of W1 (and W2 for SwiGLU): [H2, d], contraction over the b tokens:
             // sum_t dU_t (x) (-K_t x_t), A = dU shared by both accumulators
            GemmShape s{H2, d, b, B};
            Operand A = opnd(dU, H2, (int64_t)b * H2, 0, b);
            Operand B1 = opnd(aw + (int64_t)i * n * d, d, (int64_t)b * d, 0, b);
            Operand B2 = opnd(am + (int64_t)i * n * d, d, (int64_t)b * d, 0, b);
            EpiUpdate<T> ep{Wl, Ml, Sl, seqW, seqW, consts, c, p.nchunks, d, sw ? h : 0};
            LAUNCH(K_AGG_UPDATE, 4.0 * H2 * d * b * B,
                   (16.0 + e) * H2 * d * B + e * ((double)n * H2 + 2.0 * n * d),
                   TRY((gemm_dualb<T>(s, A, B1, B2, ep, st, status))));
          }
          if (conc) {
            TRY(cudaEventRecord(hd->ev_up[k], st));
            up_pend[k] = true;
          }
          {  // the output matrix (W2 for GELU, W3 for SwiGLU): [d, h]
            GemmShape s{d, h, b, B};
            Operand A = opnd(doutW[k], d, (int64_t)b * d, 0, b);
            Operand A2 = opnd(doutM[k], d, (int64_t)b * d, 0, b);
            Operand Bx = opnd(aout, h, (int64_t)b * h, 0, b);
            EpiUpdate<T> ep{Wl + (int64_t)H2 * d, Ml + (int64_t)H2 * d, Sl + (int64_t)H2 * d, seqW, seqW,
                            consts, c, p.nchunks, h, 0};
            LAUNCH(K_AGG_UPDATE, 4.0 * d * h * b * B,
                   (16.0 + e) * d * h * B + e * ((double)n * d * 2 + (double)n * h),
                   TRY((gemm<T, 2>(s, A, A2, Bx, ep, st, status))));
          }
          if (conc) {
            TRY(cudaEventRecord(hd->ev_out[k], st));
            out_pend[k] = true;
          }
        }
      }
      if (conc) {   // the next chunk's forward reads the updated shadow
        TRY(cudaEventRecord(hd->ev_join, ast));
        TRY(cudaStreamWaitEvent(st, hd->ev_join, 0));
        for (int k = 0; k < 3; ++k) up_pend[k] = out_pend[k] = false;
      }
    }
    return cudaSuccess;
  };
  err = chunks();
  // A failed launch leaves the call early: order what the aggregation stream
  // already holds before anything the caller enqueues next (best effort).
  if (err != cudaSuccess && conc) {
    cudaEventRecord(hd->ev_join, ast);
    cudaStreamWaitEvent(st, hd->ev_join, 0);
  }
  return err;
}

// ---------------------------------------------------------------------------
// The inner loop with frozen sliding-window attention in front of every
// updated block ("TTT-E2E：端到端测试时训练的长上下文语言建模": the sketch's
// TTTE2EBlock; 滑动窗口注意力): per block h <- h + Attn(LN(h)), then the static
// and dynamic MLPs.  A chunk's queries see the keys and values of earlier
// chunks inside the window (kept for the whole sequence, written when their
// chunk ran) and of their own chunk.
//
// The backward above the top block's attention is row-local, as without
// attention (the top block's MLPs aggregate with K-scaled operand copies).
// Below it attention mixes the chunk's rows, so sum_t K_t G_t is taken as the
// gradient of the K-weighted chunk loss: two cotangent streams (K_W- and
// K_M-weighted) run through the attention and MLP backward, and the lower
// blocks' aggregations pair each stream's activation gradients with the
// unscaled inputs (two A operands sharing B).
// ---------------------------------------------------------------------------
template <typename T>
static cudaError_t enqueue_prefill_swa(ttt_handle* hd, const Plan& p, const float* hidden, const int* tokens,
                                       float* W, float* M, const float* eta, const float* beta,
                                       const float* gamma, float* chunk_loss, char* ws, cudaStream_t st,
                                       Prof& prof) {
  const int B = p.B, b = p.b, n = p.n, d = p.d, h = p.h, H2 = p.H2, L = p.L;
  const int H = p.H, dh = p.dh, ldS = p.ldS;
  float* KW = reinterpret_cast<float*>(ws + p.KW);
  float* KM = reinterpret_cast<float*>(ws + p.KM);
  float* consts = reinterpret_cast<float*>(ws + p.consts);
  T* Wsh = reinterpret_cast<T*>(ws + p.Wsh);
  float* resid = reinterpret_cast<float*>(ws + p.resid);
  T* actin = reinterpret_cast<T*>(ws + p.actin);
  T* aw = reinterpret_cast<T*>(ws + p.aw);
  T* am = reinterpret_cast<T*>(ws + p.am);
  T* act = reinterpret_cast<T*>(ws + p.act);
  T* fac = reinterpret_cast<T*>(ws + p.fac);
  T* zT = reinterpret_cast<T*>(ws + p.z);            // LayerNorm output (the head reuses it later)
  float* dout = reinterpret_cast<float*>(ws + p.dout);
  T* dout_a = reinterpret_cast<T*>(ws + p.dout_a);
  T* doutW[2] = {reinterpret_cast<T*>(ws + p.doutW[0]), reinterpret_cast<T*>(ws + p.doutW[1])};
  T* doutM[2] = {reinterpret_cast<T*>(ws + p.doutM[0]), reinterpret_cast<T*>(ws + p.doutM[1])};
  T* dU = reinterpret_cast<T*>(ws + p.dU);
  const float2* rtab = reinterpret_cast<const float2*>(ws + p.rope_tab);
  float* xhat = reinterpret_cast<float*>(ws + p.xhat);
  float* lnr = reinterpret_cast<float*>(ws + p.lnr);
  float* qkv = reinterpret_cast<float*>(ws + p.qkv);
  T* qh = reinterpret_cast<T*>(ws + p.qh);
  T* kh = reinterpret_cast<T*>(ws + p.kh);
  T* vh = reinterpret_cast<T*>(ws + p.vh);
  float* spart = reinterpret_cast<float*>(ws + p.spart);
  float* slse = reinterpret_cast<float*>(ws + p.slse);
  float* sD = reinterpret_cast<float*>(ws + p.sD);
  T* Pa = reinterpret_cast<T*>(ws + p.Pa);
  float* Of = reinterpret_cast<float*>(ws + p.Of);
  T* Oc = reinterpret_cast<T*>(ws + p.Oc);
  T* dOh = reinterpret_cast<T*>(ws + p.dOh);
  T* dSa = reinterpret_cast<T*>(ws + p.dSa);
  float* dq = reinterpret_cast<float*>(ws + p.dq);
  float* dk = reinterpret_cast<float*>(ws + p.dk);
  float* dv = reinterpret_cast<float*>(ws + p.dv);
  T* dqkv = reinterpret_cast<T*>(ws + p.dqkv);
  float* da = reinterpret_cast<float*>(ws + p.da);
  float* sdout[2] = {reinterpret_cast<float*>(ws + p.sdout[0]), reinterpret_cast<float*>(ws + p.sdout[1])};
  T* sdoutT[2][2] = {{reinterpret_cast<T*>(ws + p.sdoutT[0][0]), reinterpret_cast<T*>(ws + p.sdoutT[0][1])},
                     {reinterpret_cast<T*>(ws + p.sdoutT[1][0]), reinterpret_cast<T*>(ws + p.sdoutT[1][1])}};
  T* sdU[2] = {reinterpret_cast<T*>(ws + p.sdU[0]), reinterpret_cast<T*>(ws + p.sdU[1])};
  const T* S = static_cast<const T*>(hd->S);
  const T* Wqkv = static_cast<const T*>(hd->Wqkv);
  const T* Wo = static_cast<const T*>(hd->Wo);
  int* status = hd->status;
  SplitScratch ss;
  if (p.sk_partial_bytes) {
    ss.partial = reinterpret_cast<float*>(ws + p.sk_partial);
    ss.partial_bytes = p.sk_partial_bytes;
    ss.counters = reinterpret_cast<int*>(ws + p.sk_counters);
    ss.counter_count = p.sk_counter_count;
  }
  cudaError_t err;
  const double e = (double)p.esz;
  const float scale = 1.0f / sqrtf((float)dh);
  const int64_t Tn = p.T;

  if (p.sk_counter_count) TRY(cudaMemsetAsync(ws + p.sk_counters, 0, 4 * p.sk_counter_count, st));
  LAUNCH(K_SCAN, 0, 5.0 * 4 * B * p.T,
         TRY(launch_scalar_scan(hd->cfg.update_rule, eta, beta, gamma, B, p.T, b, KW, KM, consts, st)));
  LAUNCH(K_SHADOW, 0, (4.0 + e) * B * L * p.m * h * d,
         (build_shadow_kernel<T><<<1184, 256, 0, st>>>(W, Wsh, (int64_t)B * L, h, d, p.swiglu ? 1 : 0)));
  LAUNCH(K_ATTN_ROWS, 0, 8.0 * Tn * (dh / 2),
         (rope_table_kernel<<<1184, 256, 0, st>>>(Tn, dh / 2, 10000.0, reinterpret_cast<float2*>(ws + p.rope_tab))));

  const int64_t blk = (int64_t)p.m * h * d;
  const int64_t seqW = (int64_t)L * blk;
  const bool sw = p.swiglu;
  const int per_blk = p.has_static ? 2 : 1;
  const int i_min = per_blk - 1;
  const int i_top = (L - 1) * per_blk;   // first MLP of the top block
  auto is_dyn = [&](int i) { return (i % per_blk) == per_blk - 1; };
  auto blk_of = [&](int i) { return i / per_blk; };
  const int64_t hist = (int64_t)B * H * Tn * dh;   // history elements per block
  const int64_t pblk = (int64_t)B * H * b * ldS;  // probabilities per block

  for (int c = 0; c < p.nchunks; ++c) {
    const TokenMap tm{b, p.T, c};
    const int64_t q0 = (int64_t)c * b;
    int64_t j0 = q0 - p.window + 1;
    j0 = j0 < 0 ? 0 : j0 / 8 * 8;
    const int nk = (int)(q0 + b - j0);
    LAUNCH(K_GATHER, 0, (8.0 + e) * n * d,
           (gather_chunk_kernel<T><<<592, 256, 0, st>>>(hidden, p.T, b, c, d, n, resid, actin, nullptr, nullptr, KW,
                                                        KM, p.kscale)));
    // ---- forward ----
    for (int l = 0; l < L; ++l) {
      const int i0 = l * per_blk;      // the block's first MLP
      T* qb = qh + (int64_t)l * n * d;
      T* kb = kh + l * hist;
      T* vb = vh + l * hist;
      float* ob = Of + (int64_t)l * n * d;
      LAUNCH(K_ATTN_ROWS, 0, (12.0 + e) * n * d,
             (ln_affine_fwd_kernel<T><<<(n + 7) / 8, 256, 0, st>>>(resid, hd->ln_gain + (int64_t)l * d,
                                                                   hd->ln_bias + (int64_t)l * d, hd->attn_ln_eps, n, d, zT,
                                                                   xhat + (int64_t)l * n * d, lnr + (int64_t)l * n)));
      {
        GemmShape s{n, 3 * d, d, 1};
        LAUNCH(K_ATTN_PROJ, 2.0 * n * 3 * d * d, e * ((double)n * d + 3.0 * d * d) + 12.0 * n * d,
               TRY((gemm<T, 1>(s, opnd(zT, d, 0, 1, n), opnd(zT, d, 0, 1, n),
                               opnd(Wqkv + (int64_t)l * 3 * d * d, d, 0, 1, 3 * d), EpiStoreF32{qkv, 3 * d, 0}, st,
                               status, ss))));
      }
      LAUNCH(K_ATTN_ROWS, 0, (12.0 + 3.0 * e) * n * d,
             (rope_split_kernel<T><<<592, 256, 0, st>>>(qkv, rtab, n, b, d, H, Tn, c, qb, kb, vb)));
      for (int s = 0; s < B; ++s) {
        T* qs = qb + (int64_t)s * H * b * dh;
        T* ks = kb + (int64_t)s * H * Tn * dh + j0 * dh;
        T* vs = vb + (int64_t)s * H * Tn * dh + j0 * dh;
        T* ps = Pa + l * pblk + (int64_t)s * H * b * ldS;
        {
          // pass A: masked (max, sum exp) partials per row and column part;
          // pass B recomputes the scores and writes P = exp(scale s - lse)
          GemmShape g{b, nk, dh, H};
          const int ntn = head_parts(hd->cfg.precision, nk);
          Operand Aq = opnd(qs, dh, (int64_t)b * dh, 1, b);
          Operand Bk = opnd(ks, dh, Tn * dh, 1, nk);
          LAUNCH(K_ATTN_SCORE, 2.0 * b * nk * dh * H, e * ((double)b + nk) * dh * H + 8.0 * H * b * ntn,
                 TRY((gemm<T, 1>(g, Aq, Aq, Bk, EpiScorePartial<T>{spart, b, ntn, q0, j0, p.window, scale}, st, status,
                                 ss))));
          LAUNCH(K_ATTN_ROWS, 0, 8.0 * H * b * ntn + 4.0 * H * b,
                 (attn_lse_kernel<<<(H * b + 7) / 8, 256, 0, st>>>(spart, ntn, (int64_t)H * b, slse)));
          LAUNCH(K_ATTN_SCORE, 2.0 * b * nk * dh * H, e * ((double)b + nk) * dh * H + e * H * b * nk,
                 TRY((gemm<T, 1>(g, Aq, Aq, Bk, EpiScoreP<T>{ps, slse, b, ldS, q0, j0, p.window, scale}, st, status,
                                 ss))));
        }
        {
          GemmShape g{b, dh, nk, H};
          LAUNCH(K_ATTN_SCORE, 2.0 * b * nk * dh * H, e * ((double)b * nk + (double)nk * dh) * H + 4.0 * b * d,
                 TRY((gemm<T, 1>(g, opnd(ps, ldS, (int64_t)b * ldS, 1, b), opnd(ps, ldS, (int64_t)b * ldS, 1, b),
                                 opnd(vs, dh, Tn * dh, 0, nk), EpiStoreBatched{ob + (int64_t)s * b * d, d, dh}, st,
                                 status, ss))));
        }
      }
      LAUNCH(K_ATTN_ROWS, 0, (4.0 + e) * n * d,
             (cast_kernel<T><<<592, 256, 0, st>>>(ob, Oc, (int64_t)n * d)));
      {
        // the output projection adds into the residual stream and writes the
        // block's first MLP input (with its K-scaled copies when that MLP is
        // dynamic and row-local, i.e. in the top block)
        const bool rowloc = l == L - 1 && is_dyn(i0);
        T* next = actin + (int64_t)i0 * n * d;
        GemmShape s{n, d, d, 1};
        LAUNCH(K_ATTN_PROJ, 2.0 * n * d * d, e * ((double)n * d * (rowloc ? 4 : 2) + (double)d * d) + 8.0 * n * d,
               TRY((gemm<T, 1>(s, opnd(Oc, d, 0, 1, n), opnd(Oc, d, 0, 1, n),
                               opnd(Wo + (int64_t)l * d * d, d, 0, 1, d),
                               EpiResid<T>{resid, next, rowloc ? aw + (int64_t)i0 * n * d : nullptr,
                                           rowloc ? am + (int64_t)i0 * n * d : nullptr, KW, KM, p.kscale, tm, d, n},
                               st, status, ss))));
      }
      for (int i = i0; i < i0 + per_blk; ++i) {
        const bool dyn = is_dyn(i);
        const T* w1 = dyn ? Wsh + l * blk : S + l * blk;
        const T* w2 = w1 + (int64_t)H2 * d;
        const int64_t wstride = dyn ? seqW : 0;
        const int Bz = dyn ? B : 1, Mz = dyn ? b : n;
        T* ain = actin + (int64_t)i * n * d;
        T* aout = act + (int64_t)i * n * h;
        T* fptr = i >= i_min ? fac + (int64_t)i * n * H2 : nullptr;
        {
          GemmShape s{Mz, H2, d, Bz};
          Operand A = opnd(ain, d, (int64_t)Mz * d, 1, Mz);
          Operand Bw = opnd(w1, d, wstride, 1, H2);
          const double fl = 2.0 * Mz * H2 * d * Bz;
          const double by = e * ((double)n * d + (double)H2 * d * Bz + (double)n * h + (fptr ? (double)n * H2 : 0.0));
          if (sw) LAUNCH(K_MLP_UP, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiF1<T, true>{aout, fptr, h, Mz}, st, status, ss))));
          else LAUNCH(K_MLP_UP, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiF1<T, false>{aout, fptr, h, Mz}, st, status, ss))));
        }
        {
          // the block's last MLP feeds the next block's LayerNorm (or the head)
          // through the fp32 residual stream alone
          const bool last = i == i0 + per_blk - 1;
          T* next = last ? nullptr : actin + (int64_t)(i + 1) * n * d;
          const bool next_rl = !last && l == L - 1 && is_dyn(i + 1);
          T* nw = next_rl ? aw + (int64_t)(i + 1) * n * d : nullptr;
          T* nmm = next_rl ? am + (int64_t)(i + 1) * n * d : nullptr;
          GemmShape s{Mz, d, h, Bz};
          Operand A = opnd(aout, h, (int64_t)Mz * h, 1, Mz);
          Operand Bw = opnd(w2, h, wstride, 1, d);
          LAUNCH(K_MLP_DOWN, 2.0 * Mz * d * h * Bz,
                 e * ((double)n * h + (double)d * h * Bz + (next ? (double)n * d : 0.0) + (nw ? 2.0 * n * d : 0.0)) +
                     8.0 * n * d,
                 TRY((gemm<T, 1>(s, A, A, Bw, EpiResid<T>{resid, next, nw, nmm, KW, KM, p.kscale, tm, d, Mz}, st,
                                  status, ss))));
        }
      }
    }

    // ---- head ----
    TRY(enqueue_head<T>(hd, p, tokens, chunk_loss, c, KW, KM, ws, ss, st, prof, (p.nM - 1) & 1));

    // ---- backward of the top block's MLPs (row-local) ----
    for (int i = p.nM - 1; i >= std::max(i_top, i_min); --i) {
      const bool dyn = is_dyn(i);
      const int l = blk_of(i);
      const T* w1 = dyn ? Wsh + l * blk : S + l * blk;
      const T* w2 = w1 + (int64_t)H2 * d;
      const int64_t wstride = dyn ? seqW : 0;
      const int Bz = dyn ? B : 1, Mz = dyn ? b : n;
      const bool need_dx = i > i_min;
      T* fi = fac + (int64_t)i * n * H2;
      {
        GemmShape s{Mz, h, d, Bz};
        Operand A = opnd(dout_a, d, (int64_t)Mz * d, 1, Mz);
        Operand Bw = opnd(w2, h, wstride, 0, d);
        const double fl = 2.0 * Mz * h * d * Bz;
        const double by = e * ((double)n * d + (double)d * h * Bz + 2.0 * n * H2);
        if (sw) LAUNCH(K_BWD_DA, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiB1<T, true>{fi, dU, h, Mz}, st, status, ss))));
        else LAUNCH(K_BWD_DA, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiB1<T, false>{fi, dU, h, Mz}, st, status, ss))));
      }
      if (need_dx) {
        GemmShape s{Mz, d, H2, Bz};
        Operand A = opnd(dU, H2, (int64_t)Mz * H2, 1, Mz);
        Operand Bw = opnd(w1, d, wstride, 0, H2);
        const bool below_rl = i - 1 >= i_top && is_dyn(i - 1);
        T* ow = below_rl ? doutW[(i - 1) & 1] : nullptr;
        T* om = below_rl ? doutM[(i - 1) & 1] : nullptr;
        LAUNCH(K_BWD_DX, 2.0 * Mz * d * H2 * Bz,
               e * ((double)n * H2 + (double)H2 * d * Bz + (double)n * d * (ow ? 3 : 1)) + 8.0 * n * d,
               TRY((gemm<T, 1>(s, A, A, Bw, EpiB2<T>{dout, dout_a, ow, om, KW, KM, p.kscale, tm, d, Mz}, st, status, ss))));
      }
      if (dyn) {
        T* aout = act + (int64_t)i * n * h;
        float* Wl = W + l * blk;
        float* Ml = M + l * blk;
        T* Sl = Wsh + l * blk;
        {
          GemmShape s{H2, d, b, B};
          Operand A = opnd(dU, H2, (int64_t)b * H2, 0, b);
          Operand B1 = opnd(aw + (int64_t)i * n * d, d, (int64_t)b * d, 0, b);
          Operand B2 = opnd(am + (int64_t)i * n * d, d, (int64_t)b * d, 0, b);
          EpiUpdate<T> ep{Wl, Ml, Sl, seqW, seqW, consts, c, p.nchunks, d, sw ? h : 0};
          LAUNCH(K_AGG_UPDATE, 4.0 * H2 * d * b * B, (16.0 + e) * H2 * d * B + e * ((double)n * H2 + 2.0 * n * d),
                 TRY((gemm_dualb<T>(s, A, B1, B2, ep, st, status))));
        }
        {
          GemmShape s{d, h, b, B};
          Operand A = opnd(doutW[i & 1], d, (int64_t)b * d, 0, b);
          Operand A2 = opnd(doutM[i & 1], d, (int64_t)b * d, 0, b);
          Operand Bx = opnd(aout, h, (int64_t)b * h, 0, b);
          EpiUpdate<T> ep{Wl + (int64_t)H2 * d, Ml + (int64_t)H2 * d, Sl + (int64_t)H2 * d, seqW, seqW,
                          consts, c, p.nchunks, h, 0};
          LAUNCH(K_AGG_UPDATE, 4.0 * d * h * b * B, (16.0 + e) * d * h * B + e * ((double)n * d * 2 + (double)n * h),
                 TRY((gemm<T, 2>(s, A, A2, Bx, ep, st, status))));
        }
      }
    }
    if (L == 1) continue;   // block 0's attention reads the frozen hidden rows

    // ---- the two weighted streams, through attention and the lower blocks ----
    int cur = 0;   // sdoutT[st][cur]: operand copy of stream st's cotangent
    LAUNCH(K_ATTN_ROWS, 0, (4.0 + 8.0 + 2.0 * e) * n * d,
           (stream_split_kernel<T><<<592, 256, 0, st>>>(dout, KW, KM, p.kscale, tm, n, d, sdout[0], sdout[1],
                                                        sdoutT[0][0], sdoutT[1][0])));
    for (int l = L - 1; l >= 1; --l) {
      T* qb = qh + (int64_t)l * n * d;
      T* kb = kh + l * hist;
      T* vb = vh + l * hist;
      float* ob = Of + (int64_t)l * n * d;
      const int64_t off = q0 - j0;   // the chunk's own keys start at this column
      for (int sidx = 0; sidx < 2; ++sidx) {
        {
          GemmShape s{n, d, d, 1};
          LAUNCH(K_ATTN_PROJ, 2.0 * n * d * d, e * (2.0 * n * d + (double)d * d),
                 TRY((gemm<T, 1>(s, opnd(sdoutT[sidx][cur], d, 0, 1, n), opnd(sdoutT[sidx][cur], d, 0, 1, n),
                                 opnd(Wo + (int64_t)l * d * d, d, 0, 0, d), EpiStoreHeads<T>{dOh, b, H, dh}, st,
                                 status, ss))));
        }
        for (int s = 0; s < B; ++s) {
          T* qs = qb + (int64_t)s * H * b * dh;
          T* ks = kb + (int64_t)s * H * Tn * dh + j0 * dh;
          T* vs = vb + (int64_t)s * H * Tn * dh + j0 * dh;
          T* ps = Pa + l * pblk + (int64_t)s * H * b * ldS;
          T* dos = dOh + (int64_t)s * H * b * dh;
          LAUNCH(K_ATTN_ROWS, 0, (e + 4.0) * H * b * dh + 4.0 * H * b,
                 (attn_rowdot_kernel<T><<<(H * b + 7) / 8, 256, 0, st>>>(dos, ob + (int64_t)s * b * d, H * b, b, d, dh,
                                                                         sD)));
          {
            // dP = dO V^T, turned into dS = P (dP - D) scale in the epilogue
            GemmShape g{b, nk, dh, H};
            LAUNCH(K_ATTN_SCORE, 2.0 * b * nk * dh * H, e * ((double)b + nk) * dh * H + 2.0 * e * H * b * nk,
                   TRY((gemm<T, 1>(g, opnd(dos, dh, (int64_t)b * dh, 1, b), opnd(dos, dh, (int64_t)b * dh, 1, b),
                                   opnd(vs, dh, Tn * dh, 1, nk), EpiDScore<T>{dSa, ps, sD, b, ldS, scale}, st, status,
                                   ss))));
          }
          {
            GemmShape g{b, dh, nk, H};
            LAUNCH(K_ATTN_SCORE, 2.0 * b * nk * dh * H, e * ((double)b * nk + (double)nk * dh) * H + 4.0 * b * d,
                   TRY((gemm<T, 1>(g, opnd(dSa, ldS, (int64_t)b * ldS, 1, b), opnd(dSa, ldS, (int64_t)b * ldS, 1, b),
                                   opnd(ks, dh, Tn * dh, 0, nk), EpiStoreBatched{dq + (int64_t)s * b * d, d, dh}, st,
                                   status, ss))));
          }
          {
            GemmShape g{b, dh, b, H};
            LAUNCH(K_ATTN_SCORE, 2.0 * b * b * dh * H, e * ((double)b * b + (double)b * dh) * H + 4.0 * b * d,
                   TRY((gemm<T, 1>(g, opnd(dSa + off, ldS, (int64_t)b * ldS, 0, b),
                                   opnd(dSa + off, ldS, (int64_t)b * ldS, 0, b), opnd(qs, dh, (int64_t)b * dh, 0, b),
                                   EpiStoreBatched{dk + (int64_t)s * b * d, d, dh}, st, status, ss))));
            LAUNCH(K_ATTN_SCORE, 2.0 * b * b * dh * H, e * ((double)b * b + (double)b * dh) * H + 4.0 * b * d,
                   TRY((gemm<T, 1>(g, opnd(ps + off, ldS, (int64_t)b * ldS, 0, b),
                                   opnd(ps + off, ldS, (int64_t)b * ldS, 0, b), opnd(dos, dh, (int64_t)b * dh, 0, b),
                                   EpiStoreBatched{dv + (int64_t)s * b * d, d, dh}, st, status, ss))));
          }
          LAUNCH(K_ATTN_ROWS, 0, (12.0 + 3.0 * e) * b * d,
                 (rope_bwd_pack_kernel<T><<<592, 256, 0, st>>>(dq + (int64_t)s * b * d, dk + (int64_t)s * b * d,
                                                               dv + (int64_t)s * b * d, rtab, b, d, H, c,
                                                               dqkv + (int64_t)s * b * 3 * d)));
        }
        {
          GemmShape s{n, d, 3 * d, 1};
          LAUNCH(K_ATTN_PROJ, 2.0 * n * d * 3 * d, e * ((double)n * 3 * d + 3.0 * d * d) + 4.0 * n * d,
                 TRY((gemm<T, 1>(s, opnd(dqkv, 3 * d, 0, 1, n), opnd(dqkv, 3 * d, 0, 1, n),
                                 opnd(Wqkv + (int64_t)l * 3 * d * d, d, 0, 0, 3 * d), EpiStoreF32{da, d, 0}, st,
                                 status, ss))));
        }
        LAUNCH(K_ATTN_ROWS, 0, (20.0 + e) * n * d,
               (ln_affine_bwd_kernel<T><<<(n + 7) / 8, 256, 0, st>>>(da, xhat + (int64_t)l * n * d,
                                                                     lnr + (int64_t)l * n, hd->ln_gain + (int64_t)l * d,
                                                                     n, d, sdout[sidx], sdoutT[sidx][cur ^ 1])));
      }
      cur ^= 1;
      // block l-1's MLPs, top down, both streams
      for (int i = l * per_blk - 1; i >= std::max((l - 1) * per_blk, i_min); --i) {
        const bool dyn = is_dyn(i);
        const int lb = blk_of(i);
        const T* w1 = dyn ? Wsh + lb * blk : S + lb * blk;
        const T* w2 = w1 + (int64_t)H2 * d;
        const int64_t wstride = dyn ? seqW : 0;
        const int Bz = dyn ? B : 1, Mz = dyn ? b : n;
        const bool need_dx = i > i_min;
        T* fi = fac + (int64_t)i * n * H2;
        for (int sidx = 0; sidx < 2; ++sidx) {
          GemmShape s{Mz, h, d, Bz};
          Operand A = opnd(sdoutT[sidx][cur], d, (int64_t)Mz * d, 1, Mz);
          Operand Bw = opnd(w2, h, wstride, 0, d);
          const double fl = 2.0 * Mz * h * d * Bz;
          const double by = e * ((double)n * d + (double)d * h * Bz + 2.0 * n * H2);
          if (sw) LAUNCH(K_BWD_DA, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiB1<T, true>{fi, sdU[sidx], h, Mz}, st, status, ss))));
          else LAUNCH(K_BWD_DA, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiB1<T, false>{fi, sdU[sidx], h, Mz}, st, status, ss))));
        }
        if (need_dx) {
          for (int sidx = 0; sidx < 2; ++sidx) {
            GemmShape s{Mz, d, H2, Bz};
            Operand A = opnd(sdU[sidx], H2, (int64_t)Mz * H2, 1, Mz);
            Operand Bw = opnd(w1, d, wstride, 0, H2);
            LAUNCH(K_BWD_DX, 2.0 * Mz * d * H2 * Bz, e * ((double)n * H2 + (double)H2 * d * Bz + (double)n * d) + 8.0 * n * d,
                   TRY((gemm<T, 1>(s, A, A, Bw, EpiB2<T>{sdout[sidx], sdoutT[sidx][cur ^ 1], nullptr, nullptr, KW, KM,
                                                          p.kscale, tm, d, Mz}, st, status, ss))));
          }
        }
        if (dyn) {
          T* aout = act + (int64_t)i * n * h;
          float* Wl = W + lb * blk;
          float* Ml = M + lb * blk;
          T* Sl = Wsh + lb * blk;
          {
            // rows of W1 (and W2): sum_t dU^W_t (x) x_t and sum_t dU^M_t (x) x_t
            GemmShape s{H2, d, b, B};
            Operand A = opnd(sdU[0], H2, (int64_t)b * H2, 0, b);
            Operand A2 = opnd(sdU[1], H2, (int64_t)b * H2, 0, b);
            Operand Bx = opnd(actin + (int64_t)i * n * d, d, (int64_t)b * d, 0, b);
            EpiUpdate<T> ep{Wl, Ml, Sl, seqW, seqW, consts, c, p.nchunks, d, sw ? h : 0};
            LAUNCH(K_AGG_UPDATE, 4.0 * H2 * d * b * B, (16.0 + e) * H2 * d * B + e * (2.0 * n * H2 + (double)n * d),
                   TRY((gemm<T, 2>(s, A, A2, Bx, ep, st, status))));
          }
          {
            GemmShape s{d, h, b, B};
            Operand A = opnd(sdoutT[0][cur], d, (int64_t)b * d, 0, b);
            Operand A2 = opnd(sdoutT[1][cur], d, (int64_t)b * d, 0, b);
            Operand Bx = opnd(aout, h, (int64_t)b * h, 0, b);
            EpiUpdate<T> ep{Wl + (int64_t)H2 * d, Ml + (int64_t)H2 * d, Sl + (int64_t)H2 * d, seqW, seqW,
                            consts, c, p.nchunks, h, 0};
            LAUNCH(K_AGG_UPDATE, 4.0 * d * h * b * B, (16.0 + e) * d * h * B + e * ((double)n * d * 2 + (double)n * h),
                   TRY((gemm<T, 2>(s, A, A2, Bx, ep, st, status))));
          }
        }
        if (need_dx) cur ^= 1;
      }
    }
  }
  return cudaSuccess;
}

// The LM-head inner loop: with or without frozen attention in the blocks,
// in the handle's operand precision.
static cudaError_t enqueue_lm(ttt_handle* hd, const Plan& p, const float* hidden, const int* tokens, float* W,
                              float* M, const float* eta, const float* beta, const float* gamma, float* chunk_loss,
                              char* ws, cudaStream_t st, Prof& prof) {
  const bool fp32 = hd->cfg.precision == TTT_PREC_FP32;
  if (p.H > 0)
    return fp32 ? enqueue_prefill_swa<float>(hd, p, hidden, tokens, W, M, eta, beta, gamma, chunk_loss, ws, st, prof)
                : enqueue_prefill_swa<bf16>(hd, p, hidden, tokens, W, M, eta, beta, gamma, chunk_loss, ws, st, prof);
  return fp32 ? enqueue_prefill<float>(hd, p, hidden, tokens, W, M, eta, beta, gamma, chunk_loss, ws, st, prof)
              : enqueue_prefill<bf16>(hd, p, hidden, tokens, W, M, eta, beta, gamma, chunk_loss, ws, st, prof);
}

// ---------------------------------------------------------------------------
// E2-TTT's own layer, chunk after chunk ("Rethinking Expressivity and
// Efficiency in Test-Time Training", Algorithm 1): outputs o_t = f_{W_0}(q_t)
// and per-token losses at the chunk-start weights, one backward to the
// activation gradients, the two aggregations of the chunk update.  One dynamic
// block: f_W(x) = x + LN(MLP_W(x)).
// ---------------------------------------------------------------------------
template <typename T>
static cudaError_t enqueue_recon(ttt_handle* hd, const Plan& p, const float* Kin, const float* Vin, const float* Qin,
                                 float* W, float* M, const float* eta, const float* beta, const float* gamma,
                                 float* O, float* chunk_loss, char* ws, cudaStream_t st, Prof& prof) {
  const int B = p.B, b = p.b, d = p.d, h = p.h, H2 = p.H2;
  const int64_t n = p.n;
  float* KW = reinterpret_cast<float*>(ws + p.KW);
  float* KM = reinterpret_cast<float*>(ws + p.KM);
  float* consts = reinterpret_cast<float*>(ws + p.consts);
  T* Wsh = reinterpret_cast<T*>(ws + p.Wsh);
  float* kres = reinterpret_cast<float*>(ws + p.resid);
  T* kin = reinterpret_cast<T*>(ws + p.actin);
  T* aw = reinterpret_cast<T*>(ws + p.aw);
  T* am = reinterpret_cast<T*>(ws + p.am);
  T* act_k = reinterpret_cast<T*>(ws + p.act);
  T* act_q = act_k + n * h;
  T* fac = reinterpret_cast<T*>(ws + p.fac);
  T* qin = reinterpret_cast<T*>(ws + p.z);
  float* ltok = reinterpret_cast<float*>(ws + p.ltok);
  T* dout_a = reinterpret_cast<T*>(ws + p.dout_a);
  T* doutW = reinterpret_cast<T*>(ws + p.doutW[0]);
  T* doutM = reinterpret_cast<T*>(ws + p.doutM[0]);
  T* dU = reinterpret_cast<T*>(ws + p.dU);
  float* yk = reinterpret_cast<float*>(ws + p.yk);
  float* yq = reinterpret_cast<float*>(ws + p.yq);
  float* qres = reinterpret_cast<float*>(ws + p.qres);
  int* status = hd->status;
  SplitScratch ss;
  ss.partial = reinterpret_cast<float*>(ws + p.sk_partial);
  ss.partial_bytes = p.sk_partial_bytes;
  ss.counters = reinterpret_cast<int*>(ws + p.sk_counters);
  ss.counter_count = p.sk_counter_count;
  if (!p.sk_partial_bytes) ss = SplitScratch();
  cudaError_t err;
  const double e = (double)p.esz;
  if (p.sk_counter_count) TRY(cudaMemsetAsync(ws + p.sk_counters, 0, 4 * p.sk_counter_count, st));
  LAUNCH(K_SCAN, 0, 5.0 * 4 * B * p.T,
         TRY(launch_scalar_scan(hd->cfg.update_rule, eta, beta, gamma, B, p.T, b, KW, KM, consts, st)));
  LAUNCH(K_SHADOW, 0, (4.0 + e) * B * p.m * h * d,
         (build_shadow_kernel<T><<<1184, 256, 0, st>>>(W, Wsh, (int64_t)B, h, d, p.swiglu ? 1 : 0)));
  const int64_t seqW = (int64_t)p.m * h * d;   // params per sequence (one block)
  const bool sw = p.swiglu;
  const T* w1 = Wsh;
  const T* w2 = Wsh + (int64_t)H2 * d;
  for (int c = 0; c < p.nchunks; ++c) {
    TokenMap tm{b, p.T, c};
    LAUNCH(K_GATHER, 0, (8.0 + 3 * e) * n * d,
           (gather_chunk_kernel<T><<<592, 256, 0, st>>>(Kin, p.T, b, c, d, n, kres, kin, aw, am, KW, KM, p.kscale)));
    LAUNCH(K_GATHER, 0, (8.0 + e) * n * d,
           (gather_chunk_kernel<T><<<592, 256, 0, st>>>(Qin, p.T, b, c, d, n, qres, qin, nullptr, nullptr, KW, KM,
                                                        p.kscale)));
    // forward at the chunk-start weights: keys (with the backward's factors), then queries
    for (int side = 0; side < 2; ++side) {
      T* xin = side ? qin : kin;
      T* aout = side ? act_q : act_k;
      T* fptr = side ? nullptr : fac;
      float* y = side ? yq : yk;
      {
        GemmShape s{b, H2, d, B};
        Operand A = opnd(xin, d, (int64_t)b * d, 1, b);
        Operand Bw = opnd(w1, d, seqW, 1, H2);
        const double fl = 2.0 * b * H2 * d * B;
        const double by = e * ((double)n * d + (double)H2 * d * B + (double)n * h + (fptr ? (double)n * H2 : 0.0));
        if (sw) LAUNCH(K_MLP_UP, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiF1<T, true>{aout, fptr, h, b}, st, status, ss))));
        else LAUNCH(K_MLP_UP, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiF1<T, false>{aout, fptr, h, b}, st, status, ss))));
      }
      {
        GemmShape s{b, d, h, B};
        Operand A = opnd(aout, h, (int64_t)b * h, 1, b);
        Operand Bw = opnd(w2, h, seqW, 1, d);
        LAUNCH(K_MLP_DOWN, 2.0 * b * d * h * B, e * ((double)n * h + (double)d * h * B) + 4.0 * n * d,
               TRY((gemm<T, 1>(s, A, A, Bw, EpiStoreBatched{y, d, (int64_t)b * d}, st, status, ss))));
      }
    }
    LAUNCH(K_RECON_ROWS, 0, 4.0 * n * d * 6 + 3 * e * n * d,
           (recon_rows_kernel<T><<<(unsigned)((n + 7) / 8), 256, 0, st>>>(yk, kres, Vin, yq, qres, tm, n, d,
                                                                          hd->cfg.rms_eps, KW, KM, p.kscale, ltok,
                                                                          dout_a, doutW, doutM, O)));
    LAUNCH(K_CE_MEAN, 0, 4.0 * n, (ce_mean_kernel<<<B, 256, 0, st>>>(ltok, b, chunk_loss, c, p.nchunks, status)));
    {  // dA = g_y W_down -> dU
      GemmShape s{b, h, d, B};
      Operand A = opnd(dout_a, d, (int64_t)b * d, 1, b);
      Operand Bw = opnd(w2, h, seqW, 0, d);
      const double fl = 2.0 * b * h * d * B;
      const double by = e * ((double)n * d + (double)d * h * B + 2.0 * n * H2);
      if (sw) LAUNCH(K_BWD_DA, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiB1<T, true>{fac, dU, h, b}, st, status, ss))));
      else LAUNCH(K_BWD_DA, fl, by, TRY((gemm<T, 1>(s, A, A, Bw, EpiB1<T, false>{fac, dU, h, b}, st, status, ss))));
    }
    {  // rows of W1 (and W2 for SwiGLU): sum_t dU_t (x) (-K_t k_t)
      GemmShape s{H2, d, b, B};
      Operand A = opnd(dU, H2, (int64_t)b * H2, 0, b);
      Operand B1 = opnd(aw, d, (int64_t)b * d, 0, b);
      Operand B2 = opnd(am, d, (int64_t)b * d, 0, b);
      EpiUpdate<T> ep{W, M, Wsh, seqW, seqW, consts, c, p.nchunks, d, sw ? h : 0};
      LAUNCH(K_AGG_UPDATE, 4.0 * H2 * d * b * B, (16.0 + e) * H2 * d * B + e * ((double)n * H2 + 2.0 * n * d),
             TRY((gemm_dualb<T>(s, A, B1, B2, ep, st, status))));
    }
    {  // the output matrix: sum_t (-K_t g_y,t) (x) a_t
      GemmShape s{d, h, b, B};
      Operand A = opnd(doutW, d, (int64_t)b * d, 0, b);
      Operand A2 = opnd(doutM, d, (int64_t)b * d, 0, b);
      Operand Bx = opnd(act_k, h, (int64_t)b * h, 0, b);
      EpiUpdate<T> ep{W + (int64_t)H2 * d, M + (int64_t)H2 * d, Wsh + (int64_t)H2 * d, seqW, seqW, consts, c,
                      p.nchunks, h, 0};
      LAUNCH(K_AGG_UPDATE, 4.0 * d * h * b * B, (16.0 + e) * d * h * B + e * ((double)n * d * 2 + (double)n * h),
             TRY((gemm<T, 2>(s, A, A2, Bx, ep, st, status))));
    }
  }
  return cudaSuccess;
}

// ---------------------------------------------------------------------------
// Final prediction ("TTT-E2E：端到端测试时训练的长上下文语言建模", 持续学习框架,
// the 预测 step, and the final-prediction part of its inner-loop sketch): the
// prefill's forward and CE pass A at fixed weights W, b rows per sequence at a
// time, scored by the next-token loss.  No backward, no update.
// ---------------------------------------------------------------------------
template <typename T>
static cudaError_t enqueue_predict(ttt_handle* hd, const Plan& p, const float* hidden, const int* tokens,
                                   const float* W, float* group_loss, float* token_loss, char* ws,
                                   cudaStream_t st, Prof& prof) {
  const int B = p.B, b = p.b, n = p.n, d = p.d, h = p.h, V = p.V, L = p.L;
  T* Wsh = reinterpret_cast<T*>(ws + p.Wsh);
  float* resid = reinterpret_cast<float*>(ws + p.resid);
  T* z = reinterpret_cast<T*>(ws + p.z);
  float* rstd = reinterpret_cast<float*>(ws + p.rstd);
  float* part = reinterpret_cast<float*>(ws + p.part);
  float* tgt = reinterpret_cast<float*>(ws + p.tgt);
  float* lse = reinterpret_cast<float*>(ws + p.lse);
  float* ltok = reinterpret_cast<float*>(ws + p.ltok);
  const T* E = static_cast<const T*>(hd->E);
  int* status = hd->status;
  SplitScratch ss;
  if (p.sk_partial_bytes) {
    ss.partial = reinterpret_cast<float*>(ws + p.sk_partial);
    ss.partial_bytes = p.sk_partial_bytes;
    ss.counters = reinterpret_cast<int*>(ws + p.sk_counters);
    ss.counter_count = p.sk_counter_count;
  }
  cudaError_t err;
  const double e = (double)p.esz;
  if (p.sk_counter_count) TRY(cudaMemsetAsync(ws + p.sk_counters, 0, 4 * p.sk_counter_count, st));
  LAUNCH(K_SHADOW, 0, (4.0 + e) * B * L * p.m * h * d,
         (build_shadow_kernel<T><<<1184, 256, 0, st>>>(W, Wsh, (int64_t)B * L, h, d, p.swiglu ? 1 : 0)));
  for (int c = 0; c < p.nchunks; ++c) {
    const TokenMap tm{b, p.T, c};
    TRY(enqueue_forward<T>(hd, p, hidden, Wsh, c, false, nullptr, nullptr, ws, ss, st, prof));
    LAUNCH(K_RMS_FWD, 0, (4.0 + e) * n * d,
           (rmsnorm_fwd_kernel<T><<<(n + 7) / 8, 256, 0, st>>>(resid, hd->gain, hd->cfg.rms_eps, n, d, z, rstd)));
    {
      GemmShape s{n, V, d, 1};
      Operand A = opnd(z, d, 0, 1, n);
      Operand Be = opnd(E, d, 0, 1, V);
      LAUNCH(K_CE_LSE, 2.0 * n * V * d, e * ((double)n * d + (double)V * d) + 8.0 * n * p.ntn,
             TRY((gemm<T, 1>(s, A, A, Be, EpiCEPartial<T>{part, tgt, tokens, tm, p.ntn}, st, status, ss))));
    }
    LAUNCH(K_CE_ROWS, 0, 8.0 * n * p.ntn + (token_loss ? 20.0 : 16.0) * n,
           (ce_rows_kernel<<<(n + 7) / 8, 256, 0, st>>>(part, tgt, p.ntn, tokens, tm, V, n, lse, ltok, status,
                                                        token_loss)));
    LAUNCH(K_CE_MEAN, 0, 4.0 * n, (ce_mean_kernel<<<B, 256, 0, st>>>(ltok, b, group_loss, c, p.nchunks, status)));
  }
  return cudaSuccess;
}
#undef LAUNCH
#undef TRY

// Replays the graph captured for exactly this call, capturing it first when
// the slot holds another call's graph or none; with graphs off (TTT_GRAPH=0)
// the launches go straight to the caller's stream.
template <class Enqueue>
static ttt_status run_graph(ttt_handle* h, int slot, const CallKey& key, Enqueue enqueue, cudaStream_t st) {
  if (!h->use_graph) {
    cudaError_t e = enqueue(st);
    if (e != cudaSuccess) { set_last_error("enqueue", cudaGetErrorString(e), __FILE__, __LINE__); return TTT_ERR_CUDA; }
    return TTT_OK;
  }
  GraphSlot& g = h->graph[slot];
  if (!(g.have && g.key == key && g.exec)) {
    if (g.exec) { cudaGraphExecDestroy(g.exec); g.exec = nullptr; }
    g.have = false;
    TTT_CUDA_TRY(cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal));
    cudaError_t e = enqueue(h->cap);
    cudaGraph_t graph = nullptr;
    cudaError_t e2 = cudaStreamEndCapture(h->cap, &graph);
    if (e != cudaSuccess || e2 != cudaSuccess) {
      if (graph) cudaGraphDestroy(graph);
      set_last_error("capture", cudaGetErrorString(e != cudaSuccess ? e : e2), __FILE__, __LINE__);
      return TTT_ERR_CUDA;
    }
    e = cudaGraphInstantiate(&g.exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) {
      g.exec = nullptr;
      set_last_error("cudaGraphInstantiate", cudaGetErrorString(e), __FILE__, __LINE__);
      return TTT_ERR_CUDA;
    }
    g.key = key;
    g.have = true;
  }
  TTT_CUDA_TRY(cudaGraphLaunch(g.exec, st));
  return TTT_OK;
}

// ---------------------------------------------------------------------------
// Validation
// ---------------------------------------------------------------------------
static ttt_status check_config(const ttt_config* c) {
  if (!c) return fail(TTT_ERR_INVALID_ARG, "config is NULL");
  if (c->mlp != TTT_MLP_GELU && c->mlp != TTT_MLP_SWIGLU) return fail(TTT_ERR_INVALID_ARG, "mlp must be GELU or SwiGLU");
  if (c->precision != TTT_PREC_FP32 && c->precision != TTT_PREC_BF16)
    return fail(TTT_ERR_INVALID_ARG, "precision must be FP32 or BF16");
  if (c->has_static != 0 && c->has_static != 1) return fail(TTT_ERR_INVALID_ARG, "has_static must be 0 or 1");
  if (c->loss_reduction != TTT_REDUCE_MEAN && c->loss_reduction != TTT_REDUCE_SUM)
    return fail(TTT_ERR_INVALID_ARG, "loss_reduction must be MEAN or SUM");
  if (c->update_rule != TTT_RULE_E2TTT && c->update_rule != TTT_RULE_LACT)
    return fail(TTT_ERR_INVALID_ARG, "update_rule must be E2TTT or LACT");
  if (!(c->rms_eps >= 0.f) || !std::isfinite(c->rms_eps)) return fail(TTT_ERR_INVALID_ARG, "rms_eps must be finite and >= 0");
  if (c->head != TTT_HEAD_LM && c->head != TTT_HEAD_RECON) return fail(TTT_ERR_INVALID_ARG, "head must be LM or RECON");
  const bool recon = c->head == TTT_HEAD_RECON;
  if (recon && (c->n_blocks != 1 || c->has_static))
    return fail(TTT_ERR_UNSUPPORTED, "the reconstruction head takes one dynamic block and no static MLP");
  const int vocab = recon ? 16 : c->vocab;   // unused by the reconstruction head
  if (c->d < 16 || c->hidden < 16 || vocab < 16 || c->n_blocks < 1)
    return fail(TTT_ERR_SHAPE, "d, hidden, vocab must be >= 16 and n_blocks >= 1");
  if (c->d > 16384 || c->hidden > 65536 || vocab >= (1 << 26) || c->n_blocks > 64)
    return fail(TTT_ERR_SHAPE, "size above the supported maximum");
  if (c->d % 16 || c->hidden % 16 || vocab % 16)
    return fail(TTT_ERR_UNSUPPORTED, "d, hidden and vocab must be multiples of 16");
  return TTT_OK;
}

static ttt_status check_shape(const ttt_handle* h, int batch, int T, int b) {
  if (!h) return fail(TTT_ERR_INVALID_ARG, "handle is NULL");
  if (batch < 0 || T < 0) return fail(TTT_ERR_SHAPE, "batch and T must be >= 0");
  if (b < 1) return fail(TTT_ERR_SHAPE, "chunk size b must be >= 1");
  if (T % b != 0) return fail(TTT_ERR_SHAPE, "T must be a multiple of b");
  if ((int64_t)batch * b > (1 << 24)) return fail(TTT_ERR_SHAPE, "batch * b above 2^24 tokens per step");
  if ((int64_t)batch * T > ((int64_t)1 << 31) - 1) return fail(TTT_ERR_SHAPE, "batch * T above 2^31 - 1");
  if (h->attn_heads > 0 && b % 8) return fail(TTT_ERR_SHAPE, "with attention the chunk size b must be a multiple of 8");
  return TTT_OK;
}

}  // namespace ttt

using namespace ttt;

// ---------------------------------------------------------------------------
// Allocation-free prefill: scratch in a file-scope device array.
//
// For callers that must not allocate device memory while they run: programs
// whose device memory is budgeted once at start-up, hosts that own the
// allocator and forbid raw cudaMalloc, and latency-critical loops where the
// implicit device synchronisation of cudaMalloc / cudaFree is not acceptable.
// The scratch is kNoAllocScratchBytes of static device memory that every GPU
// loading this library holds until the process exits.
// ---------------------------------------------------------------------------
static constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[64] = {};                 // device address of the scratch, per device ordinal
static unsigned long long g_noalloc_ctx[64] = {};    // id of the context that address belongs to

// Unique id of this thread's current context (0 if none is current or the
// driver cannot say).  A device reset replaces the context, and the array's
// address in the new one has to be looked up again.
static unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static bool resolved = false;
  if (!resolved) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
    resolved = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch for the current device.  In host code the
// array's name is only a stand-in, so the address comes from
// cudaGetSymbolAddress, once per device and context, with that device current.
static ttt_status noalloc_scratch(void** out) {
  int dev = 0;
  TTT_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(TTT_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  const unsigned long long ctx = current_context_id();
  if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void* ptr = nullptr;
    TTT_CUDA_TRY(cudaGetSymbolAddress(&ptr, g_noalloc_scratch));
    g_noalloc_ptr[dev] = ptr;
    g_noalloc_ctx[dev] = current_context_id();   // the lookup made the device's context current
  }
  *out = g_noalloc_ptr[dev];
  return TTT_OK;
}

// ---------------------------------------------------------------------------
// Host-buffer prefill: the sequence in segments of whole chunks, the copy of
// segment s + 1's inputs (and of s + 2's, once slot s's compute is done)
// overlapping the compute of segment s.  Chunk-end state is the only carried
// state, so running the segments one after another on the same W and M gives
// the whole call's result bit for bit.
// ---------------------------------------------------------------------------
struct HostPlan {
  int seg_chunks = 0, nseg = 0, segT = 0, nchunks = 0;
  int64_t per_seq = 0;               // fast-weight parameters per sequence
  size_t W = 0, M = 0, loss = 0;     // offsets in the device buffer
  size_t slot[2] = {0, 0};           // input slots
  size_t hid = 0, tok = 0, eta = 0, beta = 0, gamma = 0;   // offsets inside a slot
  size_t ws = 0, ws_bytes = 0, total = 0;
};

static HostPlan make_host_plan(const ttt_handle* h, int B, int T, int b, int seg_chunks) {
  HostPlan q;
  q.nchunks = b > 0 ? T / b : 0;
  if (seg_chunks <= 0) seg_chunks = std::max(1, (q.nchunks + 7) / 8);
  // with attention a chunk reads the keys of earlier chunks, kept in the
  // workspace for one call: the whole sequence is one segment
  if (h->attn_heads > 0) seg_chunks = q.nchunks;
  seg_chunks = std::max(1, std::min(seg_chunks, std::max(q.nchunks, 1)));
  q.seg_chunks = seg_chunks;
  q.segT = seg_chunks * b;
  q.nseg = q.nchunks > 0 ? (q.nchunks + seg_chunks - 1) / seg_chunks : 0;
  const int m = h->cfg.mlp == TTT_MLP_SWIGLU ? 3 : 2;
  q.per_seq = (int64_t)h->cfg.n_blocks * m * h->cfg.hidden * h->cfg.d;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  q.W = take(4ull * B * q.per_seq);
  q.M = take(4ull * B * q.per_seq);
  q.loss = take(2 * 4ull * B * seg_chunks);   // one [B][seg_chunks] block per input slot
  const size_t n = (size_t)B * q.segT;
  size_t so = 0;
  auto stake = [&](size_t bytes) { size_t o = so; so = align_up(so + bytes, 256); return o; };
  q.hid = stake(4 * n * h->cfg.d);
  q.tok = stake(4 * n);
  q.eta = stake(4 * n);
  q.beta = stake(4 * n);
  q.gamma = stake(4 * n);
  q.slot[0] = take(so);
  q.slot[1] = take(so);
  q.ws_bytes = make_plan(h, B, q.segT, b).total;
  q.ws = take(q.ws_bytes);
  q.total = off;
  return q;
}

static ttt_status prefill_host_impl(ttt_handle* h, int B, int T, int b, const float* hidden, const int32_t* tokens,
                                    const float* W0, const float* M0, float* W, float* M, const float* eta,
                                    const float* beta, const float* gamma, float* chunk_loss, char* buf,
                                    const HostPlan& q, cudaStream_t st) {
  if (!h->copy) {
    TTT_CUDA_TRY(cudaStreamCreateWithFlags(&h->copy, cudaStreamNonBlocking));
    for (int i = 0; i < 2; ++i) {
      TTT_CUDA_TRY(cudaEventCreateWithFlags(&h->ev_copied[i], cudaEventDisableTiming));
      TTT_CUDA_TRY(cudaEventCreateWithFlags(&h->ev_consumed[i], cudaEventDisableTiming));
    }
  }
  const int64_t d = h->cfg.d;
  const size_t state = 4ull * B * q.per_seq;
  float* Wd = reinterpret_cast<float*>(buf + q.W);
  float* Md = reinterpret_cast<float*>(buf + q.M);
  TTT_CUDA_TRY(cudaMemcpyAsync(Wd, W0, state, cudaMemcpyHostToDevice, st));
  TTT_CUDA_TRY(cudaMemcpyAsync(Md, M0, state, cudaMemcpyHostToDevice, st));
  // segment s: chunks [s * seg_chunks, ...), Ts tokens per sequence
  auto seg_T = [&](int s) { return std::min(q.seg_chunks, q.nchunks - s * q.seg_chunks) * b; };
  auto copy_in = [&](int s) -> ttt_status {
    const int slot = s & 1;
    char* sb = buf + q.slot[slot];
    const size_t t0 = (size_t)s * q.segT, Ts = (size_t)seg_T(s);
    TTT_CUDA_TRY(cudaMemcpy2DAsync(sb + q.hid, 4 * Ts * d, hidden + t0 * d, 4 * (size_t)T * d, 4 * Ts * d, B,
                                   cudaMemcpyHostToDevice, h->copy));
    const void* src[4] = {tokens + t0, eta + t0, beta + t0, gamma + t0};
    const size_t dst[4] = {q.tok, q.eta, q.beta, q.gamma};
    for (int i = 0; i < 4; ++i)
      TTT_CUDA_TRY(cudaMemcpy2DAsync(sb + dst[i], 4 * Ts, src[i], 4 * (size_t)T, 4 * Ts, B, cudaMemcpyHostToDevice,
                                     h->copy));
    TTT_CUDA_TRY(cudaEventRecord(h->ev_copied[slot], h->copy));
    return TTT_OK;
  };
  ttt_status s0 = copy_in(0);
  if (s0 != TTT_OK) return s0;
  if (q.nseg > 1 && (s0 = copy_in(1)) != TTT_OK) return s0;
  char* ws = buf + q.ws;
  for (int s = 0; s < q.nseg; ++s) {
    const int slot = s & 1;
    const int Ts = seg_T(s);
    const size_t nc = (size_t)Ts / b;
    char* sb = buf + q.slot[slot];
    float* loss_s = reinterpret_cast<float*>(buf + q.loss) + (size_t)slot * B * q.seg_chunks;
    TTT_CUDA_TRY(cudaStreamWaitEvent(st, h->ev_copied[slot], 0));
    Plan p = make_plan(h, B, Ts, b);
    Prof prof;
    const float* hid = reinterpret_cast<const float*>(sb + q.hid);
    const int* tok = reinterpret_cast<const int*>(sb + q.tok);
    const float* et = reinterpret_cast<const float*>(sb + q.eta);
    const float* be = reinterpret_cast<const float*>(sb + q.beta);
    const float* ga = reinterpret_cast<const float*>(sb + q.gamma);
    auto enqueue = [&](cudaStream_t qs) -> cudaError_t {
      return enqueue_lm(h, p, hid, tok, Wd, Md, et, be, ga, loss_s, ws, qs, prof);
    };
    // one cached graph per input slot (and one for a shorter last segment):
    // the same pointers every segment and every call with these sizes
    CallKey key;
    key.batch = B; key.T = Ts; key.b = b; key.ws_bytes = q.ws_bytes;
    const void* ptrs[] = {hid, tok, Wd, Md, et, be, ga, loss_s, ws};
    std::copy(std::begin(ptrs), std::end(ptrs), key.ptr);
    const int gslot = Ts != q.segT ? SLOT_HOST_LAST : (slot ? SLOT_HOST1 : SLOT_HOST0);
    ttt_status r = run_graph(h, gslot, key, enqueue, st);
    if (r != TTT_OK) return r;
    // this segment's chunk losses out before the slot's next segment overwrites them
    TTT_CUDA_TRY(cudaMemcpy2DAsync(chunk_loss + (size_t)s * q.seg_chunks, 4 * (size_t)q.nchunks, loss_s, 4 * nc,
                                   4 * nc, B, cudaMemcpyDeviceToHost, st));
    TTT_CUDA_TRY(cudaEventRecord(h->ev_consumed[slot], st));
    if (s + 2 < q.nseg) {
      TTT_CUDA_TRY(cudaStreamWaitEvent(h->copy, h->ev_consumed[slot], 0));
      if ((s0 = copy_in(s + 2)) != TTT_OK) return s0;
    }
  }
  TTT_CUDA_TRY(cudaMemcpyAsync(W, Wd, state, cudaMemcpyDeviceToHost, st));
  TTT_CUDA_TRY(cudaMemcpyAsync(M, Md, state, cudaMemcpyDeviceToHost, st));
  TTT_CUDA_TRY(cudaStreamSynchronize(st));
  return TTT_OK;
}

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
extern "C" {

const char* ttt_status_string(ttt_status s) {
  switch (s) {
    case TTT_OK: return "ok";
    case TTT_ERR_INVALID_ARG: return "invalid argument";
    case TTT_ERR_SHAPE: return "invalid shape";
    case TTT_ERR_UNSUPPORTED: return "unsupported configuration";
    case TTT_ERR_WORKSPACE: return "workspace too small";
    case TTT_ERR_TOKEN_RANGE: return "token outside [0, vocab)";
    case TTT_ERR_NONFINITE: return "non-finite loss";
    case TTT_ERR_TIMEOUT: return "bounded wait timed out";
    case TTT_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* ttt_last_error(void) { return g_last_error.c_str(); }

ttt_status ttt_create(const ttt_config* cfg, const float* lm_head, const float* rms_gain,
                      const float* static_w, ttt_handle** out) {
  ttt_status s = check_config(cfg);
  if (s != TTT_OK) return s;
  const bool recon = cfg->head == TTT_HEAD_RECON;
  if (!out || (!recon && (!lm_head || !rms_gain)))
    return fail(TTT_ERR_INVALID_ARG, "lm_head, rms_gain and out must be non-NULL");
  if (cfg->has_static && !static_w) return fail(TTT_ERR_INVALID_ARG, "static_w is NULL but has_static = 1");
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return fail(TTT_ERR_UNSUPPORTED, "no CUDA device");
  }
  ttt_handle* h = new ttt_handle();
  h->cfg = *cfg;
  const char* env = getenv("TTT_GRAPH");
  h->use_graph = !(env && env[0] == '0');
  auto bail = [&](ttt_status st) { ttt_destroy(h); return st; };
#define CTRY(x) do { cudaError_t _e = (x); if (_e != cudaSuccess) { set_last_error(#x, cudaGetErrorString(_e), __FILE__, __LINE__); return bail(TTT_ERR_CUDA); } } while (0)
  CTRY(cudaGetDevice(&h->device));
  const int64_t V = cfg->vocab, d = cfg->d, hh = cfg->hidden;
  const int m = cfg->mlp == TTT_MLP_SWIGLU ? 3 : 2;
  const size_t esz = cfg->precision == TTT_PREC_FP32 ? 4 : 2;
  CTRY(cudaMalloc(&h->status, 8));
  h->zero_flag = h->status + 1;
  CTRY(cudaMemset(h->status, 0, 8));
  CTRY(cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking));
  const char* env_agg = getenv("TTT_AGG_STREAM");   // 0: aggregations on the caller's stream (A/B timing)
  h->agg_stream = !(env_agg && env_agg[0] == '0');
  CTRY(cudaStreamCreateWithFlags(&h->agg, cudaStreamNonBlocking));
  CTRY(cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming));
  CTRY(cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming));
  for (int i = 0; i < 3; ++i) {
    CTRY(cudaEventCreateWithFlags(&h->ev_up[i], cudaEventDisableTiming));
    CTRY(cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming));
  }
  if (!recon) {   // the frozen LM head and RMSNorm gain
    CTRY(cudaMalloc(&h->E, esz * V * d));
    CTRY(cudaMalloc(&h->gain, 4 * d));
    CTRY(cudaMemcpyAsync(h->gain, rms_gain, 4 * d, cudaMemcpyDeviceToDevice, h->cap));
    if (cfg->precision == TTT_PREC_FP32) {
      CTRY(cudaMemcpyAsync(h->E, lm_head, 4 * V * d, cudaMemcpyDeviceToDevice, h->cap));
    } else {
      cast_kernel<bf16><<<1184, 256, 0, h->cap>>>(lm_head, static_cast<bf16*>(h->E), V * d);
      CTRY(cudaGetLastError());
    }
  }
  if (cfg->has_static) {
    const int64_t count = cfg->n_blocks;
    CTRY(cudaMalloc(&h->S, esz * count * m * hh * d));
    if (cfg->precision == TTT_PREC_FP32)
      build_shadow_kernel<float><<<1184, 256, 0, h->cap>>>(static_w, static_cast<float*>(h->S), count, (int)hh, (int)d, m == 3);
    else
      build_shadow_kernel<bf16><<<1184, 256, 0, h->cap>>>(static_w, static_cast<bf16*>(h->S), count, (int)hh, (int)d, m == 3);
    CTRY(cudaGetLastError());
  }
  CTRY(cudaStreamSynchronize(h->cap));
#undef CTRY
  *out = h;
  return TTT_OK;
}

void ttt_destroy(ttt_handle* h) {
  if (!h) return;
  if (h->cap) cudaStreamSynchronize(h->cap);
  for (auto& g : h->graph)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  if (h->E) cudaFree(h->E);
  if (h->gain) cudaFree(h->gain);
  if (h->S) cudaFree(h->S);
  if (h->Wqkv) cudaFree(h->Wqkv);
  if (h->Wo) cudaFree(h->Wo);
  if (h->ln_gain) cudaFree(h->ln_gain);
  if (h->ln_bias) cudaFree(h->ln_bias);
  if (h->status) cudaFree(h->status);
  if (h->copy) { cudaStreamSynchronize(h->copy); cudaStreamDestroy(h->copy); }
  for (int i = 0; i < 2; ++i) {
    if (h->ev_copied[i]) cudaEventDestroy(h->ev_copied[i]);
    if (h->ev_consumed[i]) cudaEventDestroy(h->ev_consumed[i]);
  }
  if (h->agg) { cudaStreamSynchronize(h->agg); cudaStreamDestroy(h->agg); }
  for (cudaEvent_t ev : {h->ev_fork, h->ev_join, h->ev_up[0], h->ev_up[1], h->ev_up[2], h->ev_out[0], h->ev_out[1],
                         h->ev_out[2]})
    if (ev) cudaEventDestroy(ev);
  if (h->cap) cudaStreamDestroy(h->cap);
  delete h;
}

ttt_status ttt_set_attention(ttt_handle* h, int32_t n_heads, int32_t window, const float* attn_w,
                             const float* ln_gain, const float* ln_bias, float ln_eps) {
  if (!h) return fail(TTT_ERR_INVALID_ARG, "handle is NULL");
  if (h->cfg.head != TTT_HEAD_LM) return fail(TTT_ERR_UNSUPPORTED, "attention blocks need the LM head");
  if (n_heads < 0) return fail(TTT_ERR_INVALID_ARG, "n_heads must be >= 0");
  auto release = [&]() {
    cudaFree(h->Wqkv); cudaFree(h->Wo); cudaFree(h->ln_gain); cudaFree(h->ln_bias);
    h->Wqkv = h->Wo = nullptr;
    h->ln_gain = h->ln_bias = nullptr;
    h->attn_heads = 0;
    for (auto& g : h->graph) g.have = false;   // captured graphs hold the old layout
  };
  if (n_heads == 0) { release(); return TTT_OK; }
  const int d = h->cfg.d;
  if (d % n_heads) return fail(TTT_ERR_SHAPE, "d must be a multiple of n_heads");
  const int dh = d / n_heads;
  if (dh % 16) return fail(TTT_ERR_SHAPE, "the head size d / n_heads must be a multiple of 16");
  if (window < 1) return fail(TTT_ERR_INVALID_ARG, "window must be >= 1");
  if (!(ln_eps > 0.f) || !std::isfinite(ln_eps)) return fail(TTT_ERR_INVALID_ARG, "ln_eps must be positive and finite");
  if (!attn_w || !ln_gain || !ln_bias) return fail(TTT_ERR_INVALID_ARG, "a required pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(ln_gain) | reinterpret_cast<uintptr_t>(ln_bias)) % 16)
    return fail(TTT_ERR_INVALID_ARG, "ln_gain and ln_bias must be 16-byte aligned");
  release();
  const int64_t L = h->cfg.n_blocks, dd = (int64_t)d * d;
  const size_t esz = h->cfg.precision == TTT_PREC_FP32 ? 4 : 2;
  TTT_CUDA_TRY(cudaMalloc(&h->Wqkv, esz * L * 3 * dd));
  TTT_CUDA_TRY(cudaMalloc(&h->Wo, esz * L * dd));
  TTT_CUDA_TRY(cudaMalloc(&h->ln_gain, 4 * L * d));
  TTT_CUDA_TRY(cudaMalloc(&h->ln_bias, 4 * L * d));
  TTT_CUDA_TRY(cudaMemcpyAsync(h->ln_gain, ln_gain, 4 * L * d, cudaMemcpyDeviceToDevice, h->cap));
  TTT_CUDA_TRY(cudaMemcpyAsync(h->ln_bias, ln_bias, 4 * L * d, cudaMemcpyDeviceToDevice, h->cap));
  for (int64_t l = 0; l < L; ++l) {   // attn_w[l] = Wq, Wk, Wv, Wo: the first three are the fused q|k|v rows
    const float* src = attn_w + l * 4 * dd;
    if (h->cfg.precision == TTT_PREC_FP32) {
      TTT_CUDA_TRY(cudaMemcpyAsync(static_cast<float*>(h->Wqkv) + l * 3 * dd, src, 4 * 3 * dd, cudaMemcpyDeviceToDevice, h->cap));
      TTT_CUDA_TRY(cudaMemcpyAsync(static_cast<float*>(h->Wo) + l * dd, src + 3 * dd, 4 * dd, cudaMemcpyDeviceToDevice, h->cap));
    } else {
      cast_kernel<bf16><<<1184, 256, 0, h->cap>>>(src, static_cast<bf16*>(h->Wqkv) + l * 3 * dd, 3 * dd);
      cast_kernel<bf16><<<1184, 256, 0, h->cap>>>(src + 3 * dd, static_cast<bf16*>(h->Wo) + l * dd, dd);
      TTT_CUDA_TRY(cudaGetLastError());
    }
  }
  TTT_CUDA_TRY(cudaStreamSynchronize(h->cap));
  h->attn_heads = n_heads;
  h->attn_window = window;
  h->attn_ln_eps = ln_eps;
  return TTT_OK;
}

ttt_status ttt_workspace_size(const ttt_handle* h, int32_t batch, int32_t T, int32_t b, size_t* bytes) {
  ttt_status s = check_shape(h, batch, T, b);
  if (s != TTT_OK) return s;
  if (!bytes) return fail(TTT_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = make_plan(h, batch, T, b).total;
  return TTT_OK;
}

ttt_status ttt_prefill(ttt_handle* h, int32_t batch, int32_t T, int32_t b, const float* hidden,
                       const int32_t* tokens, float* W, float* M, const float* eta, const float* beta,
                       const float* gamma, float* chunk_loss, void* workspace, size_t ws_bytes,
                       void* stream) {
  ttt_status s = check_shape(h, batch, T, b);
  if (s != TTT_OK) return s;
  if (h->cfg.head != TTT_HEAD_LM) return fail(TTT_ERR_UNSUPPORTED, "the handle's head is the reconstruction layer: use ttt_prefill_recon");
  if (batch == 0 || T == 0) return TTT_OK;
  if (!hidden || !tokens || !W || !M || !eta || !beta || !gamma || !chunk_loss)
    return fail(TTT_ERR_INVALID_ARG, "a required pointer is NULL");
  Plan p = make_plan(h, batch, T, b);
  if (!workspace || ws_bytes < p.total) return fail(TTT_ERR_WORKSPACE, "workspace missing or too small");
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(M)) % 16)
    return fail(TTT_ERR_INVALID_ARG, "hidden, W and M must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);

  Prof prof;
  auto enqueue = [&](cudaStream_t q) -> cudaError_t {
    return enqueue_lm(h, p, hidden, tokens, W, M, eta, beta, gamma, chunk_loss, ws, q, prof);
  };

  CallKey key;
  key.batch = batch; key.T = T; key.b = b; key.ws_bytes = ws_bytes;
  const void* ptrs[] = {hidden, tokens, W, M, eta, beta, gamma, chunk_loss, workspace};
  std::copy(std::begin(ptrs), std::end(ptrs), key.ptr);
  return run_graph(h, SLOT_PREFILL, key, enqueue, st);
}

ttt_status ttt_host_buffer_size(const ttt_handle* h, int32_t batch, int32_t T, int32_t b, int32_t seg_chunks,
                                size_t* bytes) {
  ttt_status s = check_shape(h, batch, T, b);
  if (s != TTT_OK) return s;
  if (!bytes) return fail(TTT_ERR_INVALID_ARG, "bytes is NULL");
  if (h->cfg.head != TTT_HEAD_LM) return fail(TTT_ERR_UNSUPPORTED, "the host-buffer prefill serves the LM head");
  *bytes = make_host_plan(h, batch, T, b, seg_chunks).total;
  return TTT_OK;
}

ttt_status ttt_prefill_host(ttt_handle* h, int32_t batch, int32_t T, int32_t b, int32_t seg_chunks,
                            const float* hidden, const int32_t* tokens, const float* W0, const float* M0, float* W,
                            float* M, const float* eta, const float* beta, const float* gamma, float* chunk_loss,
                            void* device_buffer, size_t buffer_bytes, void* stream) {
  ttt_status s = check_shape(h, batch, T, b);
  if (s != TTT_OK) return s;
  if (h->cfg.head != TTT_HEAD_LM) return fail(TTT_ERR_UNSUPPORTED, "the host-buffer prefill serves the LM head");
  if (batch == 0 || T == 0) return TTT_OK;
  if (!hidden || !tokens || !W0 || !M0 || !W || !M || !eta || !beta || !gamma || !chunk_loss)
    return fail(TTT_ERR_INVALID_ARG, "a required pointer is NULL");
  const HostPlan q = make_host_plan(h, batch, T, b, seg_chunks);
  if (!device_buffer || buffer_bytes < q.total) return fail(TTT_ERR_WORKSPACE, "device buffer missing or too small");
  if (reinterpret_cast<uintptr_t>(device_buffer) % 256)
    return fail(TTT_ERR_INVALID_ARG, "device buffer must be 256-byte aligned");
  int dev = 0;
  TTT_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != h->device) return fail(TTT_ERR_INVALID_ARG, "the current device is not the handle's device");
  return prefill_host_impl(h, batch, T, b, hidden, tokens, W0, M0, W, M, eta, beta, gamma, chunk_loss,
                           static_cast<char*>(device_buffer), q, static_cast<cudaStream_t>(stream));
}

ttt_status ttt_prefill_recon(ttt_handle* h, int32_t batch, int32_t T, int32_t b, const float* K, const float* V,
                             const float* Q, float* W, float* M, const float* eta, const float* beta,
                             const float* gamma, float* O, float* chunk_loss, void* workspace, size_t ws_bytes,
                             void* stream) {
  ttt_status s = check_shape(h, batch, T, b);
  if (s != TTT_OK) return s;
  if (h->cfg.head != TTT_HEAD_RECON) return fail(TTT_ERR_UNSUPPORTED, "the handle's head is the LM head: use ttt_prefill");
  if (batch == 0 || T == 0) return TTT_OK;
  if (!K || !V || !Q || !W || !M || !eta || !beta || !gamma || !O || !chunk_loss)
    return fail(TTT_ERR_INVALID_ARG, "a required pointer is NULL");
  Plan p = make_plan(h, batch, T, b);
  if (!workspace || ws_bytes < p.total) return fail(TTT_ERR_WORKSPACE, "workspace missing or too small");
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(Q) |
       reinterpret_cast<uintptr_t>(O) | reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(M)) % 16)
    return fail(TTT_ERR_INVALID_ARG, "K, V, Q, O, W and M must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  Prof prof;
  auto enqueue = [&](cudaStream_t q) -> cudaError_t {
    if (h->cfg.precision == TTT_PREC_FP32)
      return enqueue_recon<float>(h, p, K, V, Q, W, M, eta, beta, gamma, O, chunk_loss, ws, q, prof);
    return enqueue_recon<bf16>(h, p, K, V, Q, W, M, eta, beta, gamma, O, chunk_loss, ws, q, prof);
  };
  CallKey key;
  key.batch = batch; key.T = T; key.b = b; key.ws_bytes = ws_bytes;
  const void* ptrs[] = {K, V, Q, W, M, eta, beta, gamma, O, chunk_loss, workspace};
  std::copy(std::begin(ptrs), std::end(ptrs), key.ptr);
  return run_graph(h, SLOT_RECON, key, enqueue, st);
}

ttt_status ttt_predict(ttt_handle* h, int32_t batch, int32_t T, int32_t b, const float* hidden,
                       const int32_t* tokens, const float* W, float* group_loss, float* token_loss,
                       void* workspace, size_t ws_bytes, void* stream) {
  ttt_status s = check_shape(h, batch, T, b);
  if (s != TTT_OK) return s;
  if (h->cfg.head != TTT_HEAD_LM) return fail(TTT_ERR_UNSUPPORTED, "the handle's head is the reconstruction layer: it has no next-token prediction");
  if (h->attn_heads > 0) return fail(TTT_ERR_UNSUPPORTED, "the final prediction does not run attention blocks");
  if (batch == 0 || T == 0) return TTT_OK;
  if (!hidden || !tokens || !W || !group_loss) return fail(TTT_ERR_INVALID_ARG, "a required pointer is NULL");
  Plan p = make_plan(h, batch, T, b);
  if (!workspace || ws_bytes < p.total) return fail(TTT_ERR_WORKSPACE, "workspace missing or too small");
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(W)) % 16)
    return fail(TTT_ERR_INVALID_ARG, "hidden and W must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  Prof prof;
  auto enqueue = [&](cudaStream_t q) -> cudaError_t {
    if (h->cfg.precision == TTT_PREC_FP32)
      return enqueue_predict<float>(h, p, hidden, tokens, W, group_loss, token_loss, ws, q, prof);
    return enqueue_predict<bf16>(h, p, hidden, tokens, W, group_loss, token_loss, ws, q, prof);
  };
  CallKey key;
  key.batch = batch; key.T = T; key.b = b; key.ws_bytes = ws_bytes;
  const void* ptrs[] = {hidden, tokens, W, group_loss, token_loss, workspace};
  std::copy(std::begin(ptrs), std::end(ptrs), key.ptr);
  return run_graph(h, SLOT_PREDICT, key, enqueue, st);
}

ttt_status ttt_prefill_profiled(ttt_handle* h, int32_t batch, int32_t T, int32_t b, const float* hidden,
                                const int32_t* tokens, float* W, float* M, const float* eta, const float* beta,
                                const float* gamma, float* chunk_loss, void* workspace, size_t ws_bytes,
                                void* stream, ttt_kernel_stat* stats, int32_t max_stats, int32_t* n_stats) {
  ttt_status s = check_shape(h, batch, T, b);
  if (s != TTT_OK) return s;
  if (h->cfg.head != TTT_HEAD_LM) return fail(TTT_ERR_UNSUPPORTED, "the handle's head is the reconstruction layer: use ttt_prefill_recon");
  if (!stats || !n_stats || max_stats < 0) return fail(TTT_ERR_INVALID_ARG, "stats / n_stats missing");
  *n_stats = 0;
  if (batch == 0 || T == 0) return TTT_OK;
  if (!hidden || !tokens || !W || !M || !eta || !beta || !gamma || !chunk_loss)
    return fail(TTT_ERR_INVALID_ARG, "a required pointer is NULL");
  Plan p = make_plan(h, batch, T, b);
  if (!workspace || ws_bytes < p.total) return fail(TTT_ERR_WORKSPACE, "workspace missing or too small");
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(M)) % 16)
    return fail(TTT_ERR_INVALID_ARG, "hidden, W and M must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  Prof prof;
  prof.timing = true;
  prof.recs.reserve(1 << 16);
  cudaError_t e = enqueue_lm(h, p, hidden, tokens, W, M, eta, beta, gamma, chunk_loss, ws, st, prof);
  if (e != cudaSuccess) { set_last_error("enqueue", cudaGetErrorString(e), __FILE__, __LINE__); return TTT_ERR_CUDA; }
  TTT_CUDA_TRY(cudaStreamSynchronize(st));
  ttt_kernel_stat agg[K_NCLASS];
  memset(agg, 0, sizeof(agg));
  for (const auto& r : prof.recs) {
    float ms = 0.f;
    TTT_CUDA_TRY(cudaEventElapsedTime(&ms, r.a, r.b));
    ttt_kernel_stat& a = agg[r.cls];
    a.launches += 1;
    a.ms += ms;
    a.flops += r.flops;
    a.bytes += r.bytes;
  }
  int32_t k = 0;
  for (int c = 0; c < K_NCLASS && k < max_stats; ++c) {
    if (agg[c].launches == 0) continue;
    stats[k] = agg[c];
    snprintf(stats[k].name, sizeof(stats[k].name), "%s", kClassName[c]);
    ++k;
  }
  *n_stats = k;
  return TTT_OK;
}

ttt_status ttt_scalar_kernels(int32_t rule, int32_t batch, int32_t T, int32_t b, const float* eta,
                              const float* beta, const float* gamma, float* KW, float* KM, float* consts,
                              void* stream) {
  if (rule != TTT_RULE_E2TTT && rule != TTT_RULE_LACT) return fail(TTT_ERR_INVALID_ARG, "unknown update rule");
  if (batch < 0 || T < 0) return fail(TTT_ERR_SHAPE, "batch and T must be >= 0");
  if (b < 1 || T % b) return fail(TTT_ERR_SHAPE, "b >= 1 and T % b == 0 required");
  if (batch == 0 || T == 0) return TTT_OK;
  if (!eta || !beta || !gamma || !KW || !KM || !consts) return fail(TTT_ERR_INVALID_ARG, "a required pointer is NULL");
  TTT_CUDA_TRY(launch_scalar_scan(rule, eta, beta, gamma, batch, T, b, KW, KM, consts,
                                  static_cast<cudaStream_t>(stream)));
  return TTT_OK;
}

ttt_status ttt_scalar_heads(int32_t batch, int32_t T, int32_t d, const float* hidden, const float* heads,
                            float b_eta, float b_beta, float b_alpha, float eta_base, float alpha_base,
                            float tau, float* eta, float* beta, float* gamma, void* stream) {
  if (batch < 0 || T < 0 || d < 4 || d % 4) return fail(TTT_ERR_SHAPE, "batch, T >= 0 and d >= 4, d % 4 == 0 required");
  if (!(tau > 0.f) || !std::isfinite(tau)) return fail(TTT_ERR_INVALID_ARG, "tau must be positive and finite");
  if (batch == 0 || T == 0) return TTT_OK;
  if (!hidden || !heads || !eta || !beta || !gamma) return fail(TTT_ERR_INVALID_ARG, "a required pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(heads)) % 16)
    return fail(TTT_ERR_INVALID_ARG, "hidden and heads must be 16-byte aligned");
  const int64_t rows = (int64_t)batch * T;
  scalar_heads_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      hidden, rows, d, heads, b_eta, b_beta, b_alpha, eta_base, alpha_base, 1.f / tau, eta, beta, gamma);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

ttt_status ttt_prefill_noalloc(ttt_handle* h, int32_t batch, int32_t T, int32_t b, const float* hidden,
                               const int32_t* tokens, float* W, float* M, const float* eta, const float* beta,
                               const float* gamma, float* chunk_loss, void* stream) {
  ttt_status s = check_shape(h, batch, T, b);
  if (s != TTT_OK) return s;
  if (h->cfg.head != TTT_HEAD_LM) return fail(TTT_ERR_UNSUPPORTED, "the handle's head is the reconstruction layer: use ttt_prefill_recon");
  if (batch == 0 || T == 0) return TTT_OK;
  if (!hidden || !tokens || !W || !M || !eta || !beta || !gamma || !chunk_loss)
    return fail(TTT_ERR_INVALID_ARG, "a required pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(M)) % 16)
    return fail(TTT_ERR_INVALID_ARG, "hidden, W and M must be 16-byte aligned");
  Plan p = make_plan(h, batch, T, b);
  if (p.total > kNoAllocScratchBytes) {
    static thread_local char msg[160];
    snprintf(msg, sizeof(msg), "ttt_prefill_noalloc needs %zu bytes of scratch; its static scratch holds %zu bytes",
             p.total, kNoAllocScratchBytes);
    return fail(TTT_ERR_WORKSPACE, msg);
  }
  int dev = 0;
  TTT_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != h->device) return fail(TTT_ERR_INVALID_ARG, "the current device is not the handle's device");
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != TTT_OK) return s;
  // Every buffer of the plan is written before it is read within the call
  // (the split-K counters are cleared by the call itself), so the scratch
  // needs no clearing between calls.
  Prof prof;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(scratch);
  cudaError_t e = enqueue_lm(h, p, hidden, tokens, W, M, eta, beta, gamma, chunk_loss, ws, st, prof);
  if (e != cudaSuccess) { set_last_error("enqueue", cudaGetErrorString(e), __FILE__, __LINE__); return TTT_ERR_CUDA; }
  return TTT_OK;
}

ttt_status ttt_gemm_bf16(int32_t M, int32_t N, int32_t K, int32_t batch, const void* A, int64_t lda,
                         int64_t strideA, int32_t a_kmajor, const void* B, int64_t ldb, int64_t strideB,
                         int32_t b_kmajor, float* D, int64_t ldd, int64_t strideD, void* workspace,
                         size_t ws_bytes, void* stream) {
  if (M < 0 || N < 0 || K < 0 || batch < 0) return fail(TTT_ERR_SHAPE, "negative size");
  if (M == 0 || N == 0 || K == 0 || batch == 0) return TTT_OK;
  if (!A || !B || !D) return fail(TTT_ERR_INVALID_ARG, "a required pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B)) % 16 || lda % 8 || ldb % 8 ||
      strideA % 8 || strideB % 8)
    return fail(TTT_ERR_UNSUPPORTED, "operands need 16-byte aligned bases and strides multiple of 8 elements");
  if (lda < (a_kmajor ? K : M) || ldb < (b_kmajor ? K : N) || ldd < N)
    return fail(TTT_ERR_SHAPE, "leading dimension smaller than the matrix");
  if (batch > 1 && (strideA == 0 || strideB == 0))
    return fail(TTT_ERR_UNSUPPORTED, "batched operands need nonzero strides");
  GemmShape s{M, N, K, batch};
  Operand a = opnd(A, lda, strideA, a_kmajor ? 1 : 0, a_kmajor ? M : K);
  Operand b = opnd(B, ldb, strideB, b_kmajor ? 1 : 0, b_kmajor ? N : K);
  EpiStoreBatched e{D, ldd, strideD};
  SplitScratch ss;
  if (workspace && ws_bytes >= (size_t(1) << 20)) {
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    // counters first (zeroed here), the rest holds split-K partial tiles
    ss.counters = static_cast<int*>(workspace);
    ss.counter_count = 65536;
    ss.partial = reinterpret_cast<float*>(static_cast<char*>(workspace) + 4 * ss.counter_count);
    ss.partial_bytes = ws_bytes - 4 * ss.counter_count;
    TTT_CUDA_TRY(cudaMemsetAsync(ss.counters, 0, 4 * ss.counter_count, static_cast<cudaStream_t>(stream)));
  }
  TTT_CUDA_TRY((tc::launch_gemm_tc<1, EpiStoreBatched>(s, a, a, b, e, static_cast<cudaStream_t>(stream), nullptr, ss)));
  return TTT_OK;
}

ttt_status ttt_get_device_status(ttt_handle* h, void* stream) {
  if (!h) return fail(TTT_ERR_INVALID_ARG, "handle is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  TTT_CUDA_TRY(cudaStreamSynchronize(st));
  int v = 0;
  TTT_CUDA_TRY(cudaMemcpy(&v, h->status, 4, cudaMemcpyDeviceToHost));
  TTT_CUDA_TRY(cudaMemset(h->status, 0, 4));
  return static_cast<ttt_status>(v);
}

ttt_status ttt_selftest_bounded_wait(ttt_handle* h, uint32_t spin_limit, void* stream) {
  if (!h) return fail(TTT_ERR_INVALID_ARG, "handle is NULL");
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(h->zero_flag, spin_limit, h->status);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

}  // extern "C"
