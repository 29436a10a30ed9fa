// C ABI of libmla.so (declared in include/mla.h): validation, workspace layout, dispatch.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <new>

#include "mla.h"
#include "common.cuh"
#include "simt.cuh"
#include "tc.cuh"

struct mla_handle {
  mla_dims_t dims;
  mla_dtype_t dtype;
  int device;
  mla_weights_t w;
  bool has_weights;
  uint32_t* d_err;         // device error word (sticky until mla_sync_status)
  uint32_t last_err_bits;  // last word read by mla_sync_status
  int num_sms;
  mla::LayerOpts opts;     // RMSNorm gains and the RoPE (plain or YaRN)
};

namespace mla {
static std::atomic<unsigned long long> g_launches{0};
void note_launch(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// Kernel timing: one event pair per timed kernel, created on the device of the first bracketed launch.
static std::atomic<bool> g_timing{false};
static cudaEvent_t g_ev[TIMED_KERNELS][2];
static bool g_ev_made = false;
static bool g_ev_recorded[TIMED_KERNELS] = {false, false};
static std::mutex g_timing_mu;
void timer_begin(TimedKernel k, cudaStream_t st) {
  if (!g_timing.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lock(g_timing_mu);
  if (!g_ev_made) {
    for (int i = 0; i < TIMED_KERNELS; ++i)
      for (int j = 0; j < 2; ++j) cudaEventCreate(&g_ev[i][j]);
    g_ev_made = true;
  }
  cudaEventRecord(g_ev[k][0], st);
}
void timer_end(TimedKernel k, cudaStream_t st) {
  if (!g_timing.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lock(g_timing_mu);
  if (!g_ev_made) return;
  cudaEventRecord(g_ev[k][1], st);
  g_ev_recorded[k] = true;
}
}  // namespace mla

namespace {

using mla::SimtAttnArgs;
using mla::SimtGemmArgs;

constexpr size_t kAlign = 1024;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t elem_size(const mla_handle* h) { return h->dtype == MLA_BF16 ? 2 : 4; }

// The sizes the tcgen05/TMA kernels are built for: the DeepSeek-V3 head layout, d and d_c'
// multiples of 64. BF16 handles exist only at these sizes (mla_create).
bool v3_dims(const mla_dims_t& d) {
  return d.n_h == 128 && d.d_h == 128 && d.d_c == 512 && d.d_r == 64 && d.d_cq % 64 == 0 && d.d % 64 == 0;
}

// BF16 handles run on the tcgen05/TMA kernels; FP32 handles on the generic CUDA-core kernels.
bool tc_dims(const mla_handle* h) { return h->dtype == MLA_BF16; }

// Makes the handle's device current for the life of the guard and restores the caller's device
// afterwards, so that no entry point changes the calling thread's current device.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int device) {
    if (cudaGetDevice(&prev) != cudaSuccess) return;
    ok = prev == device || cudaSetDevice(device) == cudaSuccess;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

struct Layout {
  size_t off[9];
  bool has[9];
  size_t pos_off;     // int64 positions [T]
  size_t slot_off;    // int64 cache rows [T] (chunked prefill only)
  size_t tc_off;      // tensor-core attention scratch
  size_t total;
};

// Workspace layout of one call; every region starts on a 1024-byte boundary. A chunked prefill
// (kv_rows >= 0) takes the decode layout (absorbed form, B sequences of tq tokens) or the prefill
// layout with k^C / v^C over kv_rows key rows (unabsorbed form), plus the chunk's cache rows.
Layout layout(const mla_handle* h, mla_op_t op, int64_t B, int32_t tq, int64_t total_tokens,
              int64_t kv_rows = -1) {
  Layout L;
  memset(&L, 0, sizeof(L));
  const mla_dims_t& d = h->dims;
  const size_t es = elem_size(h);
  const int64_t T = (op == MLA_OP_DECODE || op == MLA_OP_ATTN_DECODE_LATENT) ? B * tq : total_tokens;
  size_t cur = 0;
  auto take = [&](int which, size_t bytes) {
    L.off[which] = cur;
    L.has[which] = true;
    cur = align_up(cur + bytes);
  };
  if (op == MLA_OP_DECODE || op == MLA_OP_PREFILL) {
    take(MLA_BUF_CQ, (size_t)T * d.d_cq * es);
    take(MLA_BUF_QC, (size_t)T * d.n_h * d.d_h * es);
    take(MLA_BUF_QR, (size_t)T * d.n_h * d.d_r * es);
    take(MLA_BUF_O, (size_t)T * d.n_h * d.d_h * es);
  }
  if (op == MLA_OP_DECODE) {
    take(MLA_BUF_QABS, (size_t)T * d.n_h * d.d_c * es);
    take(MLA_BUF_OLAT, (size_t)T * d.n_h * d.d_c * es);
    take(MLA_BUF_LSE, (size_t)T * d.n_h * sizeof(float));
  }
  if (op == MLA_OP_PREFILL) {
    const int64_t KV = kv_rows >= 0 ? kv_rows : T;
    take(MLA_BUF_KC, (size_t)KV * d.n_h * d.d_h * es);
    take(MLA_BUF_VC, (size_t)KV * d.n_h * d.d_h * es);
  }
  if (op != MLA_OP_CACHE_APPEND) {
    L.pos_off = cur;
    cur = align_up(cur + (size_t)(T > 0 ? T : 1) * sizeof(int64_t));
  }
  if (kv_rows >= 0) {
    L.slot_off = cur;
    cur = align_up(cur + (size_t)(T > 0 ? T : 1) * sizeof(int64_t));
  }
  if (tc_dims(h)) {
    L.tc_off = cur;
    if (op == MLA_OP_DECODE && kv_rows >= 0) {
      // the chunk's cache rows are written first, with the same scratch
      const size_t a = mla::tc_decode_scratch_bytes(d, B, tq), b = mla::tc_append_scratch_bytes(d, T);
      cur = align_up(cur + (a > b ? a : b));
    }
    if (op == MLA_OP_DECODE && kv_rows < 0) cur = align_up(cur + mla::tc_decode_scratch_bytes(d, B, tq));
    if (op == MLA_OP_ATTN_DECODE_LATENT) cur = align_up(cur + mla::tc_core_scratch_bytes(d, B, tq));
    if (op == MLA_OP_CACHE_APPEND)
      cur = align_up(cur + mla::tc_append_scratch_bytes(d, total_tokens, h->opts.cache_fp8 != 0));
  }
  L.total = cur;
  return L;
}

mla_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

#define MLA_TRY(expr)                              \
  do {                                             \
    cudaError_t _e = (expr);                       \
    if (_e != cudaSuccess) return MLA_ERR_CUDA;    \
  } while (0)

// Allocates the handle's error word on first use. The caller holds a DeviceGuard for h->device.
mla_status_t ensure_device(mla_handle* h) {
  if (!h->d_err) {
    MLA_TRY(cudaMalloc(&h->d_err, sizeof(uint32_t)));
    MLA_TRY(cudaMemset(h->d_err, 0, sizeof(uint32_t)));
    int sms = 0;
    MLA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, h->device));
    h->num_sms = sms;
  }
  return MLA_OK;
}

// --- generic (CUDA-core) building blocks ----------------------------------------------------
SimtGemmArgs gemm_args() {
  SimtGemmArgs a;
  memset(&a, 0, sizeof(a));
  a.batch = 1;
  return a;
}

// C[M, N] = A[M, K] . W[N, K]^T with dense row-major A (row stride lda) and W.
SimtGemmArgs dense_nt(const void* A, int64_t lda, const void* W, void* C, int64_t ldc, int64_t M, int64_t N,
                      int64_t K) {
  SimtGemmArgs a = gemm_args();
  a.A = A; a.sam = lda; a.sak = 1;
  a.B = W; a.sbn = K; a.sbk = 1;
  a.C = C; a.scm = ldc; a.scn = 1;
  a.M = M; a.N = N; a.K = K;
  return a;
}

mla_status_t run_simt_gemm(const mla_handle* h, SimtGemmArgs a, cudaStream_t st) {
  a.err = h->d_err;
  return cuda_status(mla::simt_gemm(a, st));
}

// Steps (5), (7) + cache write: rows [c^KV | RoPE(W^KR h)] scattered to cache[rowmap[t]].
mla_status_t simt_cache_rows(const mla_handle* h, const void* hidden, const int64_t* pos, const int64_t* rowmap,
                             int64_t T, void* cache, int64_t capacity, cudaStream_t st) {
  const mla_dims_t& d = h->dims;
  const size_t es = elem_size(h);
  const int64_t R = d.d_c + d.d_r;
  SimtGemmArgs a = dense_nt(hidden, d.d, h->w.w_dkv, cache, R, T, d.d_c, d.d);
  a.rowmap = rowmap; a.rowmap_limit = capacity;
  mla_status_t s = run_simt_gemm(h, a, st);
  if (s != MLA_OK) return s;
  if (h->opts.g_kv)
    MLA_TRY(mla::rmsnorm_rows(cache, h->dtype == MLA_BF16, R, rowmap, capacity, T, d.d_c, h->opts.g_kv, h->opts.eps,
                              st));
  SimtGemmArgs b = dense_nt(hidden, d.d, h->w.w_kr, (char*)cache + (size_t)d.d_c * es, R, T, d.d_r, d.d);
  b.rowmap = rowmap; b.rowmap_limit = capacity;
  b.pos = pos; b.rope_col0 = 0; b.d_r = d.d_r; b.rope = h->opts.rope;
  return run_simt_gemm(h, b, st);
}

// Steps (1)-(3): c^Q, q^C and the rotated q^R of T tokens at positions pos.
mla_status_t simt_queries(const mla_handle* h, const void* hidden, const int64_t* pos, int64_t T, void* cq,
                          void* qc, void* qr, cudaStream_t st) {
  const mla_dims_t& d = h->dims;
  mla_status_t s = run_simt_gemm(h, dense_nt(hidden, d.d, h->w.w_dq, cq, d.d_cq, T, d.d_cq, d.d), st);
  if (s != MLA_OK) return s;
  if (h->opts.g_q)
    MLA_TRY(mla::rmsnorm_rows(cq, h->dtype == MLA_BF16, d.d_cq, nullptr, T, T, d.d_cq, h->opts.g_q, h->opts.eps, st));
  s = run_simt_gemm(h, dense_nt(cq, d.d_cq, h->w.w_uq, qc, (int64_t)d.n_h * d.d_h, T, (int64_t)d.n_h * d.d_h,
                                d.d_cq), st);
  if (s != MLA_OK) return s;
  SimtGemmArgs a = dense_nt(cq, d.d_cq, h->w.w_qr, qr, (int64_t)d.n_h * d.d_r, T, (int64_t)d.n_h * d.d_r, d.d_cq);
  a.pos = pos; a.rope_col0 = 0; a.d_r = d.d_r; a.rope = h->opts.rope;
  return run_simt_gemm(h, a, st);
}

// Step (10), second equation: u = W^O [o_1; ...; o_nh].
mla_status_t simt_output(const mla_handle* h, const void* o, int64_t T, void* u, cudaStream_t st) {
  const mla_dims_t& d = h->dims;
  const int64_t HD = (int64_t)d.n_h * d.d_h;
  return run_simt_gemm(h, dense_nt(o, HD, h->w.w_o, u, d.d, T, d.d, HD), st);
}

// Latent attention core by CUDA cores: q~ [T, n_h, d_c], q^R [T, n_h, d_r] over the cache.
mla_status_t simt_latent_core(const mla_handle* h, const void* q_abs, const void* q_rope, int64_t B, int32_t tq,
                              const int64_t* cu, const void* cache, int64_t capacity, void* o_lat, bool o_f32,
                              float* lse, cudaStream_t st) {
  const mla_dims_t& d = h->dims;
  const size_t es = elem_size(h);
  const int64_t R = d.d_c + d.d_r;
  SimtAttnArgs a;
  memset(&a, 0, sizeof(a));
  a.q1 = q_abs; a.sq1t = (int64_t)d.n_h * d.d_c; a.sq1h = d.d_c; a.d1 = d.d_c;
  a.q2 = q_rope; a.sq2t = (int64_t)d.n_h * d.d_r; a.sq2h = d.d_r; a.d2 = d.d_r;
  a.k1 = cache; a.sk1 = R; a.sk1h = 0;
  a.k2 = (const char*)cache + (size_t)d.d_c * es; a.sk2 = R;
  a.v = cache; a.sv = R; a.svh = 0; a.dv = d.d_c;
  a.o = o_lat; a.sot = (int64_t)d.n_h * d.d_c; a.soh = d.d_c;
  a.lse = lse;
  a.cu = cu; a.B = B; a.tq = tq; a.T = B * tq; a.n_h = d.n_h; a.capacity = capacity;
  a.scale = (float)(1.0 / sqrt((double)(d.d_h + d.d_r)));
  a.err = h->d_err;
  (void)o_f32;
  return cuda_status(mla::simt_attention(a, st));
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: null pointer, bad size or bad enum";
    case MLA_ERR_ALIGNMENT: return "MLA_ERR_ALIGNMENT: device pointer not 16-byte aligned";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: no kernel for these dims/dtype";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace smaller than mla_workspace_size()";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: a CUDA runtime call failed";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT: a bounded device-side wait gave up";
    case MLA_ERR_DEVICE_CHECK: return "MLA_ERR_DEVICE_CHECK: device-side argument check failed";
    case MLA_ERR_NO_WEIGHTS: return "MLA_ERR_NO_WEIGHTS: mla_set_weights() not called";
    case MLA_ERR_SCRATCH_LIMIT:
      return "MLA_ERR_SCRATCH_LIMIT: the call needs more than the 4 MiB fixed scratch of mla_cache_append_noalloc";
  }
  return "MLA_ERR_UNKNOWN";
}

mla_status_t mla_create(const mla_dims_t* dims, mla_dtype_t dtype, int device, mla_handle_t** out) {
  if (!dims || !out) return MLA_ERR_INVALID_ARG;
  *out = nullptr;
  const mla_dims_t& d = *dims;
  if (d.d <= 0 || d.n_h <= 0 || d.d_h <= 0 || d.d_c <= 0 || d.d_cq <= 0 || d.d_r <= 0 || (d.d_r & 1) ||
      !(d.rope_base > 1.0) || device < 0)
    return MLA_ERR_INVALID_ARG;
  if (dtype != MLA_BF16 && dtype != MLA_FP32) return MLA_ERR_INVALID_ARG;
  // BF16 runs on the tcgen05 kernels, which are built for the DeepSeek-V3 head layout only.
  if (dtype == MLA_BF16 && !v3_dims(d)) return MLA_ERR_UNSUPPORTED;
  // Generic kernels hold one latent row of q in shared memory and up to 512 value columns.
  if (d.d_c > 512 || d.d_h > 512 || d.d_c + d.d_r > 1024 || d.d_h + d.d_r > 1024) return MLA_ERR_UNSUPPORTED;
  mla_handle* h = new (std::nothrow) mla_handle;
  if (!h) return MLA_ERR_INVALID_ARG;
  memset(h, 0, sizeof(*h));
  h->dims = d;
  h->dtype = dtype;
  h->device = device;
  h->opts.eps = 1e-6f;
  h->opts.rope = mla::RopeSpec{d.rope_base, 1.0, 1.0, 32.0, 4096.0};
  *out = h;
  return MLA_OK;
}

mla_status_t mla_set_rmsnorm(mla_handle_t* h, const void* g_q, const void* g_kv, double eps) {
  if (!h || (!g_q) != (!g_kv) || !(eps >= 0.0)) return MLA_ERR_INVALID_ARG;
  if ((g_q && !aligned16(g_q)) || (g_kv && !aligned16(g_kv))) return MLA_ERR_ALIGNMENT;
  h->opts.g_q = g_q;
  h->opts.g_kv = g_kv;
  h->opts.eps = (float)eps;
  return MLA_OK;
}

mla_status_t mla_set_cache_format(mla_handle_t* h, mla_cache_format_t format) {
  if (!h || (format != MLA_CACHE_BF16 && format != MLA_CACHE_FP8)) return MLA_ERR_INVALID_ARG;
  if (format == MLA_CACHE_FP8 && !tc_dims(h)) return MLA_ERR_UNSUPPORTED;
  h->opts.cache_fp8 = format == MLA_CACHE_FP8 ? 1 : 0;
  return MLA_OK;
}

mla_status_t mla_cache_quantize_fp8(mla_handle_t* h, const void* rows, int64_t n, void* out, mla_stream_t stream) {
  if (!h || !rows || !out || n <= 0) return MLA_ERR_INVALID_ARG;
  if (!tc_dims(h)) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(rows) || !aligned16(out)) return MLA_ERR_ALIGNMENT;
  DeviceGuard g(h->device);
  if (!g.ok) return MLA_ERR_CUDA;
  mla_status_t s = ensure_device(h);
  if (s != MLA_OK) return s;
  return cuda_status(mla::fp8_quantize_rows(rows, n, nullptr, n, out, h->d_err, (cudaStream_t)stream));
}

mla_status_t mla_set_yarn(mla_handle_t* h, double s, double alpha, double beta, double original_len) {
  if (!h || !(s >= 1.0) || !(beta > alpha) || !(original_len > 0.0)) return MLA_ERR_INVALID_ARG;
  h->opts.rope = mla::RopeSpec{h->dims.rope_base, s, alpha, beta, original_len};
  return MLA_OK;
}

mla_status_t mla_set_weights(mla_handle_t* h, const mla_weights_t* w) {
  if (!h || !w) return MLA_ERR_INVALID_ARG;
  const void* ps[8] = {w->w_dq, w->w_uq, w->w_qr, w->w_dkv, w->w_kr, w->w_uk, w->w_uv, w->w_o};
  for (const void* p : ps) {
    if (!p) return MLA_ERR_INVALID_ARG;
    if (!aligned16(p)) return MLA_ERR_ALIGNMENT;
  }
  DeviceGuard g(h->device);
  if (!g.ok) return MLA_ERR_CUDA;
  mla_status_t s = ensure_device(h);
  if (s != MLA_OK) return s;
  h->w = *w;
  h->has_weights = true;
  return MLA_OK;
}

mla_status_t mla_workspace_size(const mla_handle_t* h, mla_op_t op, int64_t num_seqs, int32_t tq,
                                int64_t total_tokens, size_t* bytes) {
  if (!h || !bytes) return MLA_ERR_INVALID_ARG;
  if (op < MLA_OP_CACHE_APPEND || op > MLA_OP_ATTN_DECODE_LATENT) return MLA_ERR_INVALID_ARG;
  if (op == MLA_OP_DECODE || op == MLA_OP_ATTN_DECODE_LATENT) {
    if (num_seqs <= 0 || (tq != 1 && tq != 2)) return MLA_ERR_INVALID_ARG;
  } else if (total_tokens <= 0) {
    return MLA_ERR_INVALID_ARG;
  }
  *bytes = layout(h, op, num_seqs, tq, total_tokens).total;
  return MLA_OK;
}

mla_status_t mla_workspace_offset(const mla_handle_t* h, mla_op_t op, int64_t num_seqs, int32_t tq,
                                  int64_t total_tokens, mla_buffer_t which, size_t* offset) {
  size_t total = 0;
  mla_status_t s = mla_workspace_size(h, op, num_seqs, tq, total_tokens, &total);
  if (s != MLA_OK) return s;
  if (!offset || which < MLA_BUF_CQ || which > MLA_BUF_LSE) return MLA_ERR_INVALID_ARG;
  Layout L = layout(h, op, num_seqs, tq, total_tokens);
  if (!L.has[which]) return MLA_ERR_INVALID_ARG;
  *offset = L.off[which];
  return MLA_OK;
}

namespace {

constexpr int64_t kAbsorbedChunkMax = 64;   // the latent core runs one row of clusters per chunk token

// Resolves the form of a chunked prefill; false if the arguments or the forced form do not fit.
bool chunk_form(int64_t B, int64_t total_q, int64_t max_q, int64_t total_kv, mla_chunk_form_t form,
                mla_chunk_form_t* chosen) {
  if (B <= 0 || total_q <= 0 || max_q <= 0 || total_kv < total_q) return false;
  if (form != MLA_CHUNK_AUTO && form != MLA_CHUNK_ABSORBED && form != MLA_CHUNK_UNABSORBED) return false;
  const bool uniform = total_q == B * max_q && max_q <= kAbsorbedChunkMax;
  if (form == MLA_CHUNK_ABSORBED && !uniform) return false;
  if (form == MLA_CHUNK_AUTO) form = (uniform && total_kv >= 2 * total_q) ? MLA_CHUNK_ABSORBED : MLA_CHUNK_UNABSORBED;
  *chosen = form;
  return true;
}

Layout chunk_layout(const mla_handle* h, int64_t B, int64_t total_q, int64_t max_q, int64_t total_kv,
                    mla_chunk_form_t chosen) {
  return chosen == MLA_CHUNK_ABSORBED ? layout(h, MLA_OP_DECODE, B, (int32_t)max_q, 0, total_kv)
                                      : layout(h, MLA_OP_PREFILL, B, 0, total_q, total_kv);
}

}  // namespace

mla_status_t mla_prefill_chunk_workspace(const mla_handle_t* h, int64_t B, int64_t total_q, int64_t max_q,
                                         int64_t total_kv, mla_chunk_form_t form, mla_chunk_form_t* chosen,
                                         size_t* bytes) {
  mla_chunk_form_t f;
  if (!h || !bytes || !chunk_form(B, total_q, max_q, total_kv, form, &f)) return MLA_ERR_INVALID_ARG;
  if (chosen) *chosen = f;
  *bytes = chunk_layout(h, B, total_q, max_q, total_kv, f).total;
  return MLA_OK;
}

mla_status_t mla_prefill_chunk_offset(const mla_handle_t* h, int64_t B, int64_t total_q, int64_t max_q,
                                      int64_t total_kv, mla_chunk_form_t form, mla_buffer_t which,
                                      size_t* offset) {
  mla_chunk_form_t f;
  if (!h || !offset || !chunk_form(B, total_q, max_q, total_kv, form, &f)) return MLA_ERR_INVALID_ARG;
  if (which < MLA_BUF_CQ || which > MLA_BUF_LSE) return MLA_ERR_INVALID_ARG;
  Layout L = chunk_layout(h, B, total_q, max_q, total_kv, f);
  if (!L.has[which]) return MLA_ERR_INVALID_ARG;
  *offset = L.off[which];
  return MLA_OK;
}

int mla_uses_tensor_cores(const mla_handle_t* h, mla_op_t op) {
  if (!h || op < MLA_OP_CACHE_APPEND || op > MLA_OP_ATTN_DECODE_LATENT) return 0;
  return tc_dims(h) ? 1 : 0;
}

mla_status_t mla_cache_append(mla_handle_t* h, const void* hidden, const int64_t* positions, const int64_t* slots,
                              int64_t T, void* cache, int64_t capacity, void* ws, size_t ws_bytes,
                              mla_stream_t stream) {
  if (!h || !hidden || !positions || !slots || !cache || T <= 0 || capacity <= 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(cache) || !aligned16(positions) || !aligned16(slots) ||
      (ws && !aligned16(ws)))
    return MLA_ERR_ALIGNMENT;
  Layout L = layout(h, MLA_OP_CACHE_APPEND, 0, 1, T);
  if (ws_bytes < L.total || (L.total > 0 && !ws)) return MLA_ERR_WORKSPACE;
  if (!h->has_weights) return MLA_ERR_NO_WEIGHTS;
  DeviceGuard g(h->device);
  if (!g.ok) return MLA_ERR_CUDA;
  mla_status_t s = ensure_device(h);
  if (s != MLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (tc_dims(h))
    return cuda_status(mla::tc_cache_append(h->dims, h->w, h->opts, hidden, positions, slots, T, cache, capacity,
                                            (char*)ws + L.tc_off, L.total - L.tc_off, h->d_err, st));
  return simt_cache_rows(h, hidden, positions, slots, T, cache, capacity, st);
}

mla_status_t mla_attn_decode_latent(mla_handle_t* h, const void* q_abs, const void* q_rope, int64_t B, int32_t Tq,
                                    const int64_t* cu_seqlens, const void* cache, int64_t capacity, float* o_lat,
                                    float* lse, void* ws, size_t ws_bytes, mla_stream_t stream) {
  if (!h || !q_abs || !q_rope || !cu_seqlens || !cache || !o_lat || !lse || B <= 0 || capacity <= 0)
    return MLA_ERR_INVALID_ARG;
  if (Tq != 1 && Tq != 2) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_abs) || !aligned16(q_rope) || !aligned16(cache) || !aligned16(o_lat) || !aligned16(lse) ||
      !aligned16(cu_seqlens) || (ws && !aligned16(ws)))
    return MLA_ERR_ALIGNMENT;
  Layout L = layout(h, MLA_OP_ATTN_DECODE_LATENT, B, Tq, 0);
  if (ws_bytes < L.total || (L.total > 0 && !ws)) return MLA_ERR_WORKSPACE;
  DeviceGuard g(h->device);
  if (!g.ok) return MLA_ERR_CUDA;
  mla_status_t s = ensure_device(h);  // the core needs no weights
  if (s != MLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  char* w = (char*)ws;
  if (tc_dims(h)) {
    // the device checks ride in the core's plan launch
    MLA_TRY(mla::tc_core_prepare(cu_seqlens, B, Tq, capacity, nullptr, w + L.tc_off, h->num_sms, h->d_err, st));
    return cuda_status(mla::tc_core_run(q_abs, q_rope, B, Tq, cu_seqlens, cache, capacity, h->opts.cache_fp8 != 0,
                                        o_lat, true, lse, w + L.tc_off, h->num_sms, h->d_err, st));
  }
  MLA_TRY(mla::check_and_positions(cu_seqlens, B, Tq, B * Tq, capacity, 0, (int64_t*)(w + L.pos_off), h->d_err,
                                   st));
  return simt_latent_core(h, q_abs, q_rope, B, Tq, cu_seqlens, cache, capacity, o_lat, true, lse, st);
}

namespace {

// Decode steps after the position check (absorbed form, Tq tokens per sequence, positions in pos).
mla_status_t decode_steps(mla_handle* h, const void* h_q, int64_t B, int32_t Tq, const int64_t* cu,
                          const int64_t* pos, const void* cache, int64_t capacity, void* u_out, char* w,
                          const Layout& L, cudaStream_t st) {
  const mla_dims_t& d = h->dims;
  const int64_t T = B * Tq;
  void* cq = w + L.off[MLA_BUF_CQ];
  void* qc = w + L.off[MLA_BUF_QC];
  void* qr = w + L.off[MLA_BUF_QR];
  void* qabs = w + L.off[MLA_BUF_QABS];
  void* olat = w + L.off[MLA_BUF_OLAT];
  void* o = w + L.off[MLA_BUF_O];
  float* lse = (float*)(w + L.off[MLA_BUF_LSE]);
  if (tc_dims(h))
    return cuda_status(mla::tc_decode(d, h->w, h->opts, h_q, B, Tq, cu, pos, cache, capacity, u_out, cq, qc, qr, qabs,
                                      olat, o, lse, w + L.tc_off, h->num_sms, h->d_err, st));
  // Steps (1)-(3)
  mla_status_t s = simt_queries(h, h_q, pos, T, cq, qc, qr, st);
  if (s != MLA_OK) return s;
  // q~_i = W_i^UK^T q^C_i (batched over heads): A(t, k) = q^C[t, i d_h + k], B(c, k) = W^UK[i d_h + k, c]
  SimtGemmArgs a = gemm_args();
  a.A = qc; a.sam = (int64_t)d.n_h * d.d_h; a.sak = 1; a.sab = d.d_h;
  a.B = h->w.w_uk; a.sbn = 1; a.sbk = d.d_c; a.sbb = (int64_t)d.d_h * d.d_c;
  a.C = qabs; a.scm = (int64_t)d.n_h * d.d_c; a.scn = 1; a.scb = d.d_c;
  a.M = T; a.N = d.d_c; a.K = d.d_h; a.batch = d.n_h;
  s = run_simt_gemm(h, a, st);
  if (s != MLA_OK) return s;
  s = simt_latent_core(h, qabs, qr, B, Tq, cu, cache, capacity, olat, h->dtype == MLA_FP32, lse, st);
  if (s != MLA_OK) return s;
  // o_i = W_i^UV o^lat_i: A(t, c) = o^lat[t, i, c], B(k, c) = W^UV[i d_h + k, c]
  SimtGemmArgs v = gemm_args();
  v.A = olat; v.sam = (int64_t)d.n_h * d.d_c; v.sak = 1; v.sab = d.d_c;
  v.B = h->w.w_uv; v.sbn = d.d_c; v.sbk = 1; v.sbb = (int64_t)d.d_h * d.d_c;
  v.C = o; v.scm = (int64_t)d.n_h * d.d_h; v.scn = 1; v.scb = d.d_h;
  v.M = T; v.N = d.d_h; v.K = d.d_c; v.batch = d.n_h;
  s = run_simt_gemm(h, v, st);
  if (s != MLA_OK) return s;
  return simt_output(h, o, T, u_out, st);
}

// Unabsorbed prefill steps after the position check: T query tokens packed by cu at positions pos,
// their cache rows at slots (nullptr: row t); key rows packed by cu_kv (nullptr: cu_kv = cu).
mla_status_t prefill_steps(mla_handle* h, const void* hidden, int64_t B, const int64_t* cu, const int64_t* cu_kv,
                           int64_t T, int64_t T_kv, int64_t max_q, const int64_t* pos, const int64_t* slots,
                           void* cache, int64_t capacity, void* u_out, char* w, const Layout& L, cudaStream_t st) {
  const mla_dims_t& d = h->dims;
  const size_t es = elem_size(h);
  const int64_t R = d.d_c + d.d_r, HD = (int64_t)d.n_h * d.d_h;
  if (!cu_kv) T_kv = T;
  void* cq = w + L.off[MLA_BUF_CQ];
  void* qc = w + L.off[MLA_BUF_QC];
  void* qr = w + L.off[MLA_BUF_QR];
  void* o = w + L.off[MLA_BUF_O];
  void* kc = w + L.off[MLA_BUF_KC];
  void* vc = w + L.off[MLA_BUF_VC];
  if (tc_dims(h))
    return cuda_status(mla::tc_prefill(d, h->w, h->opts, hidden, B, cu, cu_kv, T, T_kv, max_q, pos, slots, cache,
                                       capacity, u_out, cq, qc, qr, kc, vc, o, h->num_sms, h->d_err, st));
  // Steps (5), (7): the tokens' cache rows
  mla_status_t s = simt_cache_rows(h, hidden, pos, slots, T, cache, capacity, st);
  if (s != MLA_OK) return s;
  s = simt_queries(h, hidden, pos, T, cq, qc, qr, st);
  if (s != MLA_OK) return s;
  // Steps (6), (9): k^C = W^UK c^KV, v^C = W^UV c^KV from every key row
  s = run_simt_gemm(h, dense_nt(cache, R, h->w.w_uk, kc, HD, T_kv, HD, d.d_c), st);
  if (s != MLA_OK) return s;
  s = run_simt_gemm(h, dense_nt(cache, R, h->w.w_uv, vc, HD, T_kv, HD, d.d_c), st);
  if (s != MLA_OK) return s;
  // Steps (4), (8), (10): causal attention per head with keys [k^C_i; k^R], values v^C_i
  SimtAttnArgs a;
  memset(&a, 0, sizeof(a));
  a.q1 = qc; a.sq1t = HD; a.sq1h = d.d_h; a.d1 = d.d_h;
  a.q2 = qr; a.sq2t = (int64_t)d.n_h * d.d_r; a.sq2h = d.d_r; a.d2 = d.d_r;
  a.k1 = kc; a.sk1 = HD; a.sk1h = d.d_h;
  a.k2 = (const char*)cache + (size_t)d.d_c * es; a.sk2 = R;
  a.v = vc; a.sv = HD; a.svh = d.d_h; a.dv = d.d_h;
  a.o = o; a.sot = HD; a.soh = d.d_h;
  a.lse = nullptr;
  a.cu = cu; a.cu_kv = cu_kv; a.B = B; a.tq = 0; a.T = T; a.n_h = d.n_h; a.capacity = capacity;
  a.scale = (float)(1.0 / sqrt((double)(d.d_h + d.d_r)));
  a.err = h->d_err;
  MLA_TRY(mla::simt_attention(a, st));
  return simt_output(h, o, T, u_out, st);
}

}  // namespace

mla_status_t mla_decode(mla_handle_t* h, const void* h_q, int64_t B, int32_t Tq, const int64_t* cu_seqlens,
                        const void* cache, int64_t capacity, void* u_out, void* ws, size_t ws_bytes,
                        mla_stream_t stream) {
  if (!h || !h_q || !cu_seqlens || !cache || !u_out || !ws || B <= 0 || capacity <= 0) return MLA_ERR_INVALID_ARG;
  if (Tq != 1 && Tq != 2) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h_q) || !aligned16(cache) || !aligned16(u_out) || !aligned16(ws) || !aligned16(cu_seqlens))
    return MLA_ERR_ALIGNMENT;
  Layout L = layout(h, MLA_OP_DECODE, B, Tq, 0);
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  if (!h->has_weights) return MLA_ERR_NO_WEIGHTS;
  DeviceGuard g(h->device);
  if (!g.ok) return MLA_ERR_CUDA;
  mla_status_t s = ensure_device(h);
  if (s != MLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  char* w = (char*)ws;
  int64_t* pos = (int64_t*)(w + L.pos_off);
  // the tensor-core path runs the device checks and writes the positions in its core's plan launch
  if (!tc_dims(h)) MLA_TRY(mla::check_and_positions(cu_seqlens, B, Tq, B * Tq, capacity, 0, pos, h->d_err, st));
  return decode_steps(h, h_q, B, Tq, cu_seqlens, pos, cache, capacity, u_out, w, L, st);
}

mla_status_t mla_prefill(mla_handle_t* h, const void* hidden, int64_t B, const int64_t* cu_seqlens,
                         int64_t total_tokens, int64_t max_seqlen, void* cache, int64_t capacity, void* u_out,
                         void* ws, size_t ws_bytes, mla_stream_t stream) {
  if (h && h->opts.cache_fp8) return MLA_ERR_UNSUPPORTED;   // FP8 caches: append and decode only
  if (!h || !hidden || !cu_seqlens || !cache || !u_out || !ws || B <= 0 || total_tokens <= 0 || max_seqlen <= 0 ||
      capacity < total_tokens)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(cache) || !aligned16(u_out) || !aligned16(ws) || !aligned16(cu_seqlens))
    return MLA_ERR_ALIGNMENT;
  Layout L = layout(h, MLA_OP_PREFILL, B, 0, total_tokens);
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  if (!h->has_weights) return MLA_ERR_NO_WEIGHTS;
  DeviceGuard g(h->device);
  if (!g.ok) return MLA_ERR_CUDA;
  mla_status_t s = ensure_device(h);
  if (s != MLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  char* w = (char*)ws;
  int64_t* pos = (int64_t*)(w + L.pos_off);
  MLA_TRY(mla::check_and_positions(cu_seqlens, B, 0, total_tokens, capacity, max_seqlen, pos, h->d_err, st));
  return prefill_steps(h, hidden, B, cu_seqlens, nullptr, total_tokens, total_tokens, max_seqlen, pos, nullptr, cache,
                       capacity, u_out, w, L, st);
}

mla_status_t mla_prefill_chunk(mla_handle_t* h, const void* hidden, int64_t B, const int64_t* cu_q, int64_t total_q,
                               int64_t max_q, const int64_t* cu_kv, int64_t total_kv, void* cache, int64_t capacity,
                               mla_chunk_form_t form, void* u_out, void* ws, size_t ws_bytes, mla_stream_t stream) {
  if (h && h->opts.cache_fp8) return MLA_ERR_UNSUPPORTED;   // FP8 caches: append and decode only
  mla_chunk_form_t f;
  if (!h || !hidden || !cu_q || !cu_kv || !cache || !u_out || !ws || capacity < total_kv ||
      !chunk_form(B, total_q, max_q, total_kv, form, &f))
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(cache) || !aligned16(u_out) || !aligned16(ws) || !aligned16(cu_q) ||
      !aligned16(cu_kv))
    return MLA_ERR_ALIGNMENT;
  Layout L = chunk_layout(h, B, total_q, max_q, total_kv, f);
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  if (!h->has_weights) return MLA_ERR_NO_WEIGHTS;
  DeviceGuard g(h->device);
  if (!g.ok) return MLA_ERR_CUDA;
  mla_status_t s = ensure_device(h);
  if (s != MLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  char* w = (char*)ws;
  int64_t* pos = (int64_t*)(w + L.pos_off);
  int64_t* slots = (int64_t*)(w + L.slot_off);
  MLA_TRY(mla::check_chunk_positions(cu_q, cu_kv, B, total_q, total_kv, capacity, max_q, pos, slots, h->d_err, st));
  if (f == MLA_CHUNK_UNABSORBED)
    return prefill_steps(h, hidden, B, cu_q, cu_kv, total_q, total_kv, max_q, pos, slots, cache, capacity, u_out, w,
                         L, st);
  // Absorbed: the chunk's cache rows first (steps (5), (7)), then the decode steps with Tq = Tc,
  // whose query k of sequence b sits at position len_b - Tc + k, the same position as above.
  const int32_t tc = (int32_t)max_q;
  if (tc_dims(h)) {
    const size_t scratch = mla::tc_append_scratch_bytes(h->dims, total_q);
    MLA_TRY(mla::tc_cache_append(h->dims, h->w, h->opts, hidden, pos, slots, total_q, cache, capacity, w + L.tc_off,
                                 scratch, h->d_err, st));
  } else {
    s = simt_cache_rows(h, hidden, pos, slots, total_q, cache, capacity, st);
    if (s != MLA_OK) return s;
  }
  return decode_steps(h, hidden, B, tc, cu_kv, pos, cache, capacity, u_out, w, L, st);
}

mla_status_t mla_attn_prefill(mla_handle_t* h, const void* q_c, const void* q_rope, const void* k_c, const void* v_c,
                              int64_t B, const int64_t* cu_seqlens, int64_t total_tokens, int64_t max_seqlen,
                              const void* cache, int64_t capacity, void* o, mla_stream_t stream) {
  if (h && h->opts.cache_fp8) return MLA_ERR_UNSUPPORTED;   // FP8 caches: append and decode only
  if (!h || !q_c || !q_rope || !k_c || !v_c || !cu_seqlens || !cache || !o || B <= 0 || total_tokens <= 0 ||
      max_seqlen <= 0 || capacity < total_tokens)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_c) || !aligned16(q_rope) || !aligned16(k_c) || !aligned16(v_c) || !aligned16(cache) ||
      !aligned16(o) || !aligned16(cu_seqlens))
    return MLA_ERR_ALIGNMENT;
  DeviceGuard g(h->device);
  if (!g.ok) return MLA_ERR_CUDA;
  mla_status_t s = ensure_device(h);  // the core needs no weights
  if (s != MLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  const mla_dims_t& d = h->dims;
  const int64_t T = total_tokens, R = d.d_c + d.d_r, HD = (int64_t)d.n_h * d.d_h;
  MLA_TRY(mla::check_and_positions(cu_seqlens, B, 0, T, capacity, max_seqlen, nullptr, h->d_err, st));
  if (tc_dims(h))
    return cuda_status(mla::tc_prefill_attention(q_c, q_rope, k_c, v_c, cache, capacity, cu_seqlens, nullptr, B, T, T,
                                                 max_seqlen, o, h->num_sms, h->d_err, st));
  SimtAttnArgs a;
  memset(&a, 0, sizeof(a));
  a.q1 = q_c; a.sq1t = HD; a.sq1h = d.d_h; a.d1 = d.d_h;
  a.q2 = q_rope; a.sq2t = (int64_t)d.n_h * d.d_r; a.sq2h = d.d_r; a.d2 = d.d_r;
  a.k1 = k_c; a.sk1 = HD; a.sk1h = d.d_h;
  a.k2 = (const char*)cache + (size_t)d.d_c * elem_size(h); a.sk2 = R;
  a.v = v_c; a.sv = HD; a.svh = d.d_h; a.dv = d.d_h;
  a.o = o; a.sot = HD; a.soh = d.d_h;
  a.lse = nullptr;
  a.cu = cu_seqlens; a.B = B; a.tq = 0; a.T = T; a.n_h = d.n_h; a.capacity = capacity;
  a.scale = (float)(1.0 / sqrt((double)(d.d_h + d.d_r)));
  a.err = h->d_err;
  return cuda_status(mla::simt_attention(a, st));
}

mla_status_t mla_sync_status(mla_handle_t* h, mla_stream_t stream) {
  if (!h) return MLA_ERR_INVALID_ARG;
  if (!h->d_err) return MLA_OK;
  DeviceGuard g(h->device);
  if (!g.ok) return MLA_ERR_CUDA;
  MLA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
  uint32_t bits = 0;
  MLA_TRY(cudaMemcpy(&bits, h->d_err, sizeof(bits), cudaMemcpyDeviceToHost));
  MLA_TRY(cudaMemset(h->d_err, 0, sizeof(uint32_t)));
  h->last_err_bits = bits;
  if (bits & mla::DEVERR_TIMEOUT) return MLA_ERR_TIMEOUT;
  if (bits) return MLA_ERR_DEVICE_CHECK;
  return MLA_OK;
}

uint32_t mla_device_error_bits(const mla_handle_t* h) { return h ? h->last_err_bits : 0u; }

uint64_t mla_kernel_launches(void) { return mla::g_launches.load(std::memory_order_relaxed); }

void mla_test_arm_stall(void) { mla::tc_latent_core_arm_stall(); }

mla_status_t mla_set_kernel_timing(int enabled) {
  mla::g_timing.store(enabled != 0, std::memory_order_relaxed);
  return MLA_OK;
}

mla_status_t mla_kernel_time_ms(int which, float* ms) {
  if (!ms || which < 0 || which >= mla::TIMED_KERNELS) return MLA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(mla::g_timing_mu);
  if (!mla::g_ev_made || !mla::g_ev_recorded[which]) return MLA_ERR_INVALID_ARG;
  MLA_TRY(cudaEventSynchronize(mla::g_ev[which][1]));
  MLA_TRY(cudaEventElapsedTime(ms, mla::g_ev[which][0], mla::g_ev[which][1]));
  return MLA_OK;
}

void mla_destroy(mla_handle_t* h) {
  if (!h) return;
  if (h->d_err) {
    DeviceGuard g(h->device);
    cudaFree(h->d_err);
  }
  delete h;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// mla_cache_append_noalloc: the cache append for callers that cannot allocate. Its split-K
// scratch is this fixed device array; host code never touches the array's name as an address
// but asks the runtime for the device address once per device.
// ---------------------------------------------------------------------------------------------

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_noalloc_addr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on `device` (which must be current), looked up once.
mla_status_t noalloc_scratch(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return MLA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[device]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
    g_noalloc_addr[device] = p;
  }
  *out = g_noalloc_addr[device];
  return MLA_OK;
}

}  // namespace

extern "C" mla_status_t mla_cache_append_noalloc(mla_handle_t* h, const void* hidden, const int64_t* positions,
                                                 const int64_t* slots, int64_t T, void* cache, int64_t capacity,
                                                 mla_stream_t stream) {
  if (h && h->opts.cache_fp8) return MLA_ERR_UNSUPPORTED;   // FP8 caches: append and decode only
  if (!h || !hidden || !positions || !slots || !cache || T <= 0 || capacity <= 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(cache) || !aligned16(positions) || !aligned16(slots))
    return MLA_ERR_ALIGNMENT;
  // mla_set_weights() already allocated the error word; this call allocates nothing itself.
  if (!h->has_weights || !h->d_err) return MLA_ERR_NO_WEIGHTS;
  Layout L = layout(h, MLA_OP_CACHE_APPEND, 0, 1, T);
  if (L.total > kNoAllocScratchBytes) return MLA_ERR_SCRATCH_LIMIT;
  DeviceGuard g(h->device);
  if (!g.ok) return MLA_ERR_CUDA;
  void* scratch = nullptr;
  mla_status_t s = noalloc_scratch(h->device, &scratch);
  if (s != MLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (tc_dims(h))
    return cuda_status(mla::tc_cache_append(h->dims, h->w, h->opts, hidden, positions, slots, T, cache, capacity,
                                            (char*)scratch + L.tc_off, L.total - L.tc_off, h->d_err, st));
  return simt_cache_rows(h, hidden, positions, slots, T, cache, capacity, st);
}
