// Tensor-core op sequences (BF16, DeepSeek-V3 sizes): the projection GEMMs on tcgen05, the
// latent attention core, the output projection. Steps follow section 一(一) of the DeepSeek-V3
// notes: (1)-(3) queries, (5)/(7) cache rows, the absorbed core, then W^UV and W^O.
#include <string.h>

#include "simt.cuh"
#include "tc.cuh"
#include "tc_gemm.cuh"

namespace mla {
namespace {

constexpr size_t kAlign = 1024;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

TcMatrix mat(const void* p, int64_t rows, int64_t cols, int64_t ld) {
  TcMatrix m;
  m.ptr = p; m.rows = rows; m.cols = cols; m.ld = ld;
  return m;
}

TcEpiSeg epi(void* out, int64_t so_t, int64_t so_f, int64_t f_rows) {
  TcEpiSeg e;
  memset(&e, 0, sizeof(e));
  e.out = out; e.so_t = so_t; e.so_f = so_f; e.f_rows = f_rows;
  return e;
}

TcGemmDesc desc(const TcMatrix& x, int64_t T, int64_t K, uint32_t* err) {
  TcGemmDesc g;
  memset(&g, 0, sizeof(g));
  g.x = x; g.T = T; g.K = K; g.batch = 1; g.err = err;
  return g;
}

int64_t tiles128(int64_t n) { return (n + 127) / 128; }

size_t decode_gemm_partials(const mla_dims_t& d, int64_t T) {
  const int64_t HD = (int64_t)d.n_h * d.d_h, HR = (int64_t)d.n_h * d.d_r;
  const size_t a = tc_gemm_partial_bytes(T, tiles128(d.d_cq), d.d_cq, d.d, 1);                      // W^DQ
  const size_t b = tc_gemm_partial_bytes(T, tiles128(HD) + tiles128(HR), HD + HR, d.d_cq, 1);       // [W^UQ; W^QR]
  const size_t c = tc_gemm_partial_bytes(T, tiles128(d.d), d.d, HD, 1);                             // W^O
  const size_t ab = a > b ? a : b;
  return align_up(ab > c ? ab : c);
}

// Steps (5) and (7) with the cache write: rows [c^KV | RoPE(W^KR h)] -> cache[rowmap[t]], then the
// optional RMSNorm of c^KV in place. With an FP8 cache the rows go to `staging` ([T][576] bf16) first,
// are normalised there, and are quantized into the cache rows.
cudaError_t cache_rows(const mla_dims_t& d, const mla_weights_t& w, const LayerOpts& o, const void* hidden,
                       const int64_t* pos, const int64_t* rowmap, int64_t T, void* cache, int64_t capacity,
                       void* scratch, size_t scratch_bytes, void* staging, uint32_t* err, cudaStream_t st) {
  const int64_t R = d.d_c + d.d_r;
  const bool fp8 = o.cache_fp8 && staging;
  void* dst = fp8 ? staging : cache;
  const int64_t* map = fp8 ? nullptr : rowmap;
  const int64_t limit = fp8 ? T : capacity;
  TcGemmDesc g = desc(mat(hidden, T, d.d, d.d), T, d.d, err);
  g.nseg = 2;
  g.seg[0].w = mat(w.w_dkv, d.d_c, d.d, d.d);
  g.seg[0].epi = epi(dst, R, 1, d.d_c);
  g.seg[1].w = mat(w.w_kr, d.d_r, d.d, d.d);
  g.seg[1].epi = epi((char*)dst + (size_t)d.d_c * 2, R, 1, d.d_r);
  g.seg[1].epi.rope = 1;
  for (int s = 0; s < 2; ++s) {
    g.seg[s].epi.rowmap = map;
    g.seg[s].epi.rowmap_limit = limit;
  }
  g.pos = pos; g.d_r = d.d_r; g.rope = o.rope;
  g.partial = (float*)scratch; g.partial_bytes = scratch_bytes;
  cudaError_t e = tc_gemm(g, st);
  if (e != cudaSuccess) return e;
  if (o.g_kv && (e = rmsnorm_rows(dst, true, R, map, limit, T, d.d_c, o.g_kv, o.eps, st)) != cudaSuccess) return e;
  // the projection wrote the staged rows without the slots, so the quantizer checks them
  return fp8 ? fp8_quantize_rows(staging, T, rowmap, capacity, cache, err, st) : cudaSuccess;
}

// Steps (1)-(3): c^Q = W^DQ h (then the optional RMSNorm); q^C = W^UQ c^Q; q^R = RoPE(W^QR c^Q).
cudaError_t queries(const mla_dims_t& d, const mla_weights_t& w, const LayerOpts& o, const void* hidden,
                    const int64_t* pos, int64_t T, void* cq, void* qc, void* qr, void* scratch, size_t scratch_bytes,
                    uint32_t* err, cudaStream_t st) {
  const int64_t HD = (int64_t)d.n_h * d.d_h, HR = (int64_t)d.n_h * d.d_r;
  TcGemmDesc a = desc(mat(hidden, T, d.d, d.d), T, d.d, err);
  a.nseg = 1;
  a.seg[0].w = mat(w.w_dq, d.d_cq, d.d, d.d);
  a.seg[0].epi = epi(cq, d.d_cq, 1, d.d_cq);
  a.partial = (float*)scratch; a.partial_bytes = scratch_bytes;
  cudaError_t e = tc_gemm(a, st);
  if (e != cudaSuccess) return e;
  if (o.g_q && (e = rmsnorm_rows(cq, true, d.d_cq, nullptr, T, T, d.d_cq, o.g_q, o.eps, st)) != cudaSuccess) return e;
  TcGemmDesc b = desc(mat(cq, T, d.d_cq, d.d_cq), T, d.d_cq, err);
  b.nseg = 2;
  b.seg[0].w = mat(w.w_uq, HD, d.d_cq, d.d_cq);
  b.seg[0].epi = epi(qc, HD, 1, HD);
  b.seg[1].w = mat(w.w_qr, HR, d.d_cq, d.d_cq);
  b.seg[1].epi = epi(qr, HR, 1, HR);
  b.seg[1].epi.rope = 1;
  b.pos = pos; b.d_r = d.d_r; b.rope = o.rope;
  b.partial = (float*)scratch; b.partial_bytes = scratch_bytes;
  return tc_gemm(b, st);
}

// Step (10), second equation: u = W^O [o_1; ...; o_nh].
cudaError_t output(const mla_dims_t& d, const mla_weights_t& w, const void* o, int64_t T, void* u, void* scratch,
                   size_t scratch_bytes, uint32_t* err, cudaStream_t st) {
  const int64_t HD = (int64_t)d.n_h * d.d_h;
  TcGemmDesc g = desc(mat(o, T, HD, HD), T, HD, err);
  g.nseg = 1;
  g.seg[0].w = mat(w.w_o, d.d, HD, HD);
  g.seg[0].epi = epi(u, d.d, 1, d.d);
  g.partial = (float*)scratch; g.partial_bytes = scratch_bytes;
  return tc_gemm(g, st);
}

}  // namespace

size_t tc_decode_scratch_bytes(const mla_dims_t& d, int64_t B, int32_t tq) {
  return decode_gemm_partials(d, B * tq) + align_up(tc_core_scratch_bytes(d, B, tq));
}

size_t tc_append_scratch_bytes(const mla_dims_t& d, int64_t T, bool fp8) {
  return align_up(tc_gemm_partial_bytes(T, tiles128(d.d_c) + tiles128(d.d_r), d.d_c + d.d_r, d.d, 1)) +
         (fp8 ? align_up(fp8_staging_bytes(T)) : 0);
}

cudaError_t tc_cache_append(const mla_dims_t& d, const mla_weights_t& w, const LayerOpts& o, const void* hidden,
                            const int64_t* positions, const int64_t* slots, int64_t T, void* cache,
                            int64_t capacity, void* scratch, size_t scratch_bytes, uint32_t* err,
                            cudaStream_t st) {
  // FP8: the bf16 rows are staged at the end of the scratch, after the split-K partials
  const size_t stage = o.cache_fp8 ? align_up(fp8_staging_bytes(T)) : 0;
  if (scratch_bytes < stage) return cudaErrorInvalidValue;
  void* staging = o.cache_fp8 ? (char*)scratch + (scratch_bytes - stage) : nullptr;
  return cache_rows(d, w, o, hidden, positions, slots, T, cache, capacity, scratch, scratch_bytes - stage, staging, err,
                    st);
}

cudaError_t tc_decode(const mla_dims_t& d, const mla_weights_t& w, const LayerOpts& lo, const void* h_q, int64_t B,
                      int32_t tq,
                      const int64_t* cu, const int64_t* pos, const void* cache, int64_t capacity, void* u_out,
                      void* cq, void* qc, void* qr, void* qabs, void* olat, void* o, float* lse, void* scratch,
                      int num_sms, uint32_t* err, cudaStream_t st) {
  const int64_t T = B * tq, HD = (int64_t)d.n_h * d.d_h, HC = (int64_t)d.n_h * d.d_c;
  const size_t part_bytes = decode_gemm_partials(d, T);
  void* core_scratch = (char*)scratch + part_bytes;
  // device checks of cu_seqlens, the query positions and the latent core's plan: one launch
  cudaError_t e = tc_core_prepare(cu, B, tq, capacity, const_cast<int64_t*>(pos), core_scratch, num_sms, err, st);
  if (e != cudaSuccess) return e;
  e = queries(d, w, lo, h_q, pos, T, cq, qc, qr, scratch, part_bytes, err, st);
  if (e != cudaSuccess) return e;
  // q~_i = W_i^UK^T q^C_i for every head i: the weight operand is W^UK read MN-major. The
  // head-batched GEMM streams weights with the tokens on the MMA's N side, so it runs on chunks of
  // at most kSwapMaxTokens tokens.
  for (int64_t t0 = 0; t0 < T; t0 += kSwapMaxTokens) {
    const int64_t n = T - t0 < kSwapMaxTokens ? T - t0 : kSwapMaxTokens;
    TcGemmDesc a = desc(mat((const char*)qc + (size_t)t0 * HD * 2, n, HD, HD), n, d.d_h, err);
    a.nseg = 1;
    a.w_mn = true;
    a.seg[0].w = mat(w.w_uk, HD, d.d_c, d.d_c);
    a.seg[0].epi = epi((char*)qabs + (size_t)t0 * HC * 2, HC, 1, d.d_c);
    a.seg[0].epi.so_z = d.d_c;
    a.batch = d.n_h; a.w_row_z = d.d_h; a.x_col_z = d.d_h;
    if ((e = tc_gemm(a, st)) != cudaSuccess) return e;
  }
  e = tc_core_run(qabs, qr, B, tq, cu, cache, capacity, lo.cache_fp8 != 0, olat, false, lse, core_scratch, num_sms,
                  err, st);
  if (e != cudaSuccess) return e;
  // o_i = W_i^UV o^lat_i for every head i, in the same token chunks.
  for (int64_t t0 = 0; t0 < T; t0 += kSwapMaxTokens) {
    const int64_t n = T - t0 < kSwapMaxTokens ? T - t0 : kSwapMaxTokens;
    TcGemmDesc v = desc(mat((const char*)olat + (size_t)t0 * HC * 2, n, HC, HC), n, d.d_c, err);
    v.nseg = 1;
    v.seg[0].w = mat(w.w_uv, HD, d.d_c, d.d_c);
    v.seg[0].epi = epi((char*)o + (size_t)t0 * HD * 2, HD, 1, d.d_h);
    v.seg[0].epi.so_z = d.d_h;
    v.batch = d.n_h; v.w_row_z = d.d_h; v.x_col_z = d.d_c;
    if ((e = tc_gemm(v, st)) != cudaSuccess) return e;
  }
  return output(d, w, o, T, u_out, scratch, part_bytes, err, st);
}

cudaError_t tc_prefill(const mla_dims_t& d, const mla_weights_t& w, const LayerOpts& lo, const void* hidden, int64_t B,
                       const int64_t* cu, const int64_t* cu_kv, int64_t T, int64_t T_kv, int64_t max_seqlen,
                       const int64_t* pos, const int64_t* slots, void* cache, int64_t capacity, void* u_out,
                       void* cq, void* qc, void* qr, void* kc, void* vc, void* o, int num_sms, uint32_t* err,
                       cudaStream_t st) {
  const int64_t R = d.d_c + d.d_r, HD = (int64_t)d.n_h * d.d_h;
  if (!cu_kv) T_kv = T;
  cudaError_t e = cache_rows(d, w, lo, hidden, pos, slots, T, cache, capacity, nullptr, 0, nullptr, err, st);
  if (e != cudaSuccess) return e;
  e = queries(d, w, lo, hidden, pos, T, cq, qc, qr, nullptr, 0, err, st);
  if (e != cudaSuccess) return e;
  // Steps (6), (9): [k^C; v^C] = [W^UK; W^UV] c^KV from every key row (a chunk's cached prefix and
  // the rows just written).
  TcGemmDesc p3 = desc(mat(cache, T_kv, d.d_c, R), T_kv, d.d_c, err);
  p3.nseg = 2;
  p3.seg[0].w = mat(w.w_uk, HD, d.d_c, d.d_c);
  p3.seg[0].epi = epi(kc, HD, 1, HD);
  p3.seg[1].w = mat(w.w_uv, HD, d.d_c, d.d_c);
  p3.seg[1].epi = epi(vc, HD, 1, HD);
  e = tc_gemm(p3, st);
  if (e != cudaSuccess) return e;
  // Steps (4), (8), (10): causal attention per head, keys [k^C_i; k^R], values v^C_i.
  e = tc_prefill_attention(qc, qr, kc, vc, cache, capacity, cu, cu_kv, B, T, T_kv, max_seqlen, o, num_sms, err, st);
  if (e != cudaSuccess) return e;
  return output(d, w, o, T, u_out, nullptr, 0, err, st);
}

}  // namespace mla
