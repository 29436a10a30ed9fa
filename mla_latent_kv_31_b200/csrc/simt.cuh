// Generic CUDA-core kernels (any MLA sizes, fp32 storage and arithmetic). They serve the FP32
// configuration, where tcgen05's tf32 rounding would miss a 1e-5 bound. BF16 runs only on the
// tcgen05 kernels (DeepSeek-V3 sizes); these kernels are not instantiated for it.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace mla {

// C(m, n) = sum_k A(m, k) B(n, k) over a batch z, with strided operands (elements):
//   A(m, k) = A[z*sab + m*sam + k*sak], B(n, k) = B[z*sbb + n*sbn + k*sbk],
//   C(r, n) = C[z*scb + r*scm + n*scn] with r = rowmap ? rowmap[m] : m.
// Optional epilogue: columns n >= rope_col0 are RoPE'd in (2m, 2m+1) pairs of d_r-wide blocks
// at position pos[m] (section 一(一)3 of the DeepSeek-V3 notes).
struct SimtGemmArgs {
  const void* A; int64_t sam, sak, sab;
  const void* B; int64_t sbn, sbk, sbb;
  void* C; int64_t scm, scn, scb;
  int64_t M, N, K, batch;
  const int64_t* rowmap; int64_t rowmap_limit;
  const int64_t* pos; int64_t rope_col0; int32_t d_r; RopeSpec rope;
  uint32_t* err;
};

// Attention over latent-cache rows for one (query token, head) per block (section 一(一)3,
// step (10)): s_j = (q1.k1_j + q2.k2_j) * scale over the rows j of the token's sequence up to
// its position, o = sum_j softmax(s)_j v_j, lse = log sum_j exp(s_j).
struct SimtAttnArgs {
  const void* q1; int64_t sq1t, sq1h; int32_t d1;
  const void* q2; int64_t sq2t, sq2h; int32_t d2;
  const void* k1; int64_t sk1, sk1h;
  const void* k2; int64_t sk2;
  const void* v; int64_t sv, svh; int32_t dv;
  void* o; int64_t sot, soh;
  float* lse;
  const int64_t* cu; int64_t B; int32_t tq;  // tq > 0: decode (token t of seq t/tq); tq == 0: prefill
  const int64_t* cu_kv;  // prefill only, optional: key rows of each sequence, its query tokens the last ones
  int64_t T; int32_t n_h; int64_t capacity;
  float scale;
  uint32_t* err;
};

cudaError_t simt_gemm(const SimtGemmArgs& a, cudaStream_t st);
cudaError_t simt_attention(const SimtAttnArgs& a, cudaStream_t st);

// Device-side checks of cu_seqlens; also writes per-token positions when pos_out != nullptr:
// decode (tq > 0): pos = len_b - tq + k; prefill (tq == 0): pos = t - cu[b].
cudaError_t check_and_positions(const int64_t* cu, int64_t B, int32_t tq, int64_t total_tokens,
                                int64_t capacity, int64_t max_seqlen, int64_t* pos_out, uint32_t* err,
                                cudaStream_t st);

// Device-side checks of a chunked prefill's cu_q / cu_kv (chunk b = the last cu_q[b+1] - cu_q[b] of
// sequence b's cu_kv[b+1] - cu_kv[b] rows) and, per chunk token t of sequence b, its position
// pos = len_kv_b - len_q_b + (t - cu_q[b]) and its cache row cu_kv[b] + pos.
cudaError_t check_chunk_positions(const int64_t* cu_q, const int64_t* cu_kv, int64_t B, int64_t total_q,
                                  int64_t total_kv, int64_t capacity, int64_t max_q, int64_t* pos_out,
                                  int64_t* slot_out, uint32_t* err, cudaStream_t st);

}  // namespace mla
