// Generic CUDA-core kernels: strided GEMM with RoPE / row-scatter epilogue, attention over
// latent-cache rows, and the cu_seqlens checks. fp32 arithmetic throughout.
#include "simt.cuh"

namespace mla {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <typename TA, typename TC>
__global__ void __launch_bounds__(256) simt_gemm_kernel(SimtGemmArgs a) {
  __shared__ float As[TK][TM + 1];
  __shared__ float Bs[TK][TN + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = (int64_t)blockIdx.y * TM, n0 = (int64_t)blockIdx.x * TN, z = blockIdx.z;
  const TA* A = reinterpret_cast<const TA*>(a.A) + z * a.sab;
  const TA* B = reinterpret_cast<const TA*>(a.B) + z * a.sbb;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < a.K; k0 += TK) {
    for (int idx = threadIdx.x; idx < TM * TK; idx += 256) {
      const int mm = idx / TK, kk = idx % TK;
      const int64_t m = m0 + mm, k = k0 + kk;
      As[kk][mm] = (m < a.M && k < a.K) ? to_f(A[m * a.sam + k * a.sak]) : 0.f;
      const int64_t n = n0 + mm;
      Bs[kk][mm] = (n < a.N && k < a.K) ? to_f(B[n * a.sbn + k * a.sbk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  TC* C = reinterpret_cast<TC*>(a.C) + z * a.scb;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= a.M) continue;
    int64_t r = m;
    if (a.rowmap) {
      r = a.rowmap[m];
      if (r < 0 || r >= a.rowmap_limit) {
        if (blockIdx.x == 0 && tx == 0) flag_error(a.err, DEVERR_SLOT);
        continue;
      }
    }
    int64_t p = 0;
    if (a.pos) {
      p = a.pos[m];
      if (p < 0) {
        if (blockIdx.x == 0 && tx == 0) flag_error(a.err, DEVERR_POSITION);
        continue;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
      const int64_t n = n0 + tx * 4 + j;  // even
      float x0 = acc[i][j], x1 = acc[i][j + 1];
      if (a.pos && n >= a.rope_col0) {
        const int pair = (int)(((n - a.rope_col0) % a.d_r) >> 1);
        float c, s;
        rope_cos_sin(p, pair, a.d_r, a.rope, &c, &s);
        const float mul = rope_mul(a.rope);
        const float y0 = (x0 * c - x1 * s) * mul, y1 = (x0 * s + x1 * c) * mul;
        x0 = y0; x1 = y1;
      }
      if (n < a.N) C[r * a.scm + n * a.scn] = from_f<TC>(x0);
      if (n + 1 < a.N) C[r * a.scm + (n + 1) * a.scn] = from_f<TC>(x1);
    }
  }
}

constexpr int ATT_THREADS = 128;
constexpr int ATT_MAX_DV = 512;
constexpr int ATT_MAX_Q = 1024;

template <typename TI, typename TO>
__global__ void __launch_bounds__(ATT_THREADS) simt_attention_kernel(SimtAttnArgs a) {
  __shared__ float qs[ATT_MAX_Q];
  __shared__ float ps[ATT_THREADS];
  __shared__ float red[32];
  const int64_t t = blockIdx.x;
  const int head = blockIdx.y;
  const int tid = threadIdx.x;
  int64_t b, pos, row0;
  if (a.tq > 0) {
    b = t / a.tq;
    pos = (a.cu[b + 1] - a.cu[b]) - a.tq + (t % a.tq);
    row0 = a.cu[b];
  } else if (a.cu_kv) {
    // a chunk: the sequence's query tokens are the last ones of its key rows
    b = seq_of_token(a.cu, a.B, t);
    row0 = a.cu_kv[b];
    pos = (a.cu_kv[b + 1] - row0) - (a.cu[b + 1] - a.cu[b]) + (t - a.cu[b]);
  } else {
    b = seq_of_token(a.cu, a.B, t);
    pos = t - a.cu[b];
    row0 = a.cu[b];
  }
  const int64_t n = pos + 1;
  const bool bad = pos < 0 || row0 < 0 || row0 + n > a.capacity;
  TO* o = reinterpret_cast<TO*>(a.o) + t * a.sot + (int64_t)head * a.soh;
  if (bad) {  // flagged by the cu_seqlens check; write zeros so outputs stay finite
    for (int c = tid; c < a.dv; c += ATT_THREADS) o[c] = from_f<TO>(0.f);
    if (a.lse && tid == 0) a.lse[t * a.n_h + head] = -INFINITY;
    return;
  }
  const TI* q1 = reinterpret_cast<const TI*>(a.q1) + t * a.sq1t + (int64_t)head * a.sq1h;
  const TI* q2 = reinterpret_cast<const TI*>(a.q2) + t * a.sq2t + (int64_t)head * a.sq2h;
  for (int c = tid; c < a.d1; c += ATT_THREADS) qs[c] = to_f(q1[c]);
  for (int c = tid; c < a.d2; c += ATT_THREADS) qs[a.d1 + c] = to_f(q2[c]);
  __syncthreads();
  const TI* k1 = reinterpret_cast<const TI*>(a.k1) + (int64_t)head * a.sk1h;
  const TI* k2 = reinterpret_cast<const TI*>(a.k2);
  const TI* v = reinterpret_cast<const TI*>(a.v) + (int64_t)head * a.svh;
  float m = -INFINITY, l = 0.f;
  float acc[ATT_MAX_DV / ATT_THREADS] = {};
  for (int64_t c0 = 0; c0 < n; c0 += ATT_THREADS) {
    const int64_t j = c0 + tid;
    float s = -INFINITY;
    if (j < n) {
      const int64_t row = row0 + j;
      float d = 0.f;
      for (int c = 0; c < a.d1; ++c) d = fmaf(qs[c], to_f(k1[row * a.sk1 + c]), d);
      for (int c = 0; c < a.d2; ++c) d = fmaf(qs[a.d1 + c], to_f(k2[row * a.sk2 + c]), d);
      s = d * a.scale;
    }
    const float mc = block_max(s, red);
    const float m_new = fmaxf(m, mc);
    const float alpha = (m == -INFINITY) ? 0.f : __expf(m - m_new);
    const float p = (j < n) ? __expf(s - m_new) : 0.f;
    ps[tid] = p;
    const float sc = block_sum(p, red);
    l = l * alpha + sc;
#pragma unroll
    for (int i = 0; i < ATT_MAX_DV / ATT_THREADS; ++i) acc[i] *= alpha;
    __syncthreads();
    const int64_t cnt = min((int64_t)ATT_THREADS, n - c0);
    for (int64_t jj = 0; jj < cnt; ++jj) {
      const float pj = ps[jj];
      const TI* vr = v + (row0 + c0 + jj) * a.sv;
#pragma unroll
      for (int i = 0; i < ATT_MAX_DV / ATT_THREADS; ++i) {
        const int c = tid + i * ATT_THREADS;
        if (c < a.dv) acc[i] = fmaf(pj, to_f(vr[c]), acc[i]);
      }
    }
    m = m_new;
    __syncthreads();
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int i = 0; i < ATT_MAX_DV / ATT_THREADS; ++i) {
    const int c = tid + i * ATT_THREADS;
    if (c < a.dv) o[c] = from_f<TO>(acc[i] * inv);
  }
  if (a.lse && tid == 0) a.lse[t * a.n_h + head] = m + logf(l);
}

__global__ void check_positions_kernel(const int64_t* cu, int64_t B, int32_t tq, int64_t total,
                                       int64_t capacity, int64_t max_seqlen, int64_t* pos_out,
                                       uint32_t* err) {
  check_seqs_and_positions(cu, B, tq, total, capacity, max_seqlen, pos_out, err);
}

__global__ void check_chunk_kernel(const int64_t* cu_q, const int64_t* cu_kv, int64_t B, int64_t total_q,
                                   int64_t total_kv, int64_t capacity, int64_t max_q, int64_t* pos_out,
                                   int64_t* slot_out, uint32_t* err) {
  // One block: sequence checks by a strided loop, then per-token positions and cache rows.
  for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
    const int64_t q0 = cu_q[b], q1 = cu_q[b + 1], k0 = cu_kv[b], k1 = cu_kv[b + 1];
    if (b == 0 && (q0 != 0 || k0 != 0)) flag_error(err, DEVERR_CU_SEQLENS);
    if (q1 < q0 || k1 < k0 || k1 > capacity) flag_error(err, DEVERR_CU_SEQLENS);
    if (q1 - q0 > k1 - k0) flag_error(err, DEVERR_SHORT_SEQ);
    if (q1 - q0 > max_q) flag_error(err, DEVERR_SEQ_TOO_LONG);
  }
  if (threadIdx.x == 0 && (cu_q[B] != total_q || cu_kv[B] != total_kv)) flag_error(err, DEVERR_TOTAL);
  for (int64_t t = threadIdx.x; t < total_q; t += blockDim.x) {
    const int64_t b = seq_of_token(cu_q, B, t);
    const int64_t kb = cu_kv[b], qb = cu_q[b];
    const int64_t pos = (cu_kv[b + 1] - kb) - (cu_q[b + 1] - qb) + (t - qb);
    pos_out[t] = pos;
    slot_out[t] = pos >= 0 ? kb + pos : -1;   // a negative row is skipped by the writers
  }
}

}  // namespace

cudaError_t simt_gemm(const SimtGemmArgs& a, cudaStream_t st) {
  if (a.M <= 0 || a.N <= 0) return cudaSuccess;
  dim3 grid((unsigned)((a.N + TN - 1) / TN), (unsigned)((a.M + TM - 1) / TM), (unsigned)a.batch);
  simt_gemm_kernel<float, float><<<grid, 256, 0, st>>>(a);
  note_launch();
  return cudaGetLastError();
}

cudaError_t simt_attention(const SimtAttnArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  if (a.dv > ATT_MAX_DV || a.d1 + a.d2 > ATT_MAX_Q) return cudaErrorInvalidValue;
  dim3 grid((unsigned)a.T, (unsigned)a.n_h);
  simt_attention_kernel<float, float><<<grid, ATT_THREADS, 0, st>>>(a);
  note_launch();
  return cudaGetLastError();
}

cudaError_t check_and_positions(const int64_t* cu, int64_t B, int32_t tq, int64_t total_tokens,
                                int64_t capacity, int64_t max_seqlen, int64_t* pos_out, uint32_t* err,
                                cudaStream_t st) {
  check_positions_kernel<<<1, 512, 0, st>>>(cu, B, tq, total_tokens, capacity, max_seqlen, pos_out, err);
  note_launch();
  return cudaGetLastError();
}

cudaError_t check_chunk_positions(const int64_t* cu_q, const int64_t* cu_kv, int64_t B, int64_t total_q,
                                  int64_t total_kv, int64_t capacity, int64_t max_q, int64_t* pos_out,
                                  int64_t* slot_out, uint32_t* err, cudaStream_t st) {
  check_chunk_kernel<<<1, 512, 0, st>>>(cu_q, cu_kv, B, total_q, total_kv, capacity, max_q, pos_out, slot_out, err);
  note_launch();
  return cudaGetLastError();
}

}  // namespace mla
