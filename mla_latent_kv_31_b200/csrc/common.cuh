// Shared device helpers for libmla: error word bits, dtype conversion, block reductions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

// Bits of the handle's sticky device error word.
enum : uint32_t {
  DEVERR_CU_SEQLENS = 1u << 0,    // cu_seqlens[0] != 0, decreasing, or past the cache capacity
  DEVERR_SHORT_SEQ = 1u << 1,     // a sequence holds fewer rows than its query tokens (decode Tq, chunk)
  DEVERR_SLOT = 1u << 2,          // a cache slot outside [0, capacity)
  DEVERR_POSITION = 1u << 3,      // a negative position
  DEVERR_SEQ_TOO_LONG = 1u << 4,  // a prefill sequence (or chunk) longer than max_seqlen (max_q)
  DEVERR_TOTAL = 1u << 5,         // cu_seqlens[B] differs from the token count given on the host
  DEVERR_TIMEOUT = 1u << 6,       // a bounded mbarrier wait gave up
};

// Host-side count of kernels this library has launched (mla_kernel_launches()).
void note_launch(unsigned n = 1);
// Optional event brackets around the attention-core launches (see mla_set_kernel_timing).
enum TimedKernel { TIMED_LATENT_CORE = 0, TIMED_PREFILL_CORE = 1, TIMED_KERNELS = 2 };
void timer_begin(TimedKernel k, cudaStream_t st);
void timer_end(TimedKernel k, cudaStream_t st);

// The decoupled RoPE of a layer (section 一(一)3 of the DeepSeek-V3 notes): pair m of a d_r-wide block
// turns at theta_m = base^(-2m/d_r). With YaRN (section 三(二)3, yarn_s > 1) the frequencies are
// interpolated by parts: pair m turns r_m = L0 theta_m / (2 pi) times over the original context
// L0; gamma = clamp((r_m - alpha) / (beta - alpha), 0, 1) and theta'_m = (1 - gamma) theta_m / s +
// gamma theta_m; each rotated vector (q^R and k^R) is multiplied by 0.1 ln s + 1.
struct RopeSpec {
  double base;
  double yarn_s, yarn_alpha, yarn_beta, yarn_l0;   // yarn_s <= 1: plain RoPE
};
__host__ __device__ inline double rope_theta(const RopeSpec& r, int m, int d_r) {
  const double theta = pow(r.base, -2.0 * (double)m / (double)d_r);
  if (!(r.yarn_s > 1.0)) return theta;
  const double turns = r.yarn_l0 * theta / 6.283185307179586;
  double g = (turns - r.yarn_alpha) / (r.yarn_beta - r.yarn_alpha);
  g = g < 0.0 ? 0.0 : (g > 1.0 ? 1.0 : g);
  return (1.0 - g) * theta / r.yarn_s + g * theta;
}
__host__ __device__ inline float rope_mul(const RopeSpec& r) {
  return r.yarn_s > 1.0 ? (float)(0.1 * log(r.yarn_s) + 1.0) : 1.0f;
}

// Opt-in parts of a layer: the RMSNorm after the latent compression (section 三(二)1 of the notes:
// c^Q = RMSNorm(W^DQ h), c^KV = RMSNorm(W^DKV h), y = x / sqrt(mean(x^2) + eps) * g) and the RoPE.
struct LayerOpts {
  const void* g_q;    // [d_c'] gains of c^Q in the handle dtype; nullptr: no norm
  const void* g_kv;   // [d_c] gains of c^KV
  float eps;
  RopeSpec rope;
  int cache_fp8;      // the latent cache holds FP8 rows (656 bytes) instead of bf16 rows
};

__device__ __forceinline__ void flag_error(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide reductions for blockDim.x a multiple of 32 (<= 1024); `scratch` holds 32 floats.
__device__ __forceinline__ float block_max(float v, float* scratch) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float r = lane < nw ? scratch[lane] : -INFINITY;
  return warp_max(r);
}
__device__ __forceinline__ float block_sum(float v, float* scratch) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float r = lane < nw ? scratch[lane] : 0.f;
  return warp_sum(r);
}

// RoPE angle for pair m of a d_r-wide block at position pos: pos * theta_m, in double, then
// sine/cosine in double (CUDA's sincos) so long positions keep their precision.
__device__ __forceinline__ void rope_cos_sin(int64_t pos, int m, int d_r, const RopeSpec& r, float* c, float* s) {
  const double theta = rope_theta(r, m, d_r);
  double sd, cd;
  sincos((double)pos * theta, &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

// In-place RMSNorm of `rows` rows of `cols` elements (row r at x + row(r) * ld, row(r) = rowmap ?
// rowmap[r] : r; rows mapped outside [0, rowmap_limit) are skipped) with gains g.
cudaError_t rmsnorm_rows(void* x, bool bf16, int64_t ld, const int64_t* rowmap, int64_t rowmap_limit, int64_t rows,
                         int cols, const void* g, float eps, cudaStream_t st);

// Sequence of a packed token t: the b with cu[b] <= t < cu[b+1] (cu non-decreasing, B >= 1).
__device__ __forceinline__ int64_t seq_of_token(const int64_t* cu, int64_t B, int64_t t) {
  int64_t lo = 0, hi = B;  // answer in [lo, hi)
  while (hi - lo > 1) {
    int64_t mid = (lo + hi) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid;
  }
  return lo;
}

// Device-side checks of cu_seqlens by one block (strided loops), and per-token positions when
// pos_out != nullptr: decode (tq > 0): pos = len_b - tq + k for token k of sequence b; prefill
// (tq == 0): pos = t - cu[b]. Offending sequences set bits of the error word.
__device__ inline void check_seqs_and_positions(const int64_t* cu, int64_t B, int32_t tq, int64_t total,
                                                int64_t capacity, int64_t max_seqlen, int64_t* pos_out,
                                                uint32_t* err) {
  for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
    const int64_t lo = cu[b], hi = cu[b + 1];
    if (b == 0 && lo != 0) flag_error(err, DEVERR_CU_SEQLENS);
    if (hi < lo || hi > capacity) flag_error(err, DEVERR_CU_SEQLENS);
    if (tq > 0 && hi - lo < tq) flag_error(err, DEVERR_SHORT_SEQ);
    if (tq == 0 && max_seqlen > 0 && hi - lo > max_seqlen) flag_error(err, DEVERR_SEQ_TOO_LONG);
  }
  if (threadIdx.x == 0 && tq == 0 && total >= 0 && cu[B] != total) flag_error(err, DEVERR_TOTAL);
  if (!pos_out) return;
  if (tq > 0) {
    for (int64_t t = threadIdx.x; t < B * tq; t += blockDim.x) {
      const int64_t b = t / tq;
      pos_out[t] = (cu[b + 1] - cu[b]) - tq + (t % tq);
    }
  } else {
    for (int64_t t = threadIdx.x; t < total; t += blockDim.x) {
      const int64_t b = seq_of_token(cu, B, t);
      pos_out[t] = t - cu[b];
    }
  }
}

}  // namespace mla
