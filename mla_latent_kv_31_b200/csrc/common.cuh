// Shared device helpers for libmla: error word bits, dtype conversion, block reductions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

// Bits of the handle's sticky device error word.
enum : uint32_t {
  DEVERR_CU_SEQLENS = 1u << 0,    // cu_seqlens[0] != 0, decreasing, or past the cache capacity
  DEVERR_SHORT_SEQ = 1u << 1,     // a decode sequence holds fewer rows than its Tq query tokens
  DEVERR_SLOT = 1u << 2,          // a cache slot outside [0, capacity)
  DEVERR_POSITION = 1u << 3,      // a negative position
  DEVERR_SEQ_TOO_LONG = 1u << 4,  // a prefill sequence longer than max_seqlen
  DEVERR_TOTAL = 1u << 5,         // cu_seqlens[B] differs from the token count given on the host
  DEVERR_TIMEOUT = 1u << 6,       // a bounded mbarrier wait gave up
};

// Host-side count of kernels this library has launched (mla_kernel_launches()).
void note_launch(unsigned n = 1);
// Optional event brackets around the attention-core launches (see mla_set_kernel_timing).
enum TimedKernel { TIMED_LATENT_CORE = 0, TIMED_PREFILL_CORE = 1, TIMED_KERNELS = 2 };
void timer_begin(TimedKernel k, cudaStream_t st);
void timer_end(TimedKernel k, cudaStream_t st);

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

// RoPE angle for pair m of a d_r-wide block at position pos: pos * base^(-2m/d_r), in double,
// then sine/cosine in double (CUDA's sincos) so long positions keep their precision.
__device__ __forceinline__ void rope_cos_sin(int64_t pos, int m, int d_r, double base, float* c, float* s) {
  const double theta = pow(base, -2.0 * (double)m / (double)d_r);
  double sd, cd;
  sincos((double)pos * theta, &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

// Sequence of a packed token t: the b with cu[b] <= t < cu[b+1] (cu non-decreasing, B >= 1).
__device__ __forceinline__ int64_t seq_of_token(const int64_t* cu, int64_t B, int64_t t) {
  int64_t lo = 0, hi = B;  // answer in [lo, hi)
  while (hi - lo > 1) {
    int64_t mid = (lo + hi) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid;
  }
  return lo;
}

}  // namespace mla
