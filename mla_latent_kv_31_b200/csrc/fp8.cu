// FP8 (e4m3) latent cache rows. The DeepSeek-V3 notes (section 二（三）"FP8训练") store e4m3 values
// with fp32 scales; the cache uses one scale per cached row:
//   s = max(amax(c^KV) / 448, amax(k^R) / 32768)   (1 for an all-zero row), in fp32;
//   bytes [0, 512):   e4m3 codes of c^KV / s (round to nearest even, saturating at 448);
//   bytes [512, 640): f16 of k^R / s (round to nearest even);
//   bytes [640, 644): s as fp32; bytes [644, 656): zero.
// Every division is an IEEE fp32 division, so the codes are the same bytes whoever computes them.
// The k^R term carries the same scale as c^KV, so a score over a quantized row is s times the score
// over (codes, k^R / s), and the latent core applies s once per key.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc.cuh"

namespace mla {
namespace {

constexpr int kRowsPerBlock = 8;

// Two fp32 values to e4m3 (round to nearest even, saturating): `lo` in the low byte.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(32 * kRowsPerBlock)
    quantize_rows_kernel(const __nv_bfloat16* rows, int64_t n, const int64_t* rowmap, int64_t limit,
                         uint8_t* out, uint32_t* err) {
  const int64_t r = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= n) return;
  int64_t dst = r;
  if (rowmap) {
    dst = rowmap[r];
    if (dst < 0 || dst >= limit) {         // a slot outside the cache: reported, nothing written
      if (lane == 0) flag_error(err, DEVERR_SLOT);
      return;
    }
  }
  const __nv_bfloat16* src = rows + r * kFp8RowLatent;
  // lane: c^KV columns 16 lane .. 16 lane + 15, k^R columns 2 lane, 2 lane + 1
  float c[16];
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(src + 16 * lane + e);
    c[e] = __bfloat162float(v.x);
    c[e + 1] = __bfloat162float(v.y);
  }
  const __nv_bfloat162 kv = *reinterpret_cast<const __nv_bfloat162*>(src + 512 + 2 * lane);
  const float k0 = __bfloat162float(kv.x), k1 = __bfloat162float(kv.y);
  float ac = 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) ac = fmaxf(ac, fabsf(c[e]));
  float ar = fmaxf(fabsf(k0), fabsf(k1));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ac = fmaxf(ac, __shfl_xor_sync(0xffffffffu, ac, o));
    ar = fmaxf(ar, __shfl_xor_sync(0xffffffffu, ar, o));
  }
  float s = fmaxf(__fdiv_rn(ac, 448.f), __fdiv_rn(ar, 32768.f));
  if (!(s > 0.f)) s = 1.f;
  uint8_t* row = out + dst * kFp8RowBytes;
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t a = e4m3x2(__fdiv_rn(c[4 * e], s), __fdiv_rn(c[4 * e + 1], s));
    const uint32_t b = e4m3x2(__fdiv_rn(c[4 * e + 2], s), __fdiv_rn(c[4 * e + 3], s));
    w[e] = a | (b << 16);
  }
  *reinterpret_cast<uint4*>(row + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
  const __half2 kh = __halves2half2(__float2half_rn(__fdiv_rn(k0, s)), __float2half_rn(__fdiv_rn(k1, s)));
  *reinterpret_cast<__half2*>(row + kFp8KrOffset + 4 * lane) = kh;
  if (lane == 0) *reinterpret_cast<uint4*>(row + kFp8ScaleOffset) = make_uint4(__float_as_uint(s), 0u, 0u, 0u);
}

}  // namespace

cudaError_t fp8_quantize_rows(const void* rows, int64_t n, const int64_t* rowmap, int64_t limit, void* out,
                              uint32_t* err, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((n + kRowsPerBlock - 1) / kRowsPerBlock);
  quantize_rows_kernel<<<grid, 32 * kRowsPerBlock, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(rows), n, rowmap,
                                                            limit, reinterpret_cast<uint8_t*>(out), err);
  note_launch();
  return cudaGetLastError();
}

}  // namespace mla
