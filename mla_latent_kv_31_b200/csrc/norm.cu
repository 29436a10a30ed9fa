// RMSNorm after the latent compression (section 三(二)1 of the DeepSeek-V3 notes):
// c <- c / sqrt(mean(c^2) + eps) * g over the d_c' columns of c^Q or the d_c columns of c^KV.
// One warp per row, in place; the sum of squares is taken in fp32 in a fixed order (each lane
// strides the row, then a fixed xor tree), so the result does not depend on timing.
#include <cuda_bf16.h>

#include "common.cuh"

namespace mla {
namespace {

constexpr int kRowsPerBlock = 8;

template <typename T>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
    rmsnorm_rows_kernel(T* x, int64_t ld, const int64_t* rowmap, int64_t limit, int64_t rows, int cols,
                        const T* g, float eps) {
  const int64_t r = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  int64_t row = r;
  if (rowmap) {
    row = rowmap[r];
    if (row < 0 || row >= limit) return;   // the writer of the row flagged it
  }
  T* p = x + row * ld;
  float ss = 0.f;
  for (int c = lane; c < cols; c += 32) {
    const float v = to_f(p[c]);
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  const float inv = 1.f / sqrtf(ss / (float)cols + eps);
  for (int c = lane; c < cols; c += 32) p[c] = from_f<T>(to_f(p[c]) * inv * to_f(g[c]));
}

}  // namespace

cudaError_t rmsnorm_rows(void* x, bool bf16, int64_t ld, const int64_t* rowmap, int64_t rowmap_limit, int64_t rows,
                         int cols, const void* g, float eps, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock);
  if (bf16)
    rmsnorm_rows_kernel<__nv_bfloat16><<<grid, 32 * kRowsPerBlock, 0, st>>>(
        reinterpret_cast<__nv_bfloat16*>(x), ld, rowmap, rowmap_limit, rows, cols,
        reinterpret_cast<const __nv_bfloat16*>(g), eps);
  else
    rmsnorm_rows_kernel<float><<<grid, 32 * kRowsPerBlock, 0, st>>>(reinterpret_cast<float*>(x), ld, rowmap,
                                                                     rowmap_limit, rows, cols,
                                                                     reinterpret_cast<const float*>(g), eps);
  note_launch();
  return cudaGetLastError();
}

}  // namespace mla
