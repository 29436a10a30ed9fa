// tcgen05 GEMM for the MLA projections: D[f, t] = sum_k W[f, k] X[t, k] over a batch of heads.
//
// W is a weight operand (rows = output features f), X the activations (rows = tokens t), both
// bf16. Two orientations share one kernel: "swap" puts the weights on the MMA's M side
// (128 features per tile, tokens as N), which streams weights at small token counts (decode);
// otherwise tokens are M and 256 features are N (prefill). The weight may be given MN-major
// (W stored [k, f], i.e. W_i^UK used transposed for the absorbed query). Up to two weight
// segments with their own output and epilogue share one launch (e.g. [W^DKV; W^KR]).
// Epilogue: optional RoPE on feature pairs (2m, 2m+1) of d_r-wide blocks at pos[t], bf16/fp32
// store at out + z*so_z + row(t)*so_t + f*so_f with row(t) = rowmap ? rowmap[t] : t.
// Split-K writes fp32 partials that a reduce pass sums in a fixed order (deterministic).
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "common.cuh"

namespace mla {

// Largest token count of the weight-streaming ("swap") orientation; head-batched and MN-major weight
// launches exist only in that orientation, so their callers split larger token counts into chunks.
constexpr int64_t kSwapMaxTokens = 256;

struct TcMatrix {       // row-major bf16 matrix [rows, cols] with a row stride in elements
  const void* ptr;
  int64_t rows, cols, ld;
};

struct TcEpiSeg {
  void* out;
  int64_t so_t, so_f, so_z;
  int32_t out_f32;
  int32_t rope;
  const int64_t* rowmap;
  int64_t rowmap_limit;
  int64_t f_rows;       // valid features of this segment
  int64_t f_base;       // offset of the segment on the split-K partial's feature axis
  int32_t tiles;        // weight tiles of this segment
};

struct TcGemmSeg {
  TcMatrix w;           // K-major: [f_rows, K] ; MN-major: [K, f_rows]
  TcEpiSeg epi;
};

struct TcGemmDesc {
  TcGemmSeg seg[2];
  int nseg;
  bool w_mn;            // weights MN-major (only with swap)
  TcMatrix x;           // [T, K] (K-major), per-batch column offset x_col_z
  int64_t T, K;
  int32_t batch;
  int64_t w_row_z, w_col_z;   // per-batch offsets of the weight operand (elements)
  int64_t x_col_z;            // per-batch column offset of X
  const int64_t* pos; int32_t d_r; RopeSpec rope;   // RoPE epilogue (segments with epi.rope)
  float* partial;             // split-K scratch (fp32), may be null when splits == 1
  size_t partial_bytes;
  uint32_t* err;
};

// Split-K scratch bytes tc_gemm uses for T tokens against f_tiles 128-row weight tiles holding
// f_total features over reduction length K (0 when it will not split).
size_t tc_gemm_partial_bytes(int64_t T, int64_t f_tiles, int64_t f_total, int64_t K, int32_t batch);

// 2-D bf16 TMA map over a row-major [outer, inner] matrix (row stride ld elements), box
// {box_inner, box_outer}, 128-byte swizzle (64-byte with swizzle_bytes = 64, for boxes of
// 32 bf16 columns), zero fill out of bounds.
cudaError_t make_tmap_bf16(CUtensorMap* m, const void* ptr, int64_t inner, int64_t outer, int64_t ld, int box_inner,
                           int box_outer, int swizzle_bytes = 128);

// 2-D byte TMA map over a row-major [outer, inner] byte matrix (row stride ld bytes, a multiple of
// 16), box {box_inner <= 128, box_outer}, 128-byte swizzle, zero fill out of bounds.
cudaError_t make_tmap_u8(CUtensorMap* m, const void* ptr, int64_t inner, int64_t outer, int64_t ld, int box_inner,
                         int box_outer);

cudaError_t tc_gemm(const TcGemmDesc& g, cudaStream_t st);

}  // namespace mla
