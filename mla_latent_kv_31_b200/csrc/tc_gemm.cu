// tcgen05 GEMM kernel (TMA -> shared memory ring -> tcgen05.mma into TMEM -> epilogue), the
// split-K reduce pass, and the host launcher that encodes the TMA tensor maps.
#include <cuda_bf16.h>
#include <stdio.h>
#include <string.h>

#include "sm100.cuh"
#include "tc_gemm.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int BK = 64;           // k-block: one 128-byte swizzle row of bf16
constexpr int kThreads = 192;    // warp 0: TMA producer, warp 1: TMEM owner + MMA issuer, warps 2-5: epilogue
constexpr int kMaxSplits = 64;

struct GemmParams {
  CUtensorMap wmap[2];
  CUtensorMap xmap;
  TcEpiSeg seg[2];
  int32_t nseg;
  int32_t splits, kb_total, kb_per_split;
  int64_t T;
  int32_t w_row_z, w_col_z, x_col_z;
  const int64_t* pos;
  int32_t d_r;
  double rope_base;
  float* partial;
  int64_t f_total;
  uint32_t* err;
};

__device__ __forceinline__ void store_out(const TcEpiSeg& E, uint32_t* err, int z, int64_t f, int64_t t,
                                          float v) {
  int64_t row = t;
  if (E.rowmap) {
    row = E.rowmap[t];
    if (row < 0 || row >= E.rowmap_limit) {
      flag_error(err, DEVERR_SLOT);
      return;
    }
  }
  const int64_t idx = (int64_t)z * E.so_z + row * E.so_t + f * E.so_f;
  if (E.out_f32) reinterpret_cast<float*>(E.out)[idx] = v;
  else reinterpret_cast<__nv_bfloat16*>(E.out)[idx] = __float2bfloat16_rn(v);
}

// RoPE of one element of the pair (2m, 2m+1) holding feature f (segment-local): `own` is x_f,
// `partner` is x_{f^1}.
__device__ __forceinline__ float rope_one(int64_t f, int64_t pos, float own, float partner, int d_r,
                                          double base) {
  float c, s;
  rope_cos_sin(pos, (int)((f % d_r) >> 1), d_r, base, &c, &s);
  return (f & 1) ? (partner * s + own * c) : (own * c - partner * s);
}

template <int BN, bool SWAP, bool W_MN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  constexpr uint32_t A_BYTES = 128 * 128;
  constexpr uint32_t B_BYTES = BN * 128;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = BN <= 32 ? 32 : BN;
  constexpr int W_TILE = SWAP ? 128 : BN;
  constexpr int X_TILE = SWAP ? BN : 128;
  constexpr int CH = BN < 32 ? BN : 32;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);  // full[S], empty[S], done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int wt = blockIdx.x, s = 0;
  if (p.nseg > 1 && wt >= p.seg[0].tiles) {
    s = 1;
    wt -= p.seg[0].tiles;
  }
  const TcEpiSeg& E = p.seg[s];
  const int z = blockIdx.z / p.splits, split = blockIdx.z % p.splits;
  const int kb0 = split * p.kb_per_split;
  const int nkb = min(p.kb_total, kb0 + p.kb_per_split) - kb0;
  const int64_t f0 = (int64_t)wt * W_TILE;
  const int64_t t0 = (int64_t)blockIdx.y * X_TILE;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * STAGES + 1; ++i) mbar_init(smem_addr(&bars[i]), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    prefetch_tmap(&p.wmap[s]);
    prefetch_tmap(&p.xmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t done_bar = smem_addr(&bars[2 * STAGES]);

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap* wm = &p.wmap[s];
      const CUtensorMap* xm = &p.xmap;
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int st = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(smem_addr(&bars[STAGES + st]), ph ^ 1)) {
          ok = false;
          break;
        }
        const uint32_t full = smem_addr(&bars[st]);
        mbar_expect_tx(full, STAGE_BYTES);
        const int k0 = (kb0 + i) * BK;
        const uint32_t a_dst = smem_addr(sA + st * A_BYTES), b_dst = smem_addr(sB + st * B_BYTES);
        const uint32_t w_dst = SWAP ? a_dst : b_dst, x_dst = SWAP ? b_dst : a_dst;
        if (W_MN) {
#pragma unroll
          for (int j = 0; j < W_TILE / 64; ++j)
            tma_load_2d(w_dst + j * 8192, wm, (int)(f0 + 64 * j) + z * p.w_col_z, k0 + z * p.w_row_z, full);
        } else {
          tma_load_2d(w_dst, wm, k0 + z * p.w_col_z, (int)f0 + z * p.w_row_z, full);
        }
        tma_load_2d(x_dst, xm, k0 + z * p.x_col_z, (int)t0, full);
        issued = i + 1;
      }
      if (!ok) {
        flag_error(p.err, DEVERR_TIMEOUT);
        // let the loads already issued land before the CTA can exit
        for (int i = max(0, issued - STAGES); i < issued; ++i)
          mbar_wait(smem_addr(&bars[i % STAGES]), (i / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BN, (SWAP && W_MN) ? 1 : 0, (!SWAP && W_MN) ? 1 : 0);
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int st = i % STAGES;
        if (!mbar_wait(smem_addr(&bars[st]), (i / STAGES) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_addr(sA + st * A_BYTES), b_base = smem_addr(sB + st * B_BYTES);
#pragma unroll
        for (int j = 0; j < BK / 16; ++j) {
          const uint64_t ad = (SWAP && W_MN) ? sw128_desc(a_base + j * 2048, 8192, 1024)
                                             : sw128_desc(a_base + j * 32, 0, 1024);
          const uint64_t bd = (!SWAP && W_MN) ? sw128_desc(b_base + j * 2048, 8192, 1024)
                                              : sw128_desc(b_base + j * 32, 0, 1024);
          mma_bf16_ss(tmem, ad, bd, idesc, (i > 0 || j > 0) ? 1u : 0u);
        }
        mma_commit(smem_addr(&bars[STAGES + st]));
      }
      if (ok) {
        mma_commit(done_bar);
      } else {
        flag_error(p.err, DEVERR_TIMEOUT);
        mbar_arrive(done_bar);
      }
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;  // accumulator row = TMEM lane
    if (!mbar_wait(done_bar, 0)) flag_error(p.err, DEVERR_TIMEOUT);
    tc_fence_after();
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
    for (int c = 0; c < BN; c += CH) {
      uint32_t v[32];
      if (CH == 32) tmem_ld32(trow + c, v);
      else tmem_ld16(trow + c, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        const float x = __uint_as_float(v[j]);
        int64_t f, t;
        if (SWAP) { f = f0 + r; t = t0 + c + j; }
        else { f = f0 + c + j; t = t0 + r; }
        float partner = 0.f;
        if (SWAP) partner = __shfl_xor_sync(0xffffffffu, x, 1);
        else partner = __uint_as_float(v[j ^ 1]);
        if (f >= E.f_rows || t >= p.T) continue;
        if (p.splits > 1) {
          p.partial[((int64_t)split * p.T + t) * p.f_total + E.f_base + f] = x;
          continue;
        }
        float y = x;
        if (E.rope) {
          const int64_t ps = p.pos[t];
          if (ps < 0) {
            flag_error(p.err, DEVERR_POSITION);
            continue;
          }
          y = rope_one(f, ps, x, partner, p.d_r, p.rope_base);
        }
        store_out(E, p.err, z, f, t, y);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

struct ReduceParams {
  TcEpiSeg seg[2];
  int32_t nseg, splits;
  int64_t T, f_total;
  const float* partial;
  const int64_t* pos;
  int32_t d_r;
  double rope_base;
  uint32_t* err;
};

// Sums the split-K partials of feature pairs (f, f+1) in split order, then applies the epilogue.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const ReduceParams p) {
  const int64_t f = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  const int64_t t = blockIdx.y;
  if (f >= p.f_total) return;
  const int s = (p.nseg > 1 && f >= p.seg[1].f_base) ? 1 : 0;
  const TcEpiSeg& E = p.seg[s];
  const int64_t fl = f - E.f_base;
  float a = 0.f, b = 0.f;
  for (int k = 0; k < p.splits; ++k) {
    const float* src = p.partial + ((int64_t)k * p.T + t) * p.f_total + f;
    a += src[0];
    if (fl + 1 < E.f_rows) b += src[1];
  }
  if (E.rope) {
    const int64_t ps = p.pos[t];
    if (ps < 0) {
      flag_error(p.err, DEVERR_POSITION);
      return;
    }
    const float a2 = rope_one(fl, ps, a, b, p.d_r, p.rope_base);
    const float b2 = rope_one(fl + 1, ps, b, a, p.d_r, p.rope_base);
    a = a2;
    b = b2;
  }
  store_out(E, p.err, 0, fl, t, a);
  if (fl + 1 < E.f_rows) store_out(E, p.err, 0, fl + 1, t, b);
}

// ---- host side ------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

// 2-D bf16 tensor map over a row-major [outer, inner] matrix with row stride ld (elements),
// box {box_inner, box_outer}, 128-byte swizzle, zero fill out of bounds.
cudaError_t make_tmap_bf16(CUtensorMap* m, const void* ptr, int64_t inner, int64_t outer, int64_t ld, int box_inner,
                           int box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

template <int BN, bool SWAP, bool W_MN, int STAGES>
cudaError_t launch_gemm(const GemmParams& p, dim3 grid, cudaStream_t st) {
  constexpr size_t smem = (size_t)STAGES * (128 * 128 + BN * 128) + 1024 + 256;
  static bool configured = false;
  auto kern = gemm_kernel<BN, SWAP, W_MN, STAGES>;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  kern<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

int swap_bn(int64_t T) { return T <= 16 ? 16 : T <= 32 ? 32 : T <= 64 ? 64 : 128; }

}  // namespace

// Split-K factor for a swap-orientation launch of `ctas` CTAs over kb_total k-blocks: enough
// splits to cover the 148 SMs once; returns (splits, k-blocks per split).
static void choose_splits(int64_t ctas, int kb_total, int* splits_out, int* kbps_out) {
  int splits = (int)((148 + ctas - 1) / ctas);
  splits = splits < kb_total ? splits : kb_total;
  splits = splits < kMaxSplits ? splits : kMaxSplits;
  splits = splits < 1 ? 1 : splits;
  const int kbps = (kb_total + splits - 1) / splits;
  *splits_out = (kb_total + kbps - 1) / kbps;
  *kbps_out = kbps;
}

size_t tc_gemm_partial_bytes(int64_t T, int64_t f_tiles, int64_t f_total, int64_t K, int32_t batch) {
  if (T <= 0 || T > 256 || batch != 1) return 0;
  const int64_t ctas = f_tiles * ((T + swap_bn(T) - 1) / swap_bn(T));
  if (ctas >= 120) return 0;
  int splits, kbps;
  choose_splits(ctas, (int)(K / BK), &splits, &kbps);
  return splits > 1 ? (size_t)splits * T * f_total * sizeof(float) : 0;
}

cudaError_t tc_gemm(const TcGemmDesc& g, cudaStream_t st) {
  if (g.T <= 0) return cudaSuccess;
  if (g.K % BK != 0 || g.nseg < 1 || g.nseg > 2) return cudaErrorInvalidValue;
  const bool swap = g.T <= 256;
  if (g.w_mn && !swap) return cudaErrorInvalidValue;
  const int BN = swap ? swap_bn(g.T) : 256;
  const int w_tile = swap ? 128 : BN, x_tile = swap ? BN : 128;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.nseg = g.nseg;
  int64_t f_total = 0;
  int wtiles = 0;
  for (int s = 0; s < g.nseg; ++s) {
    const TcMatrix& w = g.seg[s].w;
    p.seg[s] = g.seg[s].epi;
    p.seg[s].f_base = f_total;
    p.seg[s].tiles = (int)((p.seg[s].f_rows + w_tile - 1) / w_tile);
    f_total += p.seg[s].f_rows;
    wtiles += p.seg[s].tiles;
    cudaError_t e = g.w_mn ? make_tmap_bf16(&p.wmap[s], w.ptr, w.cols, w.rows, w.ld, 64, 64)
                           : make_tmap_bf16(&p.wmap[s], w.ptr, w.cols, w.rows, w.ld, 64, w_tile);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = make_tmap_bf16(&p.xmap, g.x.ptr, g.x.cols, g.x.rows, g.x.ld, 64, x_tile);
  if (e != cudaSuccess) return e;
  const int ttiles = (int)((g.T + x_tile - 1) / x_tile);
  p.kb_total = (int)(g.K / BK);
  p.splits = 1;
  p.kb_per_split = p.kb_total;
  const int64_t ctas = (int64_t)wtiles * ttiles * g.batch;
  if (swap && g.batch == 1 && ctas < 120 && g.partial) {
    int splits, kbps;
    choose_splits(ctas, p.kb_total, &splits, &kbps);
    if ((size_t)splits * g.T * f_total * sizeof(float) <= g.partial_bytes && splits > 1) {
      p.splits = splits;
      p.kb_per_split = kbps;
    }
  }
  p.T = g.T;
  p.w_row_z = (int32_t)g.w_row_z;
  p.w_col_z = (int32_t)g.w_col_z;
  p.x_col_z = (int32_t)g.x_col_z;
  p.pos = g.pos;
  p.d_r = g.d_r;
  p.rope_base = g.rope_base;
  p.partial = g.partial;
  p.f_total = f_total;
  p.err = g.err;
  dim3 grid((unsigned)wtiles, (unsigned)ttiles, (unsigned)(g.batch * p.splits));
  if (!swap) e = launch_gemm<256, false, false, 4>(p, grid, st);
  else if (g.w_mn) {
    switch (BN) {
      case 16: e = launch_gemm<16, true, true, 8>(p, grid, st); break;
      case 32: e = launch_gemm<32, true, true, 8>(p, grid, st); break;
      case 64: e = launch_gemm<64, true, true, 8>(p, grid, st); break;
      default: e = launch_gemm<128, true, true, 6>(p, grid, st); break;
    }
  } else {
    switch (BN) {
      case 16: e = launch_gemm<16, true, false, 8>(p, grid, st); break;
      case 32: e = launch_gemm<32, true, false, 8>(p, grid, st); break;
      case 64: e = launch_gemm<64, true, false, 8>(p, grid, st); break;
      default: e = launch_gemm<128, true, false, 6>(p, grid, st); break;
    }
  }
  if (e != cudaSuccess || p.splits == 1) return e;
  ReduceParams r;
  memset(&r, 0, sizeof(r));
  r.seg[0] = p.seg[0];
  r.seg[1] = p.seg[1];
  r.nseg = p.nseg;
  r.splits = p.splits;
  r.T = g.T;
  r.f_total = f_total;
  r.partial = g.partial;
  r.pos = g.pos;
  r.d_r = g.d_r;
  r.rope_base = g.rope_base;
  r.err = g.err;
  dim3 rg((unsigned)((f_total / 2 + 255) / 256), (unsigned)g.T);
  splitk_reduce_kernel<<<rg, 256, 0, st>>>(r);
  return cudaGetLastError();
}

}  // namespace mla
