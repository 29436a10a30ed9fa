// tcgen05 GEMM kernel (TMA -> shared-memory ring -> tcgen05.mma into TMEM -> epilogue), the
// split-K reduce pass, and the host launcher that encodes the TMA tensor maps.
//
// The kernel is persistent: each CTA walks output tiles blockIdx.x, +gridDim.x, ... The TMA
// producer streams k-blocks of consecutive tiles through one ring; the MMA issuer alternates
// between two TMEM accumulators so the epilogue of one tile overlaps the MMAs of the next.
#include <cuda_bf16.h>
#include <math.h>
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
constexpr int kMaxRopePairs = 64;
constexpr int kRasterW = 8;      // weight tiles per raster group (large token counts)
constexpr int kIssuers = 4;      // TMA issuing lanes of the producer warp (every ring has 4 stages)

struct GemmParams {
  CUtensorMap wmap[2];
  CUtensorMap xmap;
  TcEpiSeg seg[2];
  int32_t nseg;
  int32_t splits, kb_total, kb_per_split;
  int32_t wtiles, ttiles, tiles;   // weight tiles (all segments), token tiles, total tiles
  int64_t T;
  int32_t w_row_z, w_col_z, x_col_z;
  const int64_t* pos;
  int32_t d_r;
  double theta[kMaxRopePairs];     // RoPE frequencies theta_m (plain or YaRN)
  float rope_mul;                  // factor on each rotated vector (YaRN; else 1)
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

// RoPE of one element of the pair (2m, 2m+1) that holds feature f (segment-local): `own` is x_f,
// `partner` is x_{f^1}. The angle pos * theta_m is reduced modulo 2 pi in double, then sincosf;
// the rotated value is multiplied by `mul`.
__device__ __forceinline__ float rope_one(int64_t f, int64_t pos, float own, float partner, int d_r,
                                          const double* theta, float mul) {
  const double a = (double)pos * theta[(f % d_r) >> 1];
  const double red = a - 6.283185307179586 * rint(a * 0.15915494309189535);
  float s, c;
  sincosf((float)red, &s, &c);
  return ((f & 1) ? (partner * s + own * c) : (own * c - partner * s)) * mul;
}

// Weight-streaming launches stage each epilogue warp's [16 tokens x 32 features] blocks in shared
// memory (8 KB per CTA) and store them as 16-byte vectors (per-element stores were issue-bound, about
// 150 to 300 ns each once the store queue filled).
constexpr int kEpiRows = 16;
template <int BN, bool SWAP>
__host__ __device__ constexpr uint32_t epi_stage_bytes() {
  return SWAP ? 4u * kEpiRows * 32u * 4u : 0u;
}

template <int BN, bool SWAP, bool W_MN, int STAGES>
__global__ void __launch_bounds__(kThreads) gemm_kernel(const __grid_constant__ GemmParams p) {
  constexpr uint32_t A_BYTES = 128 * 128;
  constexpr uint32_t B_BYTES = BN * 128;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t ACC_COLS = BN < 32 ? 32 : BN;     // one accumulator
  constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;          // double-buffered
  constexpr int W_TILE = SWAP ? 128 : BN;
  constexpr int X_TILE = SWAP ? BN : 128;
  constexpr int CH = BN < 32 ? BN : 32;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  // barriers: full[S], empty[S], acc_full[2], acc_empty[2]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  constexpr uint32_t EPI_STAGE = epi_stage_bytes<BN, SWAP>();
  float* epi_stage = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES + 256);   // [4 warps][16][32]
  auto bar = [&](int i) { return smem_addr(&bars[i]); };
  const int B_FULL = 0, B_EMPTY = STAGES, B_ACCF = 2 * STAGES, B_ACCE = 2 * STAGES + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * STAGES + 2; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(B_ACCE), 128);
    mbar_init(bar(B_ACCE + 1), 128);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    prefetch_tmap(&p.wmap[0]);
    if (p.nseg > 1) prefetch_tmap(&p.wmap[1]);
    prefetch_tmap(&p.xmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // tile index -> (segment, weight tile within it, token tile, batch z, split)
  struct Tile {
    int s, wt, tt, z, split, kb0, nkb;
  };
  auto decode_tile = [&](int idx) {
    Tile d;
    int wt, rest;
    if (!SWAP) {
      // large token counts: groups of kRasterW weight tiles x all token tiles, weight tile fastest,
      // so the CTAs running at the same time share a few weight tiles and a few token tiles in L2
      // (one batch, one split on this path)
      const int group = idx / (kRasterW * p.ttiles), local = idx % (kRasterW * p.ttiles);
      const int gw = min(kRasterW, p.wtiles - group * kRasterW);
      wt = group * kRasterW + local % gw;
      d.tt = local / gw;
      rest = 0;
    } else {
      d.tt = idx % p.ttiles;
      rest = idx / p.ttiles;
      wt = rest % p.wtiles;
      rest /= p.wtiles;
    }
    d.z = rest / p.splits;
    d.split = rest % p.splits;
    d.s = 0;
    if (p.nseg > 1 && wt >= p.seg[0].tiles) {
      d.s = 1;
      wt -= p.seg[0].tiles;
    }
    d.wt = wt;
    d.kb0 = d.split * p.kb_per_split;
    d.nkb = min(p.kb_total, d.kb0 + p.kb_per_split) - d.kb0;
    return d;
  };

  if (warp == 0) {
    // One TMA issuing thread streams only about 40 GB/s, so lanes 0 .. kIssuers-1 issue: lane l
    // loads the k-blocks it = l mod kIssuers (ring stages l, l + kIssuers, ...).
    if (lane < kIssuers) {
      int it = 0, last = -1;
      bool ok = true;
      for (int idx = blockIdx.x; ok && idx < p.tiles; idx += gridDim.x) {
        const Tile d = decode_tile(idx);
        const CUtensorMap* wm = &p.wmap[d.s];
        const int64_t f0 = (int64_t)d.wt * W_TILE, t0 = (int64_t)d.tt * X_TILE;
        for (int i = 0; i < d.nkb; ++i, ++it) {
          if ((it % kIssuers) != lane) continue;
          const int st = it % STAGES;
          if (!mbar_wait(bar(B_EMPTY + st), ((it / STAGES) & 1) ^ 1)) { ok = false; break; }
          const uint32_t full = bar(B_FULL + st);
          mbar_expect_tx(full, STAGE_BYTES);
          const int k0 = (d.kb0 + i) * BK;
          const uint32_t a_dst = smem_addr(sA + st * A_BYTES), b_dst = smem_addr(sB + st * B_BYTES);
          const uint32_t w_dst = SWAP ? a_dst : b_dst, x_dst = SWAP ? b_dst : a_dst;
          if (W_MN) {
#pragma unroll
            for (int jb = 0; jb < W_TILE / 64; ++jb)
              tma_load_2d(w_dst + jb * 8192, wm, (int)(f0 + 64 * jb) + d.z * p.w_col_z, k0 + d.z * p.w_row_z, full);
          } else {
            tma_load_2d(w_dst, wm, k0 + d.z * p.w_col_z, (int)f0 + d.z * p.w_row_z, full);
          }
          tma_load_2d(x_dst, &p.xmap, k0 + d.z * p.x_col_z, (int)t0, full);
          last = it;
        }
      }
      if (!ok) {
        flag_error(p.err, DEVERR_TIMEOUT);
        for (int i = max(lane, last - STAGES + 1); i <= last; ++i)
          if ((i % kIssuers) == lane) mbar_wait(bar(B_FULL + i % STAGES), (i / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BN, (SWAP && W_MN) ? 1 : 0, (!SWAP && W_MN) ? 1 : 0);
      int it = 0, n = 0;
      bool ok = true;
      for (int idx = blockIdx.x; ok && idx < p.tiles; idx += gridDim.x, ++n) {
        const Tile d = decode_tile(idx);
        const int acc = n & 1;
        if (!mbar_wait(bar(B_ACCE + acc), ((n >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem + acc * ACC_COLS;
        for (int i = 0; i < d.nkb; ++i, ++it) {
          const int st = it % STAGES;
          if (!mbar_wait(bar(B_FULL + st), (it / STAGES) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_addr(sA + st * A_BYTES), b_base = smem_addr(sB + st * B_BYTES);
          // base descriptors, advanced by (byte offset >> 4) in the start-address field per K step
          const uint64_t ad0 = (SWAP && W_MN) ? sw128_desc(a_base, 8192, 1024) : sw128_desc(a_base, 0, 1024);
          const uint64_t bd0 = (!SWAP && W_MN) ? sw128_desc(b_base, 8192, 1024) : sw128_desc(b_base, 0, 1024);
          constexpr uint32_t a_step = ((SWAP && W_MN) ? 2048 : 32) >> 4, b_step = ((!SWAP && W_MN) ? 2048 : 32) >> 4;
#pragma unroll
          for (int j = 0; j < BK / 16; ++j)
            mma_bf16_ss(dt, ad0 + j * a_step, bd0 + j * b_step, idesc, (i > 0 || j > 0) ? 1u : 0u);
          mma_commit(bar(B_EMPTY + st));
        }
        if (!ok) break;
        mma_commit(bar(B_ACCF + acc));
      }
      if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;  // accumulator row = TMEM lane
    int n = 0;
    bool ok = true;
    for (int idx = blockIdx.x; ok && idx < p.tiles; idx += gridDim.x, ++n) {
      const Tile d = decode_tile(idx);
      const TcEpiSeg E = d.s ? p.seg[1] : p.seg[0];   // in registers (see the swap path below)
      const int acc = n & 1;
      if (!mbar_wait(bar(B_ACCF + acc), (n >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t trow = tmem + acc * ACC_COLS + ((uint32_t)(q * 32) << 16);
      const int64_t f0 = (int64_t)d.wt * W_TILE, t0 = (int64_t)d.tt * X_TILE;
      // tile orientation: this thread's token row, through the row map (cache slots) when there is one
      int64_t row_r = t0 + r;
      bool row_ok = !SWAP && t0 + r < p.T;
      if (!SWAP && row_ok && E.rowmap) {
        row_r = E.rowmap[t0 + r];
        row_ok = row_r >= 0 && row_r < E.rowmap_limit;
      }
#pragma unroll 1
      for (int c = 0; c < BN; c += CH) {
        uint32_t v[32];
        if (CH == 32) tmem_ld32(trow + c, v);
        else tmem_ld16(trow + c, v);
        tmem_wait_ld();
        if (!SWAP && CH == 32) {
          // a token row's 32 consecutive features: bf16, 16-byte stores, when the layout allows
          const int64_t t = t0 + r, f = f0 + c;
          if (p.splits == 1 && !E.out_f32 && E.so_f == 1 && d.z == 0 && f + 32 <= E.f_rows && t < p.T &&
              ((row_r * E.so_t + f) & 7) == 0 && (reinterpret_cast<uintptr_t>(E.out) & 15) == 0) {
            if (!row_ok) {
              flag_error(p.err, DEVERR_SLOT);
              continue;
            }
            int64_t ps = 0;
            if (E.rope) {
              ps = p.pos[t];
              if (ps < 0) {
                flag_error(p.err, DEVERR_POSITION);
                continue;
              }
            }
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              float a = __uint_as_float(v[j]), b2 = __uint_as_float(v[j + 1]);
              if (E.rope) {
                const float a2 = rope_one(f + j, ps, a, b2, p.d_r, p.theta, p.rope_mul);
                const float b3 = rope_one(f + j + 1, ps, b2, a, p.d_r, p.theta, p.rope_mul);
                a = a2;
                b2 = b3;
              }
              pk[j / 2] = pack_bf16(a, b2);
            }
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(E.out) + row_r * E.so_t + f);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
            continue;
          }
        }
        if constexpr (SWAP) {
          // weight-streaming orientation: this thread holds feature f0 + r for CH consecutive tokens.
          // The segment's fields are plain scalars read once per tile at fixed parameter offsets, and
          // the stores go through shared memory as 16-byte vectors where the layout allows (below).
          const bool s1 = d.s != 0;
          char* const out = reinterpret_cast<char*>(s1 ? p.seg[1].out : p.seg[0].out);
          const int64_t so_t = s1 ? p.seg[1].so_t : p.seg[0].so_t;
          const int64_t so_f = s1 ? p.seg[1].so_f : p.seg[0].so_f;
          const int64_t so_z = s1 ? p.seg[1].so_z : p.seg[0].so_z;
          const bool out_f32 = (s1 ? p.seg[1].out_f32 : p.seg[0].out_f32) != 0;
          const bool rope = (s1 ? p.seg[1].rope : p.seg[0].rope) != 0;
          const int64_t* const rowmap = s1 ? p.seg[1].rowmap : p.seg[0].rowmap;
          const int64_t rowmap_limit = s1 ? p.seg[1].rowmap_limit : p.seg[0].rowmap_limit;
          const int64_t f_rows = s1 ? p.seg[1].f_rows : p.seg[0].f_rows;
          const int64_t f_base = s1 ? p.seg[1].f_base : p.seg[0].f_base;
          const int64_t f = f0 + r, T = p.T;
          const bool fok = f < f_rows;
          if constexpr (EPI_STAGE > 0) {
            // this warp's features fw .. fw + 31 for the CH tokens of this chunk, through shared memory
            const int64_t fw = f0 + 32 * q;
            const bool part = p.splits > 1;
            const bool vec = (f_rows & (part ? 3 : 7)) == 0 &&   // a vector is all valid or all past f_rows
                             (part ? ((p.f_total & 3) == 0 && (f_base & 3) == 0)
                                   : (!rope && !rowmap && !out_f32 && so_f == 1 && (so_t & 7) == 0 &&
                                      (((int64_t)d.z * so_z + fw) & 7) == 0 &&
                                      (reinterpret_cast<uintptr_t>(out) & 15) == 0));
            if (vec) {
              float* stg = epi_stage + q * (kEpiRows * 32);
#pragma unroll
              for (int h = 0; h < CH / kEpiRows; ++h) {   // 16 tokens at a time
                const int64_t tb = t0 + c + kEpiRows * h;
                __syncwarp();
#pragma unroll
                for (int j = 0; j < kEpiRows; ++j) stg[j * 32 + lane] = __uint_as_float(v[kEpiRows * h + j]);
                __syncwarp();
                if (part) {
                  // rows of 32 fp32 = 8 vectors of 4; 16 rows over the 32 lanes
#pragma unroll
                  for (int i = 0; i < kEpiRows / 4; ++i) {
                    const int cid = i * 32 + lane, j = cid >> 3, c4 = cid & 7;
                    const int64_t t = tb + j, fe = fw + 4 * c4;
                    if (t < T && fe < f_rows)
                      *reinterpret_cast<float4*>(p.partial + ((int64_t)d.split * T + t) * p.f_total + f_base + fe) =
                          *reinterpret_cast<const float4*>(stg + j * 32 + 4 * c4);
                  }
                } else {
                  // rows of 32 bf16 = 4 vectors of 8; 16 rows over the 32 lanes
#pragma unroll
                  for (int i = 0; i < kEpiRows / 8; ++i) {
                    const int cid = i * 32 + lane, j = cid >> 2, c8 = cid & 3;
                    const int64_t t = tb + j, fe = fw + 8 * c8;
                    if (t < T && fe < f_rows) {
                      const float* x = stg + j * 32 + 8 * c8;
                      *reinterpret_cast<uint4*>(out + 2 * ((int64_t)d.z * so_z + fe + t * so_t)) =
                          make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                                     pack_bf16(x[6], x[7]));
                    }
                  }
                }
              }
              continue;
            }
          }
          if (p.splits > 1) {
            float* dst = p.partial + ((int64_t)d.split * T + t0 + c) * p.f_total + f_base + f;
            const int64_t step = p.f_total;
#pragma unroll
            for (int j = 0; j < CH; ++j)
              if (fok && t0 + c + j < T) dst[j * step] = __uint_as_float(v[j]);
            continue;
          }
          const int64_t base = (int64_t)d.z * so_z + f * so_f;
#pragma unroll
          for (int j = 0; j < CH; ++j) {
            const int64_t t = t0 + c + j;
            float y = __uint_as_float(v[j]);
            if (rope) {
              const float partner = __shfl_xor_sync(0xffffffffu, y, 1);
              if (!fok || t >= T) continue;
              const int64_t ps = p.pos[t];
              if (ps < 0) {
                flag_error(p.err, DEVERR_POSITION);
                continue;
              }
              y = rope_one(f, ps, y, partner, p.d_r, p.theta, p.rope_mul);
            }
            if (!fok || t >= T) continue;
            int64_t row = t;
            if (rowmap) {
              row = rowmap[t];
              if (row < 0 || row >= rowmap_limit) {
                flag_error(p.err, DEVERR_SLOT);
                continue;
              }
            }
            const int64_t idx = base + row * so_t;
            if (out_f32) reinterpret_cast<float*>(out)[idx] = y;
            else reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(y);
          }
        } else {
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          const float x = __uint_as_float(v[j]);
          const int64_t f = f0 + c + j, t = t0 + r;
          const float partner = __uint_as_float(v[j ^ 1]);
          if (f >= E.f_rows || t >= p.T) continue;
          if (p.splits > 1) {
            p.partial[((int64_t)d.split * p.T + t) * p.f_total + E.f_base + f] = x;
            continue;
          }
          float y = x;
          if (E.rope) {
            const int64_t ps = p.pos[t];
            if (ps < 0) {
              flag_error(p.err, DEVERR_POSITION);
              continue;
            }
            y = rope_one(f, ps, x, partner, p.d_r, p.theta, p.rope_mul);
          }
          store_out(E, p.err, d.z, f, t, y);
        }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_ACCE + acc));
    }
    if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
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
  double theta[kMaxRopePairs];
  float rope_mul;
  uint32_t* err;
};

// Sums the split-K partials of feature pairs (f, f+1), then applies the epilogue. L lanes per (token,
// feature pair), L = 1, 2 or 4 so that each lane has at most 8 splits: lane l issues the loads of splits
// l, l + L, ... at once and adds them in order, then the group adds its lanes by a fixed xor tree, so
// the result does not depend on timing. (One lane per split needed thousands of blocks for a few MB of
// L2-resident partials and was bound by the waves of blocks; one thread per pair serialised up to four
// rounds of loads when there are 28 splits.)
constexpr int kReduceBatch = 8;
template <int L>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const __grid_constant__ ReduceParams p) {
  const int64_t npairs = p.f_total / 2;
  const int64_t gid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / L;
  const int l = threadIdx.x & (L - 1);
  const bool active = gid < npairs * p.T;
  const int64_t t = active ? gid / npairs : 0, f = active ? 2 * (gid % npairs) : 0;
  const float* src = p.partial + t * p.f_total + f;
  const int64_t kstride = p.T * p.f_total;
  float a = 0.f, b = 0.f;
  if (active) {
    for (int k0 = l; k0 < p.splits; k0 += kReduceBatch * L) {
      float2 v[kReduceBatch];
#pragma unroll
      for (int u = 0; u < kReduceBatch; ++u)
        v[u] = k0 + u * L < p.splits ? *reinterpret_cast<const float2*>(src + (int64_t)(k0 + u * L) * kstride)
                                     : make_float2(0.f, 0.f);
#pragma unroll
      for (int u = 0; u < kReduceBatch; ++u) {
        a += v[u].x;
        b += v[u].y;
      }
    }
  }
#pragma unroll
  for (int o = L / 2; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  if (!active || l != 0) return;
  const int s = (p.nseg > 1 && f >= p.seg[1].f_base) ? 1 : 0;
  const TcEpiSeg E = s ? p.seg[1] : p.seg[0];   // in registers, not read through the parameters
  const int64_t fl = f - E.f_base;
  if (E.rope) {
    const int64_t ps = p.pos[t];
    if (ps < 0) {
      flag_error(p.err, DEVERR_POSITION);
      return;
    }
    const float a2 = rope_one(fl, ps, a, b, p.d_r, p.theta, p.rope_mul);
    const float b2 = rope_one(fl + 1, ps, b, a, p.d_r, p.theta, p.rope_mul);
    a = a2;
    b = b2;
  }
  if (E.so_f == 1 && fl + 1 < E.f_rows && ((E.so_t | fl) & 1) == 0 && (reinterpret_cast<uintptr_t>(E.out) & 7) == 0) {
    // the pair is contiguous: one 4-byte (bf16) or 8-byte (fp32) store
    int64_t row = t;
    if (E.rowmap) {
      row = E.rowmap[t];
      if (row < 0 || row >= E.rowmap_limit) {
        flag_error(p.err, DEVERR_SLOT);
        return;
      }
    }
    const int64_t idx = row * E.so_t + fl;
    if (E.out_f32) *reinterpret_cast<float2*>(reinterpret_cast<float*>(E.out) + idx) = make_float2(a, b);
    else *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(E.out) + idx) = pack_bf16(a, b);
    return;
  }
  store_out(E, p.err, 0, fl, t, a);
  if (fl + 1 < E.f_rows) store_out(E, p.err, 0, fl + 1, t, b);
}

// The same for at most 8 splits with four consecutive features per thread (segments and feature counts
// in multiples of 4): float4 loads of every split at once, in split order, and one 8-byte (bf16) or
// 16-byte (fp32) store; half the threads and blocks of a thread per pair.
__global__ void __launch_bounds__(256) splitk_reduce4_kernel(const __grid_constant__ ReduceParams p) {
  const int64_t nquads = p.f_total / 4;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= nquads * p.T) return;
  const int64_t t = gid / nquads, f = 4 * (gid % nquads);
  const float* src = p.partial + t * p.f_total + f;
  const int64_t kstride = p.T * p.f_total;
  float4 v[kReduceBatch];
#pragma unroll
  for (int u = 0; u < kReduceBatch; ++u)
    v[u] = u < p.splits ? *reinterpret_cast<const float4*>(src + (int64_t)u * kstride) : make_float4(0.f, 0.f, 0.f, 0.f);
  float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int u = 0; u < kReduceBatch; ++u) {
    x[0] += v[u].x;
    x[1] += v[u].y;
    x[2] += v[u].z;
    x[3] += v[u].w;
  }
  const int s = (p.nseg > 1 && f >= p.seg[1].f_base) ? 1 : 0;
  const TcEpiSeg E = s ? p.seg[1] : p.seg[0];
  const int64_t fl = f - E.f_base;
  if (E.rope) {
    const int64_t ps = p.pos[t];
    if (ps < 0) {
      flag_error(p.err, DEVERR_POSITION);
      return;
    }
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const float a2 = rope_one(fl + e, ps, x[e], x[e + 1], p.d_r, p.theta, p.rope_mul);
      const float b2 = rope_one(fl + e + 1, ps, x[e + 1], x[e], p.d_r, p.theta, p.rope_mul);
      x[e] = a2;
      x[e + 1] = b2;
    }
  }
  int64_t row = t;
  if (E.rowmap) {
    row = E.rowmap[t];
    if (row < 0 || row >= E.rowmap_limit) {
      flag_error(p.err, DEVERR_SLOT);
      return;
    }
  }
  if (E.so_f == 1 && fl + 3 < E.f_rows && ((E.so_t | fl) & 3) == 0 && (reinterpret_cast<uintptr_t>(E.out) & 15) == 0) {
    const int64_t idx = row * E.so_t + fl;
    if (E.out_f32) *reinterpret_cast<float4*>(reinterpret_cast<float*>(E.out) + idx) = make_float4(x[0], x[1], x[2], x[3]);
    else *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(E.out) + idx) = make_uint2(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]));
    return;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (fl + e < E.f_rows) store_out(E, p.err, 0, fl + e, t, x[e]);
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

cudaError_t make_tmap_bf16(CUtensorMap* m, const void* ptr, int64_t inner, int64_t outer, int64_t ld, int box_inner,
                           int box_outer, int swizzle_bytes) {
  if (swizzle_bytes != 128 && swizzle_bytes != 64) return cudaErrorInvalidValue;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_u8(CUtensorMap* m, const void* ptr, int64_t inner, int64_t outer, int64_t ld, int box_inner,
                         int box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)ld};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

int g_num_sms = 0;

int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_num_sms = n > 0 ? n : 148;
  }
  return g_num_sms;
}

template <int BN, bool SWAP, bool W_MN, int STAGES>
cudaError_t launch_gemm(const GemmParams& p, int ctas_per_sm, cudaStream_t st) {
  constexpr size_t smem = (size_t)STAGES * (128 * 128 + BN * 128) + 1024 + 256 + epi_stage_bytes<BN, SWAP>();
  static bool configured = false;
  auto kern = gemm_kernel<BN, SWAP, W_MN, STAGES>;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  int grid = num_sms() * ctas_per_sm;
  if (grid > p.tiles) grid = p.tiles;
  kern<<<grid, kThreads, smem, st>>>(p);
  note_launch();
  return cudaGetLastError();
}

int swap_bn(int64_t T) { return T <= 16 ? 16 : T <= 32 ? 32 : T <= 64 ? 64 : 128; }

// CTA slots of a weight-streaming launch on a 148-SM B200 (two CTAs per SM up to BN = 64). The
// split decision uses this fixed count so that workspace sizing and launches always agree.
int swap_slots(int BN) { return BN <= 64 ? 2 * 148 : 148; }

// Split-K factor for a swap-orientation launch of `ctas` output tiles over kb_total k-blocks on
// `slots` resident CTAs: going up from 1, a factor is taken when it cuts the k-blocks the busiest
// CTA streams (ceil(items / slots) * ceil(kb_total / splits)) by at least 10% against the best so
// far (more splits also mean more fp32 partials to write and sum), with at least four k-blocks
// (256 of K) per split. Returns (splits, k-blocks per split).
void choose_splits(int64_t ctas, int kb_total, int slots, int* splits_out, int* kbps_out) {
  int max_splits = kb_total / 4;
  max_splits = max_splits < kMaxSplits ? max_splits : kMaxSplits;
  int best = 1;
  int64_t best_load = ((ctas + slots - 1) / slots) * (int64_t)kb_total;
  for (int sp = 2; sp <= max_splits; ++sp) {
    const int kbps = (kb_total + sp - 1) / sp;
    const int real = (kb_total + kbps - 1) / kbps;
    const int64_t load = ((ctas * real + slots - 1) / slots) * (int64_t)kbps;
    if (load * 10 < best_load * 9) {
      best_load = load;
      best = real;
    }
  }
  const int kbps = (kb_total + best - 1) / best;
  *splits_out = (kb_total + kbps - 1) / kbps;
  *kbps_out = kbps;
}

}  // namespace

size_t tc_gemm_partial_bytes(int64_t T, int64_t f_tiles, int64_t f_total, int64_t K, int32_t batch) {
  if (T <= 0 || T > kSwapMaxTokens || batch != 1) return 0;
  const int64_t ctas = f_tiles * ((T + swap_bn(T) - 1) / swap_bn(T));
  const int slots = swap_slots(swap_bn(T));
  int splits, kbps;
  choose_splits(ctas, (int)(K / BK), slots, &splits, &kbps);
  return splits > 1 ? (size_t)splits * T * f_total * sizeof(float) : 0;
}

cudaError_t tc_gemm(const TcGemmDesc& g, cudaStream_t st) {
  if (g.T <= 0) return cudaSuccess;
  if (g.K % BK != 0 || g.nseg < 1 || g.nseg > 2 || g.d_r > 2 * kMaxRopePairs) return cudaErrorInvalidValue;
  const bool swap = g.T <= kSwapMaxTokens;
  // head batching and MN-major weights exist only in the swap orientation
  if ((g.w_mn || g.batch != 1) && !swap) return cudaErrorInvalidValue;
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
  if (swap && g.batch == 1 && g.partial) {
    int splits, kbps;
    choose_splits(ctas, p.kb_total, swap_slots(BN), &splits, &kbps);
    if ((size_t)splits * g.T * f_total * sizeof(float) <= g.partial_bytes && splits > 1) {
      p.splits = splits;
      p.kb_per_split = kbps;
    }
  }
  p.wtiles = wtiles;
  p.ttiles = ttiles;
  p.tiles = wtiles * ttiles * g.batch * p.splits;
  p.T = g.T;
  p.w_row_z = (int32_t)g.w_row_z;
  p.w_col_z = (int32_t)g.w_col_z;
  p.x_col_z = (int32_t)g.x_col_z;
  p.pos = g.pos;
  p.d_r = g.d_r;
  for (int m = 0; m < g.d_r / 2; ++m) p.theta[m] = rope_theta(g.rope, m, g.d_r);
  p.rope_mul = rope_mul(g.rope);
  p.partial = g.partial;
  p.f_total = f_total;
  p.err = g.err;
  // weight streaming (swap): 4 stages, two CTAs per SM; large token counts: 128x256 tiles, 4 stages
  if (!swap) e = launch_gemm<256, false, false, 4>(p, 1, st);
  else if (g.w_mn) {
    switch (BN) {
      case 16: e = launch_gemm<16, true, true, 4>(p, 2, st); break;
      case 32: e = launch_gemm<32, true, true, 4>(p, 2, st); break;
      case 64: e = launch_gemm<64, true, true, 4>(p, 2, st); break;
      default: e = launch_gemm<128, true, true, 4>(p, 1, st); break;
    }
  } else {
    switch (BN) {
      case 16: e = launch_gemm<16, true, false, 4>(p, 2, st); break;
      case 32: e = launch_gemm<32, true, false, 4>(p, 2, st); break;
      case 64: e = launch_gemm<64, true, false, 4>(p, 2, st); break;
      default: e = launch_gemm<128, true, false, 4>(p, 1, st); break;
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
  memcpy(r.theta, p.theta, sizeof(r.theta));
  r.rope_mul = p.rope_mul;
  r.err = g.err;
  const int L = p.splits <= kReduceBatch ? 1 : p.splits <= 2 * kReduceBatch ? 2 : 4;
  const unsigned rg = (unsigned)(((f_total / 2) * g.T * L + 255) / 256);
  bool quads = L == 1 && f_total % 4 == 0;
  for (int sgi = 0; sgi < p.nseg; ++sgi) quads = quads && p.seg[sgi].f_rows % 4 == 0 && p.seg[sgi].f_base % 4 == 0;
  if (quads) splitk_reduce4_kernel<<<(unsigned)((f_total / 4 * g.T + 255) / 256), 256, 0, st>>>(r);
  else if (L == 1) splitk_reduce_kernel<1><<<rg, 256, 0, st>>>(r);
  else if (L == 2) splitk_reduce_kernel<2><<<rg, 256, 0, st>>>(r);
  else splitk_reduce_kernel<4><<<rg, 256, 0, st>>>(r);
  note_launch();
  return cudaGetLastError();
}

}  // namespace mla
