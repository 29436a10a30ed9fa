// Causal prefill attention core at the DeepSeek-V3 sizes (n_h = 128, d_h = 128, d_h^R = 64), bf16
// inputs, fp32 accumulation, tcgen05 + TMA on sm_100a.
//
// It computes step (10) of section 一(一) of the DeepSeek-V3 notes in the unabsorbed form: for every
// head i and query token t at position p of its sequence,
//   q = [q^C_t,i ; q^R_t,i] (192),  k_j = [k^C_j,i ; k^R_j] (192, k^R shared by the heads),
//   o_t,i = sum_{j <= p} softmax_j(q . k_j / sqrt(d_h + d_h^R)) v^C_j,i   (128).
// The query tokens of sequence b may be the last Tc_b of its len_b key rows (a chunk after a cached
// prefix of P_b = len_b - Tc_b rows, whose keys are reused as they are): query token r of the chunk
// sits at position P_b + r. A whole-sequence prefill is the case P_b = 0.
//
// Work unit: one head and one tile of 128 query rows of one sequence; it walks the key tiles of
// 128 rows up to the last one its rows can see (flash-attention online softmax), masking the keys
// past each row's position. The kernel is persistent (one CTA
// per SM); units run head-major with query tiles in descending order, so that the CTAs running at
// the same time share one head's k^C / v^C in L2 and the long units start first.
//
// Per CTA: q (128 x 192 bf16) sits in TMEM as the A operand of QK^T; scores S go to one of two
// 128-column TMEM buffers; P is written back as bf16 into the first 64 columns of the buffer it
// came from and is the A operand of P.V; O takes 128 TMEM columns. Key tiles stream through a
// 3-stage ring (k^C two 64-column boxes + k^R one box, 48 KB) and value tiles through a 2-stage
// ring (two 64-column boxes, 32 KB), all loaded by TMA with 128-byte swizzle.
//
// Roles (192 threads): warps 0-3 softmax/epilogue (thread i = query row i = TMEM lane i), warp 4 TMA
// producer, warp 5 TMEM owner + MMA issuer. Every wait is bounded.
#include <cuda_bf16.h>
#include <string.h>

#include "sm100.cuh"
#include "tc.cuh"
#include "tc_gemm.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int H = 128, DH = 128, DR = 64, DQK = DH + DR, CROW = 512 + DR;
constexpr int BM = 128, BN = 128;             // query rows and key rows per tile
constexpr int KSTAGES = 3, VSTAGES = 2;
constexpr int kThreads = 192;
constexpr float kRescaleLog2 = 8.f;           // lazy rescale threshold of the running max (log2 units)

constexpr uint32_t BOX = BN * 128;            // [128 rows x 64 cols] bf16, 128-byte swizzle: 16 KB
constexpr uint32_t K_BYTES = 3 * BOX;         // k^C cols 0-63, 64-127, k^R
constexpr uint32_t V_BYTES = 2 * BOX;         // v^C cols 0-63, 64-127
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = OFF_K + KSTAGES * K_BYTES;
constexpr uint32_t OFF_BAR = OFF_V + VSTAGES * V_BYTES;

constexpr int B_KFULL = 0, B_KEMPTY = B_KFULL + KSTAGES, B_VFULL = B_KEMPTY + KSTAGES, B_VEMPTY = B_VFULL + VSTAGES,
              B_SFULL = B_VEMPTY + VSTAGES, B_PFULL = B_SFULL + 2, B_PVDONE = B_PFULL + 2, B_QFULL = B_PVDONE + 1,
              B_QEMPTY = B_QFULL + 1, B_OFREE = B_QEMPTY + 1;
constexpr int NBAR = B_OFREE + 1;
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns: S0 [0, 128), S1 [128, 256) (P as bf16 pairs in the first 64 of each), O [256, 384),
// q as bf16 pairs [384, 480): q^C cols 0-63, 64-127, then q^R.
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_O = 256, T_Q = 384;

struct PrefillParams {
  CUtensorMap kc_map;   // k^C as [T_kv, H * 128], box {64, 128}
  CUtensorMap kr_map;   // cache as [capacity, 576], box {64, 128} (k^R at column 512)
  CUtensorMap vc_map;   // v^C as [T_kv, H * 128], box {64, 128}
  const __nv_bfloat16* qc;   // [T][H][128]
  const __nv_bfloat16* qr;   // [T][H][64]
  __nv_bfloat16* o;          // [T][H][128]
  const int64_t* cu;         // [B + 1] query tokens of each sequence
  const int64_t* cu_kv;      // [B + 1] key rows of each sequence (k^C, v^C and cache rows)
  int32_t B, M;              // sequences; query tiles of the longest sequence
  int64_t T;
  float scale_log2;          // log2(e) / sqrt(d_h + d_h^R)
  uint32_t* err;
};

// Unit u -> head, query tile (descending), sequence; false when the sequence has no such tile.
struct Unit {
  int h, m, b;
  int nt;               // key tiles the unit's rows see
  int64_t row0, len;    // first packed query row of the sequence, its query count
  int64_t kv0, pre;     // first key row of the sequence, its prefix (position of query row 0)
};
__device__ __forceinline__ bool unit_of(const PrefillParams& p, int64_t u, Unit& x) {
  const int64_t per_head = (int64_t)p.B * p.M;
  x.h = (int)(u / per_head);
  const int64_t rem = u % per_head;
  x.m = p.M - 1 - (int)(rem / p.B);
  x.b = (int)(rem % p.B);
  x.row0 = p.cu[x.b];
  x.len = p.cu[x.b + 1] - x.row0;
  x.kv0 = p.cu_kv[x.b];
  x.pre = (p.cu_kv[x.b + 1] - x.kv0) - x.len;
  const int64_t r_last = min((int64_t)x.m * BM + BM - 1, x.len - 1);   // the tile's last valid row
  x.nt = (int)((x.pre + r_last) / BN) + 1;
  return (int64_t)x.m * BM < x.len && x.pre >= 0;
}

__global__ void __launch_bounds__(kThreads, 1) prefill_attn_kernel(const __grid_constant__ PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  const uint32_t sbase = smem_addr(smem);
  auto bar = [&](int i) { return smem_addr(&bars[i]); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t U = (int64_t)H * p.B * p.M;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) {
      const bool many = i == B_PFULL || i == B_PFULL + 1 || i == B_QFULL || i == B_OFREE;
      mbar_init(bar(i), many ? 128 : 1);
    }
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    prefetch_tmap(&p.kc_map);
    prefetch_tmap(&p.kr_map);
    prefetch_tmap(&p.vc_map);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    // lane 0 streams the key tiles, lane 1 the value tiles, each through its own ring
    if (lane < 2) {
      const bool keys = lane == 0;
      const int nst = keys ? KSTAGES : VSTAGES;
      const uint32_t bytes = keys ? K_BYTES : V_BYTES;
      const int b_full = keys ? B_KFULL : B_VFULL, b_empty = keys ? B_KEMPTY : B_VEMPTY;
      const uint32_t base = sbase + (keys ? OFF_K : OFF_V);
      int j = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; ok && u < U; u += gridDim.x) {
        Unit x;
        if (!unit_of(p, u, x)) continue;
        for (int n = 0; n < x.nt; ++n, ++j) {
          const int s = j % nst;
          if (!mbar_wait(bar(b_empty + s), ((j / nst) & 1) ^ 1)) { ok = false; break; }
          mbar_expect_tx(bar(b_full + s), bytes);
          const int32_t y = (int32_t)(x.kv0 + (int64_t)n * BN);
          const uint32_t dst = base + s * bytes;
          const CUtensorMap* map = keys ? &p.kc_map : &p.vc_map;
          tma_load_2d(dst, map, DH * x.h, y, bar(b_full + s));
          tma_load_2d(dst + BOX, map, DH * x.h + 64, y, bar(b_full + s));
          if (keys) tma_load_2d(dst + 2 * BOX, &p.kr_map, 512, y, bar(b_full + s));
        }
      }
      if (!ok) {
        flag_error(p.err, DEVERR_TIMEOUT);
        for (int i = max(0, j - nst); i < j; ++i) mbar_wait(bar(b_full + i % nst), (i / nst) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    // Per unit: QK^T(0); then for each key tile n: QK^T(n + 1) (so that the tensor pipe works on it
    // while the softmax takes tile n), then P.V(n).
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(BM, DH, 0, 1);
      int J = 0, jk = 0, jv = 0, g = 0;
      bool ok = true;
      // QK^T of global tile JJ from key stage jk into score buffer JJ & 1
      auto qk = [&](int JJ, bool last) -> bool {
        const int ks = jk % KSTAGES;
        if (!mbar_wait(bar(B_KFULL + ks), (jk / KSTAGES) & 1)) return false;
        tc_fence_after();
        const uint32_t kst = sbase + OFF_K + ks * K_BYTES;
        const uint32_t d = tmem + BN * (JJ & 1);
        // descriptors advance by adding (byte offset >> 4) to the start-address field (bits 0-13)
        const uint64_t bk = sw128_desc(kst, 0, 1024);
#pragma unroll
        for (int k = 0; k < DQK / 16; ++k)
          mma_bf16_ts(d, tmem + T_Q + 8 * k, bk + ((((k >> 2) * BOX) + (k & 3) * 32) >> 4), idesc_qk, k ? 1u : 0u);
        mma_commit(bar(B_SFULL + (JJ & 1)));
        mma_commit(bar(B_KEMPTY + ks));
        if (last) mma_commit(bar(B_QEMPTY));
        ++jk;
        return true;
      };
      for (int64_t u = blockIdx.x; ok && u < U; u += gridDim.x) {
        Unit x;
        if (!unit_of(p, u, x)) continue;
        if (!mbar_wait(bar(B_QFULL), g & 1)) { ok = false; break; }
        if (!qk(J, x.nt == 1)) { ok = false; break; }
        for (int n = 0; n < x.nt; ++n, ++J) {
          if (n + 1 < x.nt && !qk(J + 1, n + 2 == x.nt)) { ok = false; break; }
          const int vs = jv % VSTAGES;
          if (!mbar_wait(bar(B_PFULL + (J & 1)), (J >> 1) & 1) || !mbar_wait(bar(B_VFULL + vs), (jv / VSTAGES) & 1) ||
              (n == 0 && !mbar_wait(bar(B_OFREE), (g & 1) ^ 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t vst = sbase + OFF_V + vs * V_BYTES;
          const uint32_t pa = tmem + BN * (J & 1);
          const uint64_t bv = sw128_desc(vst, BOX, 1024);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_bf16_ts(tmem + T_O, pa + 8 * kk, bv + (kk * 2048 >> 4), idesc_pv, (n > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(B_PVDONE));
          mma_commit(bar(B_VEMPTY + vs));
          ++jv;
        }
        ++g;
      }
      if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int i = threadIdx.x;                       // query row within the tile
    const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
    const float c2 = p.scale_log2;
    const float thr_raw = kRescaleLog2 / c2;
    auto wait_u = [](uint32_t b, uint32_t par) { return __all_sync(0xffffffffu, mbar_wait(b, par)) != 0; };
    int J = 0, g = 0;
    bool ok = true;
    // q of unit x -> TMEM (row i of the tile; rows past the sequence read as zero), once the previous
    // unit's last QK^T is done with it.
    auto load_q = [&](const Unit& x, int gg) -> bool {
      if (!wait_u(bar(B_QEMPTY), (gg & 1) ^ 1)) return false;
      tc_fence_after();
      const int64_t r = (int64_t)x.m * BM + i;
      const bool valid = r < x.len;
      const int64_t t = x.row0 + r;
      const uint4* src = reinterpret_cast<const uint4*>(p.qc + (t * H + x.h) * DH);
      const uint4* rsrc = reinterpret_cast<const uint4*>(p.qr + (t * H + x.h) * DR);
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        uint32_t v[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 w = valid ? __ldg(c < 2 ? src + 8 * c + e : rsrc + e) : make_uint4(0, 0, 0, 0);
          v[4 * e] = w.x; v[4 * e + 1] = w.y; v[4 * e + 2] = w.z; v[4 * e + 3] = w.w;
        }
        tmem_st32(trow + T_Q + 32 * c, v);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_QFULL));
      return true;
    };
    // the first valid unit at or after u
    auto next_unit = [&](int64_t u, Unit& x) -> int64_t {
      for (; u < U; u += gridDim.x)
        if (unit_of(p, u, x)) return u;
      return U;
    };
    Unit x;
    int64_t u = next_unit(blockIdx.x, x);
    if (u < U && !load_q(x, 0)) ok = false;
    for (; ok && u < U; ++g) {
      float m_ref = -INFINITY, l = 0.f;              // running max (raw score units) and row sum
      // row i sits at position pre + 128 m + i: key c of tile n is visible while 128 n + c <= that
      const int64_t rpos = x.pre + (int64_t)x.m * BM + i;
      for (int n = 0; n < x.nt; ++n, ++J) {
        const int sb = J & 1;
        if (!wait_u(bar(B_SFULL + sb), (J >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        float s[BN];
#pragma unroll
        for (int c = 0; c < BN; c += 32) tmem_ld32(trow + BN * sb + c, reinterpret_cast<uint32_t*>(s + c));
        tmem_wait_ld();
        const int64_t lim = rpos - (int64_t)n * BN;   // the last visible key column of this tile
        if (lim < BN - 1) {
          const int li = (int)max(lim, (int64_t)-1);
#pragma unroll
          for (int c = 0; c < BN; ++c) s[c] = c <= li ? s[c] : -INFINITY;
        }
        float mx[BN / 2];
#pragma unroll
        for (int c = 0; c < BN / 2; ++c) mx[c] = fmaxf(s[2 * c], s[2 * c + 1]);
#pragma unroll
        for (int w2 = BN / 4; w2 > 0; w2 >>= 1)
#pragma unroll
          for (int c = 0; c < w2; ++c) mx[c] = fmaxf(mx[c], mx[c + w2]);
        const float tmax = mx[0];
        if (tmax > -INFINITY && (m_ref == -INFINITY || tmax > m_ref + thr_raw)) {
          const float alpha = ex2_approx((m_ref - tmax) * c2);
          if (n > 0) {
            // O must be at rest: P.V of the previous tile done
            if (!wait_u(bar(B_PVDONE), (J - 1) & 1)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < DH; c += 32) {
              uint32_t v[32];
              tmem_ld32(trow + T_O + c, v);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
              tmem_st32(trow + T_O + c, v);
            }
          }
          l *= alpha;
          m_ref = tmax;
        }
        // P = 2^((s - m_ref) c2) as bf16 pairs over the first 64 columns of this score buffer
        const uint64_t cc = f2_pack(c2, c2), off = f2_pack(-m_ref * c2, -m_ref * c2);
        uint64_t acc2[8];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int k2 = 32 * h2 + c;
            float a0, a1;
            f2_unpack(f2_fma(f2_pack(s[2 * k2], s[2 * k2 + 1]), cc, off), a0, a1);
            const float e0 = ex2_approx(a0), e1 = ex2_approx(a1);
            pk[c] = pack_bf16(e0, e1);
            if (k2 < 8) acc2[k2] = f2_pack(e0, e1);
            else acc2[k2 & 7] = f2_add(acc2[k2 & 7], f2_pack(e0, e1));
          }
          tmem_st32(trow + BN * sb + 32 * h2, pk);
        }
#pragma unroll
        for (int w2 = 4; w2 > 0; w2 >>= 1)
#pragma unroll
          for (int c = 0; c < w2; ++c) acc2[c] = f2_add(acc2[c], acc2[c + w2]);
        float l0, l1;
        f2_unpack(acc2[0], l0, l1);
        l += l0 + l1;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL + sb));
      }
      if (!ok) break;
      // the next unit's q goes in now, so that its first QK^T overlaps this epilogue
      Unit nx;
      const int64_t un = next_unit(u + gridDim.x, nx);
      if (un < U && !load_q(nx, g + 1)) { ok = false; break; }
      // epilogue: O / l of this unit's rows
      if (!wait_u(bar(B_PVDONE), (J - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const int64_t r = (int64_t)x.m * BM + i;
      const bool valid = r < x.len;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(p.o + ((x.row0 + r) * H + x.h) * DH);
#pragma unroll 1
      for (int c = 0; c < DH; c += 32) {
        uint32_t v[32];
        tmem_ld32(trow + T_O + c, v);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[c / 8 + e] =
                make_uint4(pack_bf16(__uint_as_float(v[8 * e]) * inv, __uint_as_float(v[8 * e + 1]) * inv),
                           pack_bf16(__uint_as_float(v[8 * e + 2]) * inv, __uint_as_float(v[8 * e + 3]) * inv),
                           pack_bf16(__uint_as_float(v[8 * e + 4]) * inv, __uint_as_float(v[8 * e + 5]) * inv),
                           pack_bf16(__uint_as_float(v[8 * e + 6]) * inv, __uint_as_float(v[8 * e + 7]) * inv));
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_OFREE));
      u = un;
      x = nx;
    }
    if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t tc_prefill_attention(const void* qc, const void* qr, const void* kc, const void* vc, const void* cache,
                                 int64_t capacity, const int64_t* cu, const int64_t* cu_kv, int64_t B, int64_t T,
                                 int64_t T_kv, int64_t max_seqlen, void* o, int num_sms, uint32_t* err,
                                 cudaStream_t st) {
  if (B <= 0 || T <= 0 || max_seqlen <= 0) return cudaSuccess;
  if (!cu_kv) { cu_kv = cu; T_kv = T; }
  if (T > INT32_MAX || T_kv > INT32_MAX || T_kv <= 0 || capacity > INT32_MAX || B > INT32_MAX)
    return cudaErrorInvalidValue;
  PrefillParams p;
  memset(&p, 0, sizeof(p));
  cudaError_t e;
  if ((e = make_tmap_bf16(&p.kc_map, kc, (int64_t)H * DH, T_kv, (int64_t)H * DH, 64, BN)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&p.vc_map, vc, (int64_t)H * DH, T_kv, (int64_t)H * DH, 64, BN)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&p.kr_map, cache, CROW, capacity, CROW, 64, BN)) != cudaSuccess) return e;
  p.qc = reinterpret_cast<const __nv_bfloat16*>(qc);
  p.qr = reinterpret_cast<const __nv_bfloat16*>(qr);
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.cu = cu;
  p.cu_kv = cu_kv;
  p.B = (int32_t)B;
  p.M = (int32_t)((max_seqlen + BM - 1) / BM);
  p.T = T;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)(DH + DR)));
  p.err = err;
  static bool configured = false;
  if (!configured) {
    if ((e = cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)SMEM_BYTES)) != cudaSuccess)
      return e;
    configured = true;
  }
  const int64_t units = (int64_t)H * B * p.M;
  const int grid = (int)(units < num_sms ? units : num_sms);
  timer_begin(TIMED_PREFILL_CORE, st);
  prefill_attn_kernel<<<grid, kThreads, SMEM_BYTES, st>>>(p);
  timer_end(TIMED_PREFILL_CORE, st);
  note_launch();
  return cudaGetLastError();
}

}  // namespace mla
