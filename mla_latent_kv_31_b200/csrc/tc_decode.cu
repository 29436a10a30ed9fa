// Split-KV latent attention core for decode at the DeepSeek-V3 sizes (n_h = 128, d_c = 512,
// d_h^R = 64), bf16 inputs, fp32 accumulation, tcgen05 + TMA on sm_100a.
//
// It computes, for every query token t of sequence b and head i, the absorbed score of the
// DeepSeek-V3 notes (section 一(一)2 【思考】 and 3 "解耦RoPE"):
//   s_j = (q~_t,i . c_j + q^R_t,i . k^R_j) / sqrt(d_h + d_h^R),  j <= pos_t,
//   o^lat_t,i = sum_j softmax(s)_j c_j,   lse_t,i = log sum_j exp(s_j).
//
// Work split. Each sequence's cache rows form tiles of 64 keys; all tiles of all sequences are
// cut into equal contiguous ranges, one per CTA pair (a 2-CTA cluster); a pair whose range
// crosses a sequence boundary emits one partial result per sequence piece, and a final pass
// merges the pieces of a sequence exactly (log-sum-exp). Within a pair, CTA r owns latent
// columns [256 r, 256 r + 256) and k^R columns [32 r, 32 r + 32): it streams only those 288
// columns of every cache row, computes the partial score over them, swaps the 128 x 64 partial
// (as fp16) with its peer through distributed shared memory, and then both run the same softmax
// and accumulate P . c into their own 256 TMEM columns of O. The 128 heads form the MMA M
// dimension; one TMA-loaded cache tile is read K-major by QK^T and MN-major by P.V.
//
// Pipelining. Scores are double-buffered in TMEM and the peer's partials in shared memory, so QK^T
// of tile j + 1 and the copy of its partial run while the softmax works on tile j; P.V of tile j
// reads P from shared memory, which the softmax of tile j + 1 rewrites once that P.V is done.
// Sending this CTA's partial scores to the peer has warps of its own: they read a tile's partial out
// of TMEM as soon as QK^T is done, stage it in shared memory and copy it in bulk to the peer, while
// the softmax warps work on the tile before it; the softmax adds the peer's partial to its own.
//
// Roles per CTA (448 threads): warps 0-3 and 10-13 softmax/epilogue (two warps per TMEM lane
// quarter, thread = head = TMEM lane, one warp per half of a tile's keys), warp 4 TMA producer,
// warp 5 TMEM owner + MMA issuer, warps 6-9 send this CTA's partial scores (warp w on TMEM lanes
// 32 (w % 4) + [0, 32)). Every wait is bounded.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <string.h>

#include "sm100.cuh"
#include "tc.cuh"
#include "tc_gemm.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int H = 128, DC = 512, DR = 64, ROW = DC + DR;
constexpr int NK = 64;                       // keys per tile (the N of QK^T, the K of P.V)
// Partial scores cross to the peer CTA as fp16; both CTAs add the same two fp16-rounded halves, so
// they see identical scores (relative rounding 2^-11 per half, far inside the bf16 error budget).
// Half the bytes of fp32 leave room for two receive buffers and four cache stages.
constexpr bool kXHalf = true;
constexpr int STAGES = 4;
constexpr int kThreads = 448;
constexpr int kMaxPairs = 74;
constexpr float kRescaleLog2 = 8.f;          // lazy rescale: keep the running max until it grows by 2^8

constexpr uint32_t KV_BOX = NK * 128;        // [64 keys x 64 latent cols] bf16, 128-byte swizzle: 8 KB
constexpr uint32_t R_BOX = NK * 64;          // [64 keys x 32 k^R cols] bf16, 64-byte swizzle: 4 KB
constexpr uint32_t STAGE_BYTES = 4 * KV_BOX + R_BOX;   // 36 KB
constexpr uint32_t XE = kXHalf ? 2 : 4;      // bytes per exchanged score
constexpr uint32_t X_BYTES = H * NK * XE;    // [128 x 64] partial scores: 32 KB (fp32) / 16 KB (fp16)
constexpr int XPER = 16 / XE;                // scores per 16-byte chunk
constexpr int XCH = NK / XPER;               // 16-byte chunks per head
constexpr uint32_t P_BYTES = H * NK * 2;     // [128 x 64] bf16 probabilities, K-major, 128-byte swizzle
constexpr uint32_t QR_BYTES = H * 32 * 2;    // [128 x 32] bf16 q^R half, K-major, 64-byte swizzle
constexpr uint32_t OFF_KV = 0;
constexpr uint32_t OFF_X = OFF_KV + STAGES * STAGE_BYTES;
constexpr uint32_t OFF_XO = OFF_X + 2 * X_BYTES;  // two receive buffers, then this CTA's staged partial
constexpr uint32_t OFF_P = OFF_XO + X_BYTES;
constexpr uint32_t OFF_QR = OFF_P + P_BYTES;
constexpr uint32_t OFF_RED = OFF_QR + QR_BYTES;   // per-head maxima / sums swapped between softmax halves
constexpr uint32_t OFF_BAR = OFF_RED + 3 * 2 * H * 4;
static_assert(STAGE_BYTES % 1024 == 0 && OFF_P % 1024 == 0 && OFF_QR % 1024 == 0, "swizzle atom alignment");

// barrier indices
constexpr int B_FULL = 0, B_EMPTY = STAGES, B_SFULL = 2 * STAGES, B_SEMPTY = B_SFULL + 2, B_PFULL = B_SEMPTY + 2,
              B_PVDONE = B_PFULL + 1, B_XFULL = B_PVDONE + 1, B_XFREE = B_XFULL + 2, B_QFULL = B_XFREE + 2,
              B_QEMPTY = B_QFULL + 1, B_OFREE = B_QEMPTY + 1, B_XOFREE = B_OFREE + 1, B_XORDY = B_XOFREE + 1,
              B_TMAX = B_XORDY + 1;
constexpr int NBAR = B_TMAX + 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns: O half [0, 256); q~ half as bf16 pairs [256, 384) (the A operand of QK^T);
// two score buffers S0 [384, 448), S1 [448, 512).
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_Q = 256, T_S = 384;
static_assert(T_S + 2 * NK <= TMEM_COLS, "TMEM budget");

struct CoreParams {
  CUtensorMap cmap;   // cache as [capacity, ROW], box {64, NK}, 128-byte swizzle (latent columns)
  CUtensorMap rmap;   // cache as [capacity, ROW], box {32, NK}, 64-byte swizzle (k^R columns)
  const __nv_bfloat16* q_abs;   // [T][H][DC]
  const __nv_bfloat16* q_rope;  // [T][H][DR]
  const int64_t* cu;
  const int32_t* tile_start;  // [B+1]: first global tile of each sequence
  const int32_t* slot_base;   // [B+1]: first partial slot of each sequence
  int32_t B, tq, pairs, s_max;
  float* part_o;     // [tq][s_max][H][DC]
  float* part_lse;   // [tq][s_max][H]
  void* o_lat;       // [T][H][DC] (fp32 or bf16)
  float* lse;        // [T][H]
  float scale_log2;  // log2(e) / sqrt(d_h + d_h^R)
  uint32_t* err;
};

__device__ __forceinline__ int32_t range_start(int64_t p, int64_t NT, int64_t P) { return (int32_t)(p * NT / P); }

template <int V>
struct IC {
  static constexpr int value = V;
};

// The last sequence b in [0, B) with tile_start[b] <= x.
__device__ __forceinline__ int find_seq(const int32_t* ts, int B, int32_t x) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ts[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Iterates the sequence pieces of a tile range [x, end): b, [x, seg_end).
struct SegWalk {
  const int32_t* ts;
  int B;
  int32_t x, end;
  int b;
  __device__ void init(const int32_t* ts_, int B_, int32_t x0, int32_t x1) {
    ts = ts_; B = B_; x = x0; end = x1;
    b = x < end ? find_seq(ts, B, x) : 0;
  }
  __device__ bool valid() const { return x < end; }
  __device__ int32_t seg_end() const { return min(end, ts[b + 1]); }
  __device__ void next() {
    x = seg_end();
    ++b;
    while (b < B && ts[b + 1] <= x) ++b;
  }
};

// Walks the tiles of a range one by one: j (tile count), g (piece count), first/last of a piece.
struct TileCursor {
  SegWalk w;
  int32_t xt;
  int j, g;
  __device__ void init(const int32_t* ts, int B, int32_t x0, int32_t x1) {
    w.init(ts, B, x0, x1);
    xt = w.x;
    j = 0;
    g = 0;
  }
  __device__ bool valid() const { return w.valid(); }
  __device__ bool first() const { return xt == w.x; }
  __device__ bool last() const { return xt == w.seg_end() - 1; }
  __device__ void advance() {
    ++j;
    if (++xt >= w.seg_end()) {
      w.next();
      ++g;
      xt = w.x;
    }
  }
};

template <bool OUT_F32>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    latent_core_kernel(const __grid_constant__ CoreParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  const uint32_t sbase = smem_addr(smem);
  auto bar = [&](int i) { return smem_addr(&bars[i]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t r = cluster_rank();
  const uint32_t peer = r ^ 1u;
  const int k = blockIdx.y;                          // query token within the sequence window
  const int pair = blockIdx.x >> 1;
  const int64_t NT = p.tile_start[p.B];
  // Active pairs: never more than tiles, so that every active range holds at least one tile.
  const int64_t npairs = NT < p.pairs ? NT : p.pairs;
  const int32_t t_begin = pair < npairs ? range_start(pair, NT, npairs) : 0;
  const int32_t t_end = pair < npairs ? range_start(pair + 1, NT, npairs) : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) {
      // counts: the 256 softmax threads (P, O, q hand-offs); SEMPTY: those plus the 128 exchange threads
      // that also read a score buffer; XORDY: the exchange threads; XFREE: one arrival per softmax
      // warp of the peer; TMAX: the two softmax warps of one TMEM lane quarter
      uint32_t cnt = 1;
      if (i == B_PFULL || i == B_OFREE || i == B_QFULL) cnt = 256;
      else if (i >= B_SEMPTY && i < B_SEMPTY + 2) cnt = 384;
      else if (i == B_XORDY) cnt = 128;
      else if (i == B_XFREE || i == B_XFREE + 1) cnt = 8;
      else if (i >= B_TMAX && i < B_TMAX + 4) cnt = 64;
      mbar_init(bar(i), cnt);
    }
    // the exchange buffers' first phases: one arrival plus the bytes the peer's copy will bring
    mbar_expect_tx(bar(B_XFULL), X_BYTES);
    mbar_expect_tx(bar(B_XFULL + 1), X_BYTES);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    prefetch_tmap(&p.cmap);
    prefetch_tmap(&p.rmap);
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  SegWalk w;
  w.init(p.tile_start, p.B, t_begin, t_end);

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int j = 0, issued = 0;
      bool ok = true;
      const int xr = DC + 32 * (int)r;               // this CTA's k^R columns
      for (; ok && w.valid(); w.next()) {
        const int b = w.b;
        const int32_t ts_b = p.tile_start[b];
        const int32_t row_base = (int32_t)p.cu[b];
        for (int32_t xt = w.x; xt < w.seg_end(); ++xt, ++j) {
          const int st = j % STAGES;
          if (!mbar_wait(bar(B_EMPTY + st), ((j / STAGES) & 1) ^ 1)) { ok = false; break; }
          mbar_expect_tx(bar(B_FULL + st), STAGE_BYTES);
          const int32_t row0 = row_base + (xt - ts_b) * NK;
          const uint32_t dst = sbase + OFF_KV + st * STAGE_BYTES;
          for (int c = 0; c < 4; ++c)
            tma_load_2d(dst + c * KV_BOX, &p.cmap, 256 * (int)r + 64 * c, row0, bar(B_FULL + st));
          tma_load_2d(dst + 4 * KV_BOX, &p.rmap, xr, row0, bar(B_FULL + st));
          issued = j + 1;
        }
      }
      if (!ok) {
        flag_error(p.err, DEVERR_TIMEOUT);
        for (int i = max(0, issued - STAGES); i < issued; ++i) mbar_wait(bar(B_FULL + i % STAGES), (i / STAGES) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    // Greedy: P.V for the oldest tile whose P is ready, else QK^T of the next tile once its cache
    // tile has landed and its score buffer has been read out by the softmax. QK^T goes out in two
    // halves of 9 MMAs, so that a P.V that becomes ready meanwhile does not wait for all of it.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, NK, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 256, 0, 1);
      const uint32_t qr = sbase + OFF_QR;
      TileCursor cq, cp;
      cq.init(p.tile_start, p.B, t_begin, t_end);
      cp.init(p.tile_start, p.B, t_begin, t_end);
      uint64_t stall_since = 0;
      bool ok = true;
      int qk_half = 0;                               // halves of QK^T(cq.j) issued so far
      while (cp.valid()) {
        bool did = false;
        if (cp.j < cq.j && mbar_test(bar(B_PFULL), cp.j & 1) &&
            (!cp.first() || mbar_test(bar(B_OFREE), (cp.g & 1) ^ 1))) {
          tc_fence_after();
          const int st = cp.j % STAGES;
          const uint32_t kv = sbase + OFF_KV + st * STAGE_BYTES;
          const bool first = cp.first();
          // descriptors advance by adding (byte offset >> 4) to the start-address field (bits 0-13,
          // shared-memory addresses stay below 2^18): one add per MMA instead of a full encode
          const uint64_t ap = sw128_desc(sbase + OFF_P, 0, 1024), bp = sw128_desc(kv, KV_BOX, 1024);
#pragma unroll
          for (int kk = 0; kk < NK / 16; ++kk)
            mma_bf16_ss(tmem, ap + (kk * 32 >> 4), bp + (kk * 2048 >> 4), idesc_pv, (first && kk == 0) ? 0u : 1u);
          mma_commit(bar(B_PVDONE));
          mma_commit(bar(B_EMPTY + st));
          cp.advance();
          did = true;
        }
        if (!did && cq.valid()) {
          const int st = cq.j % STAGES, sb = cq.j & 1;
          if (qk_half == 1 ||
              (mbar_test(bar(B_FULL + st), (cq.j / STAGES) & 1) && mbar_test(bar(B_SEMPTY + sb), ((cq.j >> 1) & 1) ^ 1) &&
               (!cq.first() || mbar_test(bar(B_QFULL), cq.g & 1)))) {
            if (qk_half == 0) tc_fence_after();
            const uint32_t kv = sbase + OFF_KV + st * STAGE_BYTES;
            const uint32_t d = tmem + T_S + NK * sb;
            // MMA m < 16: latent chunk m / 4, K step m % 4 (A from TMEM); m = 16, 17: the k^R half
            // (A from shared memory). Descriptors: base + (byte offset >> 4), as for P.V.
            const uint64_t bq = sw128_desc(kv, 0, 1024);
            auto issue = [&](auto m_c) {
              constexpr int m = decltype(m_c)::value;
              if (m < 16)
                mma_bf16_ts(d, tmem + T_Q + 8 * m, bq + (((m >> 2) * KV_BOX + (m & 3) * 32) >> 4), idesc_qk,
                            m ? 1u : 0u);
              else
                mma_bf16_ss(d, sw64_desc(qr, 512) + (((m - 16) * 32) >> 4),
                            sw64_desc(kv + 4 * KV_BOX, 512) + (((m - 16) * 32) >> 4), idesc_qk, 1u);
            };
            if (qk_half == 0) {
              issue(IC<0>{}); issue(IC<1>{}); issue(IC<2>{}); issue(IC<3>{}); issue(IC<4>{});
              issue(IC<5>{}); issue(IC<6>{}); issue(IC<7>{}); issue(IC<8>{});
            } else {
              issue(IC<9>{}); issue(IC<10>{}); issue(IC<11>{}); issue(IC<12>{}); issue(IC<13>{});
              issue(IC<14>{}); issue(IC<15>{}); issue(IC<16>{}); issue(IC<17>{});
            }
            if (qk_half == 1) {
              mma_commit(bar(B_SFULL + sb));
              if (cq.last()) mma_commit(bar(B_QEMPTY));
              cq.advance();
            }
            qk_half ^= 1;
            did = true;
          }
        }
        if (did) {
          stall_since = 0;
        } else {
          // back off so this polling warp leaves the issue slots of its sub-partition to the
          // softmax warp that shares it
          __nanosleep(40);
          if (stall_since == 0) {
            stall_since = globaltimer();
          } else if (globaltimer() - stall_since > kWaitTimeoutNs) {
            ok = false;
            break;
          }
        }
      }
      if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
    }
  } else if (warp >= 6 && warp < 10) {
    // ------------------------------------------------------------------ score exchange (send side)
    // Per tile: this CTA's partial scores TMEM -> registers -> the local staging buffer (chunk-major:
    // chunk c of head i at (c * 128 + i) * 16), which one thread copies in bulk into the peer's
    // exchange buffer once the peer's softmax has read the previous tile out of it (counted on the
    // peer's x_full barrier). The staging buffer is rewritten only once the previous copy has read it.
    const int e = threadIdx.x - 192;                 // exchange thread 0..127
    const int i = 32 * (warp & 3) + lane;            // head = TMEM lane
    const bool leader = e == 0;
    const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    const uint32_t xin_peer = map_peer(sbase + OFF_X, peer);
    const uint32_t xfull_peer = map_peer(bar(B_XFULL), peer);
    uint4* xo = reinterpret_cast<uint4*>(smem + OFF_XO) + i;
    auto wait_u = [](uint32_t b, uint32_t par) { return __all_sync(0xffffffffu, mbar_wait(b, par)) != 0; };
    const int ntiles = t_end - t_begin;
    bool ok = true;
    for (int jj = 0; jj < ntiles; ++jj) {
      const int sb = jj & 1;
      const uint32_t taddr = trow + T_S + NK * sb;
      if (leader && jj > 0) {
        bulk_wait_read0();                           // the previous copy has read the staging buffer
        mbar_arrive(bar(B_XOFREE));
      }
      if (!wait_u(bar(B_SFULL + sb), (jj >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      uint32_t v[NK];
      tmem_ld32(taddr, v);
      tmem_ld32(taddr + 32, v + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_SEMPTY + sb));
      if (!wait_u(bar(B_XOFREE), (jj & 1) ^ 1)) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < XCH; ++c) {
        uint32_t w4[4];
        if (kXHalf) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int k2 = XPER * c + 2 * q;
            const __half2 h2 = __floats2half2_rn(__uint_as_float(v[k2]), __uint_as_float(v[k2 + 1]));
            w4[q] = *reinterpret_cast<const uint32_t*>(&h2);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) w4[q] = v[XPER * c + q];
        }
        xo[c * 128] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(B_XORDY));
      if (leader) {
        // all 128 rows staged, and the peer's softmax has read the previous tile out of its buffer
        const int xb = jj & 1;
        if (mbar_wait(bar(B_XORDY), jj & 1) && mbar_wait_cluster(bar(B_XFREE + xb), ((jj >> 1) & 1) ^ 1)) {
          bulk_copy_to_peer(xin_peer + xb * X_BYTES, sbase + OFF_XO, X_BYTES, xfull_peer + 8 * xb);
          bulk_commit();
        } else {
          ok = false;
        }
      }
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
    }
    if (leader) bulk_wait_read0();
    if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    // Two warps per TMEM lane quarter: half 0 (warps 0-3) takes keys [0, 32) of every tile, half 1
    // (warps 10-13) keys [32, 64), for the same 32 heads; they agree on each tile's max through
    // shared memory and a per-quarter barrier. O columns (rescale, epilogue) and the query load are
    // split between the halves the same way.
    const int quarter = warp & 3, half = warp >= 10 ? 1 : 0;
    const int i = 32 * quarter + lane;               // head
    const int tid = 128 * half + i;                  // 0..255 over both halves
    const int kc0 = 32 * half;                       // first key of this half within a tile
    const uint32_t trow = tmem + ((uint32_t)(32 * quarter) << 16);
    const uint32_t xfree_peer = map_peer(bar(B_XFREE), peer);
    const uint32_t tmax_bar = bar(B_TMAX + quarter);
    float* redbuf = reinterpret_cast<float*>(smem + OFF_RED);   // [2 parity][2 half][128] maxima, then [2][128] sums
    const float c2 = p.scale_log2;                   // raw score -> log2 units
    const float thr_raw = kRescaleLog2 / c2;
    // waits of the softmax warps are warp-uniform: a timeout on any lane fails the whole warp, so
    // no lane can be left behind at a .sync.aligned tcgen05 instruction
    auto wait_u = [](uint32_t b, uint32_t par) { return __all_sync(0xffffffffu, mbar_wait(b, par)) != 0; };
    auto wait_uc = [](uint32_t b, uint32_t par) { return __all_sync(0xffffffffu, mbar_wait_cluster(b, par)) != 0; };
    int gq = 0, j = 0, tph = 0;
    // one exchange of a value per head with the other half of this quarter: the partner's value in
    // y; false if the wait gave up
    auto swap_half = [&](float x, int slot, float& y) -> bool {
      redbuf[(slot * 2 + half) * 128 + i] = x;
      mbar_arrive(tmax_bar);
      const bool okw = wait_u(tmax_bar, tph & 1);
      ++tph;
      y = redbuf[(slot * 2 + (half ^ 1)) * 128 + i];
      return okw;
    };
    // q~ half -> TMEM (this half's 64 columns) and q^R half -> shared memory (64-byte swizzle, this
    // half's two chunks) for the piece of sequence bq, once the previous piece's last QK^T is done.
    auto load_q = [&](int bq) -> bool {
      const int64_t t = (int64_t)bq * p.tq + k;
      if (!wait_u(bar(B_QEMPTY), (gq & 1) ^ 1)) return false;
      tc_fence_after();
      const uint4* src = reinterpret_cast<const uint4*>(p.q_abs + (t * H + i) * DC + 256 * r + 128 * half);
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 u = __ldg(src + 8 * c + e);
          v[4 * e] = u.x; v[4 * e + 1] = u.y; v[4 * e + 2] = u.z; v[4 * e + 3] = u.w;
        }
        tmem_st32(trow + T_Q + 64 * half + 32 * c, v);
      }
      const uint4* rsrc = reinterpret_cast<const uint4*>(p.q_rope + (t * H + i) * DR + 32 * r);
      uint8_t* qrow = smem + OFF_QR + i * 64;
#pragma unroll
      for (int c = 2 * half; c < 2 * half + 2; ++c)
        *reinterpret_cast<uint4*>(qrow + ((c ^ ((i >> 1) & 3)) << 4)) = __ldg(rsrc + c);
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_QFULL));
      ++gq;
      return true;
    };
    bool ok = !w.valid() || load_q(w.b);
    for (; ok && w.valid(); w.next()) {
      const int b = w.b;
      const int64_t len = p.cu[b + 1] - p.cu[b];
      const int64_t vis = len - p.tq + k + 1;        // keys visible to this query token
      const int32_t ts_b = p.tile_start[b];
      const int32_t send = w.seg_end();
      float m_ref = -INFINITY, l = 0.f;              // running max (raw score units); this half's sum
      const int jfirst = j;
      for (int32_t xt = w.x; xt < send; ++xt) {
        // scores of this half's 32 keys: this CTA's partial (TMEM) plus the peer's (exchange buffer)
        const int sb = j & 1, xb = j & 1;
        if (!wait_u(bar(B_SFULL + sb), (j >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        float s[32];
        tmem_ld32(trow + T_S + NK * sb + kc0, reinterpret_cast<uint32_t*>(s));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(B_SEMPTY + sb));
        if (!wait_uc(bar(B_XFULL + xb), (j >> 1) & 1)) { ok = false; break; }
        {
          const uint4* xi = reinterpret_cast<const uint4*>(smem + OFF_X + xb * X_BYTES) + i;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 q = xi[(4 * half + c) * 128];
            const uint32_t q4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              // both CTAs add the two fp16-rounded partials, so they see the same scores
              const int k2 = 8 * c + 2 * u;
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&q4[u]));
              const float2 o = __half22float2(__floats2half2_rn(s[k2], s[k2 + 1]));
              s[k2] = o.x + f.x;
              s[k2 + 1] = o.y + f.y;
            }
          }
        }
        // re-arm the buffer's next phase (one arrival + the bytes), then tell the peer it is free
        if (tid == 0) mbar_expect_tx(bar(B_XFULL + xb), X_BYTES);
        __syncwarp();
        if (lane == 0) mbar_arrive_peer(xfree_peer + 8 * xb);
        const int64_t key0 = (int64_t)(xt - ts_b) * NK;
        const int nvis = (int)max((int64_t)0, min((int64_t)NK, vis - key0)) - kc0;
        if (nvis < 32) {
#pragma unroll
          for (int c = 0; c < 32; ++c) s[c] = c < nvis ? s[c] : -INFINITY;
        }
        float mx[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) mx[c] = fmaxf(s[2 * c], s[2 * c + 1]);
#pragma unroll
        for (int w2 = 8; w2 > 0; w2 >>= 1)
#pragma unroll
          for (int c = 0; c < w2; ++c) mx[c] = fmaxf(mx[c], mx[c + w2]);
        float pmax;
        if (!swap_half(mx[0], j & 1, pmax)) { ok = false; break; }
        const float tmax = fmaxf(mx[0], pmax);
        // rows of this stage past the sequence end: zero the latent half before P.V reads it
        const int nrows = (int)max((int64_t)0, min((int64_t)NK, len - key0));
        if (nrows < NK) {
          uint8_t* kvs = smem + OFF_KV + (j % STAGES) * STAGE_BYTES;
          const int chunks = (NK - nrows) * 4 * 8;   // 16-byte chunks over 4 boxes
          for (int q = tid; q < chunks; q += 256) {
            const int row = nrows + q / 32, box = (q / 8) & 3, c16 = q & 7;
            *reinterpret_cast<uint4*>(kvs + box * KV_BOX + row * 128 + c16 * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        // lazy rescale of the running max (identical decision in both halves and both CTAs); O must
        // be at rest, so P.V of the previous tile has to be done first
        if (tmax > -INFINITY && (m_ref == -INFINITY || tmax > m_ref + thr_raw)) {
          const float alpha = ex2_approx((m_ref - tmax) * c2);
          if (j > jfirst) {
            if (!wait_u(bar(B_PVDONE), (j - 1) & 1)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int c = 128 * half; c < 128 * half + 128; c += 32) {
              uint32_t v[32];
              tmem_ld32(trow + c, v);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
              tmem_st32(trow + c, v);
            }
            tmem_wait_st();
            tc_fence_before();
          }
          l *= alpha;
          m_ref = tmax;
        }
        // P = 2^((s - m_ref) c2) in bf16: this half's 4 chunks of row i of the K-major P tile
        uint32_t pk[16];
        if (m_ref > -INFINITY) {
          const uint64_t cc = f2_pack(c2, c2), off = f2_pack(-m_ref * c2, -m_ref * c2);
          uint64_t acc2[8];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            float a0, a1;
            f2_unpack(f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), cc, off), a0, a1);
            const float e0 = ex2_approx(a0), e1 = ex2_approx(a1);
            pk[c] = pack_bf16(e0, e1);
            if (c < 8) acc2[c] = f2_pack(e0, e1);
            else acc2[c & 7] = f2_add(acc2[c & 7], f2_pack(e0, e1));
          }
#pragma unroll
          for (int w2 = 4; w2 > 0; w2 >>= 1)
#pragma unroll
            for (int c = 0; c < w2; ++c) acc2[c] = f2_add(acc2[c], acc2[c + w2]);
          float l0, l1;
          f2_unpack(acc2[0], l0, l1);
          l += l0 + l1;
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) pk[c] = 0u;
        }
        // the P tile was last read by P.V of tile j - 1
        if (!wait_u(bar(B_PVDONE), (j - 1) & 1)) { ok = false; break; }
        uint8_t* prow = smem + OFF_P + i * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(prow + (((4 * half + c) ^ (i & 7)) << 4)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_smem();
        mbar_arrive(bar(B_PFULL));
        ++j;
      }
      if (!ok) break;
      // the next piece's query goes in now, so that its first QK^T overlaps this epilogue
      {
        SegWalk nx = w;
        nx.next();
        if (nx.valid() && !load_q(nx.b)) { ok = false; break; }
      }
      // piece epilogue: O / l for this half's 128 of this CTA's 256 columns (+ lse from CTA 0)
      float lp;
      if (!swap_half(l, 2, lp)) { ok = false; break; }
      const float lt = l + lp;                       // both halves' sums
      const int jl = j - 1;
      const float m_log2 = m_ref * c2;
      if (!wait_u(bar(B_PVDONE), jl & 1)) { ok = false; break; }
      tc_fence_after();
      const int64_t t = (int64_t)b * p.tq + k;
      const int32_t nseg = p.slot_base[b + 1] - p.slot_base[b];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float lse_v = lt > 0.f ? (m_log2 + log2f(lt)) * 0.69314718055994531f : -INFINITY;
      float* po = nullptr;
      if (nseg > 1) {
        const int64_t slot = (int64_t)p.slot_base[b] + (pair - (int)(((int64_t)(ts_b + 1) * npairs - 1) / NT));
        const int64_t row = ((int64_t)k * p.s_max + slot) * H + i;
        po = p.part_o + row * DC + 256 * r;
        if (r == 0 && half == 0) p.part_lse[row] = lse_v;
      } else if (r == 0 && half == 0) {
        p.lse[t * H + i] = lse_v;
      }
#pragma unroll 1
      for (int c = 128 * half; c < 128 * half + 128; c += 32) {
        uint32_t v[32];
        tmem_ld32(trow + c, v);
        tmem_wait_ld();
        if (po) {
          float4* dst = reinterpret_cast<float4*>(po + c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]) * inv, __uint_as_float(v[4 * e + 1]) * inv,
                                 __uint_as_float(v[4 * e + 2]) * inv, __uint_as_float(v[4 * e + 3]) * inv);
        } else if (OUT_F32) {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.o_lat) + (t * H + i) * DC + 256 * r + c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]) * inv, __uint_as_float(v[4 * e + 1]) * inv,
                                 __uint_as_float(v[4 * e + 2]) * inv, __uint_as_float(v[4 * e + 3]) * inv);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.o_lat) + (t * H + i) * DC +
                                                256 * r + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pack_bf16(__uint_as_float(v[8 * e]) * inv, __uint_as_float(v[8 * e + 1]) * inv),
                                pack_bf16(__uint_as_float(v[8 * e + 2]) * inv, __uint_as_float(v[8 * e + 3]) * inv),
                                pack_bf16(__uint_as_float(v[8 * e + 4]) * inv, __uint_as_float(v[8 * e + 5]) * inv),
                                pack_bf16(__uint_as_float(v[8 * e + 6]) * inv, __uint_as_float(v[8 * e + 7]) * inv));
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_OFREE));
    }
    if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
  }
  tc_fence_before();
  cluster_sync();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}


// Tile prefix and partial-slot bases of every sequence (one block). Tiles per sequence are
// counted on the cache length len_b (the last query token sees all of them). A sequence gets
// one slot per active pair whose tile range meets it.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_tot, int32_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int32_t t = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < (int)(blockDim.x >> 5)) warp_tot[lane] = t;   // inclusive warp prefix
    if (lane == (int)(blockDim.x >> 5) - 1) *total = t;
  }
  __syncthreads();
  const int32_t r = x - v + (wid > 0 ? warp_tot[wid - 1] : 0);
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(256) plan_kernel(const int64_t* cu, int32_t B, int32_t pairs, int32_t* ts,
                                                   int32_t* sb) {
  __shared__ int32_t warp_tot[8];
  __shared__ int32_t total;
  const int tid = threadIdx.x;
  const int per = (B + 255) / 256;
  const int lo = min(B, tid * per), hi = min(B, lo + per);
  auto ntiles = [&](int b) -> int32_t {
    const int64_t len = cu[b + 1] - cu[b];
    return len > 0 ? (int32_t)((len + NK - 1) / NK) : 0;
  };
  int32_t acc = 0;
  for (int b = lo; b < hi; ++b) acc += ntiles(b);
  acc = block_exclusive_scan(acc, warp_tot, &total);
  for (int b = lo; b < hi; ++b) { ts[b] = acc; acc += ntiles(b); }
  if (tid == 0) ts[B] = total;
  __syncthreads();
  const int64_t NT = total;
  const int64_t npairs = NT < pairs ? NT : pairs;   // every active pair holds >= 1 tile
  auto pair_of = [&](int64_t x) -> int64_t { return ((x + 1) * npairs - 1) / NT; };
  auto nseg = [&](int b) -> int32_t {
    const int32_t a = ts[b], e = ts[b + 1];
    return e > a ? (int32_t)(pair_of(e - 1) - pair_of(a) + 1) : 0;
  };
  acc = 0;
  for (int b = lo; b < hi; ++b) acc += nseg(b);
  acc = block_exclusive_scan(acc, warp_tot, &total);
  for (int b = lo; b < hi; ++b) { sb[b] = acc; acc += nseg(b); }
  if (tid == 0) sb[B] = total;
}

// Exact merge of a sequence's pieces: lse = log sum_s e^{lse_s}, o = sum_s e^{lse_s - lse} o_s.
// One block of 128 threads per (token, head); sequences in a single piece were written directly.
template <bool OUT_F32>
__global__ void __launch_bounds__(128) combine_kernel(const int32_t* sb, int32_t tq, int32_t s_max,
                                                      const float* part_o, const float* part_lse, void* o_lat,
                                                      float* lse) {
  __shared__ float wts[kMaxPairs + 64];
  __shared__ float red[32];
  const int64_t t = blockIdx.x;
  const int h = blockIdx.y;
  const int b = (int)(t / tq), k = (int)(t % tq);
  const int32_t s0 = sb[b], ns = min(sb[b + 1] - s0, kMaxPairs + 64);
  if (ns == 1) return;
  const int64_t row0 = ((int64_t)k * s_max + s0) * H + h;
  float lmax = -INFINITY;
  for (int s = threadIdx.x; s < ns; s += 128) {
    const float v = part_lse[row0 + (int64_t)s * H];
    wts[s] = v;
    lmax = fmaxf(lmax, v);
  }
  const float mx = block_max(lmax, red);
  float wpart = 0.f;
  for (int s = threadIdx.x; s < ns; s += 128) {
    const float wv = mx > -INFINITY ? __expf(wts[s] - mx) : 0.f;
    wts[s] = wv;
    wpart += wv;
  }
  const float wsum = block_sum(wpart, red);   // includes a __syncthreads: wts[] is complete
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int s = 0; s < ns; ++s) {
    const float wgt = wts[s];
    const float4 v = reinterpret_cast<const float4*>(part_o + (row0 + (int64_t)s * H) * DC)[threadIdx.x];
    acc.x += wgt * v.x; acc.y += wgt * v.y; acc.z += wgt * v.z; acc.w += wgt * v.w;
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
  if (OUT_F32) {
    reinterpret_cast<float4*>(reinterpret_cast<float*>(o_lat) + (t * H + h) * DC)[threadIdx.x] = acc;
  } else {
    uint2 v2 = make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
    reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(o_lat) + (t * H + h) * DC)[threadIdx.x] = v2;
  }
  if (threadIdx.x == 0) lse[t * H + h] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

size_t align1k(size_t x) { return (x + 1023) / 1024 * 1024; }

struct CoreScratch {
  int32_t* ts;
  int32_t* sb;
  float* part_lse;
  float* part_o;
  int32_t s_max;
};

CoreScratch carve(void* scratch, int64_t B, int32_t tq) {
  CoreScratch c;
  char* p = (char*)scratch;
  c.s_max = (int32_t)(kMaxPairs + B);
  c.ts = (int32_t*)p;
  p += align1k((B + 1) * 4);
  c.sb = (int32_t*)p;
  p += align1k((B + 1) * 4);
  c.part_lse = (float*)p;
  p += align1k((size_t)tq * c.s_max * H * 4);
  c.part_o = (float*)p;
  return c;
}

template <bool OUT_F32>
cudaError_t launch_core(const CoreParams& p, dim3 grid, cudaStream_t st) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(latent_core_kernel<OUT_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  timer_begin(TIMED_LATENT_CORE, st);
  latent_core_kernel<OUT_F32><<<grid, kThreads, SMEM_BYTES, st>>>(p);
  timer_end(TIMED_LATENT_CORE, st);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

size_t tc_core_scratch_bytes(const mla_dims_t& d, int64_t B, int32_t tq) {
  (void)d;
  const int64_t s_max = kMaxPairs + B;
  return 2 * align1k((B + 1) * 4) + align1k((size_t)tq * s_max * H * 4) + (size_t)tq * s_max * H * DC * 4;
}

cudaError_t tc_latent_core_impl(const void* q_abs, const void* q_rope, int64_t B, int32_t tq, const int64_t* cu,
                                const void* cache, int64_t capacity, void* o_lat, bool o_f32, float* lse,
                                void* scratch, int num_sms, uint32_t* err, cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  if (B > (int64_t)1 << 20 || capacity > INT32_MAX || B * tq * H > INT32_MAX) return cudaErrorInvalidValue;
  const int64_t T = B * tq;
  CoreScratch c = carve(scratch, B, tq);
  int pairs = num_sms / (2 * tq);
  pairs = pairs < kMaxPairs ? pairs : kMaxPairs;
  pairs = pairs < 1 ? 1 : pairs;
  plan_kernel<<<1, 256, 0, st>>>(cu, (int32_t)B, pairs, c.ts, c.sb);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CoreParams p;
  memset(&p, 0, sizeof(p));
  p.q_abs = reinterpret_cast<const __nv_bfloat16*>(q_abs);
  p.q_rope = reinterpret_cast<const __nv_bfloat16*>(q_rope);
  if ((e = make_tmap_bf16(&p.cmap, cache, ROW, capacity, ROW, 64, NK)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&p.rmap, cache, ROW, capacity, ROW, 32, NK, 64)) != cudaSuccess) return e;
  p.cu = cu;
  p.tile_start = c.ts;
  p.slot_base = c.sb;
  p.B = (int32_t)B;
  p.tq = tq;
  p.pairs = pairs;
  p.s_max = c.s_max;
  p.part_o = c.part_o;
  p.part_lse = c.part_lse;
  p.o_lat = o_lat;
  p.lse = lse;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt(128.0 + 64.0));
  p.err = err;
  dim3 grid((unsigned)(2 * pairs), (unsigned)tq);
  e = o_f32 ? launch_core<true>(p, grid, st) : launch_core<false>(p, grid, st);
  if (e != cudaSuccess) return e;
  dim3 cg((unsigned)T, (unsigned)H);
  if (o_f32) combine_kernel<true><<<cg, 128, 0, st>>>(c.sb, tq, c.s_max, c.part_o, c.part_lse, o_lat, lse);
  else combine_kernel<false><<<cg, 128, 0, st>>>(c.sb, tq, c.s_max, c.part_o, c.part_lse, o_lat, lse);
  note_launch();
  return cudaGetLastError();
}

}  // namespace mla
