// Split-KV latent attention core for decode at the DeepSeek-V3 sizes (n_h = 128, d_c = 512,
// d_h^R = 64), bf16 inputs, fp32 accumulation, tcgen05 + TMA on sm_100a.
//
// It computes, for every query token t of sequence b and head i, the absorbed score of the
// DeepSeek-V3 notes (section 一(一)2 【思考】 and 3 "解耦RoPE"):
//   s_j = (q~_t,i . c_j + q^R_t,i . k^R_j) / sqrt(d_h + d_h^R),  j <= pos_t,
//   o^lat_t,i = sum_j softmax(s)_j c_j,   lse_t,i = log sum_j exp(s_j).
//
// Work split. Each sequence's cache rows form tiles of 128 keys; all tiles of all sequences are
// cut into equal contiguous ranges, one per 2-CTA cluster; a cluster whose range crosses a
// sequence boundary emits one partial result per sequence piece, and a final pass merges the
// pieces of a sequence exactly (log-sum-exp).
//
// Roles inside a cluster. The 128 heads are the MMA's M rows, and O = P.C for 128 heads and 512
// latent columns fills the whole TMEM (512 columns of fp32) of one SM, so a cluster pairs:
//   * the score CTA (rank 0): q~ in TMEM (256 columns of bf16 pairs, the A operand), two
//     128 x 128 fp32 score buffers; QK^T over the 576 cache columns (32 TS MMAs over the latent
//     part, 4 SS MMAs over k^R with q^R in shared memory), N = 128 keys; the softmax (lazy
//     rescale of the running max); the softmax warps store P (bf16) and the per-head rescale
//     factors straight into the value CTA's shared memory (st.async, counted on its mbarrier);
//   * the value CTA (rank 1): O in all 512 TMEM columns; per tile 16 SS MMAs (N = 256 latent
//     columns, K = 16 keys) read P and the latent columns of the cache tile, which this CTA loads
//     itself (the second read of the tile hits L2); it rescales O when the score CTA's running max
//     moved, and writes the piece's normalised partial o^lat at its end.
// Each producer issues its TMA loads from four lanes: one issuing thread streams only about 40 GB/s.
// The score CTA's ring holds 12 boxes (192 KB): at the 2-3 us of HBM latency under load, the bytes
// in flight per SM set its streaming rate (Little's law), so the ring takes all the shared memory
// the P hand-off no longer needs.
//
// Queries. A piece's q~ (8 boxes of [128 heads x 64 columns]) and q^R (1 box) enter the score CTA's
// ring ahead of its first tile, like a tile's boxes; the softmax warps copy q~ into TMEM and q^R
// into its own shared-memory tile.
//
// Outputs. Every piece writes a partial: O = sum_j 2^((s_j - m) c) c_j unnormalised, its reference
// m in natural units and its lse, O in a head-interleaved layout [token k][slot][column/8][head][8]
// bf16 (fp32 accumulation, one rounding before the merge), so that the 32 heads of a warp store 512
// contiguous bytes per instruction. The merge pass
// weights each partial by e^{m_s - lse} with lse = log sum_s e^{lse_s} and writes o^lat [T][H][DC]
// and lse [T][H] (a one-piece sequence is a weighted copy).
// The score CTA's tensor work per tile is 36 MMAs at N = 128 (about 2300 cycles), the value CTA's
// 16 MMAs at N = 256 (about 2050), so the two stay busy together. Data flows one way (P), so the
// two CTAs pipeline freely: two P buffers on the value side; the score side writes P of tile j
// once the value CTA's P.V of tile j - 2 (the same buffer) is done.
//
// Every wait is bounded (a timeout sets the error word and the role returns).
#include <cuda_bf16.h>
#include <string.h>

#include "sm100.cuh"
#include "tc.cuh"
#include "tc_gemm.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int H = 128, DC = 512, DR = 64, ROW = DC + DR;
constexpr int NK = 128;                        // keys per tile
constexpr int kThreads = 384;
constexpr int kConvThreads = 64;               // FP8 cache: warps 2-3 convert the codes to f16
constexpr int kMaxPairs = 74;
constexpr float kRescaleLog2 = 8.f;            // keep the running max until it grows by 2^8
constexpr int kIssuers = 4;                    // TMA issuing lanes per producer warp
constexpr int kStartCost = 3;                  // a sequence piece's fixed cost, in half tiles (plan)

// score CTA: ring of [128 keys x 64 columns] boxes (8 latent + 1 k^R per tile)
constexpr uint32_t BOX = NK * 128;             // 16 KB, 128-byte swizzle, K-major rows of 64 bf16
constexpr int S_BOXES = 9;
constexpr int S_RING = 12;
constexpr uint32_t P_BYTES = H * NK * 2;       // P [128 heads x 128 keys] bf16, K-major SW128: 2 blocks of 16 KB
constexpr uint32_t HDR_BYTES = 2 * H * 4;      // alpha[128] (+ reserve)
constexpr uint32_t PMSG = P_BYTES + HDR_BYTES; // one P buffer: 33 KB
constexpr uint32_t PMSG_TX = P_BYTES + H * 4;  // the bytes stored into it per tile: P and alpha
constexpr uint32_t QR_BYTES = H * DR * 2;      // q^R [128 x 64] bf16, K-major SW128
// value CTA: ring of [64 keys x 256 columns] groups (4 boxes of [64 keys x 64 columns])
constexpr uint32_t VBOX = 64 * 128;            // 8 KB
constexpr uint32_t VGRP = 4 * VBOX;            // 32 KB
constexpr int V_RING = 4;                      // one tile: (N-half, key-half) = 4 groups

// Shared memory, from a 1024-byte aligned base (the same layout offsets in both CTAs for the
// barrier block, which the value CTA's multicast commits and remote arrivals rely on).
constexpr uint32_t OFF_BAR = 0;
constexpr uint32_t OFF_RED = 1024;             // score CTA: per-head maxima / sums swapped between halves
constexpr uint32_t S_OFF_RING = 4096;
constexpr uint32_t S_OFF_QR = S_OFF_RING + S_RING * BOX;
constexpr uint32_t S_END = S_OFF_QR + QR_BYTES;
constexpr uint32_t S_OFF_SC = S_END;           // FP8: per-key s, log2 s, 1/s of the two tiles in flight
constexpr uint32_t SC_BYTES = 3 * NK * 4;
constexpr uint32_t S_END8 = S_OFF_SC + 2 * SC_BYTES;
constexpr uint32_t V_OFF_PBUF = 4096;
constexpr uint32_t V_OFF_RING = V_OFF_PBUF + 2 * PMSG;
constexpr uint32_t V_END = V_OFF_RING + V_RING * VGRP;
constexpr uint32_t SMEM_BYTES = (S_END > V_END ? S_END : V_END) + 1024;
constexpr uint32_t SMEM_BYTES8 = (S_END8 > V_END ? S_END8 : V_END) + 1024;
static_assert(SMEM_BYTES <= 232448 && SMEM_BYTES8 <= 232448, "shared memory budget");
static_assert(S_OFF_RING % 1024 == 0 && S_OFF_QR % 1024 == 0 && PMSG % 1024 == 0 && V_OFF_RING % 1024 == 0,
              "swizzle atom alignment");
static_assert(OFF_RED + 3 * 2 * H * 4 <= S_OFF_RING, "reduction buffer");
static_assert(S_RING % kIssuers == 0 && V_RING % kIssuers == 0 && (kIssuers & (kIssuers - 1)) == 0,
              "issuing lanes own whole ring slots");

// barrier indices (one numbering for both CTAs)
enum : int {
  B_PVD = 0,                          // [2] value CTA's P.V of the tile in P buffer b done (multicast to both)
  B_SFULL = 2,                        // [S_RING] score CTA ring
  B_SEMPTY = B_SFULL + S_RING,        // [S_RING]
  B_SCF = B_SEMPTY + S_RING,          // [2] scores ready
  B_SCE = B_SCF + 2,                  // [2] scores read (256 softmax threads)
  B_QFULL = B_SCE + 2,                // q^R of a piece copied into its tile (256)
  B_QEMPTY = B_QFULL + 1,             // last QK^T of a piece done (q~ TMEM and q^R tile free)
  B_TMAX = B_QEMPTY + 1,              // [4] the two softmax warps of a TMEM lane quarter (64)
  B_GFULL = B_TMAX + 4,               // [V_RING] value CTA ring
  B_GEMPTY = B_GFULL + V_RING,        // [V_RING]
  B_PFULL = B_GEMPTY + V_RING,        // [2] P and alpha of a tile landed (bytes stored by the score CTA)
  B_OREADY = B_PFULL + 2,             // [2] O rescaled for the tile / nothing to rescale (128)
  B_OFREE = B_OREADY + 2,             // O read out by the piece epilogue (256: both column halves)
  B_ODONE = B_OFREE + 1,              // the last P.V of a piece done (one phase per piece)
  // FP8 cache only
  B_CF = B_ODONE + 1,                 // [8] code box m of a tile of parity t converted to f16: m + 4 t (64)
  B_SCR = B_CF + 8,                   // [2] per-key scale values of the tile written (64)
  B_SCX = B_SCR + 2,                  // [2] per-key scale values of the tile read (256 softmax threads)
  B_VCF = B_SCX + 2,                  // [V_RING] value CTA: group converted to f16 (64)
  NBAR = B_VCF + V_RING
};
static_assert(NBAR * 8 + 16 <= OFF_RED, "barrier block");

struct CoreParams {
  // bf16 cache: [capacity, ROW] bf16, kmap box {64, 128}, vmap box {64, 64};
  // FP8 cache: [capacity, 656] bytes, kmap box {128, 128}, vmap box {128, 64}; 128-byte swizzle
  CUtensorMap kmap;   // score CTA
  CUtensorMap vmap;   // value CTA
  CUtensorMap qmap;   // q~ as [T * H, DC], box {64, 128}, 128-byte swizzle
  CUtensorMap qrmap;  // q^R as [T * H, DR], box {64, 128}, 128-byte swizzle
  const int64_t* cu;
  const uint8_t* cache8;        // FP8: the cache rows (the scale of row r at byte 656 r + 640)
  const int32_t* tile_start;    // [B+1]: first global tile of each sequence
  const int32_t* slot_base;     // [B+1]: first partial slot of each sequence
  const int4* pinfo;            // [pairs]: tile range [x, y), first sequence z, its partial slot w
  int32_t B, tq, pairs, s_max;
  uint4* part_o;      // [tq][s_max][DC/8][H] x 8 bf16, unnormalised
  float* part_lse;    // [tq][s_max][H]
  float* part_m;      // [tq][s_max][H], the reference of part_o in natural units
  float scale_log2;   // log2(e) / sqrt(d_h + d_h^R)
  uint64_t wait_ns;   // bounded-wait limit
  int32_t stall;      // test hook: the score-side producer of the cluster holding tile 0 skips its first box
  uint32_t* err;
};


// Bounded waits with the launch's limit.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, uint64_t limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > limit) return false;
  }
}
__device__ __forceinline__ bool wait_bar_cluster(uint32_t bar, uint32_t parity, uint64_t limit) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (globaltimer() - t0 > limit) return false;
  }
}
// Iterates the sequence pieces of a tile range [x, end): b, [x, seg_end).
struct SegWalk {
  const int32_t* ts;
  int B;
  int32_t x, end;
  int b;
  // starts at tile x0, which belongs to sequence b0
  __device__ void init_at(const int32_t* ts_, int B_, int32_t x0, int32_t x1, int b0) {
    ts = ts_; B = B_; x = x0; end = x1; b = b0;
  }
  __device__ bool valid() const { return x < end; }
  __device__ int32_t seg_end() const { return min(end, ts[b + 1]); }
  __device__ void next() {
    x = seg_end();
    ++b;
    while (b < B && ts[b + 1] <= x) ++b;
  }
};

// FP8 cache: row r of a [rows x 128 codes] box (128-byte swizzle, the layout TMA writes) becomes
// the 128 f16 values of those codes: columns 0-63 go to row r of box `lo`, columns 64-127 over the
// codes' own row (both 128-byte swizzled K-major rows of 64 f16, the layout the MMA reads). The
// thread reads its whole row before writing, and rows are 128-byte lines of their own, so the
// in-place half is safe. `zero` writes zeros instead (cache rows that belong to no sequence).
__device__ __forceinline__ void convert_code_row(uint8_t* codes, uint8_t* lo, int r, bool zero) {
  uint8_t* crow = codes + r * 128;
  uint8_t* lrow = lo + r * 128;
  const int sw = r & 7;
  uint4 in[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) in[c] = *reinterpret_cast<const uint4*>(crow + ((c ^ sw) << 4));
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    // codes 16 c .. 16 c + 15: f16 columns 16 c .. 16 c + 15, output chunks 2 c and 2 c + 1
    uint4 o0 = make_uint4(0u, 0u, 0u, 0u), o1 = o0;
    if (!zero) {
      o0 = make_uint4(e4m3x2_to_f16x2(in[c].x & 0xffffu), e4m3x2_to_f16x2(in[c].x >> 16),
                      e4m3x2_to_f16x2(in[c].y & 0xffffu), e4m3x2_to_f16x2(in[c].y >> 16));
      o1 = make_uint4(e4m3x2_to_f16x2(in[c].z & 0xffffu), e4m3x2_to_f16x2(in[c].z >> 16),
                      e4m3x2_to_f16x2(in[c].w & 0xffffu), e4m3x2_to_f16x2(in[c].w >> 16));
    }
    uint8_t* dst = c < 4 ? lrow : crow;
    const int q0 = (2 * c) & 7;
    *reinterpret_cast<uint4*>(dst + ((q0 ^ sw) << 4)) = o0;
    *reinterpret_cast<uint4*>(dst + (((q0 + 1) ^ sw) << 4)) = o1;
  }
}

// F8 = the FP8 cache (e4m3 codes with one fp32 scale per row, k^R / s in f16). The codes are
// converted to f16 in shared memory (exactly) and the MMAs run in f16: q~ and q^R of a head are
// scaled by one power of two into f16's range, and the score of key j is s_j times the score over
// (codes_j, k^R_j / s_j). The softmax tracks w_j = log2(p_j s_j) (p_j the unnormalised softmax
// weight), so that P'_j = 2^(w_j - m) = p_j s_j 2^-m is the f16 weight of the codes in P'.C, and
// the sum l = sum_j P'_j / s_j = sum_j p_j 2^-m shares the reference m.
template <bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    latent_core_kernel(const __grid_constant__ CoreParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  const uint32_t sbase = smem_addr(smem);
  auto bar = [&](int i) { return sbase + OFF_BAR + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t r = cluster_rank();
  const int k = blockIdx.y;                          // query token within the sequence window
  const int pair = blockIdx.x >> 1;
  const uint64_t lim = p.wait_ns;
  // partial slot of this cluster's piece of sequence b: the first piece's comes with the plan; a
  // sequence that starts inside this cluster's range has this cluster as its first
  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) {
      uint32_t cnt = 1;
      if (i == B_SCE || i == B_SCE + 1 || i == B_QFULL) cnt = 256;
      else if (i >= B_TMAX && i < B_TMAX + 4) cnt = 64;
      else if (i == B_OREADY || i == B_OREADY + 1) cnt = 128;
      else if (i == B_OFREE) cnt = 256;
      else if (i >= B_CF && i < B_SCX) cnt = kConvThreads;
      else if (i == B_SCX || i == B_SCX + 1) cnt = 256;
      else if (i >= B_VCF && i < B_VCF + V_RING) cnt = kConvThreads;
      mbar_init(bar(i), cnt);
    }
    if (r == 1) {
      // the P buffers' first phases: one arrival plus the bytes of one tile
      mbar_expect_tx(bar(B_PFULL), PMSG_TX);
      mbar_expect_tx(bar(B_PFULL + 1), PMSG_TX);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    prefetch_tmap(r == 0 ? &p.kmap : &p.vmap);
    if (r == 0) {
      prefetch_tmap(&p.qmap);
      prefetch_tmap(&p.qrmap);
    }
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int4 pi = p.pinfo[pair];
  const int32_t t_begin = pi.x, t_end = pi.y;
  auto piece_slot = [&](int b) -> int64_t { return b == pi.z ? (int64_t)pi.w : (int64_t)p.slot_base[b]; };

  SegWalk w;
  w.init_at(p.tile_start, p.B, t_begin, t_end, pi.z);
  bool ok = true;

  if (r == 0) {
    // =========================================================== score CTA
    if (warp == 0) {
      // ------------------------------------------------ TMA producer: 9 entries per piece start and per tile
      // A TMA issuing thread streams at most about 40 GB/s, so lanes 0-3 issue (lane l takes the
      // entries n = l mod 4, slots l and l + 4 of the ring). Per piece: q~ in 8 boxes of
      // [128 heads x 64 columns] and q^R in 1 box, then per tile the 8 latent boxes and the k^R box.
      if (lane < kIssuers) {
        int n = 0, last = -1;
        const bool stall = p.stall && k == 0 && t_begin == 0 && t_end > 0;
        // map == nullptr (FP8): no load; the free slot is handed to the code converters, which write
        // the low half of a code box's f16 columns into it
        auto issue = [&](const CUtensorMap* map, int x, int y) -> bool {
          const int cur = n++;
          if ((cur & (kIssuers - 1)) != lane) return true;
          const int slot = cur % S_RING;
          if (!wait_bar(bar(B_SEMPTY + slot), ((cur / S_RING) & 1) ^ 1, lim)) return false;
          if (stall && cur == 0) return true;     // test hook: entry 0 never arrives
          if (map == nullptr) {
            mbar_arrive(bar(B_SFULL + slot));
            return true;
          }
          mbar_expect_tx(bar(B_SFULL + slot), BOX);
          tma_load_2d(sbase + S_OFF_RING + slot * BOX, map, x, y, bar(B_SFULL + slot));
          last = cur;
          return true;
        };
        for (SegWalk sw = w; ok && sw.valid(); sw.next()) {
          const int32_t ts_b = p.tile_start[sw.b];
          const int32_t row_base = (int32_t)p.cu[sw.b];
          const int32_t qrow = (sw.b * p.tq + k) * H;
          for (int c = 0; ok && c < 8; ++c) ok = issue(&p.qmap, 64 * c, qrow);
          if (ok) ok = issue(&p.qrmap, 0, qrow);
          for (int32_t xt = sw.x; ok && xt < sw.seg_end(); ++xt) {
            const int32_t row0 = row_base + (xt - ts_b) * NK;
            if (F8) {
              // entries 2m, 2m + 1: code box m (columns 128 m .. 128 m + 127) lands in entry 2m + 1's
              // slot; entry 8: k^R / s (f16, bytes 512 .. 639 of the row)
              for (int c = 0; ok && c < S_BOXES; ++c)
                ok = c == 8 ? issue(&p.kmap, DC, row0) : (c & 1) ? issue(&p.kmap, 128 * (c >> 1), row0)
                                                                  : issue(nullptr, 0, 0);
            } else {
              for (int c = 0; ok && c < S_BOXES; ++c) ok = issue(&p.kmap, c < 8 ? 64 * c : DC, row0);
            }
          }
        }
        if (!ok) {
          flag_error(p.err, DEVERR_TIMEOUT);
          // this lane's entries still in flight: the last S_RING / kIssuers it issued
          for (int i2 = max(lane, last - S_RING + 1); i2 <= last; ++i2)
            if ((i2 & (kIssuers - 1)) == lane && !(stall && i2 == 0))
              wait_bar(bar(B_SFULL + i2 % S_RING), (i2 / S_RING) & 1, lim);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------ MMA issuer: S = [q~ | q^R] [c | k^R]^T
      if (lane == 0) {
        constexpr uint32_t idesc = F8 ? idesc_f16(128, NK, 0, 0) : idesc_bf16(128, NK, 0, 0);
        const uint64_t qr_desc = sw128_desc(sbase + S_OFF_QR, 0, 1024);
        int j = 0, g = 0, n = 0;
        for (; ok && w.valid(); w.next(), ++g) {
          // the piece's q~ / q^R entries are taken by the softmax warps (TMEM q~, q^R tile)
          n += 9;
          if (!wait_bar(bar(B_QFULL), g & 1, lim)) { ok = false; break; }
          const int32_t send = w.seg_end();
          for (int32_t xt = w.x; xt < send; ++xt, ++j) {
            const int sb = j & 1;
            if (!wait_bar(bar(B_SCE + sb), ((j >> 1) & 1) ^ 1, lim)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d = tmem + 256 + 128 * sb;
            for (int c = 0; c < S_BOXES; ++c, ++n) {
              const int slot = n % S_RING;
              if (F8 && c < 8) {
                // both f16 halves of code box c / 2 written by the converters
                if ((c & 1) == 0 && !wait_bar(bar(B_CF + (c >> 1) + 4 * sb), (j >> 1) & 1, lim)) { ok = false; break; }
              } else if (!wait_bar(bar(B_SFULL + slot), (n / S_RING) & 1, lim)) {
                ok = false;
                break;
              }
              tc_fence_after();
              // descriptors advance by (byte offset >> 4) in the start-address field: 32 bytes per
              // K step of 16 bf16 inside the 128-byte swizzled row
              const uint64_t bdesc = sw128_desc(sbase + S_OFF_RING + slot * BOX, 0, 1024);
              if (c < 8) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_bf16_ts(d, tmem + 32 * c + 8 * kk, bdesc + 2 * kk, idesc, (c | kk) ? 1u : 0u);
              } else {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(d, qr_desc + 2 * kk, bdesc + 2 * kk, idesc, 1u);
              }
              mma_commit(bar(B_SEMPTY + slot));
            }
            if (!ok) break;
            mma_commit(bar(B_SCF + sb));
          }
          if (!ok) break;
          mma_commit(bar(B_QEMPTY));
        }
        if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
      }
    } else if (F8 && (warp == 2 || warp == 3)) {
      // ------------------------------------------------ FP8 code converters (64 threads, key rows ct, ct + 64)
      // Per tile: the scales of its two keys (s, log2 s, 1/s into the tile's scale buffer; a row past
      // the last sequence gets s = 0: weight 0), then the 4 code boxes of the tile, its two rows of
      // each, into f16 in place (the low half into the slot of the box's even entry).
      const int ct = threadIdx.x - 64;
      float* scb = reinterpret_cast<float*>(smem + S_OFF_SC);
      const int64_t total_rows = p.cu[p.B];
      int j = 0, n = 0;
      for (; ok && w.valid(); w.next()) {
        n += 9;                                      // the piece's q~ / q^R entries
        const int b = w.b;
        const int32_t ts_b = p.tile_start[b];
        const int64_t row_base = p.cu[b];
        const int32_t send = w.seg_end();
        for (int32_t xt = w.x; xt < send; ++xt, ++j, n += S_BOXES) {
          const int sb = j & 1;
          const int64_t row = row_base + (int64_t)(xt - ts_b) * NK + ct;
          float sv[2];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int64_t r2 = row + 64 * h2;
            sv[h2] = r2 < total_rows ? *reinterpret_cast<const float*>(p.cache8 + r2 * kFp8RowBytes + kFp8ScaleOffset) : 0.f;
            if (!(sv[h2] > 0.f && sv[h2] < INFINITY)) sv[h2] = 0.f;
          }
          if (!wait_bar(bar(B_SCX + sb), ((j >> 1) & 1) ^ 1, lim)) { ok = false; break; }
          float* sc = scb + sb * (3 * NK);
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int key = ct + 64 * h2;
            sc[key] = sv[h2];
            sc[NK + key] = sv[h2] > 0.f ? log2f(sv[h2]) : -INFINITY;
            sc[2 * NK + key] = sv[h2] > 0.f ? 1.f / sv[h2] : 0.f;
          }
          mbar_arrive(bar(B_SCR + sb));
          for (int m = 0; m < 4; ++m) {
            const int e0 = n + 2 * m, e1 = e0 + 1;
            const int s0 = e0 % S_RING, s1 = e1 % S_RING;
            if (!wait_bar(bar(B_SFULL + s0), (e0 / S_RING) & 1, lim) ||
                !wait_bar(bar(B_SFULL + s1), (e1 / S_RING) & 1, lim)) {
              ok = false;
              break;
            }
            convert_code_row(smem + S_OFF_RING + s1 * BOX, smem + S_OFF_RING + s0 * BOX, ct, false);
            convert_code_row(smem + S_OFF_RING + s1 * BOX, smem + S_OFF_RING + s0 * BOX, ct + 64, false);
            fence_proxy_async_smem();
            mbar_arrive(bar(B_CF + m + 4 * sb));
          }
          if (!ok) break;
        }
      }
      if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
    } else if (warp >= 4) {
      // ------------------------------------------------ softmax: 8 warps, two per TMEM lane quarter
      // Half 0 (warps 4-7) takes keys [0, 64) of every tile, half 1 (warps 8-11) keys [64, 128),
      // for the same 32 heads (thread = head = TMEM lane); they agree on each tile's max through
      // shared memory and a per-quarter barrier.
      const int quarter = warp & 3, half = (warp - 4) >> 2;
      const int i = 32 * quarter + lane;
      const uint32_t trow = tmem + ((uint32_t)(32 * quarter) << 16);
      const uint32_t tmax_bar = bar(B_TMAX + quarter);
      float* redbuf = reinterpret_cast<float*>(smem + OFF_RED);   // [3 slots][2 halves][128]
      const float c2 = p.scale_log2;
      // bf16: the running max is in raw score units and P = 2^((s - m) c2); FP8: the softmax works on
      // w = log2(p s) directly (c2 and the head's q scale folded into kq), P' = 2^(w - m)
      const float cw = F8 ? 1.f : c2;
      const float thr_raw = kRescaleLog2 / cw;
      float kq = c2;
      const float* scb = reinterpret_cast<const float*>(smem + S_OFF_SC);
      const uint32_t pbuf_peer = map_peer(sbase + V_OFF_PBUF, 1);
      const uint32_t pfull_peer = map_peer(bar(B_PFULL), 1);
      auto wait_u = [&](uint32_t b, uint32_t par) { return __all_sync(0xffffffffu, wait_bar(b, par, lim)) != 0; };
      int tph = 0;
      auto swap_half = [&](float x, int slot, float& y) -> bool {
        redbuf[(slot * 2 + half) * 128 + i] = x;
        mbar_arrive(tmax_bar);
        const bool okw = wait_u(tmax_bar, tph & 1);
        ++tph;
        y = redbuf[(slot * 2 + (half ^ 1)) * 128 + i];
        return okw;
      };
      // q~ and q^R of a piece from its 9 ring entries, once the previous piece's last QK^T is done with
      // them: this half's 4 q~ boxes (its 256 latent columns) -> TMEM columns [128 half, +128) of row
      // i as bf16 pairs; then this half's 4 chunks of q^R row i -> the q^R tile (the same swizzled
      // offsets). The entries are released after a barrier over the 8 softmax warps. Both halves
      // reach each barrier even when one of their waits gave up, and leave together if any did.
      int gq = 0, nq = 0;                            // pieces seen; ring index of the next piece's q~
      auto load_q = [&](int ntiles_prev) -> bool {
        nq += ntiles_prev * S_BOXES;
        const int n0 = nq;
        nq += 9;
        bool okq = wait_u(bar(B_QEMPTY), (gq & 1) ^ 1);
        tc_fence_after();
        if constexpr (F8) {
          // f16 operands: q~ and q^R of head i scaled by fq = 2^(14 - e), e the exponent of the row's
          // largest magnitude, so that the row's values are f16 normals up to 2^15 (exact for bf16
          // values down to 2^-14 of the largest); the scores are multiplied back by kq = c2 / fq
          for (int c = 0; okq && c < 9; ++c) okq = wait_u(bar(B_SFULL + (n0 + c) % S_RING), ((n0 + c) / S_RING) & 1);
          float amax = 0.f;
          if (okq) {
            for (int c = 0; c < 9; ++c) {
              const uint8_t* src = smem + S_OFF_RING + ((n0 + c) % S_RING) * BOX + i * 128;
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const uint4 u = *reinterpret_cast<const uint4*>(src + 16 * q);
                amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(u.x)), fabsf(bf16_hi(u.x))),
                                         fmaxf(fabsf(bf16_lo(u.y)), fabsf(bf16_hi(u.y)))));
                amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(u.z)), fabsf(bf16_hi(u.z))),
                                         fmaxf(fabsf(bf16_lo(u.w)), fabsf(bf16_hi(u.w)))));
              }
            }
          }
          int e = amax > 0.f ? (int)((__float_as_uint(amax) >> 23) & 0xffu) - 127 : 0;
          e = max(-100, min(100, e));
          const float fq = __uint_as_float((uint32_t)(127 + 14 - e) << 23);
          kq = c2 * __uint_as_float((uint32_t)(127 - 14 + e) << 23);
          if (okq) {
            for (int c = 4 * half; c < 4 * half + 4; ++c) {
              const uint8_t* src = smem + S_OFF_RING + ((n0 + c) % S_RING) * BOX + i * 128;
              uint32_t v[32];
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const uint4 u = *reinterpret_cast<const uint4*>(src + ((q ^ (i & 7)) << 4));
                v[4 * q] = pack_f16(bf16_lo(u.x) * fq, bf16_hi(u.x) * fq);
                v[4 * q + 1] = pack_f16(bf16_lo(u.y) * fq, bf16_hi(u.y) * fq);
                v[4 * q + 2] = pack_f16(bf16_lo(u.z) * fq, bf16_hi(u.z) * fq);
                v[4 * q + 3] = pack_f16(bf16_lo(u.w) * fq, bf16_hi(u.w) * fq);
              }
              tmem_st32(trow + 32 * c, v);
            }
            tmem_wait_st();
            const uint8_t* src = smem + S_OFF_RING + ((n0 + 8) % S_RING) * BOX + i * 128;
            uint8_t* dst = smem + S_OFF_QR + i * 128;
#pragma unroll
            for (int c = 4 * half; c < 4 * half + 4; ++c) {
              const int o = (c ^ (i & 7)) << 4;
              const uint4 u = *reinterpret_cast<const uint4*>(src + o);
              *reinterpret_cast<uint4*>(dst + o) =
                  make_uint4(pack_f16(bf16_lo(u.x) * fq, bf16_hi(u.x) * fq), pack_f16(bf16_lo(u.y) * fq, bf16_hi(u.y) * fq),
                             pack_f16(bf16_lo(u.z) * fq, bf16_hi(u.z) * fq), pack_f16(bf16_lo(u.w) * fq, bf16_hi(u.w) * fq));
            }
            fence_proxy_async_smem();
          }
          if (bar_sync_or(1, 256, !okq)) return false;   // all 9 entries read (or a wait gave up)
          if (threadIdx.x == 128)
            for (int c = 0; c < 9; ++c) mbar_arrive(bar(B_SEMPTY + (n0 + c) % S_RING));
        } else {
          for (int c = 4 * half; okq && c < 4 * half + 4; ++c) {
            const int e = n0 + c, slot = e % S_RING;
            okq = wait_u(bar(B_SFULL + slot), (e / S_RING) & 1);
            if (!okq) break;
            const uint8_t* src = smem + S_OFF_RING + slot * BOX + i * 128;
            uint32_t v[32];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint4 u = *reinterpret_cast<const uint4*>(src + ((q ^ (i & 7)) << 4));
              v[4 * q] = u.x; v[4 * q + 1] = u.y; v[4 * q + 2] = u.z; v[4 * q + 3] = u.w;
            }
            tmem_st32(trow + 32 * c, v);
          }
          tmem_wait_st();
          if (bar_sync_or(1, 256, !okq)) return false;   // all 8 q~ boxes read (or a wait gave up)
          if (threadIdx.x == 128)
            for (int c = 0; c < 8; ++c) mbar_arrive(bar(B_SEMPTY + (n0 + c) % S_RING));
          const int e = n0 + 8, slot = e % S_RING;
          okq = wait_u(bar(B_SFULL + slot), (e / S_RING) & 1);
          if (okq) {
            const uint8_t* src = smem + S_OFF_RING + slot * BOX + i * 128;
            uint8_t* dst = smem + S_OFF_QR + i * 128;
#pragma unroll
            for (int c = 4 * half; c < 4 * half + 4; ++c) {
              const int o = (c ^ (i & 7)) << 4;
              *reinterpret_cast<uint4*>(dst + o) = *reinterpret_cast<const uint4*>(src + o);
            }
            fence_proxy_async_smem();
          }
          if (bar_sync_or(1, 256, !okq)) return false;   // the q^R entry read
          if (threadIdx.x == 128) mbar_arrive(bar(B_SEMPTY + slot));
        }
        tc_fence_before();
        mbar_arrive(bar(B_QFULL));
        ++gq;
        return true;
      };
      ok = !w.valid() || load_q(0);
      int j = 0;
      for (; ok && w.valid(); w.next()) {
        const int b = w.b;
        const int64_t len = p.cu[b + 1] - p.cu[b];
        const int64_t vis = len - p.tq + k + 1;       // keys visible to this query token
        const int32_t ts_b = p.tile_start[b];
        const int32_t send = w.seg_end();
        float m_ref = -INFINITY, l = 0.f;             // running max (raw score units); this half's sum
        for (int32_t xt = w.x; xt < send; ++xt, ++j) {
          const int sb = j & 1;
          const bool first = xt == w.x, last = xt == send - 1;
          if (!wait_u(bar(B_SCF + sb), (j >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          float s[64];
          tmem_ld32(trow + 256 + 128 * sb + 64 * half, reinterpret_cast<uint32_t*>(s));
          tmem_ld32(trow + 256 + 128 * sb + 64 * half + 32, reinterpret_cast<uint32_t*>(s) + 32);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar(B_SCE + sb));
          const float* sc = scb + sb * (3 * NK) + 64 * half;   // FP8: this half's keys' s, log2 s, 1/s
          if constexpr (F8) {
            // w_j = s_j S'_j kq + log2 s_j (S' the score over the codes and k^R / s in f16 units)
            if (!wait_u(bar(B_SCR + sb), (j >> 1) & 1)) { ok = false; break; }
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const float2 sv = *reinterpret_cast<const float2*>(sc + c);
              const float2 lv = *reinterpret_cast<const float2*>(sc + NK + c);
              s[c] = fmaf(s[c] * sv.x, kq, lv.x);
              s[c + 1] = fmaf(s[c + 1] * sv.y, kq, lv.y);
            }
          }
          const int64_t key0 = (int64_t)(xt - ts_b) * NK + 64 * half;
          const int nvis = (int)max((int64_t)0, min((int64_t)64, vis - key0));
          if (nvis < 64) {
#pragma unroll
            for (int c = 0; c < 64; ++c) s[c] = c < nvis ? s[c] : -INFINITY;
          }
          float mx[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) mx[c] = fmaxf(fmaxf(s[4 * c], s[4 * c + 1]), fmaxf(s[4 * c + 2], s[4 * c + 3]));
#pragma unroll
          for (int w2 = 8; w2 > 0; w2 >>= 1)
#pragma unroll
            for (int c = 0; c < w2; ++c) mx[c] = fmaxf(mx[c], mx[c + w2]);
          float pmax;
          if (!swap_half(mx[0], j & 1, pmax)) { ok = false; break; }
          const float tmax = fmaxf(mx[0], pmax);
          // lazy rescale of the running max: the same decision in both halves (same tmax, m_ref)
          float alpha = 1.f;
          if (tmax > -INFINITY && (m_ref == -INFINITY || tmax > m_ref + thr_raw)) {
            alpha = m_ref == -INFINITY ? 0.f : ex2_approx((m_ref - tmax) * cw);
            l *= alpha;
            m_ref = tmax;
          }
          // P = 2^((s - m_ref) c2) in bf16 (FP8: P' = 2^(w - m_ref) in f16, l sums P' / s), packed in pairs
          uint32_t pk[32];
          if (m_ref > -INFINITY) {
            const uint64_t cc = f2_pack(cw, cw), off = f2_pack(-m_ref * cw, -m_ref * cw);
            uint64_t acc2[8];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              float a0, a1;
              f2_unpack(f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), cc, off), a0, a1);
              const float e0 = ex2_approx(a0), e1 = ex2_approx(a1);
              uint64_t le = f2_pack(e0, e1);
              if constexpr (F8) {
                pk[c] = pack_f16(e0, e1);
                const float2 iv = *reinterpret_cast<const float2*>(sc + 2 * NK + 2 * c);
                le = f2_mul(le, f2_pack(iv.x, iv.y));
              } else {
                pk[c] = pack_bf16(e0, e1);
              }
              if (c < 8) acc2[c] = le;
              else acc2[c & 7] = f2_add(acc2[c & 7], le);
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
            for (int c = 0; c < 32; ++c) pk[c] = 0u;
          }
          if (F8) mbar_arrive(bar(B_SCX + sb));      // done with the tile's scale values
          // the value CTA's P buffer sb: its P.V of tile j - 2 is done; this half's 64 keys of row i
          // go straight into it (the same 128-byte swizzle the MMA descriptor reads), alpha too
          if (!wait_u(bar(B_PVD + sb), ((j >> 1) & 1) ^ 1)) { ok = false; break; }
          const uint32_t pbuf = pbuf_peer + sb * PMSG, pfull = pfull_peer + 8 * sb;
          const uint32_t prow = pbuf + 16384 * half + i * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_async_v4(prow + ((c ^ (i & 7)) << 4), make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]),
                        pfull);
          if (half == 0) st_async_b32(pbuf + P_BYTES + 4 * i, __float_as_uint(first ? 1.f : alpha), pfull);
          if (last) {
            // piece end: lse of the piece and the reference of its unnormalised partial
            float lp;
            if (!swap_half(l, 2, lp)) { ok = false; break; }
            const float lt = l + lp;
            if (half == 0) {
              const int64_t row = ((int64_t)k * p.s_max + piece_slot(b)) * H + i;
              p.part_lse[row] = lt > 0.f ? (m_ref * cw + log2f(lt)) * 0.69314718055994531f : -INFINITY;
              p.part_m[row] = lt > 0.f ? m_ref * cw * 0.69314718055994531f : -INFINITY;
            }
          }
        }
        if (!ok) break;
        // the next piece's q^R goes in now, so that its first QK^T overlaps the value CTA's epilogue
        SegWalk nx = w;
        nx.next();
        if (nx.valid() && !load_q(send - w.x)) { ok = false; break; }
      }
      if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
    }
  } else {
    // =========================================================== value CTA
    if (warp == 0) {
      // ------------------------------------------------ TMA producer: 4 groups per tile
      // lanes 0-3 issue, lane l the group (N-half l & 1, key-half l >> 1) of every tile (ring slot l)
      if (lane < kIssuers) {
        int n = 0, last = -1;
        // The first tile's groups wait for the first P message: at launch the score CTAs' q~ and
        // first boxes then have the memory system to themselves, and these loads hit L2 behind them.
        if (w.valid() && !wait_bar_cluster(bar(B_PFULL), 0, lim)) ok = false;
        for (SegWalk sw = w; ok && sw.valid(); sw.next()) {
          const int32_t ts_b = p.tile_start[sw.b];
          const int32_t row_base = (int32_t)p.cu[sw.b];
          for (int32_t xt = sw.x; ok && xt < sw.seg_end(); ++xt) {
            const int32_t row0 = row_base + (xt - ts_b) * NK;
            for (int s = 0; s < 4; ++s, ++n) {
              if ((n & (kIssuers - 1)) != lane) continue;
              const int g = n % V_RING;
              if (!wait_bar(bar(B_GEMPTY + g), ((n / V_RING) & 1) ^ 1, lim)) { ok = false; break; }
              const int nh = s & 1, kh = s >> 1;
              const uint32_t dst = sbase + V_OFF_RING + g * VGRP;
              if (F8) {
                // the group's 256 columns as two code boxes of [64 keys x 128 codes], into boxes 1 and 3
                // (the converters spread them over all four as f16)
                mbar_expect_tx(bar(B_GFULL + g), VGRP / 2);
                tma_load_2d(dst + VBOX, &p.vmap, 256 * nh, row0 + 64 * kh, bar(B_GFULL + g));
                tma_load_2d(dst + 3 * VBOX, &p.vmap, 256 * nh + 128, row0 + 64 * kh, bar(B_GFULL + g));
              } else {
                mbar_expect_tx(bar(B_GFULL + g), VGRP);
#pragma unroll
                for (int bx = 0; bx < 4; ++bx)
                  tma_load_2d(dst + bx * VBOX, &p.vmap, 256 * nh + 64 * bx, row0 + 64 * kh, bar(B_GFULL + g));
              }
              last = n;
            }
          }
        }
        if (!ok) {
          flag_error(p.err, DEVERR_TIMEOUT);
          for (int i = max(lane, last - V_RING + 1); i <= last; ++i)
            if ((i & (kIssuers - 1)) == lane) wait_bar(bar(B_GFULL + i % V_RING), (i / V_RING) & 1, lim);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------ MMA issuer: O += P . C
      if (lane == 0) {
        constexpr uint32_t idesc = F8 ? idesc_f16(128, 256, 0, 1) : idesc_bf16(128, 256, 0, 1);
        int j = 0, g = 0, n = 0;
        for (; ok && w.valid(); w.next(), ++g) {
          const int32_t send = w.seg_end();
          for (int32_t xt = w.x; xt < send; ++xt, ++j) {
            const int pb = j & 1;
            const bool first = xt == w.x;
            if (!wait_bar_cluster(bar(B_PFULL + pb), (j >> 1) & 1, lim)) { ok = false; break; }
            // re-arm the buffer's next phase (tile j + 2: the score CTA writes it after this tile's P.V)
            mbar_expect_tx(bar(B_PFULL + pb), PMSG_TX);
            if (!wait_bar(bar(B_OREADY + pb), (j >> 1) & 1, lim)) { ok = false; break; }
            if (first && !wait_bar(bar(B_OFREE), (g & 1) ^ 1, lim)) { ok = false; break; }
            tc_fence_after();
            // P came in through the score CTA's generic stores: order them before the MMAs' reads
            fence_proxy_async_smem();
            const uint32_t pmsg = sbase + V_OFF_PBUF + pb * PMSG;
            for (int s = 0; s < 4; ++s, ++n) {
              const int gi = n % V_RING;
              if (!wait_bar(bar((F8 ? B_VCF : B_GFULL) + gi), (n / V_RING) & 1, lim)) { ok = false; break; }
              tc_fence_after();
              const int nh = s & 1, kh = s >> 1;
              const uint64_t adesc = sw128_desc(pmsg + 16384 * kh, 0, 1024);
              const uint64_t bdesc = sw128_desc(sbase + V_OFF_RING + gi * VGRP, VBOX, 1024);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + 256 * nh, adesc + 2 * kk, bdesc + ((kk * 2048) >> 4), idesc,
                            (first && kh == 0 && kk == 0) ? 0u : 1u);
              mma_commit(bar(B_GEMPTY + gi));
            }
            if (!ok) break;
            // P buffer pb free again / this tile's P.V done: both CTAs' B_PVD + pb
            mma_commit_mc(bar(B_PVD + pb), 0x3);
          }
          if (!ok) break;
          mma_commit(bar(B_ODONE));
        }
        if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
      }
    } else if (F8 && (warp == 2 || warp == 3)) {
      // ------------------------------------------------ FP8 code converters (64 threads)
      // Thread rr converts row rr of both code boxes of every group into f16 (zeros for cache rows past
      // the last sequence, which may hold anything).
      const int rr = threadIdx.x - 64;
      const int64_t total_rows = p.cu[p.B];
      int n = 0;
      for (; ok && w.valid(); w.next()) {
        const int32_t ts_b = p.tile_start[w.b];
        const int64_t row_base = p.cu[w.b];
        const int32_t send = w.seg_end();
        for (int32_t xt = w.x; ok && xt < send; ++xt) {
          const int64_t row0 = row_base + (int64_t)(xt - ts_b) * NK;
          for (int s = 0; s < 4; ++s, ++n) {
            const int gi = n % V_RING, kh = s >> 1;
            if (!wait_bar(bar(B_GFULL + gi), (n / V_RING) & 1, lim)) { ok = false; break; }
            uint8_t* grp = smem + V_OFF_RING + gi * VGRP;
            const bool past = row0 + 64 * kh + rr >= total_rows;
            convert_code_row(grp + VBOX, grp, rr, past);
            convert_code_row(grp + 3 * VBOX, grp + 2 * VBOX, rr, past);
            fence_proxy_async_smem();
            mbar_arrive(bar(B_VCF + gi));
          }
        }
      }
      if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
    } else if (warp >= 4) {
      // ------------------------------------------------ rescale + piece epilogue (thread = head = TMEM lane)
      // Warps 4-7 rescale O when the running max moved and zero cache rows past the last sequence
      // (per tile); at a piece's end warps 4-7 write O's columns [0, 256) and warps 8-11 columns
      // [256, 512) as the unnormalised partial.
      const int quarter = warp & 3, ehalf = warp >= 8 ? 1 : 0;
      const int i = 32 * quarter + lane;
      const uint32_t trow = tmem + ((uint32_t)(32 * quarter) << 16);
      const int64_t total_rows = p.cu[p.B];
      auto wait_u = [&](uint32_t b, uint32_t par) { return __all_sync(0xffffffffu, wait_bar(b, par, lim)) != 0; };
      // the piece's partial, once its last P.V is done (B_ODONE moves once per piece, so neither half
      // can see a stale phase however far behind it runs)
      auto dump = [&](int b, int g) -> bool {
        if (!wait_u(bar(B_ODONE), g & 1)) return false;
        tc_fence_after();
        // 16-byte stores: the 32 heads of a warp write 512 contiguous bytes per instruction
        uint4* po = p.part_o + ((int64_t)k * p.s_max + piece_slot(b)) * (DC / 8) * H + i;
#pragma unroll 1
        for (int c = 256 * ehalf; c < 256 * ehalf + 256; c += 32) {
          uint32_t v[32];
          tmem_ld32(trow + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 4; ++e)
            po[(c / 8 + e) * H] = make_uint4(pack_bf16(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1])),
                                             pack_bf16(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
                                             pack_bf16(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
                                             pack_bf16(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
        }
        tc_fence_before();
        mbar_arrive(bar(B_OFREE));
        return true;
      };
      int j = 0, n = 0;
      for (int g = 0; ok && w.valid(); w.next(), ++g) {
        const int b = w.b;
        const int32_t ts_b = p.tile_start[b];
        const int32_t send = w.seg_end();
        if (ehalf) {
          // columns [256, 512) of the piece's partial
          if (!dump(b, g)) { ok = false; break; }
          continue;
        }
        const int64_t row_base = p.cu[b];
        for (int32_t xt = w.x; xt < send; ++xt, ++j, n += 4) {
          const int pb = j & 1;
          const bool first = xt == w.x, last = xt == send - 1;
          if (!__all_sync(0xffffffffu, wait_bar_cluster(bar(B_PFULL + pb), (j >> 1) & 1, lim))) { ok = false; break; }
          const float* hdr = reinterpret_cast<const float*>(smem + V_OFF_PBUF + pb * PMSG + P_BYTES);
          const float alpha = hdr[i];
          if (__any_sync(0xffffffffu, !first && alpha != 1.f)) {
            // O holds the previous tiles' sum at the old max: rescale once their P.V is done
            if (!wait_u(bar(B_PVD + ((j - 1) & 1)), ((j - 1) >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < DC; c += 32) {
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
          // cache rows past the last sequence may hold anything (even NaN): zero them in this tile's
          // groups before P.V reads them (their P is zero, but 0 * NaN is not)
          const int64_t row0 = row_base + (int64_t)(xt - ts_b) * NK;
          if (!F8 && row0 + NK > total_rows) {   // (FP8: the converters write those rows as zeros)
            const int nrows = (int)max((int64_t)0, total_rows - row0);
            for (int s2 = 0; s2 < 4; ++s2) {
              const int gi = (n + s2) % V_RING;
              if (!wait_u(bar(B_GFULL + gi), ((n + s2) / V_RING) & 1)) { ok = false; break; }
              uint8_t* grp = smem + V_OFF_RING + gi * VGRP;
              const int kh = s2 >> 1;
              // rows 64 kh + rr >= nrows, 4 boxes x 8 chunks of 16 bytes each
              for (int q = i; q < 64 * 32; q += 128) {
                const int rr = q >> 5, bx = (q >> 3) & 3, c16 = q & 7;
                if (64 * kh + rr >= nrows)
                  *reinterpret_cast<uint4*>(grp + bx * VBOX + rr * 128 + c16 * 16) = make_uint4(0, 0, 0, 0);
              }
            }
            if (!ok) break;
            fence_proxy_async_smem();
          }
          mbar_arrive(bar(B_OREADY + pb));
          if (last && !dump(b, g)) { ok = false; break; }
        }
        if (!ok) break;
      }
      if (!ok) flag_error(p.err, DEVERR_TIMEOUT);
    }
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
  const int32_t res = x - v + (wid > 0 ? warp_tot[wid - 1] : 0);
  __syncthreads();
  return res;
}

// The same block first runs the device checks of cu_seqlens and writes the decode positions
// (len_b - tq + k), so that a decode step needs one small launch for both. The plan is a chain of
// dependent lookups, so up to kPlanShSeqs sequences keep their tile and slot prefixes in (dynamic)
// shared memory besides the global copies the core reads.
constexpr int kPlanShSeqs = 4096;
static_assert(kMaxPairs < 96, "the active-cluster ranks take three ballots");
__global__ void __launch_bounds__(256) plan_kernel(const int64_t* cu, int32_t B, int32_t pairs, int32_t* ts,
                                                   int32_t* sb, int4* pinfo, int32_t tq, int64_t capacity,
                                                   int64_t* pos_out, uint32_t* err) {
  check_seqs_and_positions(cu, B, tq, (int64_t)B * tq, capacity, 0, pos_out, err);
  __shared__ int32_t warp_tot[8];
  __shared__ int32_t total;
  const int tid = threadIdx.x;
  const int per = (B + 255) / 256;
  const int lo = min(B, tid * per), hi = min(B, lo + per);
  auto ntiles = [&](int b) -> int32_t {
    const int64_t len = cu[b + 1] - cu[b];
    return len > 0 ? (int32_t)((len + NK - 1) / NK) : 0;
  };
  extern __shared__ int32_t plan_sh[];
  const bool in_sh = B + 1 <= kPlanShSeqs;
  int32_t* tsr = in_sh ? plan_sh : ts;
  int32_t* sbr = in_sh ? plan_sh + (B + 1) : sb;
  int32_t acc = 0;
  for (int b = lo; b < hi; ++b) acc += ntiles(b);
  acc = block_exclusive_scan(acc, warp_tot, &total);
  for (int b = lo; b < hi; ++b) { ts[b] = acc; tsr[b] = acc; acc += ntiles(b); }
  if (tid == 0) { ts[B] = total; tsr[B] = total; }
  __syncthreads();
  const int64_t NT = total;
  // Cost-aware ranges. Besides its tiles, a cluster pays once per sequence piece (the piece's q load
  // and its partial write, about kStartCost / 2 tiles), so every sequence start weighs kStartCost
  // half-tiles: in half-tile units sequence b starts at vs(b) = 2 ts[b] + kStartCost b and its tile
  // x covers [vs(b) + kStartCost + 2 (x - ts[b]), +2). The clusters split [0, V) evenly; cluster
  // pp's range begins at the first tile at or after half-unit pp V / pairs. A range can be empty.
  const int64_t V = 2 * NT + kStartCost * (int64_t)B;
  auto bound = [&](int pp) -> int32_t {
    const int64_t v = (int64_t)pp * V / pairs;
    int b0 = 0, b1 = B;                       // the last b in [0, B] with vs(b) <= v
    while (b0 < b1) {
      const int mid = (b0 + b1 + 1) >> 1;
      if (2 * (int64_t)tsr[mid] + kStartCost * (int64_t)mid <= v) b0 = mid; else b1 = mid - 1;
    }
    if (b0 == B) return tsr[B];
    const int64_t off = v - (2 * (int64_t)tsr[b0] + kStartCost * (int64_t)b0) - kStartCost;
    const int64_t x = tsr[b0] + (off <= 0 ? 0 : (off + 1) / 2);
    return (int32_t)min(x, (int64_t)tsr[b0 + 1]);
  };
  // every cluster's first tile, one thread each (each a binary search over the sequences)
  __shared__ int32_t bnd[kMaxPairs + 1];
  for (int pp = tid; pp <= pairs; pp += blockDim.x) bnd[pp] = bound(pp);
  __syncthreads();
  // the cluster owning tile x: the last pp with bnd[pp] <= x (empty clusters never win a tie)
  auto pair_of = [&](int32_t x) -> int {
    int p0 = 0, p1 = pairs - 1;
    while (p0 < p1) {
      const int mid = (p0 + p1 + 1) >> 1;
      if (bnd[mid] <= x) p0 = mid; else p1 = mid - 1;
    }
    return p0;
  };
  // rank of each cluster among the clusters with a non-empty range: a ballot of the non-empty ones
  __shared__ int32_t arank[kMaxPairs + 1];
  __shared__ uint32_t active[3];
  if (tid < 96) {
    const uint32_t m = __ballot_sync(0xffffffffu, tid < pairs && bnd[tid + 1] > bnd[tid]);
    if ((tid & 31) == 0) active[tid >> 5] = m;
  }
  __syncthreads();
  for (int pp = tid; pp <= pairs; pp += blockDim.x) {
    int32_t r = __popc(active[pp >> 5] & ((1u << (pp & 31)) - 1u));
    for (int w = 0; w < (pp >> 5); ++w) r += __popc(active[w]);
    arank[pp] = r;
  }
  __syncthreads();
  auto nseg = [&](int b) -> int32_t {
    const int32_t a = tsr[b], e = tsr[b + 1];
    return e > a ? arank[pair_of(e - 1)] - arank[pair_of(a)] + 1 : 0;
  };
  acc = 0;
  for (int b = lo; b < hi; ++b) acc += nseg(b);
  acc = block_exclusive_scan(acc, warp_tot, &total);
  for (int b = lo; b < hi; ++b) { sb[b] = acc; sbr[b] = acc; acc += nseg(b); }
  if (tid == 0) { sb[B] = total; sbr[B] = total; }
  __syncthreads();
  // per cluster: its tile range, the sequence of its first tile and that piece's partial slot
  for (int pp = tid; pp < pairs; pp += blockDim.x) {
    int4 v = make_int4(0, 0, 0, 0);
    const int32_t x0 = bnd[pp], x1 = bnd[pp + 1];
    if (x1 > x0) {
      v.x = x0;
      v.y = x1;
      int lo2 = 0, hi2 = B - 1;               // the last b with ts[b] <= x0
      while (lo2 < hi2) {
        const int mid = (lo2 + hi2 + 1) >> 1;
        if (tsr[mid] <= x0) lo2 = mid; else hi2 = mid - 1;
      }
      // the first sequence with tiles: skip empty sequences that share the start
      while (lo2 < B - 1 && tsr[lo2 + 1] <= x0) ++lo2;
      v.z = lo2;
      v.w = sbr[lo2] + arank[pp] - arank[pair_of(tsr[lo2])];
    }
    pinfo[pp] = v;
  }
}

// Exact merge of a sequence's pieces: lse = log sum_s e^{lse_s}, o = sum_s e^{m_s - lse} O_s from the
// unnormalised head-interleaved bf16 partials O_s (O_s / l_s is the piece's own softmax average and
// e^{lse_s} = e^{m_s} l_s, so the weight e^{lse_s - lse} / l_s is e^{m_s - lse}). One block per (token,
// group of 32 heads, group of 128 columns): the reads of a (piece, 8-column group) are 512 contiguous
// bytes over the 32 heads; the block's [32 heads x 128 columns] result goes through shared memory so
// that each head's row is written as contiguous runs. The kernel is latency-bound (a few MB of L2-hot
// partials), so the partials of up to kCombBatch pieces are in flight at once, the first batch issued
// before the pieces' m and lse are staged, and the staging takes one parallel pass over the pieces.
constexpr int kCombHeads = 32, kCombCols = 128, kCombBatch = 8;
template <bool OUT_F32>
__global__ void __launch_bounds__(256) combine_kernel(const int32_t* sb, int32_t tq, int32_t s_max,
                                                      const uint4* part_o, const float* part_lse,
                                                      const float* part_m, void* o_lat, float* lse) {
  __shared__ float s_lse[kMaxPairs][kCombHeads];
  __shared__ float s_m[kMaxPairs][kCombHeads];
  __shared__ float tile[kCombHeads][kCombCols + 4];
  const int64_t t = blockIdx.x;
  const int h0 = kCombHeads * blockIdx.y, c0 = kCombCols * blockIdx.z;
  const int b = (int)(t / tq), k = (int)(t % tq);
  const int32_t s0 = sb[b], ns = min(sb[b + 1] - s0, kMaxPairs);
  const int tid = threadIdx.x, lane = tid & 31, grp = tid >> 5;
  const int64_t slot0 = (int64_t)k * s_max + s0;
  // thread (lane = head, grp): 8-column groups c8 = c0/8 + 2 grp + q, q = 0, 1 (16 columns)
  const uint4* src = part_o + (slot0 * (DC / 8) + c0 / 8 + 2 * grp) * H + h0 + lane;
  uint4 v[kCombBatch][2];
  auto load_batch = [&](int sl0) {
#pragma unroll
    for (int j = 0; j < kCombBatch; ++j)
      if (sl0 + j < ns) {
        const uint4* ps = src + (int64_t)(sl0 + j) * (DC / 8) * H;
#pragma unroll
        for (int q = 0; q < 2; ++q) v[j][q] = ps[q * H];
      }
  };
  load_batch(0);
  for (int sl = grp; sl < ns; sl += 8) {
    s_lse[sl][lane] = part_lse[(slot0 + sl) * H + h0 + lane];
    s_m[sl][lane] = part_m[(slot0 + sl) * H + h0 + lane];
  }
  __syncthreads();
  // lse over all pieces of head h0 + lane
  float mx = -INFINITY;
  for (int sl = 0; sl < ns; ++sl) mx = fmaxf(mx, s_lse[sl][lane]);
  float sum = 0.f;
  for (int sl = 0; sl < ns; ++sl) sum += mx > -INFINITY ? __expf(s_lse[sl][lane] - mx) : 0.f;
  const float tot = sum > 0.f ? mx + logf(sum) : -INFINITY;
  if (blockIdx.z == 0 && grp == 0) lse[t * H + h0 + lane] = tot;
  float4 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sl0 = 0; sl0 < ns; sl0 += kCombBatch) {
    if (sl0 > 0) load_batch(sl0);
#pragma unroll
    for (int j = 0; j < kCombBatch; ++j)
      if (sl0 + j < ns) {
        const float ms = s_m[sl0 + j][lane];
        const float wgt = (tot > -INFINITY && ms > -INFINITY) ? __expf(ms - tot) : 0.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint4 u = v[j][q];
          acc[2 * q].x += wgt * bf16_lo(u.x); acc[2 * q].y += wgt * bf16_hi(u.x);
          acc[2 * q].z += wgt * bf16_lo(u.y); acc[2 * q].w += wgt * bf16_hi(u.y);
          acc[2 * q + 1].x += wgt * bf16_lo(u.z); acc[2 * q + 1].y += wgt * bf16_hi(u.z);
          acc[2 * q + 1].z += wgt * bf16_lo(u.w); acc[2 * q + 1].w += wgt * bf16_hi(u.w);
        }
      }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) *reinterpret_cast<float4*>(&tile[lane][16 * grp + 4 * q]) = acc[q];
  __syncthreads();
  // row h0 + r, columns c0 .. c0 + 127: 8 threads per row, 16 columns each
  const int r = tid >> 3, cc = 16 * (tid & 7);
  const int64_t dst = (t * H + h0 + r) * DC + c0 + cc;
  if (OUT_F32) {
    float4* d4 = reinterpret_cast<float4*>(reinterpret_cast<float*>(o_lat) + dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) d4[q] = *reinterpret_cast<const float4*>(&tile[r][cc + 4 * q]);
  } else {
    uint4* d4 = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(o_lat) + dst);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float* x = &tile[r][cc + 8 * q];
      d4[q] = make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
    }
  }
}

size_t align1k(size_t x) { return (x + 1023) / 1024 * 1024; }

// Clusters per query token: each query token k takes its own row of clusters, and all rows
// together hold at most kMaxPairs clusters (one CTA per SM).
int32_t pairs_cap(int32_t tq) { return kMaxPairs / tq > 1 ? kMaxPairs / tq : 1; }

struct CoreScratch {
  int32_t* ts;
  int32_t* sb;
  int4* pinfo;
  float* part_lse;
  float* part_m;
  uint4* part_o;
  int32_t s_max;
};

CoreScratch carve(void* scratch, int64_t B, int32_t tq) {
  CoreScratch c;
  char* ptr = (char*)scratch;
  c.s_max = (int32_t)(pairs_cap(tq) + B);
  c.ts = (int32_t*)ptr;
  ptr += align1k((B + 1) * 4);
  c.sb = (int32_t*)ptr;
  ptr += align1k((B + 1) * 4);
  c.pinfo = (int4*)ptr;
  ptr += align1k(kMaxPairs * sizeof(int4));
  c.part_lse = (float*)ptr;
  ptr += align1k((size_t)tq * c.s_max * H * 4);
  c.part_m = (float*)ptr;
  ptr += align1k((size_t)tq * c.s_max * H * 4);
  c.part_o = (uint4*)ptr;
  return c;
}

template <bool F8>
cudaError_t launch_core(const CoreParams& p, dim3 grid, cudaStream_t st) {
  static bool configured = false;
  constexpr uint32_t smem = F8 ? SMEM_BYTES8 : SMEM_BYTES;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(latent_core_kernel<F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  timer_begin(TIMED_LATENT_CORE, st);
  latent_core_kernel<F8><<<grid, kThreads, smem, st>>>(p);
  timer_end(TIMED_LATENT_CORE, st);
  note_launch();
  return cudaGetLastError();
}

// Test hook state (mla_test_arm_stall): consumed by the next launch.
int g_stall_next = 0;

}  // namespace

void tc_latent_core_arm_stall() { g_stall_next = 1; }

size_t tc_core_scratch_bytes(const mla_dims_t& d, int64_t B, int32_t tq) {
  (void)d;
  const int64_t s_max = pairs_cap(tq) + B;
  return 2 * align1k((B + 1) * 4) + align1k(kMaxPairs * sizeof(int4)) + 2 * align1k((size_t)tq * s_max * H * 4) +
         (size_t)tq * s_max * H * DC * 2;
}

namespace {
int32_t core_pairs(int32_t tq, int num_sms) {
  int pairs = num_sms / (2 * tq);
  pairs = pairs < pairs_cap(tq) ? pairs : pairs_cap(tq);
  return pairs < 1 ? 1 : pairs;
}
}  // namespace

cudaError_t tc_core_prepare(const int64_t* cu, int64_t B, int32_t tq, int64_t capacity, int64_t* pos, void* scratch,
                            int num_sms, uint32_t* err, cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  if (B > (int64_t)1 << 20 || tq < 1 || tq > kMaxPairs) return cudaErrorInvalidValue;
  CoreScratch c = carve(scratch, B, tq);
  const size_t plan_sh = B + 1 <= kPlanShSeqs ? 2 * (size_t)(B + 1) * sizeof(int32_t) : 0;
  plan_kernel<<<1, 256, plan_sh, st>>>(cu, (int32_t)B, core_pairs(tq, num_sms), c.ts, c.sb, c.pinfo, tq, capacity, pos, err);
  note_launch();
  return cudaGetLastError();
}

cudaError_t tc_core_run(const void* q_abs, const void* q_rope, int64_t B, int32_t tq, const int64_t* cu,
                        const void* cache, int64_t capacity, bool cache_fp8, void* o_lat, bool o_f32, float* lse,
                        void* scratch, int num_sms, uint32_t* err, cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  if (B > (int64_t)1 << 20 || tq < 1 || tq > kMaxPairs || capacity > INT32_MAX || B * tq * H > INT32_MAX)
    return cudaErrorInvalidValue;
  const int64_t T = B * tq;
  CoreScratch c = carve(scratch, B, tq);
  const int pairs = core_pairs(tq, num_sms);
  cudaError_t e;
  CoreParams p;
  memset(&p, 0, sizeof(p));
  if (cache_fp8) {
    if ((e = make_tmap_u8(&p.kmap, cache, kFp8RowBytes, capacity, kFp8RowBytes, 128, NK)) != cudaSuccess) return e;
    if ((e = make_tmap_u8(&p.vmap, cache, kFp8RowBytes, capacity, kFp8RowBytes, 128, 64)) != cudaSuccess) return e;
    p.cache8 = reinterpret_cast<const uint8_t*>(cache);
  } else {
    if ((e = make_tmap_bf16(&p.kmap, cache, ROW, capacity, ROW, 64, NK)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&p.vmap, cache, ROW, capacity, ROW, 64, 64)) != cudaSuccess) return e;
  }
  if ((e = make_tmap_bf16(&p.qmap, q_abs, DC, T * H, DC, 64, H)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&p.qrmap, q_rope, DR, T * H, DR, 64, H)) != cudaSuccess) return e;
  p.cu = cu;
  p.tile_start = c.ts;
  p.slot_base = c.sb;
  p.pinfo = c.pinfo;
  p.B = (int32_t)B;
  p.tq = tq;
  p.pairs = pairs;
  p.s_max = c.s_max;
  p.part_o = c.part_o;
  p.part_lse = c.part_lse;
  p.part_m = c.part_m;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt(128.0 + 64.0));
  p.wait_ns = kWaitTimeoutNs;
  if (g_stall_next) {
    p.stall = 1;
    p.wait_ns = 20000000ull;   // 20 ms, so that the stalled launch gives up quickly
    g_stall_next = 0;
  }
  p.err = err;
  dim3 grid((unsigned)(2 * pairs), (unsigned)tq);
  e = cache_fp8 ? launch_core<true>(p, grid, st) : launch_core<false>(p, grid, st);
  if (e != cudaSuccess) return e;
  dim3 cg((unsigned)T, (unsigned)(H / kCombHeads), (unsigned)(DC / kCombCols));
  if (o_f32) combine_kernel<true><<<cg, 256, 0, st>>>(c.sb, tq, c.s_max, c.part_o, c.part_lse, c.part_m, o_lat, lse);
  else combine_kernel<false><<<cg, 256, 0, st>>>(c.sb, tq, c.s_max, c.part_o, c.part_lse, c.part_m, o_lat, lse);
  note_launch();
  return cudaGetLastError();
}

}  // namespace mla
