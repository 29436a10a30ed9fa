// Tensor-core (tcgen05 / TMEM / TMA) kernels for BF16 at the DeepSeek-V3 MLA sizes
// (n_h = 128, d_h = 128, d_c = 512, d_h^R = 64; d and d_c' multiples of 64).
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "mla.h"

namespace mla {

// Scratch bytes of the tensor-core decode path (split-K partials of the projections and the
// split-KV partials of the latent core) for B sequences of tq query tokens.
size_t tc_decode_scratch_bytes(const mla_dims_t& d, int64_t B, int32_t tq);
// Scratch bytes of the latent core alone.
size_t tc_core_scratch_bytes(const mla_dims_t& d, int64_t B, int32_t tq);
// Scratch bytes of mla_cache_append for T tokens (split-K partials when T is small; with an FP8 cache,
// then the bf16 rows staged before quantization).
size_t tc_append_scratch_bytes(const mla_dims_t& d, int64_t T, bool fp8 = false);

// FP8 latent cache rows (mla_set_cache_format): 656 bytes = 512 e4m3 codes of c^KV / s, 64 f16 of
// k^R / s, the fp32 scale s and 12 zero bytes.
constexpr int kFp8RowBytes = 656;
constexpr int kFp8RowLatent = 576;   // bf16 elements of the cache row it is made from
constexpr int kFp8KrOffset = 512;    // byte offsets of k^R / s and of s in the row
constexpr int kFp8ScaleOffset = 640;
// bf16 cache rows [n][576] -> FP8 rows at out + row(r) * 656, row(r) = rowmap ? rowmap[r] : r (rows
// mapped outside [0, limit) are not written and set DEVERR_SLOT in *err).
cudaError_t fp8_quantize_rows(const void* rows, int64_t n, const int64_t* rowmap, int64_t limit, void* out,
                              uint32_t* err, cudaStream_t st);
// Scratch bytes of the bf16 rows an FP8 append stages before quantizing them.
inline size_t fp8_staging_bytes(int64_t T) { return (size_t)(T > 0 ? T : 1) * kFp8RowLatent * 2; }

cudaError_t tc_cache_append(const mla_dims_t& d, const mla_weights_t& w, const LayerOpts& o, const void* hidden,
                            const int64_t* positions, const int64_t* slots, int64_t T, void* cache,
                            int64_t capacity, void* scratch, size_t scratch_bytes, uint32_t* err,
                            cudaStream_t st);

// Test hook: the next latent-core launch in this process waits on a barrier that nothing signals
// (the first box of the cluster holding tile 0 is never loaded), with a 20 ms wait limit, so that its
// bounded waits give up and the launch reports a timeout.
void tc_latent_core_arm_stall();

// The split-KV tcgen05 latent core (q~, q^R -> o^lat, lse) on scratch of tc_core_scratch_bytes(), in two
// launches: tc_core_prepare (one block: the device checks of cu_seqlens, the decode positions when pos is
// not null, and the plan of the clusters' tile ranges and partial slots), then tc_core_run (the core and
// the log-sum-exp merge of the partials) with the same B, tq, scratch and num_sms.
cudaError_t tc_core_prepare(const int64_t* cu, int64_t B, int32_t tq, int64_t capacity, int64_t* pos, void* scratch,
                            int num_sms, uint32_t* err, cudaStream_t st);
// cache_fp8: the cache rows are FP8 rows of kFp8RowBytes (e4m3 codes, f16 k^R / s, fp32 s).
cudaError_t tc_core_run(const void* q_abs, const void* q_rope, int64_t B, int32_t tq, const int64_t* cu,
                        const void* cache, int64_t capacity, bool cache_fp8, void* o_lat, bool o_f32, float* lse,
                        void* scratch, int num_sms, uint32_t* err, cudaStream_t st);

cudaError_t tc_decode(const mla_dims_t& d, const mla_weights_t& w, const LayerOpts& lo, const void* h_q, int64_t B,
                      int32_t tq, const int64_t* cu, const int64_t* pos, const void* cache, int64_t capacity, void* u_out,
                      void* cq, void* qc, void* qr, void* qabs, void* olat, void* o, float* lse, void* scratch,
                      int num_sms, uint32_t* err, cudaStream_t st);

// The causal prefill attention core (unabsorbed): q^C [T][H][128], q^R [T][H][64] of the query tokens
// (packed by cu), k^C, v^C [T_kv][H][128] and k^R in column 512 of the cache rows [capacity][576] of
// the key rows (packed by cu_kv; sequence b's query tokens are its last ones) -> o [T][H][128].
// cu_kv == nullptr: the key rows are the query tokens themselves (cu_kv = cu, T_kv = T).
cudaError_t tc_prefill_attention(const void* qc, const void* qr, const void* kc, const void* vc, const void* cache,
                                 int64_t capacity, const int64_t* cu, const int64_t* cu_kv, int64_t B, int64_t T,
                                 int64_t T_kv, int64_t max_seqlen, void* o, int num_sms, uint32_t* err,
                                 cudaStream_t st);

// Unabsorbed prefill of T query tokens (hidden states packed by cu) at positions pos, their cache
// rows written at slots (nullptr: row t), k^C / v^C up-projected from the T_kv key rows packed by
// cu_kv (nullptr: whole sequences, cu_kv = cu), then attention and W^O.
cudaError_t tc_prefill(const mla_dims_t& d, const mla_weights_t& w, const LayerOpts& lo, const void* hidden, int64_t B,
                       const int64_t* cu, const int64_t* cu_kv, int64_t T, int64_t T_kv, int64_t max_seqlen,
                       const int64_t* pos, const int64_t* slots, void* cache, int64_t capacity, void* u_out,
                       void* cq, void* qc, void* qr, void* kc, void* vc, void* o, int num_sms, uint32_t* err,
                       cudaStream_t st);

}  // namespace mla
