/*
 * mla.h - C ABI of libmla.so: DeepSeek-V3 Multi-head Latent Attention (MLA) over the
 * latent KV cache, hand-written CUDA for B200 (sm_100a).
 *
 * Source of the operations: the notes "【论文解读】DeepSeek-V3"
 * (wkq9411.github.io/2026-01-01/Paper-DeepSeek-V3.html), section 一(一) "多头潜在注意力MLA":
 *   2 "低秩KV联合压缩"  c^KV = W^DKV h, k^C = W^UK c^KV, v^C = W^UV c^KV, c^Q = W^DQ h, q^C = W^UQ c^Q;
 *                       the 【思考】 block folds W_i^UK into the query and moves W_i^UV after attention;
 *   3 "解耦RoPE"        q^R = RoPE(W^QR c^Q) per head, shared k^R = RoPE(W^KR h), the score
 *                       q^C_i.k^C_j,i + q^R_i.k^R_j scaled by 1/sqrt(d_h + d_h^R), causal softmax,
 *                       o_i = sum_j p_j v^C_j,i, u = W^O [o_1; ...; o_nh]; only c^KV and k^R are
 *                       cached, (d_c + d_h^R) elements per token and layer.
 *
 * Conventions for every call
 *   - Tensors are caller-owned device memory, borrowed for the duration of the call (weights:
 *     until the handle is destroyed or given new weights). Nothing is copied to the host.
 *   - Row-major. Weights are [out, in]: W^DQ [d_cq, d], W^UQ [n_h d_h, d_cq], W^QR [n_h d_r, d_cq],
 *     W^DKV [d_c, d], W^KR [d_r, d], W^UK [n_h d_h, d_c], W^UV [n_h d_h, d_c], W^O [d, n_h d_h].
 *     Multi-head vectors are head-major concatenations [x_1; ...; x_nh], so W_i^UK is rows
 *     [i d_h, (i+1) d_h) of W^UK.
 *   - The latent cache is [capacity, d_c + d_r] in the handle's dtype: c^KV in columns [0, d_c),
 *     the rotated k^R in columns [d_c, d_c + d_r). At the V3 sizes a row is 1152 bytes in bf16.
 *   - Sequences are packed and addressed by cu_seqlens: device int64 [B + 1], cu[0] = 0,
 *     non-decreasing; sequence b owns cache rows [cu[b], cu[b+1]). Positions are 0-based
 *     within a sequence. RoPE rotates interleaved pairs (2m, 2m+1) by pos * base^(-2m/d_r)
 *     (or YaRN's frequencies, mla_set_yarn).
 *   - Every call is asynchronous on the given stream and returns a status; it never throws.
 *     Host-side validation (null pointers, sizes, alignment, workspace) runs before any launch:
 *     on failure nothing is launched and nothing is written. Device-side checks (cu_seqlens
 *     order, lengths, slots, positions) set a sticky error word in the handle and skip the
 *     offending rows or elements; mla_sync_status() reports it. Outputs that depend on a flagged
 *     input are not valid (see each call for what is written).
 *   - Device pointers must be 16-byte aligned (MLA_ERR_ALIGNMENT otherwise).
 *   - Calls make the handle's device current while they run and restore the calling thread's
 *     current device before they return.
 *   - A handle may be used from several streams for different calls as long as calls that
 *     share a workspace or output buffer are ordered by the caller (they also share the handle's
 *     error word, which then reports the union of their device-side errors).
 */
#ifndef MLA_H
#define MLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; callers need no CUDA header. NULL is the legacy default stream. */
typedef struct CUstream_st *mla_stream_t;

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, Tq outside {1, 2}, bad op        */
  MLA_ERR_ALIGNMENT = 2,     /* a device pointer is not 16-byte aligned                         */
  MLA_ERR_UNSUPPORTED = 3,   /* dims/dtype combination the library has no kernel for            */
  MLA_ERR_WORKSPACE = 4,     /* ws_bytes below mla_workspace_size()                              */
  MLA_ERR_CUDA = 5,          /* a CUDA runtime call failed (the CUDA error is not cleared)       */
  MLA_ERR_TIMEOUT = 6,       /* a device-side bounded wait gave up (kernel returned early)       */
  MLA_ERR_DEVICE_CHECK = 7,  /* a device-side argument check failed (see mla_device_error_bits)  */
  MLA_ERR_NO_WEIGHTS = 8,    /* mla_set_weights() was not called                                  */
  MLA_ERR_SCRATCH_LIMIT = 9  /* the call needs more scratch than mla_cache_append_noalloc() holds  */
} mla_status_t;

typedef enum { MLA_BF16 = 0, MLA_FP32 = 1 } mla_dtype_t;

/* Notation of section 一(一): d, n_h, d_h, d_c, d_c' (d_cq), d_h^R (d_r); RoPE base (10000). */
typedef struct {
  int32_t d, n_h, d_h, d_c, d_cq, d_r;
  double rope_base;
} mla_dims_t;

/* Device pointers in the handle's dtype, row-major [out, in]; borrowed, not copied. */
typedef struct {
  const void *w_dq, *w_uq, *w_qr, *w_dkv, *w_kr, *w_uk, *w_uv, *w_o;
} mla_weights_t;

typedef enum {
  MLA_OP_CACHE_APPEND = 0,
  MLA_OP_DECODE = 1,
  MLA_OP_PREFILL = 2,
  MLA_OP_ATTN_DECODE_LATENT = 3
} mla_op_t;

/* Named workspace regions, readable after a call for step-level inspection. */
typedef enum {
  MLA_BUF_CQ = 0,      /* c^Q   [T, d_cq]          handle dtype (decode, prefill)               */
  MLA_BUF_QC = 1,      /* q^C   [T, n_h, d_h]      handle dtype (decode, prefill)               */
  MLA_BUF_QR = 2,      /* q^R   [T, n_h, d_r]      handle dtype, rotated (decode, prefill)      */
  MLA_BUF_QABS = 3,    /* q~    [T, n_h, d_c]      handle dtype, W^UK folded in (decode)        */
  MLA_BUF_OLAT = 4,    /* o^lat [T, n_h, d_c]      handle dtype, sum_j p_j c_j (decode)         */
  MLA_BUF_O = 5,       /* o     [T, n_h, d_h]      handle dtype (decode, prefill)               */
  MLA_BUF_KC = 6,      /* k^C   [T, n_h, d_h]      handle dtype (prefill)                       */
  MLA_BUF_VC = 7,      /* v^C   [T, n_h, d_h]      handle dtype (prefill)                       */
  MLA_BUF_LSE = 8      /* lse   [T, n_h]           fp32 (decode)                                */
} mla_buffer_t;

typedef struct mla_handle mla_handle_t;

/* Creates a handle for one device. Host-only: no CUDA call is made here.
 * dims must describe an MLA layer (all sizes > 0, d_r even); *out receives the handle.
 * MLA_BF16 runs on the tcgen05/TMA kernels, which exist for the DeepSeek-V3 head layout only
 * (n_h = 128, d_h = 128, d_c = 512, d_r = 64; d and d_cq multiples of 64): other BF16 sizes
 * return MLA_ERR_UNSUPPORTED. MLA_FP32 runs on generic CUDA-core kernels at any sizes with
 * d_c, d_h <= 512 (they exist for exact FP32 parity, not for speed). */
mla_status_t mla_create(const mla_dims_t *dims, mla_dtype_t dtype, int device, mla_handle_t **out);

/* Borrows the eight weight matrices (section 一(一)2 and 3). The first call on a device also
 * allocates the handle's 4-byte device error word. */
mla_status_t mla_set_weights(mla_handle_t *h, const mla_weights_t *w);

/* Opt-in RMSNorm after the latent compression (section 三(二)1 of the notes): c^Q = RMSNorm(W^DQ h)
 * and c^KV = RMSNorm(W^DKV h), y = x / sqrt(mean(x^2) + eps) * g, applied by every later call
 * that computes c^Q or c^KV (the cache rows hold the normalised c^KV; k^R = RoPE(W^KR h) is not
 * normalised). g_q [d_cq] and g_kv [d_c] are device pointers in the handle dtype, borrowed; both
 * NULL turns the norm off (the default). Both or neither; eps >= 0. Host-only. */
mla_status_t mla_set_rmsnorm(mla_handle_t *h, const void *g_q, const void *g_kv, double eps);

/* Opt-in YaRN context extension of the decoupled RoPE (section 三(二)3 of the notes; the
 * DeepSeek-V3 values are s = 40, alpha = 1, beta = 32 from a 4096-token original context).
 * Pair m of the d_r-wide RoPE blocks turns r_m = original_len * theta_m / (2 pi) times over the
 * original context (theta_m = rope_base^(-2m/d_r)); gamma = clamp((r_m - alpha) / (beta - alpha),
 * 0, 1) and the frequency becomes (1 - gamma) theta_m / s + gamma theta_m. Each rotated vector,
 * q^R and k^R alike, is multiplied by 0.1 ln s + 1, so the RoPE term of every score grows by its
 * square. s = 1 turns it off (the default). s >= 1, beta > alpha, original_len > 0. Host-only;
 * cache rows written under one setting must be read under the same one. */
mla_status_t mla_set_yarn(mla_handle_t *h, double s, double alpha, double beta, double original_len);

/* The format of the latent cache the handle's calls read and write. */
typedef enum {
  MLA_CACHE_BF16 = 0,   /* rows [d_c + d_r] in the handle dtype (the default)                  */
  MLA_CACHE_FP8 = 1     /* 656-byte rows at the DeepSeek-V3 sizes, see mla_set_cache_format     */
} mla_cache_format_t;

/* Opt-in FP8 (e4m3) latent cache (the notes' FP8 section 二（三） keeps e4m3 values with fp32 scales;
 * here one scale per cached row). Row layout, 656 bytes, 16-byte aligned:
 *   bytes [0, 512)    e4m3 codes of c^KV / s, round to nearest even, saturating at 448
 *   bytes [512, 640)  f16 of k^R / s, round to nearest even
 *   bytes [640, 644)  s as fp32: s = max(amax(c^KV) / 448, amax(k^R) / 32768), or 1 for a zero row
 *   bytes [644, 656)  zero
 * A row stands for [codes * s | (k^R / s) * s]; every division is an IEEE fp32 division. With FP8 the
 * cache arguments of mla_cache_append, mla_decode and mla_attn_decode_latent point to such rows
 * (capacity rows of 656 bytes), and the decode attends over the rows they stand for; the prefill
 * calls and mla_cache_append_noalloc return MLA_ERR_UNSUPPORTED. BF16 handles only
 * (MLA_ERR_UNSUPPORTED otherwise). Host-only. */
mla_status_t mla_set_cache_format(mla_handle_t *h, mla_cache_format_t format);

/* Converts n bf16 cache rows [n, 576] to FP8 rows [n, 656 bytes] (the layout above), for example to
 * move an existing cache to FP8. Device pointers, 16-byte aligned. BF16 handles at the DeepSeek-V3
 * sizes. */
mla_status_t mla_cache_quantize_fp8(mla_handle_t *h, const void *rows, int64_t n, void *out,
                                    mla_stream_t stream);

/* Workspace bytes for one call of `op` on num_seqs sequences with tq query tokens each
 * (decode, attention core) or total_tokens packed tokens (prefill, cache append).
 * Host-only arithmetic. */
mla_status_t mla_workspace_size(const mla_handle_t *h, mla_op_t op, int64_t num_seqs, int32_t tq,
                                int64_t total_tokens, size_t *bytes);

/* Byte offset of a named region inside that workspace (same arguments as mla_workspace_size).
 * MLA_ERR_INVALID_ARG if the op has no such region. Host-only arithmetic. */
mla_status_t mla_workspace_offset(const mla_handle_t *h, mla_op_t op, int64_t num_seqs, int32_t tq,
                                  int64_t total_tokens, mla_buffer_t which, size_t *offset);

/* Steps (5), (7) and the cache write of section 一(一)3: for each of the T tokens,
 * c^KV = W^DKV h_t and k^R = RoPE_pos(W^KR h_t), stored as one row at cache[slots[t]].
 *   h          [T, d]            handle dtype
 *   positions  [T] device int64  position of each token within its sequence (>= 0; a negative
 *                                one is flagged and that token's cache row is not valid after the
 *                                call: its k^R is not computed, while c^KV may be written)
 *   slots      [T] device int64  destination row, 0 <= slot < capacity (else skipped + flagged)
 *   cache      [capacity, d_c + d_r]
 * ws: mla_workspace_size(MLA_OP_CACHE_APPEND, total_tokens = T) bytes (split-K partials of the
 * projection at small T; may be 0, in which case ws may be NULL). */
mla_status_t mla_cache_append(mla_handle_t *h, const void *hidden, const int64_t *positions,
                              const int64_t *slots, int64_t T, void *cache, int64_t capacity,
                              void *ws, size_t ws_bytes, mla_stream_t stream);

/* mla_cache_append for callers that cannot allocate device memory. There is no counterpart on
 * the pages: it is a convenience of this library. Some callers cannot call cudaMalloc or hand
 * over a workspace: code running inside a stream capture that forbids allocation, runtimes
 * that own a fixed memory pool, or plain C callers that have no allocator of their own. This
 * call takes no workspace and allocates nothing; the split-K scratch it needs lives in one
 * fixed 4 MiB device array inside the library, which every GPU that loads the library holds
 * until the process exits.
 *   Same arguments, layouts and results as mla_cache_append, minus the workspace.
 *   Returns MLA_ERR_SCRATCH_LIMIT, before any launch, when the call would need more than
 *   4 MiB of scratch (at the DeepSeek-V3 sizes in bf16: 66 <= T <= 256 tokens; smaller and
 *   larger T need 4 MiB or less). MLA_ERR_NO_WEIGHTS if mla_set_weights() was not called.
 *   The first call on a device looks up the device address of the array (no allocation) and
 *   keeps it for the life of the process; make that first call outside any stream capture, and
 *   do not reset the device (cudaDeviceReset) after it, since the address belongs to the
 *   context that was current then.
 *   All calls share the one array and it keeps the last call's contents; nothing in it needs
 *   to start at zero, but calls that overlap on the GPU (different streams, no ordering)
 *   race on it. */
mla_status_t mla_cache_append_noalloc(mla_handle_t *h, const void *hidden, const int64_t *positions,
                                      const int64_t *slots, int64_t T, void *cache, int64_t capacity,
                                      mla_stream_t stream);

/* Decode step, absorbed form (section 一(一)2 【思考】 with the decoupled RoPE of section 3):
 * c^Q = W^DQ h; q^C = W^UQ c^Q; q^R = RoPE(W^QR c^Q); q~_i = W_i^UK^T q^C_i;
 * split-KV latent attention s_j = (q~_i.c_j + q^R_i.k^R_j)/sqrt(d_h + d_r) over j <= pos with an
 * exact log-sum-exp merge of the splits; o_i = W_i^UV o^lat_i; u = W^O [o_1; ...; o_nh].
 *   h_q        [B*Tq, d]          query tokens, sequence-major (token k of sequence b at b*Tq + k)
 *   cu_seqlens [B + 1] device     cache lengths INCLUDING the Tq query tokens (append first);
 *                                 query k of sequence b is at position len_b - Tq + k and sees
 *                                 cache rows cu[b] .. cu[b] + its position. len_b >= Tq.
 *   cache      [capacity, d_c + d_r]
 *   u_out      [B*Tq, d]          handle dtype
 * Tq is 1 or 2. Any B: the head-batched W^UK / W^UV projections run in chunks of 256 tokens. */
mla_status_t mla_decode(mla_handle_t *h, const void *h_q, int64_t B, int32_t Tq,
                        const int64_t *cu_seqlens, const void *cache, int64_t capacity, void *u_out,
                        void *ws, size_t ws_bytes, mla_stream_t stream);

/* Causal prefill from hidden states, unabsorbed form (section 一(一)3 steps (1)-(10)):
 * writes every token's latent row to cache[cu[b] + t], up-projects k^C, v^C from those rows,
 * runs causal attention per head (keys [k^C_i; k^R], values v^C_i) and applies W^O.
 *   hidden     [total_tokens, d]  packed by cu_seqlens (cu[B] == total_tokens)
 *   max_seqlen upper bound on any sequence length (sizes the launch; longer rows are skipped
 *              and flagged)
 *   cache      [capacity, d_c + d_r], capacity >= total_tokens
 *   u_out      [total_tokens, d]  handle dtype */
mla_status_t mla_prefill(mla_handle_t *h, const void *hidden, int64_t B, const int64_t *cu_seqlens,
                         int64_t total_tokens, int64_t max_seqlen, void *cache, int64_t capacity,
                         void *u_out, void *ws, size_t ws_bytes, mla_stream_t stream);

/* The two forms a chunked prefill can take (mla_prefill_chunk). */
typedef enum {
  MLA_CHUNK_AUTO = 0,        /* chosen by the chunk / prefix ratio (see mla_prefill_chunk)            */
  MLA_CHUNK_ABSORBED = 1,    /* the decode form: q~ = W^UK^T q^C, the latent core, W^UV; needs chunks  */
                             /* of one length Tc <= 64 (total_q == B * max_q)                          */
  MLA_CHUNK_UNABSORBED = 2   /* the prefill form: k^C, v^C = W^UK c^KV, W^UV c^KV for every key row    */
} mla_chunk_form_t;

/* Chunked prefill against an existing latent cache: step (10) of section 一(一)3 with the sum over
 * every cached position j <= t, where the rows of the earlier positions are already in the cache
 * and are reused as they are (the KV-cache reuse of mlqm.cn/news/135256, "KV Cache的核心原理").
 * Sequence b owns cache rows cu_kv[b] .. cu_kv[b+1]; its chunk is the last Tc_b = cu_q[b+1] -
 * cu_q[b] of them, at positions P_b .. P_b + Tc_b - 1 with P_b = (cu_kv[b+1] - cu_kv[b]) - Tc_b.
 * The call writes the chunk's cache rows (steps (5), (7)), computes its queries (steps (1)-(3)),
 * lets each chunk token attend to rows 0 .. its position of its sequence, and applies W^O.
 * The first P_b rows of each sequence must hold the cache rows of its earlier tokens.
 *   hidden   [total_q, d]            chunk tokens, packed by cu_q (cu_q[B] == total_q)
 *   cu_q     [B + 1] device int64    chunk tokens per sequence (a chunk may be empty)
 *   max_q    upper bound on any chunk length
 *   cu_kv    [B + 1] device int64    cache rows per sequence INCLUDING its chunk (cu_kv[B] == total_kv)
 *   cache    [capacity, d_c + d_r]   capacity >= total_kv
 *   form     MLA_CHUNK_AUTO takes the absorbed form when the chunks share one length Tc <= 64
 *            (total_q == B * max_q) and the key rows number at least twice the chunk tokens
 *            (total_kv >= 2 total_q): its cost grows with Tc x rows, the unabsorbed form's with
 *            the rows x the up-projection of every row, so short chunks on long prefixes favour it.
 *            A forced MLA_CHUNK_ABSORBED with other chunk shapes returns MLA_ERR_INVALID_ARG.
 *   u_out    [total_q, d]            handle dtype
 *   ws       mla_prefill_chunk_workspace() bytes for the same arguments
 * Device checks (MLA_ERR_DEVICE_CHECK through mla_sync_status): cu_q[0] = cu_kv[0] = 0, both
 * non-decreasing, cu_kv[B] <= capacity, Tc_b <= len_b, Tc_b <= max_q, the two totals. */
mla_status_t mla_prefill_chunk(mla_handle_t *h, const void *hidden, int64_t B, const int64_t *cu_q,
                               int64_t total_q, int64_t max_q, const int64_t *cu_kv, int64_t total_kv,
                               void *cache, int64_t capacity, mla_chunk_form_t form, void *u_out, void *ws,
                               size_t ws_bytes, mla_stream_t stream);

/* The form mla_prefill_chunk takes for these arguments (AUTO resolved) and its workspace bytes.
 * Host-only arithmetic. */
mla_status_t mla_prefill_chunk_workspace(const mla_handle_t *h, int64_t B, int64_t total_q, int64_t max_q,
                                         int64_t total_kv, mla_chunk_form_t form, mla_chunk_form_t *chosen,
                                         size_t *bytes);

/* Byte offset of a named region of that workspace: CQ, QC, QR, O in both forms; QABS, OLAT, LSE in
 * the absorbed form ([B * Tc] tokens); KC, VC in the unabsorbed form ([total_kv] key rows).
 * MLA_ERR_INVALID_ARG if the chosen form has no such region. Host-only arithmetic. */
mla_status_t mla_prefill_chunk_offset(const mla_handle_t *h, int64_t B, int64_t total_q, int64_t max_q,
                                      int64_t total_kv, mla_chunk_form_t form, mla_buffer_t which,
                                      size_t *offset);

/* The latent attention core alone (decode semantics as mla_decode):
 *   q_abs  [B*Tq, n_h, d_c]  handle dtype (q~ = W_i^UK^T q^C_i)
 *   q_rope [B*Tq, n_h, d_r]  handle dtype (rotated q^R)
 *   o_lat  [B*Tq, n_h, d_c]  fp32, sum_j p_j c_j
 *   lse    [B*Tq, n_h]       fp32, natural log of sum_j exp(s_j) */
mla_status_t mla_attn_decode_latent(mla_handle_t *h, const void *q_abs, const void *q_rope, int64_t B,
                                    int32_t Tq, const int64_t *cu_seqlens, const void *cache,
                                    int64_t capacity, float *o_lat, float *lse, void *ws,
                                    size_t ws_bytes, mla_stream_t stream);

/* The causal prefill attention core alone: step (10) of section 一(一)3 in the unabsorbed form, as
 * inside mla_prefill. For head i and packed token t at position p of its sequence,
 *   o[t, i] = sum_{j <= p} softmax_j([q^C; q^R][t, i] . [k^C[j, i]; k^R[j]] / sqrt(d_h + d_r)) v^C[j, i]
 * over the tokens j of the same sequence.
 *   q_c    [total_tokens, n_h, d_h]  handle dtype (q^C)
 *   q_rope [total_tokens, n_h, d_r]  handle dtype (rotated q^R)
 *   k_c    [total_tokens, n_h, d_h]  handle dtype (k^C = W^UK c^KV)
 *   v_c    [total_tokens, n_h, d_h]  handle dtype (v^C = W^UV c^KV)
 *   cache  [capacity, d_c + d_r]     k^R of packed token t in row t, columns [d_c, d_c + d_r)
 *   o      [total_tokens, n_h, d_h]  handle dtype
 * cu_seqlens, total_tokens and max_seqlen as for mla_prefill. No workspace, no weights. */
mla_status_t mla_attn_prefill(mla_handle_t *h, const void *q_c, const void *q_rope, const void *k_c,
                              const void *v_c, int64_t B, const int64_t *cu_seqlens, int64_t total_tokens,
                              int64_t max_seqlen, const void *cache, int64_t capacity, void *o,
                              mla_stream_t stream);

/* Synchronizes the stream, then reports (and clears) the handle's device error word:
 * MLA_ERR_TIMEOUT, MLA_ERR_DEVICE_CHECK or MLA_OK. */
mla_status_t mla_sync_status(mla_handle_t *h, mla_stream_t stream);

/* Bits of the last error word read by mla_sync_status (see MLA_DEVERR_* in the source). */
uint32_t mla_device_error_bits(const mla_handle_t *h);

/* Number of kernels this library has launched in this process (all handles, all devices). */
uint64_t mla_kernel_launches(void);

/* Which kernel family a call of `op` takes with this handle: 1 = tcgen05/TMA (BF16 at the V3
 * sizes), 0 = generic CUDA-core kernels (FP32, or other sizes). Host-only. */
int mla_uses_tensor_cores(const mla_handle_t *h, mla_op_t op);

/* Kernel timing for measurement tools. While enabled (process-wide), the library records a CUDA event
 * on the launching stream right before and right after every launch of its two attention cores;
 * mla_kernel_time_ms waits for the end event of the last bracketed launch of `which`
 * (0 = the decode latent core, 1 = the prefill attention core) and returns its elapsed ms, or
 * MLA_ERR_INVALID_ARG if there was none. Off by default; do not enable it around stream capture. */
mla_status_t mla_set_kernel_timing(int enabled);
mla_status_t mla_kernel_time_ms(int which, float *ms);

/* Test hook for the bounded device-side waits (no counterpart on the pages). Arms the next launch
 * of the decode latent core in this process (mla_attn_decode_latent or mla_decode, any handle) so
 * that the cluster holding the first cache tile waits for a box of it that is never loaded (the
 * query's first box), with a 20 ms wait limit
 * instead of 1 s. Every role of that launch gives up after its limit and returns; the launch
 * writes garbage outputs, and mla_sync_status() reports MLA_ERR_TIMEOUT. Nothing faults or hangs,
 * and later calls run normally. Not thread-safe: arm it only while no other thread launches. */
void mla_test_arm_stall(void);

const char *mla_status_string(mla_status_t s);

/* Frees the handle's own device memory (its error word). Borrowed tensors are untouched. */
void mla_destroy(mla_handle_t *h);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H */
