"""CPU float64 oracle for DeepSeek-V3 Multi-head Latent Attention (MLA) over the latent KV cache.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import or call this
module: only the tests, the package's smoke check and the benchmark's CPU
baseline leg use it. It shares no code with the CUDA path and imports nothing
from the package; callers hand it plain numpy arrays.

Source. The definitions follow the notes "【论文解读】DeepSeek-V3"
(wkq9411.github.io/2026-01-01/Paper-DeepSeek-V3.html), section 一(一)
"多头潜在注意力MLA" (multi-head latent attention):
  * 1 "回顾多头注意力MHA"      - multi-head attention, causal softmax over j <= t, W^O last;
  * 2 "低秩KV联合压缩"         - c^KV = W^DKV h, k^C = W^UK c^KV, v^C = W^UV c^KV,
                                 c^Q = W^DQ h, q^C = W^UQ c^Q, and the 【思考】 block
                                 on absorbing W^UK into the query and W^UV into W^O;
  * 3 "解耦RoPE"               - block-diagonal 2x2 RoPE, decoupled q^R = RoPE(W^QR c^Q)
                                 per head, shared k^R = RoPE(W^KR h), score scale
                                 1/sqrt(d_h + d_h^R), and the ten-step computation
                                 (1)-(10) that this file spells out.
Section 三(二) "模型超参数" / "长上下文扩展" adds the RMSNorm after the latent
compression and YaRN on the decoupled key (readings R4, R4').
Decode semantics (cache the keys/values of past tokens, compute only the new
query, attend over every cached position) follow the explainer at
mlqm.cn/news/135256, paragraph "KV Cache的核心原理".

Readings where the pages leave a step open:
  R1 RoPE pairs are the interleaved pairs (2m, 2m+1) of the block-diagonal
     form, rotated by [[cos, -sin], [sin, cos]] with angle pos * base^(-2m/d_R).
  R2 Positions are 0-based within a sequence; packing does not shift them.
  R3 The scale is 1/sqrt(d_h + d_h^R) in both the absorbed and unabsorbed forms.
  R4 RMSNorm and YaRN are opt-in (no equation of section 一(一) has them; section
     三(二) names both). RMSNorm after the latent compression, when the weights carry
     gains g_q [d_c'] and g_kv [d_c]: c^Q = RMSNorm(W^DQ h), c^KV = RMSNorm(W^DKV h)
     with y = x / sqrt(mean(x^2) + eps) * g; k^R = RoPE(W^KR h) is not normalised
     (its input is h). eps is not on the pages: 1e-6 by default.
  R4' YaRN (section 三(二)3: s = 40, alpha = 1, beta = 32, sqrt(t) = 0.1 ln s + 1,
     for the decoupled key only), when s > 1: the "NTK-by-parts" frequencies of the
     YaRN paper from the original context L0 = 4096 (the 4K pre-training length),
     r_m = L0 theta_m / (2 pi), gamma = clip((r - alpha) / (beta - alpha), 0, 1),
     theta'_m = (1 - gamma) theta_m / s + gamma theta_m; the factor 0.1 ln s + 1
     multiplies each rotated vector, q^R and k^R alike, so the RoPE term of the
     score grows by its square and the latent term is untouched.
  R15 FP8 latent cache (opt-in): one fp32 scale per cached row, s = max(amax(c^KV) / 448,
     amax(k^R) / 32768); c^KV stored as e4m3 codes of c^KV / s (round to nearest, ties to
     even, saturating at 448) and k^R as f16 of k^R / s, both divisions in fp32. Attention
     over an FP8 cache is attention over the dequantized rows [codes s | k^R' s].
  R5 Decode: a sequence's cache length includes its Tq new tokens (appended
     first); query k sits at position len - Tq + k and sees rows j <= position.
  R6 A synthetic decode cache holds c^KV and an already-rotated k^R.
  R7 lse is the natural log of sum_j exp(s_j) over the scaled scores s_j.

Arithmetic is float64 throughout; inputs are the rounded (bf16 or fp32)
values widened to float64. Library matmuls serve only as the sums that the
equations write out; there is no blocking, fusion or reordering beyond that.
"""
from __future__ import annotations

import numpy as np


def f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# RoPE (section 3, the R_m block-diagonal rotation; reading R1)
# ---------------------------------------------------------------------------
def yarn_frequencies(d_r: int, base: float, s: float, alpha: float, beta: float, l0: int) -> np.ndarray:
    """YaRN's interpolated RoPE frequencies (reading R4'), m = 0..d_r/2-1.

    Pair m turns r_m = L0 / lambda_m times over the original context, lambda_m = 2 pi / theta_m.
    Pairs that turn more than beta times keep theta_m, pairs that turn less than alpha times are
    interpolated fully (theta_m / s), and the pairs in between are blended linearly in r.
    """
    m = np.arange(d_r // 2, dtype=np.float64)
    theta = base ** (-2.0 * m / d_r)
    r = l0 * theta / (2.0 * np.pi)
    gamma = np.clip((r - alpha) / (beta - alpha), 0.0, 1.0)
    return (1.0 - gamma) * theta / s + gamma * theta


def rope_scale(dims) -> float:
    """The factor on each rotated vector: 0.1 ln s + 1 with YaRN (s > 1), else 1 (reading R4')."""
    return 0.1 * np.log(dims.yarn_s) + 1.0 if dims.yarn_s > 1.0 else 1.0


def rope_frequencies(d_r: int, dims) -> np.ndarray:
    """theta_m = base^(-2m/d_r) (reading R1), or YaRN's interpolated table when s > 1."""
    if dims.yarn_s > 1.0:
        return yarn_frequencies(d_r, dims.rope_base, dims.yarn_s, dims.yarn_alpha, dims.yarn_beta, dims.yarn_l0)
    m = np.arange(d_r // 2, dtype=np.float64)
    return dims.rope_base ** (-2.0 * m / d_r)


def rope_angles(pos, d_r: int, base: float) -> np.ndarray:
    """Angles pos * theta_m with theta_m = base^(-2m/d_r), m = 0..d_r/2-1; shape pos.shape + (d_r/2,)."""
    m = np.arange(d_r // 2, dtype=np.float64)
    theta = base ** (-2.0 * m / d_r)
    return f64(pos)[..., None] * theta


def rotate(x, ang) -> np.ndarray:
    """Rotate each pair (x_2m, x_2m+1) of the last axis by ang[..., m]."""
    x = f64(x)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    a = x0 * c - x1 * s
    b = x0 * s + x1 * c
    return np.stack([a, b], axis=-1).reshape(a.shape[:-1] + (2 * a.shape[-1],))


def rope(x, pos, base: float) -> np.ndarray:
    """Rotate each pair (x_2m, x_2m+1) of the last axis by the angle of position pos.

    pos must broadcast against x.shape[:-1].
    """
    return rotate(x, rope_angles(pos, f64(x).shape[-1], base))


def rope_dims(x, pos, dims) -> np.ndarray:
    """The decoupled RoPE of a layer: plain (rope) or, with YaRN, its frequencies and factor."""
    if dims.yarn_s <= 1.0:
        return rope(x, pos, dims.rope_base)
    ang = f64(pos)[..., None] * rope_frequencies(f64(x).shape[-1], dims)
    return rope_scale(dims) * rotate(x, ang)


def rms_norm(x, g, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g (reading R4)."""
    x = f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * f64(g)


# ---------------------------------------------------------------------------
# Projections (section 2 and section 3, steps (1)-(3), (5)-(7), (9))
# ---------------------------------------------------------------------------
def query_projections(h, W, dims, pos):
    """Steps (1)-(3): c^Q = W^DQ h; q^C = W^UQ c^Q split by heads; q^R = RoPE(W^QR c^Q) per head.

    With gains W["g_q"], c^Q = RMSNorm(W^DQ h) (reading R4); RoPE follows dims (YaRN, reading R4').

    h [T, d], pos [T] -> c_q [T, d_cq], q_c [T, n_h, d_h], q_r [T, n_h, d_r].
    """
    h = f64(h)
    T = h.shape[0]
    c_q = h @ f64(W["w_dq"]).T
    if "g_q" in W:
        c_q = rms_norm(c_q, W["g_q"], dims.rms_eps)
    q_c = (c_q @ f64(W["w_uq"]).T).reshape(T, dims.n_h, dims.d_h)
    q_r_hat = (c_q @ f64(W["w_qr"]).T).reshape(T, dims.n_h, dims.d_r)
    q_r = rope_dims(q_r_hat, f64(pos)[:, None], dims)
    return c_q, q_c, q_r


def kv_compression(h, W, dims, pos):
    """Steps (5) and (7): c^KV = W^DKV h and k^R = RoPE(W^KR h). Returns c_kv [T, d_c], k_r [T, d_r].

    With gains W["g_kv"], c^KV = RMSNorm(W^DKV h) (reading R4); RoPE follows dims (YaRN, reading R4').
    """
    h = f64(h)
    c_kv = h @ f64(W["w_dkv"]).T
    if "g_kv" in W:
        c_kv = rms_norm(c_kv, W["g_kv"], dims.rms_eps)
    k_r = rope_dims(h @ f64(W["w_kr"]).T, pos, dims)
    return c_kv, k_r


def cache_rows(c_kv, k_r) -> np.ndarray:
    """One latent-cache row per token: [c^KV | k^R], (d_c + d_h^R) elements (section 3, cache size)."""
    return np.concatenate([f64(c_kv), f64(k_r)], axis=1)


def up_project_head(c_kv, W, dims, i):
    """Steps (6) and (9) for head i: k^C_i = W_i^UK c^KV and v^C_i = W_i^UV c^KV.

    W_i^UK are rows [i d_h, (i+1) d_h) of W^UK (head-major split of section 2's 【思考】).
    c_kv [L, d_c] -> k_c_i [L, d_h], v_c_i [L, d_h].
    """
    rows = slice(i * dims.d_h, (i + 1) * dims.d_h)
    c_kv = f64(c_kv)
    return c_kv @ f64(W["w_uk"][rows]).T, c_kv @ f64(W["w_uv"][rows]).T


# ---------------------------------------------------------------------------
# Attention (step (4), (8), (10))
# ---------------------------------------------------------------------------
def causal_softmax_attend(q, k, v, lat, qpos, scale):
    """One head: s_j = q.k_j * scale for j <= qpos, p = softmax(s), returns (sum p v, sum p lat, lse, p).

    q [Tq, e], k [L, e], v [L, dv], lat [L, d_c] or None, qpos [Tq] (reading R5: key j is
    visible to a query at position qpos iff j <= qpos; masked keys are left out of the sum).
    """
    q, k, v = f64(q), f64(k), f64(v)
    Tq, L = q.shape[0], k.shape[0]
    s = (q @ k.T) * scale
    visible = np.arange(L)[None, :] <= np.asarray(qpos)[:, None]
    s_masked = np.where(visible, s, -np.inf)
    m = s_masked.max(axis=1, keepdims=True)
    e = np.where(visible, np.exp(s_masked - m), 0.0)
    z = e.sum(axis=1, keepdims=True)
    p = e / z
    o = p @ v
    o_lat = None if lat is None else p @ f64(lat)
    lse = (m + np.log(z))[:, 0]
    return o, o_lat, lse, p


def attend_unabsorbed(q_c, q_r, c_kv, k_r, W, dims, qpos, heads=None):
    """Steps (4), (6), (8), (9), (10) for one sequence, keys/values up-projected explicitly.

    q_c [Tq, n_h, d_h], q_r [Tq, n_h, d_r], c_kv [L, d_c], k_r [L, d_r] (shared by all heads).
    Returns o [Tq, H, d_h], o_lat [Tq, H, d_c] (= sum_j p_j c_j, the factor that section 2's
    【思考】 moves W_i^UV out of), lse [Tq, H] for the heads asked for (default all).
    """
    heads = range(dims.n_h) if heads is None else list(heads)
    scale = 1.0 / np.sqrt(dims.d_h + dims.d_r)
    Tq = q_c.shape[0]
    H = len(heads)
    o = np.empty((Tq, H, dims.d_h))
    o_lat = np.empty((Tq, H, dims.d_c))
    lse = np.empty((Tq, H))
    k_r = f64(k_r)
    for hi, i in enumerate(heads):
        k_c_i, v_c_i = up_project_head(c_kv, W, dims, i)           # steps (6), (9)
        q_i = np.concatenate([f64(q_c[:, i]), f64(q_r[:, i])], axis=1)   # step (4)
        k_i = np.concatenate([k_c_i, k_r], axis=1)                  # step (8)
        o[:, hi], o_lat[:, hi], lse[:, hi], _ = causal_softmax_attend(q_i, k_i, v_c_i, c_kv, qpos, scale)
    return o, o_lat, lse


def output_projection(o, W) -> np.ndarray:
    """Step (10), second equation: u_t = W^O [o_t,1; ...; o_t,n_h]. o [T, n_h, d_h] -> u [T, d]."""
    o = f64(o)
    return o.reshape(o.shape[0], -1) @ f64(W["w_o"]).T


# ---------------------------------------------------------------------------
# Whole calls
# ---------------------------------------------------------------------------
def cache_append(h, positions, W, dims) -> np.ndarray:
    """Rows [c^KV | RoPE(W^KR h)] for tokens h [T, d] at the given positions (steps (5), (7))."""
    c_kv, k_r = kv_compression(h, W, dims, positions)
    return cache_rows(c_kv, k_r)


def decode_positions(cu_seqlens, tq):
    """Reading R5: query k of sequence b sits at position len_b - Tq + k."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lens = cu[1:] - cu[:-1]
    return np.concatenate([np.arange(L - tq, L) for L in lens]).astype(np.int64)


def mla_decode(h_q, cache, cu_seqlens, tq, W, dims, seqs=None, heads=None):
    """Decode step over a latent cache, unabsorbed (steps (1)-(10) with cached c^KV, k^R).

    h_q [B*Tq, d] (sequence-major), cache [rows, d_c + d_r] holding every sequence's rows
    (including its Tq new tokens) packed by cu_seqlens. Returns a dict for the sequences
    asked for (default all): rows (token indices), o_lat, lse, o and, when all heads are
    computed, u.
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = len(cu) - 1
    seqs = range(B) if seqs is None else list(seqs)
    pos_all = decode_positions(cu, tq)
    rows, o_l, lat_l, lse_l = [], [], [], []
    for b in seqs:
        r = np.arange(b * tq, (b + 1) * tq)
        _, q_c, q_r = query_projections(f64(np.asarray(h_q)[r]), W, dims, pos_all[r])
        seq = f64(cache[cu[b]:cu[b + 1]])
        o, o_lat, lse = attend_unabsorbed(q_c, q_r, seq[:, :dims.d_c], seq[:, dims.d_c:], W, dims,
                                          pos_all[r], heads)
        rows.append(r); o_l.append(o); lat_l.append(o_lat); lse_l.append(lse)
    out = {"rows": np.concatenate(rows), "o": np.concatenate(o_l), "o_lat": np.concatenate(lat_l),
           "lse": np.concatenate(lse_l)}
    if heads is None:
        out["u"] = output_projection(out["o"], W)
    return out


def mla_prefill(h, cu_seqlens, W, dims, query_rows=None, heads=None):
    """Causal prefill from hidden states, steps (1)-(10) for every sequence packed by cu_seqlens.

    Every token's cache row is computed; attention, o and u only for query_rows (global token
    indices, default all). Returns dict with cache [T, d_c + d_r], rows, o, o_lat, lse, u.
    """
    h = f64(h)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T = h.shape[0]
    pos = np.concatenate([np.arange(cu[b + 1] - cu[b]) for b in range(len(cu) - 1)]).astype(np.int64)
    c_kv, k_r = kv_compression(h, W, dims, pos)
    rows_all = np.arange(T) if query_rows is None else np.sort(np.asarray(query_rows, dtype=np.int64))
    rows, o_l, lat_l, lse_l = [], [], [], []
    for b in range(len(cu) - 1):
        r = rows_all[(rows_all >= cu[b]) & (rows_all < cu[b + 1])]
        if len(r) == 0:
            continue
        _, q_c, q_r = query_projections(h[r], W, dims, pos[r])
        o, o_lat, lse = attend_unabsorbed(q_c, q_r, c_kv[cu[b]:cu[b + 1]], k_r[cu[b]:cu[b + 1]], W, dims,
                                          pos[r], heads)
        rows.append(r); o_l.append(o); lat_l.append(o_lat); lse_l.append(lse)
    out = {"cache": cache_rows(c_kv, k_r), "rows": np.concatenate(rows), "o": np.concatenate(o_l),
           "o_lat": np.concatenate(lat_l), "lse": np.concatenate(lse_l)}
    if heads is None:
        out["u"] = output_projection(out["o"], W)
    return out


def mla_prefill_chunk(h, cu_q, cache, cu_kv, W, dims, heads=None):
    """Chunked prefill against an existing latent cache (section 3 steps (1)-(10), with the sum of
    step (10) running over every cached position j <= t, and the KV-cache reuse of the explainer's
    "KV Cache的核心原理" paragraph).

    Sequence b owns cache rows cache[cu_kv[b] : cu_kv[b+1]]. Its last Tc_b = cu_q[b+1] - cu_q[b] rows
    belong to the chunk's new tokens h[cu_q[b] : cu_q[b+1]], at positions P_b .. P_b + Tc_b - 1 with
    P_b = (cu_kv[b+1] - cu_kv[b]) - Tc_b; the first P_b rows are the cached prefix and are used as
    given. The chunk's rows are computed by steps (5) and (7) and written into a copy of the cache;
    every chunk token then attends over its sequence's rows 0 .. its position (unabsorbed form).
    Returns dict: cache (with the chunk's rows), rows (chunk token indices), o, o_lat, lse and, when
    all heads are computed, u.
    """
    h = f64(h)
    cq = np.asarray(cu_q, dtype=np.int64)
    ck = np.asarray(cu_kv, dtype=np.int64)
    out_cache = f64(cache).copy()
    rows, o_l, lat_l, lse_l = [], [], [], []
    for b in range(len(cq) - 1):
        tc = int(cq[b + 1] - cq[b])
        if tc == 0:
            continue
        prefix = int(ck[b + 1] - ck[b]) - tc
        pos = prefix + np.arange(tc, dtype=np.int64)
        r = np.arange(cq[b], cq[b + 1])
        c_kv, k_r = kv_compression(h[r], W, dims, pos)
        out_cache[ck[b] + pos] = cache_rows(c_kv, k_r)
        seq = out_cache[ck[b]:ck[b + 1]]
        _, q_c, q_r = query_projections(h[r], W, dims, pos)
        o, o_lat, lse = attend_unabsorbed(q_c, q_r, seq[:, :dims.d_c], seq[:, dims.d_c:], W, dims, pos, heads)
        rows.append(r); o_l.append(o); lat_l.append(o_lat); lse_l.append(lse)
    out = {"cache": out_cache, "rows": np.concatenate(rows), "o": np.concatenate(o_l),
           "o_lat": np.concatenate(lat_l), "lse": np.concatenate(lse_l)}
    if heads is None:
        out["u"] = output_projection(out["o"], W)
    return out


# ---------------------------------------------------------------------------
# The latent-attention core by its own definition (absorbed score, section 2 【思考】 + section 3)
# ---------------------------------------------------------------------------
def absorb_query(q_c, W, dims) -> np.ndarray:
    """q~_t,i = W_i^UK^T q^C_t,i in R^{d_c} (section 2 【思考】: W^UK folded into the query)."""
    q_c = f64(q_c)
    w_uk = f64(W["w_uk"]).reshape(dims.n_h, dims.d_h, dims.d_c)
    return np.einsum("thk,hkc->thc", q_c, w_uk)


def attn_decode_latent(q_abs, q_rope, cache, cu_seqlens, tq, dims, seqs=None, heads=None):
    """Core over the latent cache: s_j = (q~.c_j + q^R.k^R_j)/sqrt(d_h + d_h^R), j <= pos,
    o^lat = sum_j p_j c_j and lse (section 3's split of the score into a position-free
    latent term and a RoPE term). q_abs [B*Tq, n_h, d_c], q_rope [B*Tq, n_h, d_r].
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = len(cu) - 1
    seqs = range(B) if seqs is None else list(seqs)
    heads = range(dims.n_h) if heads is None else list(heads)
    pos_all = decode_positions(cu, tq)
    scale = 1.0 / np.sqrt(dims.d_h + dims.d_r)
    lat_l, lse_l = [], []
    for b in seqs:
        r = np.arange(b * tq, (b + 1) * tq)
        seq = f64(cache[cu[b]:cu[b + 1]])
        lat = np.empty((tq, len(heads), dims.d_c))
        lse = np.empty((tq, len(heads)))
        for hi, i in enumerate(heads):
            q = np.concatenate([f64(np.asarray(q_abs)[r, i]), f64(np.asarray(q_rope)[r, i])], axis=1)
            lat[:, hi], _, lse[:, hi], _ = causal_softmax_attend(q, seq, seq[:, :dims.d_c], None,
                                                                   pos_all[r], scale)
        lat_l.append(lat); lse_l.append(lse)
    return np.concatenate(lat_l), np.concatenate(lse_l)


def value_up_projection(o_lat, W, dims) -> np.ndarray:
    """o_t,i = W_i^UV o^lat_t,i (section 2 【思考】: the value path moved after attention)."""
    w_uv = f64(W["w_uv"]).reshape(dims.n_h, dims.d_h, dims.d_c)
    return np.einsum("thc,hdc->thd", f64(o_lat), w_uv)


def mla_decode_absorbed(h_q, cache, cu_seqlens, tq, W, dims, seqs=None):
    """The absorbed form end to end: W^UK folded into the query, W^UV after attention.

    An exact rewrite of the unabsorbed definition (section 2 【思考】; the tests pin the two
    together to 1e-12). It costs O(d_c) instead of O(n_h d_h d_c) per cached row, which is what
    lets the full-size tests check u over 128K-row caches. Rows are those of `seqs` (default all).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    seqs = range(len(cu) - 1) if seqs is None else list(seqs)
    rows = np.concatenate([np.arange(b * tq, (b + 1) * tq) for b in seqs])
    pos = decode_positions(cu, tq)[rows]
    _, q_c, q_r = query_projections(np.asarray(h_q)[rows], W, dims, pos)
    q_abs = absorb_query(q_c, W, dims)
    # re-index the chosen sequences as a packed batch of their own
    sub_cache = np.concatenate([np.asarray(cache)[cu[b]:cu[b + 1]] for b in seqs])
    sub_cu = np.concatenate([[0], np.cumsum([cu[b + 1] - cu[b] for b in seqs])]).astype(np.int64)
    o_lat, lse = attn_decode_latent(q_abs, q_r, sub_cache, sub_cu, tq, dims)
    o = value_up_projection(o_lat, W, dims)
    return {"rows": rows, "o_lat": o_lat, "lse": lse, "o": o, "u": output_projection(o, W), "q_abs": q_abs,
            "q_r": q_r, "q_c": q_c}


def mla_prefill_absorbed(h, cu_seqlens, W, dims, query_rows, cache=None):
    """Prefill outputs of the given query rows (global token indices) in the absorbed form.

    The same exact rewrite as mla_decode_absorbed (section 2 【思考】), applied to prefill: the
    cache rows of every token come from steps (5) and (7) (or `cache`, if the caller already has
    them), each query row t at position p attends over its own sequence's rows 0..p through
    q~ = W_i^UK^T q^C_i, and o = W_i^UV o^lat, u = W^O [o_1; ...; o_n_h] follow. The tests pin it
    to mla_prefill to 1e-12; it costs O(d_c) per key instead of O(n_h d_h d_c) per cached row, so
    u of a few rows of a 32K-token prefill can be checked on the host.
    """
    h = f64(h)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T = h.shape[0]
    pos = np.concatenate([np.arange(cu[b + 1] - cu[b]) for b in range(len(cu) - 1)]).astype(np.int64)
    if cache is None:
        c_kv, k_r = kv_compression(h, W, dims, pos)
        cache = cache_rows(c_kv, k_r)
    rows = np.sort(np.asarray(query_rows, dtype=np.int64))
    _, q_c, q_r = query_projections(h[rows], W, dims, pos[rows])
    q_abs = absorb_query(q_c, W, dims)
    scale = 1.0 / np.sqrt(dims.d_h + dims.d_r)
    o_lat = np.empty((len(rows), dims.n_h, dims.d_c))
    lse = np.empty((len(rows), dims.n_h))
    for n, t in enumerate(rows):
        b = int(np.searchsorted(cu, t, side="right") - 1)
        seq = f64(cache[cu[b]:t + 1])                    # the row's own sequence, keys 0..p
        for i in range(dims.n_h):
            q = np.concatenate([q_abs[n, i], f64(q_r[n, i])])[None, :]
            lat, _, l, _ = causal_softmax_attend(q, seq, seq[:, :dims.d_c], None, np.array([t - cu[b]]), scale)
            o_lat[n, i], lse[n, i] = lat[0], l[0]
    o = value_up_projection(o_lat, W, dims)
    return {"rows": rows, "cache": cache, "o_lat": o_lat, "lse": lse, "o": o, "u": output_projection(o, W)}


def output_absorbed(o_lat, W, dims) -> np.ndarray:
    """u_t = sum_i W_i^O' o^lat_t,i with W_i^O' = W_i^O W_i^UV (section 2 【思考】, second absorption)."""
    w_o = f64(W["w_o"]).reshape(-1, dims.n_h, dims.d_h)          # [d, n_h, d_h]
    w_uv = f64(W["w_uv"]).reshape(dims.n_h, dims.d_h, dims.d_c)  # [n_h, d_h, d_c]
    w_o_prime = np.einsum("xhd,hdc->xhc", w_o, w_uv)              # [d, n_h, d_c]
    return np.einsum("thc,xhc->tx", f64(o_lat), w_o_prime)


# ---------------------------------------------------------------------------
# Split-KV combine (exact identity of the softmax; used by the tests' combine pin)
# ---------------------------------------------------------------------------
def lse_combine(parts):
    """Merge (o_s, lse_s) partial results over disjoint key sets: lse = log sum_s e^{lse_s},
    o = sum_s e^{lse_s - lse} o_s."""
    lses = np.stack([f64(l) for _, l in parts])
    top = lses.max(axis=0)
    lse = top + np.log(np.exp(lses - top).sum(axis=0))
    o = sum(np.exp(f64(l) - lse)[..., None] * f64(x) for x, l in parts)
    return o, lse


# ---------------------------------------------------------------------------
# Cache-size bookkeeping (section 1 MHA cache, section 3 decoupled-key cache)
# ---------------------------------------------------------------------------
def mha_cache_elements_per_token(dims, layers: int) -> int:
    """2 n_h d_h l elements per token for multi-head attention."""
    return 2 * dims.n_h * dims.d_h * layers


def mla_cache_elements_per_token(dims, layers: int) -> int:
    """(d_c + d_h^R) l elements per token for MLA with the decoupled RoPE key."""
    return (dims.d_c + dims.d_r) * layers


# ---------------------------------------------------------------------------
# FP8 (e4m3) latent cache (opt-in; reading R15). The notes' FP8 section scales 1 x 128 tiles for
# training GEMMs; the cache takes one fp32 scale per cached row.
# ---------------------------------------------------------------------------
E4M3_MAX = 448.0
KR_F16_RANGE = 32768.0


def e4m3_positive_values() -> np.ndarray:
    """The 127 non-negative finite e4m3 values in code order 0x00 .. 0x7E (1 sign, 4 exponent bits
    with bias 7, 3 mantissa bits; no infinities, 0x7F is NaN): code e * 8 + m is m/8 * 2^-6 for e = 0
    and (1 + m/8) * 2^(e - 7) otherwise. Codes increase with the value."""
    out = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        out.append(m / 8.0 * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(out)


def round_to_e4m3(x) -> np.ndarray:
    """x rounded to the nearest e4m3 value, ties to the even code (even mantissa), magnitudes past
    448 saturated to 448. Works on the magnitude and puts the sign back."""
    x = f64(x)
    grid = e4m3_positive_values()
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(grid, a, side="left"), 0, len(grid) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - grid[lo], grid[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    return np.sign(x) * np.where(pick_hi, grid[hi], grid[lo])


def round_to_f16(x) -> np.ndarray:
    """IEEE half precision, round to nearest even (numpy's float16 conversion)."""
    return f64(np.asarray(x, dtype=np.float64).astype(np.float16))


def quantize_cache_rows_fp8(rows, dims):
    """FP8 cache rows from bf16 cache rows [n, d_c + d_r] (reading R15).

    Per row: s = max(amax(c^KV) / 448, amax(k^R) / 32768) in fp32 (1 if the row is all zero);
    codes = e4m3(c^KV / s) and k^R' = f16(k^R / s), each division in fp32. Returns (codes [n, d_c] as
    the e4m3 values, kr_scaled [n, d_r] as the f16 values, s [n]) in float64.
    """
    rows = np.asarray(rows, dtype=np.float32)
    c, kr = rows[:, :dims.d_c], rows[:, dims.d_c:]
    amax_c = np.abs(c).max(axis=1).astype(np.float32)
    amax_r = np.abs(kr).max(axis=1).astype(np.float32)
    s = np.maximum(amax_c / np.float32(E4M3_MAX), amax_r / np.float32(KR_F16_RANGE)).astype(np.float32)
    s = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    codes = round_to_e4m3((c / s[:, None]).astype(np.float32))
    kr_scaled = round_to_f16((kr / s[:, None]).astype(np.float32))
    return codes, kr_scaled, f64(s)


def dequantize_cache_rows_fp8(codes, kr_scaled, s) -> np.ndarray:
    """The cache rows an FP8 cache stands for: [codes * s | k^R' * s], exactly in float64."""
    s = f64(s)[:, None]
    return np.concatenate([f64(codes) * s, f64(kr_scaled) * s], axis=1)
