"""Pins for the CPU oracle: facts fixed by the pages and by mathematics, not by the oracle itself.

Each test names the passage of the notes "【论文解读】DeepSeek-V3" (wkq9411.github.io) it rests on.
A plausible slip in the oracle (a dropped term, a wrong sign, a transposed operand, a wrong
scale or position) fails at least one of them; test_planted_mistakes_are_caught checks that.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from mla_latent_kv_31_b200 import synth
from oracle import mla_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _weights(dims, seed, dtype="fp32", scale=None):
    W = synth.weights(dims, seed=seed, dtype=dtype)
    if scale:
        W = {k: v * scale.get(k, 1.0) for k, v in W.items()}
    return W


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


SMALL = synth.Dims(d=32, n_h=3, d_h=8, d_c=12, d_cq=10, d_r=6)


# ---------------------------------------------------------------------------
# Absorption (section 一(一)2 【思考】): exact identities in float64
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dims,tq", [(synth.TINY, 1), (synth.TINY, 2), (SMALL, 2)])
def test_absorbed_equals_unabsorbed_decode(dims, tq):
    W = _weights(dims, seed=3)
    lens = np.array([5, 17, 2 * tq, 40])
    cu = synth.cu_seqlens(lens)
    cache = synth.latent_cache(dims, int(cu[-1]), seed=4, dtype="fp32")
    h_q = synth.hidden(dims, len(lens) * tq, seed=5, dtype="fp32")
    un = orc.mla_decode(h_q, cache, cu, tq, W, dims)
    ab = orc.mla_decode_absorbed(h_q, cache, cu, tq, W, dims)
    assert _rel(ab["o_lat"], un["o_lat"]) < 1e-12
    assert _rel(ab["lse"], un["lse"]) < 1e-12
    assert _rel(ab["o"], un["o"]) < 1e-12
    assert _rel(ab["u"], un["u"]) < 1e-12
    # second absorption: W^O' = W^O W^UV applied to the latent outputs
    assert _rel(orc.output_absorbed(un["o_lat"], W, dims), un["u"]) < 1e-12
    # a subset of sequences, re-packed on their own, gives the same rows
    sub = orc.mla_decode_absorbed(h_q, cache, cu, tq, W, dims, seqs=[1, 3])
    assert _rel(sub["u"], un["u"][sub["rows"]]) < 1e-12


def test_absorbed_core_matches_unabsorbed_prefill():
    dims = synth.TINY
    W = _weights(dims, seed=11)
    cu = synth.cu_seqlens([64])
    h = synth.hidden(dims, 64, seed=12, dtype="fp32")
    pre = orc.mla_prefill(h, cu, W, dims)
    pos = np.arange(64)
    _, q_c, q_r = orc.query_projections(h, W, dims, pos)
    q_abs = orc.absorb_query(q_c, W, dims)
    # treat the 64 tokens as 64 one-token "decode" queries over growing prefixes
    for t in [0, 1, 31, 63]:
        cu_t = np.array([0, t + 1])
        lat, lse = orc.attn_decode_latent(q_abs[t:t + 1], q_r[t:t + 1], pre["cache"][:t + 1], cu_t, 1, dims)
        assert _rel(lat[0], pre["o_lat"][t]) < 1e-12
        assert _rel(lse[0], pre["lse"][t]) < 1e-12


@pytest.mark.parametrize("dims", [synth.TINY, SMALL])
def test_prefill_absorbed_equals_unabsorbed(dims):
    W = _weights(dims, seed=13)
    lens = [23, 1, 40]
    cu = synth.cu_seqlens(lens)
    h = synth.hidden(dims, int(cu[-1]), seed=14, dtype="fp32")
    rows = [0, 5, 22, 23, 24, 40, 63]
    un = orc.mla_prefill(h, cu, W, dims, query_rows=rows)
    ab = orc.mla_prefill_absorbed(h, cu, W, dims, rows)
    assert np.array_equal(ab["rows"], un["rows"])
    for key in ("o_lat", "lse", "o", "u"):
        assert _rel(ab[key], un[key]) < 1e-12, key
    assert _rel(ab["cache"], un["cache"]) < 1e-15
    # handing it the cache rows gives the same result
    ab2 = orc.mla_prefill_absorbed(h, cu, W, dims, rows, cache=un["cache"])
    assert _rel(ab2["u"], un["u"]) < 1e-12


# ---------------------------------------------------------------------------
# Softmax / single key / causality (section 一(一)1: Softmax_j over j = 1..t)
# ---------------------------------------------------------------------------
def test_lse_of_a_single_key_is_its_score():
    # one visible key: the log of a one-term sum is that term's scaled score, written out here
    # as q.k / sqrt(d_h + d_h^R) over the concatenated [q^C; q^R] and [k^C; k^R]
    dims = synth.TINY
    W = _weights(dims, seed=24)
    h = synth.hidden(dims, 1, seed=25, dtype="fp32")
    out = orc.mla_prefill(h, synth.cu_seqlens([1]), W, dims)
    h64 = np.asarray(h[0], np.float64)
    c_q = np.asarray(W["w_dq"], np.float64) @ h64
    c_kv = np.asarray(W["w_dkv"], np.float64) @ h64
    q_r = np.asarray(W["w_qr"], np.float64) @ c_q       # position 0: RoPE is the identity
    k_r = np.asarray(W["w_kr"], np.float64) @ h64
    for i in range(dims.n_h):
        rows = slice(i * dims.d_h, (i + 1) * dims.d_h)
        q_c = np.asarray(W["w_uq"], np.float64)[rows] @ c_q
        k_c = np.asarray(W["w_uk"], np.float64)[rows] @ c_kv
        s = (q_c @ k_c + q_r[i * dims.d_r:(i + 1) * dims.d_r] @ k_r) / math.sqrt(dims.d_h + dims.d_r)
        assert abs(out["lse"][0, i] - s) <= 1e-12 * max(1.0, abs(s))


def test_lse_equals_torch_logsumexp_of_the_scores():
    # lse against torch.logsumexp over the causal scores formed explicitly in torch (float64)
    dims = synth.TINY
    W = _weights(dims, seed=26)
    T = 20
    h = synth.hidden(dims, T, seed=27, dtype="fp32")
    ref = orc.mla_prefill(h, synth.cu_seqlens([T]), W, dims)
    h64 = torch.tensor(np.asarray(h, np.float64))
    Wt = {k: torch.tensor(np.asarray(v, np.float64)) for k, v in W.items()}
    c_q = h64 @ Wt["w_dq"].T
    c_kv = h64 @ Wt["w_dkv"].T
    q_c = (c_q @ Wt["w_uq"].T).reshape(T, dims.n_h, dims.d_h)
    k_c = (c_kv @ Wt["w_uk"].T).reshape(T, dims.n_h, dims.d_h)
    pos = np.arange(T)
    q_r = torch.tensor(orc.rope((c_q @ Wt["w_qr"].T).reshape(T, dims.n_h, dims.d_r).numpy(), pos[:, None],
                                dims.rope_base))
    k_r = torch.tensor(orc.rope((h64 @ Wt["w_kr"].T).numpy(), pos, dims.rope_base))
    s = (torch.einsum("thd,jhd->htj", q_c, k_c) + torch.einsum("thd,jd->htj", q_r, k_r)) / math.sqrt(
        dims.d_h + dims.d_r)
    s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
    lse = torch.logsumexp(s, dim=-1).transpose(0, 1).numpy()
    assert _rel(ref["lse"], lse) < 1e-13



def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((3, 10))
    k = rng.standard_normal((9, 10))
    v = rng.standard_normal((9, 4))
    _, _, _, p = orc.causal_softmax_attend(q, k, v, None, np.array([0, 4, 8]), 0.3)
    assert np.allclose(p.sum(axis=1), 1.0, atol=1e-14, rtol=0)
    assert np.all(p[0, 1:] == 0) and np.all(p[1, 5:] == 0)


def test_single_key_returns_its_value_exactly():
    dims = synth.TINY
    W = _weights(dims, seed=21)
    cache = synth.latent_cache(dims, 1, seed=22, dtype="fp32")
    h_q = synth.hidden(dims, 1, seed=23, dtype="fp32")
    out = orc.mla_decode(h_q, cache, np.array([0, 1]), 1, W, dims)
    c = cache[0, :dims.d_c].astype(np.float64)
    o_expect = (W["w_uv"].astype(np.float64) @ c).reshape(dims.n_h, dims.d_h)
    assert np.array_equal(out["o_lat"][0], np.broadcast_to(c, (dims.n_h, dims.d_c)))
    assert _rel(out["o"][0], o_expect) < 1e-15
    u_expect = W["w_o"].astype(np.float64) @ o_expect.reshape(-1)
    assert _rel(out["u"][0], u_expect) < 1e-14


def test_causality_rows_after_position_do_not_matter():
    dims = synth.TINY
    W = _weights(dims, seed=31)
    cu = synth.cu_seqlens([40])
    h = synth.hidden(dims, 40, seed=32, dtype="fp32")
    base = orc.mla_prefill(h, cu, W, dims, query_rows=[10, 20])
    h2 = h.copy()
    h2[21:] = synth.hidden(dims, 19, seed=33, dtype="fp32")
    pert = orc.mla_prefill(h2, cu, W, dims, query_rows=[10, 20])
    assert np.array_equal(base["u"], pert["u"])
    assert np.array_equal(base["o_lat"], pert["o_lat"])
    # decode: rows after the query positions of the 2-token window
    cache = synth.latent_cache(dims, 30, seed=34, dtype="fp32")
    h_q = synth.hidden(dims, 2, seed=35, dtype="fp32")
    a = orc.mla_decode(h_q, cache, np.array([0, 30]), 2, W, dims)
    cache2 = cache.copy()
    cache2[29] = 100.0        # visible to query 1 only
    b = orc.mla_decode(h_q, cache2, np.array([0, 30]), 2, W, dims)
    assert np.array_equal(a["u"][0], b["u"][0])
    assert not np.array_equal(a["u"][1], b["u"][1])


# ---------------------------------------------------------------------------
# RoPE (section 一(一)3: block-diagonal 2x2 rotations, score depends on m - n)
# ---------------------------------------------------------------------------
def test_rope_closed_form_two_dims():
    # d_R = 2: theta_0 = 1, so R_p e_0 = (cos p, sin p) and R_p e_1 = (-sin p, cos p).
    for p in [0, 1, 3, 7]:
        assert np.allclose(orc.rope(np.array([1.0, 0.0]), p, 10000.0), [math.cos(p), math.sin(p)], atol=1e-15)
        assert np.allclose(orc.rope(np.array([0.0, 1.0]), p, 10000.0), [-math.sin(p), math.cos(p)], atol=1e-15)


def test_rope_frequencies():
    # d_R = 4, base 10000: theta_1 = 10000^(-2/4) = 0.01; pair 1 is elements (2, 3).
    x = np.array([0.0, 0.0, 1.0, 0.0])
    y = orc.rope(x, 50, 10000.0)
    assert np.allclose(y, [0.0, 0.0, math.cos(0.5), math.sin(0.5)], atol=1e-15)


def test_rope_norm_identity_and_relative_position():
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(16), rng.standard_normal(16)
    assert np.array_equal(orc.rope(q, 0, 10000.0), q)
    assert abs(np.linalg.norm(orc.rope(q, 123, 10000.0)) - np.linalg.norm(q)) < 1e-12
    s1 = orc.rope(q, 40, 10000.0) @ orc.rope(k, 13, 10000.0)
    s2 = orc.rope(q, 1040, 10000.0) @ orc.rope(k, 1013, 10000.0)
    assert abs(s1 - s2) < 1e-10
    assert abs(s1 - orc.rope(q, 27, 10000.0) @ k) < 1e-10


def test_shifting_all_positions_leaves_attention_unchanged():
    # Only k^R and q^R carry position, and only through m - n (section 一(一)3).
    dims = synth.TINY
    W = _weights(dims, seed=41)
    h = synth.hidden(dims, 12, seed=42, dtype="fp32")
    pos = np.arange(12)
    outs = []
    for shift in [0, 777]:
        _, q_c, q_r = orc.query_projections(h, W, dims, pos + shift)
        c_kv, k_r = orc.kv_compression(h, W, dims, pos + shift)
        o, lat, lse = orc.attend_unabsorbed(q_c, q_r, c_kv, k_r, W, dims, pos)
        outs.append((o, lat, lse))
    for a, b in zip(*outs):
        assert _rel(a, b) < 1e-11


# ---------------------------------------------------------------------------
# Textbook reductions (torch's scaled_dot_product_attention, float64 on CPU)
# ---------------------------------------------------------------------------
def _sdpa_prefill(h, W, dims, zero_rope=False):
    h64 = torch.tensor(np.asarray(h, np.float64))
    Wt = {k: torch.tensor(np.asarray(v, np.float64)) for k, v in W.items()}
    T = h64.shape[0]
    c_q = h64 @ Wt["w_dq"].T
    q_c = (c_q @ Wt["w_uq"].T).reshape(T, dims.n_h, dims.d_h)
    c_kv = h64 @ Wt["w_dkv"].T
    k_c = (c_kv @ Wt["w_uk"].T).reshape(T, dims.n_h, dims.d_h)
    v_c = (c_kv @ Wt["w_uv"].T).reshape(T, dims.n_h, dims.d_h)
    pos = np.arange(T)
    q_r = torch.tensor(orc.rope((c_q @ Wt["w_qr"].T).reshape(T, dims.n_h, dims.d_r).numpy(), pos[:, None],
                                dims.rope_base))
    k_r = torch.tensor(orc.rope((h64 @ Wt["w_kr"].T).numpy(), pos, dims.rope_base))
    if zero_rope:
        Q, K = q_c, k_c
    else:
        Q = torch.cat([q_c, q_r], dim=-1)
        K = torch.cat([k_c, k_r[:, None, :].expand(T, dims.n_h, dims.d_r)], dim=-1)
    o = torch.nn.functional.scaled_dot_product_attention(
        Q.transpose(0, 1), K.transpose(0, 1), v_c.transpose(0, 1), is_causal=True,
        scale=1.0 / math.sqrt(dims.d_h + dims.d_r)).transpose(0, 1)
    u = o.reshape(T, -1) @ Wt["w_o"].T
    return o.numpy(), u.numpy()


def test_oracle_equals_sdpa_on_tiny_prefill():
    dims = synth.TINY
    W = _weights(dims, seed=0)
    h = synth.hidden(dims, 64, seed=0, dtype="fp32")
    ref = orc.mla_prefill(h, synth.cu_seqlens([64]), W, dims)
    o, u = _sdpa_prefill(h, W, dims)
    assert _rel(ref["o"], o) < 1e-12
    assert _rel(ref["u"], u) < 1e-12


def test_zero_rope_weights_reduce_to_plain_mha():
    # With W^QR = W^KR = 0 the RoPE halves vanish and MLA is MHA on q^C, k^C, v^C
    # (section 一(一)1 with d_h-wide keys) at scale 1/sqrt(d_h + d_h^R).
    dims = synth.TINY
    W = _weights(dims, seed=5)
    W["w_qr"] = np.zeros_like(W["w_qr"])
    W["w_kr"] = np.zeros_like(W["w_kr"])
    h = synth.hidden(dims, 33, seed=6, dtype="fp32")
    ref = orc.mla_prefill(h, synth.cu_seqlens([33]), W, dims)
    o, u = _sdpa_prefill(h, W, dims, zero_rope=True)
    assert _rel(ref["o"], o) < 1e-12
    assert _rel(ref["u"], u) < 1e-12


# ---------------------------------------------------------------------------
# Brute force: an independent pure-Python implementation on tiny shapes
# ---------------------------------------------------------------------------
def _bf_matvec(W, x):
    return [sum(W[r][c] * x[c] for c in range(len(x))) for r in range(len(W))]


def _bf_rope(x, pos, base):
    out = list(x)
    n = len(x)
    for m in range(n // 2):
        ang = pos * base ** (-2.0 * m / n)
        a, b = x[2 * m], x[2 * m + 1]
        out[2 * m] = a * math.cos(ang) - b * math.sin(ang)
        out[2 * m + 1] = a * math.sin(ang) + b * math.cos(ang)
    return out


def _bf_prefill(h, W, dm):
    Wl = {k: np.asarray(v, np.float64).tolist() for k, v in W.items()}
    T = len(h)
    hs = np.asarray(h, np.float64).tolist()
    q, k, v = [], [], []
    for t in range(T):
        cq = _bf_matvec(Wl["w_dq"], hs[t])
        qc = _bf_matvec(Wl["w_uq"], cq)
        qr = _bf_matvec(Wl["w_qr"], cq)
        ckv = _bf_matvec(Wl["w_dkv"], hs[t])
        kc = _bf_matvec(Wl["w_uk"], ckv)
        vc = _bf_matvec(Wl["w_uv"], ckv)
        kr = _bf_rope(_bf_matvec(Wl["w_kr"], hs[t]), t, dm.rope_base)
        q.append([qc[i * dm.d_h:(i + 1) * dm.d_h] + _bf_rope(qr[i * dm.d_r:(i + 1) * dm.d_r], t, dm.rope_base)
                  for i in range(dm.n_h)])
        k.append([kc[i * dm.d_h:(i + 1) * dm.d_h] + kr for i in range(dm.n_h)])
        v.append([vc[i * dm.d_h:(i + 1) * dm.d_h] for i in range(dm.n_h)])
    u = []
    for t in range(T):
        o_cat = []
        for i in range(dm.n_h):
            s = [sum(a * b for a, b in zip(q[t][i], k[j][i])) / math.sqrt(dm.d_h + dm.d_r) for j in range(t + 1)]
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            z = sum(e)
            o_cat += [sum(e[j] / z * v[j][i][c] for j in range(t + 1)) for c in range(dm.d_h)]
        u.append(_bf_matvec(Wl["w_o"], o_cat))
    return np.array(u)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_tiny_random(seed):
    rng = np.random.default_rng(seed)
    dm = synth.Dims(d=int(rng.integers(3, 8)), n_h=int(rng.integers(1, 3)), d_h=int(rng.integers(2, 5)),
                    d_c=int(rng.integers(2, 8)), d_cq=int(rng.integers(2, 6)), d_r=2 * int(rng.integers(1, 3)))
    L = int(rng.integers(1, 9))
    W = _weights(dm, seed=100 + seed)
    h = synth.hidden(dm, L, seed=200 + seed, dtype="fp32")
    ref = orc.mla_prefill(h, synth.cu_seqlens([L]), W, dm)
    assert _rel(ref["u"], _bf_prefill(h, W, dm)) < 1e-12


# ---------------------------------------------------------------------------
# Decode is the prefill's last step (KV-cache principle; reading R5)
# ---------------------------------------------------------------------------
def test_decode_over_prefill_cache_matches_prefill():
    dims = synth.TINY
    W = _weights(dims, seed=51)
    lens = [9, 30]
    cu = synth.cu_seqlens(lens)
    h = synth.hidden(dims, int(cu[-1]), seed=52, dtype="fp32")
    pre = orc.mla_prefill(h, cu, W, dims)
    for tq in (1, 2):
        rows = np.concatenate([np.arange(cu[b + 1] - tq, cu[b + 1]) for b in range(2)])
        dec = orc.mla_decode(h[rows], pre["cache"], cu, tq, W, dims)
        assert _rel(dec["u"], pre["u"][rows]) < 1e-12
        assert _rel(dec["o_lat"], pre["o_lat"][rows]) < 1e-12
    # cache_append at the sequence positions reproduces the prefill's rows
    pos = np.concatenate([np.arange(n) for n in lens])
    assert _rel(orc.cache_append(h, pos, W, dims), pre["cache"]) < 1e-15


def test_chunked_prefill_equals_prefill_of_the_whole_sequence():
    # prefill of [prefix; chunk] == prefill of the prefix, then the chunk against the cached prefix;
    # two sequences with different prefix and chunk lengths, then a second chunk on top
    dims = synth.TINY
    W = _weights(dims, seed=61)
    lens = [30, 19]
    cu = synth.cu_seqlens(lens)
    h = synth.hidden(dims, int(cu[-1]), seed=62, dtype="fp32")
    full = orc.mla_prefill(h, cu, W, dims)
    splits = [(12, 10), (5, 9)]           # per sequence: (prefix, first chunk); the rest is a second chunk
    cache = np.zeros_like(full["cache"])
    pre_rows = np.concatenate([np.arange(cu[b], cu[b] + splits[b][0]) for b in range(2)])
    cache[pre_rows] = full["cache"][pre_rows]
    step_cache = cache
    done = [s[0] for s in splits]
    for part in (0, 1):
        take = [splits[b][1] if part == 0 else lens[b] - splits[b][0] - splits[b][1] for b in range(2)]
        q_rows = np.concatenate([np.arange(cu[b] + done[b], cu[b] + done[b] + take[b]) for b in range(2)])
        kv_lens = [done[b] + take[b] for b in range(2)]
        # the cache of this call holds each sequence's first kv_lens[b] rows, packed
        idx = np.concatenate([np.arange(cu[b], cu[b] + kv_lens[b]) for b in range(2)])
        out = orc.mla_prefill_chunk(h[q_rows], synth.cu_seqlens(take), step_cache[idx], synth.cu_seqlens(kv_lens), W,
                                    dims)
        assert _rel(out["u"], full["u"][q_rows]) < 1e-12
        assert _rel(out["o_lat"], full["o_lat"][q_rows]) < 1e-12
        assert _rel(out["cache"], full["cache"][idx]) < 1e-15
        step_cache = step_cache.copy()
        step_cache[idx] = out["cache"]
        done = kv_lens
    assert done == lens


# ---------------------------------------------------------------------------
# YaRN on the decoupled RoPE (section 三(二)3 "长上下文扩展": s = 40, alpha = 1, beta = 32,
# sqrt(t) = 0.1 ln s + 1, for the decoupled key only) and the RMSNorm after the latent
# compression (section 三(二)1 "模型超参数"); both opt-in
# ---------------------------------------------------------------------------
def test_yarn_with_s_one_is_plain_rope():
    import dataclasses
    d1 = dataclasses.replace(synth.V3_YARN, yarn_s=1.0)
    x = np.random.default_rng(0).standard_normal((5, 64))
    pos = np.array([0, 1, 77, 4095, 131071])[:, None]
    assert np.array_equal(orc.rope_dims(x, pos, d1), orc.rope(x, pos, 10000.0))
    theta = 10000.0 ** (-2.0 * np.arange(32) / 64)
    assert _rel(orc.yarn_frequencies(64, 10000.0, 1.0, 1.0, 32.0, 4096), theta) < 1e-15
    assert orc.rope_scale(d1) == 1.0


def test_yarn_frequencies_by_parts_closed_form():
    # d_r = 4, base 100: theta = [1, 0.1]; L0 chosen so that pair 1 turns 16.5 times over it, the
    # middle of the ramp [1, 32]: gamma = 1/2 and theta' = (0.1 / 40 + 0.1) / 2 = 0.05125; pair 0 turns
    # 165 times (> beta) and keeps theta = 1
    l0 = 16.5 * 2.0 * math.pi / 0.1
    th = orc.yarn_frequencies(4, 100.0, 40.0, 1.0, 32.0, l0)
    assert abs(th[0] - 1.0) < 1e-15
    assert abs(th[1] - 0.05125) < 1e-15
    # the DeepSeek-V3 table: the fastest pair (lambda = 2 pi, 652 turns over 4K) unchanged, the slowest
    # (lambda ~ 4.7e4 > 4K: under one turn) divided by s exactly, and every pair in between blended
    th = orc.yarn_frequencies(64, 10000.0, 40.0, 1.0, 32.0, 4096)
    theta = 10000.0 ** (-2.0 * np.arange(32) / 64)
    turns = 4096 * theta / (2 * math.pi)
    assert th[0] == theta[0]
    assert np.all(th[turns > 32] == theta[turns > 32])
    assert np.allclose(th[turns < 1], theta[turns < 1] / 40, rtol=1e-15, atol=0)
    mid = (turns >= 1) & (turns <= 32)
    assert mid.sum() >= 3
    assert np.all((th[mid] <= theta[mid]) & (th[mid] >= theta[mid] / 40))
    # blending is linear in the number of turns
    g = (turns[mid] - 1) / 31
    assert _rel(th[mid], (1 - g) * theta[mid] / 40 + g * theta[mid]) < 1e-15


def test_yarn_scale_and_relative_position():
    dims = synth.V3_YARN
    m = orc.rope_scale(dims)
    assert abs(m - (0.1 * math.log(40.0) + 1.0)) < 1e-15 and abs(m - 1.3688879454113936) < 1e-12
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    # every rotated pair keeps its length times the factor
    rq = orc.rope_dims(q, np.array(1000), dims)
    assert _rel(np.hypot(rq[0::2], rq[1::2]), m * np.hypot(q[0::2], q[1::2])) < 1e-13
    # the RoPE score depends on the relative position only, and carries the factor squared
    s1 = orc.rope_dims(q, np.array(70000), dims) @ orc.rope_dims(k, np.array(50000), dims)
    s2 = orc.rope_dims(q, np.array(20123), dims) @ orc.rope_dims(k, np.array(123), dims)
    assert abs(s1 - s2) < 1e-9 * abs(s1)
    theta = orc.yarn_frequencies(64, 10000.0, 40.0, 1.0, 32.0, 4096)
    ref = m * m * (orc.rotate(q, 20000.0 * theta) @ k)
    assert abs(s1 - ref) < 1e-9 * abs(ref)


def test_rms_norm_closed_forms():
    # [3, 4]: mean square 12.5
    assert _rel(orc.rms_norm([3.0, 4.0], [1.0, 1.0], 0.0), [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)]) < 1e-15
    # a constant row normalises to the gains; eps enters under the root
    g = np.array([0.5, 2.0, -1.0])
    assert _rel(orc.rms_norm([7.0, 7.0, 7.0], g, 0.0), g) < 1e-15
    assert _rel(orc.rms_norm([2.0, 2.0, 2.0], g, 5.0), g * 2 / 3) < 1e-15
    x = np.random.default_rng(2).standard_normal((4, 96))
    assert _rel(orc.rms_norm(3.5 * x, np.ones(96), 0.0), orc.rms_norm(x, np.ones(96), 0.0)) < 1e-14
    y = orc.rms_norm(x, np.ones(96), 0.0)
    assert _rel(np.mean(y * y, axis=1), np.ones(4)) < 1e-14


def test_rmsnorm_sits_on_the_latent_vectors_only():
    # with the norm's gains and eps = 0, scaling h leaves c^Q, q^C, q^R and c^KV unchanged, while k^R
    # (RoPE(W^KR h), not normalised) scales with h; without gains everything scales
    import dataclasses
    dims = dataclasses.replace(synth.TINY, rms_eps=0.0)
    W = _weights(dims, seed=70)
    Wn = dict(W, **synth.gains(dims, seed=71, dtype="fp32"))
    h = synth.hidden(dims, 6, seed=72, dtype="fp32").astype(np.float64)
    pos = np.arange(6) * 11
    a, b = orc.query_projections(h, Wn, dims, pos), orc.query_projections(3.0 * h, Wn, dims, pos)
    for x, y in zip(a, b):
        assert _rel(y, x) < 1e-13
    (c1, k1), (c2, k2) = orc.kv_compression(h, Wn, dims, pos), orc.kv_compression(3.0 * h, Wn, dims, pos)
    assert _rel(c2, c1) < 1e-13
    assert _rel(k2, 3.0 * k1) < 1e-13
    # the gains act per latent column: c^KV / g_kv has mean square 1 in every row
    r = c1 / Wn["g_kv"]
    assert _rel(np.mean(r * r, axis=1), np.ones(6)) < 1e-13
    cq = a[0] / Wn["g_q"]
    assert _rel(np.mean(cq * cq, axis=1), np.ones(6)) < 1e-13
    # no gains: the projections are linear in h
    p1, p2 = orc.query_projections(h, W, dims, pos), orc.query_projections(3.0 * h, W, dims, pos)
    assert _rel(p2[0], 3.0 * p1[0]) < 1e-13


@pytest.mark.parametrize("tq", [1, 2])
def test_absorbed_equals_unabsorbed_with_rmsnorm_and_yarn(tq):
    dims = synth.TINY_YARN
    W = dict(_weights(dims, seed=73), **synth.gains(dims, seed=74, dtype="fp32"))
    lens = np.array([5, 70, 2 * tq, 40])
    cu = synth.cu_seqlens(lens)
    cache = synth.latent_cache(dims, int(cu[-1]), seed=75, dtype="fp32")
    h_q = synth.hidden(dims, len(lens) * tq, seed=76, dtype="fp32")
    un = orc.mla_decode(h_q, cache, cu, tq, W, dims)
    ab = orc.mla_decode_absorbed(h_q, cache, cu, tq, W, dims)
    assert _rel(ab["u"], un["u"]) < 1e-12
    # decode over a prefill-built cache equals the prefill, with both options on
    h = synth.hidden(dims, 90, seed=77, dtype="fp32")
    pre = orc.mla_prefill(h, synth.cu_seqlens([90]), W, dims)
    dec = orc.mla_decode(h[90 - tq:], pre["cache"], synth.cu_seqlens([90]), tq, W, dims)
    assert _rel(dec["u"], pre["u"][90 - tq:]) < 1e-12


# ---------------------------------------------------------------------------
# FP8 (e4m3) latent cache (reading R15; the notes' FP8 section, 二（三）, scales values into the
# e4m3 range with fp32 scales)
# ---------------------------------------------------------------------------
def test_e4m3_grid_matches_the_format_and_torch():
    g = orc.e4m3_positive_values()
    assert len(g) == 127 and np.all(np.diff(g) > 0)
    assert g[0x01] == 2.0 ** -9 and g[0x07] == 7 * 2.0 ** -9 and g[0x08] == 2.0 ** -6 and g[0x7E] == 448.0
    assert g[0x38] == 1.0 and g[0x39] == 1.125
    ref = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(g, ref)


def test_round_to_e4m3_is_round_to_nearest_even_and_saturates():
    g = orc.e4m3_positive_values()
    mids = (g[1:] + g[:-1]) / 2
    x = np.concatenate([mids, -mids, g, np.random.default_rng(5).uniform(-448, 448, 20000),
                        np.random.default_rng(6).standard_normal(20000) * 0.01])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(orc.round_to_e4m3(x.astype(np.float32)), ref)
    # ties go to the even code: 1 + 1/16 -> 1 (code 0x38), 1 + 3/16 -> 1.25 (0x3A)
    assert orc.round_to_e4m3([1.0625, 1.1875]).tolist() == [1.0, 1.25]
    # beyond the range: 448 (torch gives NaN past 464; the format's saturating conversion gives 448)
    assert orc.round_to_e4m3([500.0, -1e6, 464.0]).tolist() == [448.0, -448.0, 448.0]


def test_fp8_cache_rows_scale_codes_and_error_bounds():
    dims = synth.V3
    rng = np.random.default_rng(7)
    rows = synth.latent_cache(dims, 64, seed=8, dtype="bf16").astype(np.float64)
    rows[0] = 0.0                                   # an all-zero row: scale 1, codes 0
    rows[1, :dims.d_c] *= 1e-3                      # k^R sets the scale
    rows[2, dims.d_c:] *= 1e4                       # |k^R| / s would pass f16's range without the second term
    rows = rows.astype(np.float32)
    codes, krs, s = orc.quantize_cache_rows_fp8(rows, dims)
    c, kr = rows[:, :dims.d_c].astype(np.float64), rows[:, dims.d_c:].astype(np.float64)
    assert s[0] == 1.0 and np.all(codes[0] == 0) and np.all(krs[0] == 0)
    amax_c, amax_r = np.abs(c).max(1), np.abs(kr).max(1)
    expect = np.maximum(np.float32(amax_c) / np.float32(448), np.float32(amax_r) / np.float32(32768))
    assert np.array_equal(s[1:], expect[1:].astype(np.float64))
    assert np.all(np.abs(codes) <= 448) and np.all(np.abs(krs) <= 32768 * (1 + 2 ** -10))
    assert np.all(np.isin(np.abs(codes), orc.e4m3_positive_values()))
    deq = orc.dequantize_cache_rows_fp8(codes, krs, s)
    # e4m3: half an ulp, relative 2^-4 for normals, 2^-10 s absolute in the subnormal range
    err_c = np.abs(deq[:, :dims.d_c] - c)
    assert np.all(err_c <= np.maximum(2.0 ** -4 * np.abs(c), 2.0 ** -10 * s[:, None]) * (1 + 1e-6))
    # f16: relative 2^-11 for normals (|k^R| / s >= 2^-14), plus the fp32 division's own rounding
    err_r = np.abs(deq[:, dims.d_c:] - kr)
    assert np.all(err_r <= np.maximum(2.0 ** -11 * np.abs(kr), 2.0 ** -25 * s[:, None]) * (1 + 1e-6) + 1e-300)
    # the row whose k^R sets the scale keeps k^R exactly to f16 precision with codes far below 448
    assert np.abs(codes[1]).max() < 448 and np.abs(krs[1]).max() == 32768


# ---------------------------------------------------------------------------
# Split-KV combine: exact identity of the softmax over disjoint key sets
# ---------------------------------------------------------------------------
def test_lse_combine_of_any_split_equals_unsplit():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 20)) * 2
    k = rng.standard_normal((50, 20))
    v = rng.standard_normal((50, 6))
    full_o, _, full_lse, _ = orc.causal_softmax_attend(q, k, v, None, np.array([49]), 0.5)
    for cuts in ([0, 50], [0, 1, 50], [0, 13, 14, 37, 50], [0, 10, 20, 30, 40, 50]):
        parts = []
        for a, b in zip(cuts[:-1], cuts[1:]):
            o, _, lse, _ = orc.causal_softmax_attend(q, k[a:b], v[a:b], None, np.array([b - a - 1]), 0.5)
            parts.append((o, lse))
        o, lse = orc.lse_combine(parts)
        assert _rel(o, full_o) < 1e-13
        assert abs(lse[0] - full_lse[0]) < 1e-13


# ---------------------------------------------------------------------------
# Cache size (section 一(一)1 and 一(一)3 at the hyper-parameters of 三(二)1)
# ---------------------------------------------------------------------------
def test_cache_size_matches_pages():
    g = json.load(open(os.path.join(GOLDEN, "v3_cache_size.json")))
    dims = synth.V3
    assert (dims.d, dims.n_h, dims.d_h, dims.d_c, dims.d_cq, dims.d_r) == (g["d"], g["n_h"], g["d_h"], g["d_c"],
                                                                            g["d_cq"], g["d_r"])
    assert orc.mha_cache_elements_per_token(dims, 1) == g["mha_elements_per_token_per_layer"]
    assert orc.mla_cache_elements_per_token(dims, 1) == g["mla_elements_per_token_per_layer"]
    assert orc.mha_cache_elements_per_token(dims, g["layers"]) == g["mha_elements_per_token_all_layers"]
    assert orc.mla_cache_elements_per_token(dims, g["layers"]) == g["mla_elements_per_token_all_layers"]
    rows = orc.cache_rows(np.zeros((3, dims.d_c)), np.zeros((3, dims.d_r)))
    assert rows.shape[1] * 2 == g["mla_row_bytes_bf16"]


# ---------------------------------------------------------------------------
# Planted mistakes: each plausible slip in the oracle must trip a pin above
# ---------------------------------------------------------------------------
def _sign_flipped_rope(x, pos, base):
    x = np.asarray(x, np.float64)
    ang = orc.rope_angles(pos, x.shape[-1], base)
    c, s = np.cos(ang), np.sin(ang)
    a = x[..., 0::2] * c + x[..., 1::2] * s
    b = -x[..., 0::2] * s + x[..., 1::2] * c
    return np.stack([a, b], axis=-1).reshape(a.shape[:-1] + (2 * a.shape[-1],))


def _half_split_rope(x, pos, base):
    x = np.asarray(x, np.float64)
    n = x.shape[-1] // 2
    ang = orc.rope_angles(pos, x.shape[-1], base)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., :n], x[..., n:]
    return np.concatenate([x0 * c - x1 * s, x0 * s + x1 * c], axis=-1)


def _up_project_transposed_heads(c_kv, W, dims, i):
    w = np.asarray(W["w_uk"], np.float64).reshape(dims.d_h, dims.n_h, dims.d_c)[:, i]
    return np.asarray(c_kv, np.float64) @ w.T, np.asarray(c_kv, np.float64) @ np.asarray(
        W["w_uv"], np.float64)[i * dims.d_h:(i + 1) * dims.d_h].T


def _attend_wrong_scale(q, k, v, lat, qpos, scale):
    return _ORIG_ATTEND(q, k, v, lat, qpos, scale * math.sqrt(192.0 / 128.0))


def _attend_off_by_one(q, k, v, lat, qpos, scale):
    return _ORIG_ATTEND(q, k, v, lat, np.asarray(qpos) - 1 + (np.asarray(qpos) == 0), scale)


_ORIG_ATTEND = orc.causal_softmax_attend
_ORIG_YARN = orc.yarn_frequencies


def _yarn_ramp_inverted(d_r, base, s, alpha, beta, l0):
    m = np.arange(d_r // 2, dtype=np.float64)
    theta = base ** (-2.0 * m / d_r)
    gamma = np.clip((2.0 * np.pi / (l0 * theta) - alpha) / (beta - alpha), 0.0, 1.0)   # wavelength ratio upside down
    return (1.0 - gamma) * theta / s + gamma * theta


def _yarn_scale_once(dims):
    return math.sqrt(0.1 * math.log(dims.yarn_s) + 1.0) if dims.yarn_s > 1.0 else 1.0


def _round_e4m3_ties_away(x):
    x = np.asarray(x, np.float64)
    grid = orc.e4m3_positive_values()
    a = np.minimum(np.abs(x), 448.0)
    hi = np.clip(np.searchsorted(grid, a, side="left"), 0, len(grid) - 1)
    lo = np.maximum(hi - 1, 0)
    return np.sign(x) * np.where(grid[hi] - a <= a - grid[lo], grid[hi], grid[lo])


def _rms_norm_sum(x, g, eps):
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps) * np.asarray(g, np.float64)

PINS = [test_rope_closed_form_two_dims, test_rope_frequencies, lambda: test_oracle_equals_sdpa_on_tiny_prefill(),
        lambda: test_brute_force_tiny_random(0), lambda: test_brute_force_tiny_random(1),
        lambda: test_zero_rope_weights_reduce_to_plain_mha(), test_causality_rows_after_position_do_not_matter,
        test_yarn_frequencies_by_parts_closed_form, test_yarn_scale_and_relative_position, test_rms_norm_closed_forms,
        test_rmsnorm_sits_on_the_latent_vectors_only, test_round_to_e4m3_is_round_to_nearest_even_and_saturates]


@pytest.mark.parametrize("name,attr,fake", [
    ("rope sign", "rope", _sign_flipped_rope),
    ("rope half-split pairing", "rope", _half_split_rope),
    ("W^UK head split transposed", "up_project_head", _up_project_transposed_heads),
    ("scale 1/sqrt(d_h)", "causal_softmax_attend", _attend_wrong_scale),
    ("causal window off by one", "causal_softmax_attend", _attend_off_by_one),
    ("YaRN ramp on the wavelength ratio", "yarn_frequencies", _yarn_ramp_inverted),
    ("YaRN factor on the score, not on each vector", "rope_scale", _yarn_scale_once),
    ("RMSNorm over the sum of squares", "rms_norm", _rms_norm_sum),
    ("e4m3 ties away from zero", "round_to_e4m3", _round_e4m3_ties_away),
])
def test_planted_mistakes_are_caught(monkeypatch, name, attr, fake):
    monkeypatch.setattr(orc, attr, fake)
    failures = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failures += 1
    assert failures > 0, f"planted mistake '{name}' passed every pin"
