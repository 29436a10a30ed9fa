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

PINS = [test_rope_closed_form_two_dims, test_rope_frequencies, lambda: test_oracle_equals_sdpa_on_tiny_prefill(),
        lambda: test_brute_force_tiny_random(0), lambda: test_brute_force_tiny_random(1),
        lambda: test_zero_rope_weights_reduce_to_plain_mha(), test_causality_rows_after_position_do_not_matter]


@pytest.mark.parametrize("name,attr,fake", [
    ("rope sign", "rope", _sign_flipped_rope),
    ("rope half-split pairing", "rope", _half_split_rope),
    ("W^UK head split transposed", "up_project_head", _up_project_transposed_heads),
    ("scale 1/sqrt(d_h)", "causal_softmax_attend", _attend_wrong_scale),
    ("causal window off by one", "causal_softmax_attend", _attend_off_by_one),
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
