"""GPU parity on small cases that span several key tiles and ragged tails: every call of the
C ABI against the float64 oracle on the same seeded inputs (max-normalised error, see
mla_testlib.rel; bound 1e-2 for bf16 inputs with fp32 accumulation, 1e-5 for fp32)."""
import numpy as np
import pytest

from mla_testlib import TOL, dev, dev_i64, host, make_module, mla, orc, rel, synth

pytestmark = pytest.mark.gpu

V3_SMALL_SEED = 7


@pytest.fixture(scope="module")
def v3_weights():
    return synth.weights(synth.V3, seed=V3_SMALL_SEED, dtype="bf16")


@pytest.fixture(scope="module")
def v3_module(v3_weights):
    m = make_module(synth.V3, v3_weights, "bf16")
    yield m
    m.close()


def _status_ok(m):
    s = m.sync_status()
    assert s == 0, (mla.mla_status_string(s), hex(mla.mla_device_error_bits(m.handle)))


# ---------------------------------------------------------------------------
# FP32 tiny configuration: L = 64, d = 256, n_h = 4, d_h = 32, d_c = 64, d_c' = 96, d_R = 16
# ---------------------------------------------------------------------------
def test_tiny_prefill_fp32_unabsorbed_and_absorbed():
    dims = synth.TINY
    W = synth.weights(dims, seed=0, dtype="fp32")
    h = synth.hidden(dims, 64, seed=0, dtype="fp32")
    cu = synth.cu_seqlens([64])
    ref = orc.mla_prefill(h, cu, W, dims)
    m = make_module(dims, W, "fp32")
    cache = dev(np.zeros((64, dims.row)), "fp32")
    u = m.prefill(dev(h, "fp32"), 1, dev_i64(cu), 64, cache)
    _status_ok(m)
    assert rel(host(u), ref["u"]) <= TOL["fp32"]
    assert rel(host(cache), ref["cache"]) <= TOL["fp32"]
    o = m.region(mla.OP_PREFILL, mla.BUF_O, (64, dims.n_h, dims.d_h), m.torch.float32, 1, 1, 64)
    assert rel(host(o), ref["o"]) <= TOL["fp32"]
    # absorbed form over the same cache: every token as a one-query decode of its prefix is
    # the same computation; use the last two tokens (Tq = 2) of the sequence.
    u_dec = m.decode(dev(h[62:64], "fp32"), 1, 2, dev_i64(cu), cache)
    _status_ok(m)
    assert rel(host(u_dec), ref["u"][62:64]) <= TOL["fp32"]
    m.close()


@pytest.mark.parametrize("tq", [1, 2])
def test_tiny_decode_fp32_ragged(tq):
    dims = synth.TINY
    W = synth.weights(dims, seed=1, dtype="fp32")
    lens = np.array([tq, 5, 64, 65, 130, 257])
    cu = synth.cu_seqlens(lens)
    cache = synth.latent_cache(dims, int(cu[-1]), seed=2, dtype="fp32")
    h_q = synth.hidden(dims, len(lens) * tq, seed=3, dtype="fp32")
    ref = orc.mla_decode(h_q, cache, cu, tq, W, dims)
    m = make_module(dims, W, "fp32")
    u = m.decode(dev(h_q, "fp32"), len(lens), tq, dev_i64(cu), dev(cache, "fp32"))
    _status_ok(m)
    assert rel(host(u), ref["u"]) <= TOL["fp32"]
    T = len(lens) * tq
    olat = m.region(mla.OP_DECODE, mla.BUF_OLAT, (T, dims.n_h, dims.d_c), m.torch.float32, len(lens), tq)
    assert rel(host(olat), ref["o_lat"]) <= TOL["fp32"]
    lse = m.region(mla.OP_DECODE, mla.BUF_LSE, (T, dims.n_h), m.torch.float32, len(lens), tq)
    assert rel(host(lse), ref["lse"]) <= TOL["fp32"]
    m.close()


def test_tiny_cache_append_fp32_scattered_slots():
    dims = synth.TINY
    W = synth.weights(dims, seed=4, dtype="fp32")
    T, cap = 37, 100
    h = synth.hidden(dims, T, seed=5, dtype="fp32")
    pos = np.arange(T) * 3 + 11
    slots = np.random.default_rng(0).permutation(cap)[:T]
    ref = orc.cache_append(h, pos, W, dims)
    m = make_module(dims, W, "fp32")
    cache = dev(np.full((cap, dims.row), 7.0), "fp32")
    m.cache_append(dev(h, "fp32"), dev_i64(pos), dev_i64(slots), cache)
    _status_ok(m)
    got = host(cache)
    assert rel(got[slots], ref) <= TOL["fp32"]
    untouched = np.setdiff1d(np.arange(cap), slots)
    assert np.all(got[untouched] == 7.0)
    m.close()


# ---------------------------------------------------------------------------
# BF16 at the DeepSeek-V3 sizes, small batches with ragged tails
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("tq,lens", [(1, [1, 63, 64, 65, 129, 1000, 4097]), (2, [2, 63, 64, 65, 129, 1000, 4097]),
                                     (1, [127, 128, 256, 257, 383, 2]), (2, [128, 129, 255, 256, 2, 3]),
                                     (1, [1, 40, 100]), (2, [33, 2, 97])])
def test_v3_attn_core_bf16_ragged(v3_module, tq, lens):
    # the last two cases hold fewer key tiles than there are CTA pairs
    dims = synth.V3
    lens = np.array(lens)
    cu = synth.cu_seqlens(lens)
    B, T = len(lens), len(lens) * tq
    cache = synth.latent_cache(dims, int(cu[-1]), seed=10 + tq, dtype="bf16")
    q_abs = synth.normal(11, 20, (T, dims.n_h, dims.d_c), std=0.5, dtype="bf16")
    q_rope = synth.normal(11, 21, (T, dims.n_h, dims.d_r), std=1.0, dtype="bf16")
    lat_ref, lse_ref = orc.attn_decode_latent(q_abs, q_rope, cache, cu, tq, dims)
    o_lat, lse = v3_module.attn_decode_latent(dev(q_abs, "bf16"), dev(q_rope, "bf16"), B, tq, dev_i64(cu),
                                              dev(cache, "bf16"))
    _status_ok(v3_module)
    assert rel(host(o_lat), lat_ref) <= TOL["bf16"]
    assert rel(host(lse), lse_ref) <= TOL["bf16"]


@pytest.mark.parametrize("tq", [1, 2])
def test_v3_attn_core_rows_past_the_last_sequence_are_never_read(v3_module, tq):
    # the cache holds NaN in every row after the last sequence; the last key tile of that sequence
    # reaches into them, and nothing of them may reach the outputs
    dims = synth.V3
    lens = np.array([200, 77])
    cu = synth.cu_seqlens(lens)
    B, T = len(lens), len(lens) * tq
    total = int(cu[-1])
    cache = synth.latent_cache(dims, total, seed=80 + tq, dtype="bf16")
    q_abs = synth.normal(81, 20, (T, dims.n_h, dims.d_c), std=0.5, dtype="bf16")
    q_rope = synth.normal(81, 21, (T, dims.n_h, dims.d_r), std=1.0, dtype="bf16")
    lat_ref, lse_ref = orc.attn_decode_latent(q_abs, q_rope, cache, cu, tq, dims)
    padded = np.full((total + 300, dims.row), np.nan, dtype=np.float32)
    padded[:total] = cache
    o_lat, lse = v3_module.attn_decode_latent(dev(q_abs, "bf16"), dev(q_rope, "bf16"), B, tq, dev_i64(cu),
                                              dev(padded, "bf16"))
    _status_ok(v3_module)
    assert rel(host(o_lat), lat_ref) <= TOL["bf16"]
    assert rel(host(lse), lse_ref) <= TOL["bf16"]


@pytest.mark.parametrize("tq", [1, 2])
def test_v3_attn_core_many_short_sequences(v3_module, tq):
    # more sequences than CTA pairs: one pair walks many sequence pieces; lengths from Tq up
    dims = synth.V3
    lens = synth.ragged_lengths(300, tq, 70, seed=tq)
    lens[:3] = tq
    cu = synth.cu_seqlens(lens)
    B, T = len(lens), len(lens) * tq
    cache = synth.latent_cache(dims, int(cu[-1]), seed=30 + tq, dtype="bf16")
    q_abs = synth.normal(31, 20, (T, dims.n_h, dims.d_c), std=0.5, dtype="bf16")
    q_rope = synth.normal(31, 21, (T, dims.n_h, dims.d_r), std=1.0, dtype="bf16")
    seqs = [0, 1, 2, 57, 150, 299]
    lat_ref, lse_ref = orc.attn_decode_latent(q_abs, q_rope, cache, cu, tq, dims, seqs=seqs)
    o_lat, lse = v3_module.attn_decode_latent(dev(q_abs, "bf16"), dev(q_rope, "bf16"), B, tq, dev_i64(cu),
                                              dev(cache, "bf16"))
    _status_ok(v3_module)
    rows = np.concatenate([np.arange(b * tq, (b + 1) * tq) for b in seqs])
    assert rel(host(o_lat)[rows], lat_ref) <= TOL["bf16"]
    assert rel(host(lse)[rows], lse_ref) <= TOL["bf16"]
    assert np.all(np.isfinite(host(o_lat)))


@pytest.mark.parametrize("tq", [1, 2])
def test_v3_decode_bf16_steps(v3_module, v3_weights, tq):
    dims = synth.V3
    lens = np.array([tq, 64, 65, 300])
    cu = synth.cu_seqlens(lens)
    B, T = len(lens), len(lens) * tq
    cache = synth.latent_cache(dims, int(cu[-1]), seed=20 + tq, dtype="bf16")
    h_q = synth.hidden(dims, T, seed=22, dtype="bf16")
    ref = orc.mla_decode_absorbed(h_q, cache, cu, tq, v3_weights, dims)
    u = v3_module.decode(dev(h_q, "bf16"), B, tq, dev_i64(cu), dev(cache, "bf16"))
    _status_ok(v3_module)
    bf = v3_module.torch.bfloat16
    reg = lambda which, shape, dt=bf: host(v3_module.region(mla.OP_DECODE, which, shape, dt, B, tq))  # noqa: E731
    assert rel(reg(mla.BUF_QC, (T, dims.n_h, dims.d_h)), ref["q_c"]) <= TOL["bf16"]
    assert rel(reg(mla.BUF_QR, (T, dims.n_h, dims.d_r)), ref["q_r"]) <= TOL["bf16"]
    assert rel(reg(mla.BUF_QABS, (T, dims.n_h, dims.d_c)), ref["q_abs"]) <= TOL["bf16"]
    assert rel(reg(mla.BUF_OLAT, (T, dims.n_h, dims.d_c)), ref["o_lat"]) <= TOL["bf16"]
    assert rel(reg(mla.BUF_LSE, (T, dims.n_h), v3_module.torch.float32), ref["lse"]) <= TOL["bf16"]
    assert rel(reg(mla.BUF_O, (T, dims.n_h, dims.d_h)), ref["o"]) <= TOL["bf16"]
    assert rel(host(u), ref["u"]) <= TOL["bf16"]
    # the unabsorbed oracle on one sequence (explicit per-head up-projection)
    un = orc.mla_decode(h_q, cache, cu, tq, v3_weights, dims, seqs=[2])
    assert rel(host(u)[un["rows"]], un["u"]) <= TOL["bf16"]


@pytest.mark.parametrize("B,tq", [(12, 2), (20, 2), (33, 1)])
def test_v3_decode_bf16_token_counts_of_the_wider_tiles(v3_module, v3_weights, B, tq):
    # 24, 40 and 33 query tokens: the projections' weight-streaming tiles are 32 and 64 tokens wide
    # there (16 and 128 elsewhere in these tests), whose epilogue stores element by element
    dims = synth.V3
    lens = synth.ragged_lengths(B, tq, 600, seed=B)
    cu = synth.cu_seqlens(lens)
    T = B * tq
    cache = synth.latent_cache(dims, int(cu[-1]), seed=25 + B, dtype="bf16")
    h_q = synth.hidden(dims, T, seed=26 + B, dtype="bf16")
    ref = orc.mla_decode_absorbed(h_q, cache, cu, tq, v3_weights, dims)
    u = v3_module.decode(dev(h_q, "bf16"), B, tq, dev_i64(cu), dev(cache, "bf16"))
    _status_ok(v3_module)
    bf = v3_module.torch.bfloat16
    reg = lambda which, shape, dt=bf: host(v3_module.region(mla.OP_DECODE, which, shape, dt, B, tq))  # noqa: E731
    assert rel(reg(mla.BUF_QC, (T, dims.n_h, dims.d_h)), ref["q_c"]) <= TOL["bf16"]
    assert rel(reg(mla.BUF_QR, (T, dims.n_h, dims.d_r)), ref["q_r"]) <= TOL["bf16"]
    assert rel(reg(mla.BUF_QABS, (T, dims.n_h, dims.d_c)), ref["q_abs"]) <= TOL["bf16"]
    assert rel(reg(mla.BUF_O, (T, dims.n_h, dims.d_h)), ref["o"]) <= TOL["bf16"]
    assert rel(host(u), ref["u"]) <= TOL["bf16"]


def test_v3_cache_append_bf16(v3_module, v3_weights):
    dims = synth.V3
    T, cap = 45, 300
    h = synth.hidden(dims, T, seed=30, dtype="bf16")
    pos = np.array([0, 1, 4095, 131071] + list(range(100, 141)))
    slots = np.random.default_rng(1).permutation(cap)[:T]
    ref = orc.cache_append(h, pos, v3_weights, dims)
    cache = dev(np.zeros((cap, dims.row)), "bf16")
    v3_module.cache_append(dev(h, "bf16"), dev_i64(pos), dev_i64(slots), cache)
    _status_ok(v3_module)
    assert rel(host(cache)[slots], ref) <= TOL["bf16"]


def test_v3_prefill_bf16_two_sequences(v3_module, v3_weights):
    dims = synth.V3
    lens = [200, 37]
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    h = synth.hidden(dims, T, seed=40, dtype="bf16")
    ref = orc.mla_prefill(h, cu, v3_weights, dims)
    cache = dev(np.zeros((T + 5, dims.row)), "bf16")
    u = v3_module.prefill(dev(h, "bf16"), 2, dev_i64(cu), max(lens), cache)
    _status_ok(v3_module)
    assert rel(host(cache)[:T], ref["cache"]) <= TOL["bf16"]
    o = v3_module.region(mla.OP_PREFILL, mla.BUF_O, (T, dims.n_h, dims.d_h), v3_module.torch.bfloat16, 2, 1, T)
    assert rel(host(o), ref["o"]) <= TOL["bf16"]
    assert rel(host(u), ref["u"]) <= TOL["bf16"]


def test_v3_prefill_bf16_three_sequences_past_the_swap_size(v3_module, v3_weights):
    # T = 1129 > 256 tokens: every projection takes the tile orientation (128 tokens x 256 features),
    # the token tiles straddle sequence starts, and RoPE takes each token's own position
    dims = synth.V3
    lens = [700, 300, 129]
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    h = synth.hidden(dims, T, seed=41, dtype="bf16")
    ref = orc.mla_prefill(h, cu, v3_weights, dims)
    cache = dev(np.zeros((T, dims.row)), "bf16")
    u = v3_module.prefill(dev(h, "bf16"), 3, dev_i64(cu), max(lens), cache)
    _status_ok(v3_module)
    assert rel(host(cache), ref["cache"]) <= TOL["bf16"]
    o = v3_module.region(mla.OP_PREFILL, mla.BUF_O, (T, dims.n_h, dims.d_h), v3_module.torch.bfloat16, 3, 1, T)
    assert rel(host(o), ref["o"]) <= TOL["bf16"]
    assert rel(host(u), ref["u"]) <= TOL["bf16"]


def test_v3_decode_bf16_more_than_256_query_tokens(v3_module, v3_weights):
    # B * Tq = 300 query tokens: the head-batched W^UK / W^UV projections run in chunks of at most
    # 256 tokens, the other projections in the tile orientation
    dims = synth.V3
    tq = 2
    lens = synth.ragged_lengths(150, tq, 90, seed=5)
    cu = synth.cu_seqlens(lens)
    B, T = len(lens), len(lens) * tq
    cache = synth.latent_cache(dims, int(cu[-1]), seed=60, dtype="bf16")
    h_q = synth.hidden(dims, T, seed=61, dtype="bf16")
    seqs = [0, 1, 74, 127, 128, 149]
    ref = orc.mla_decode_absorbed(h_q, cache, cu, tq, v3_weights, dims, seqs=seqs)
    u = v3_module.decode(dev(h_q, "bf16"), B, tq, dev_i64(cu), dev(cache, "bf16"))
    _status_ok(v3_module)
    rows = v3_module.torch.from_numpy(ref["rows"]).to("cuda:0")
    bf = v3_module.torch.bfloat16
    qabs = v3_module.region(mla.OP_DECODE, mla.BUF_QABS, (T, dims.n_h, dims.d_c), bf, B, tq)
    olat = v3_module.region(mla.OP_DECODE, mla.BUF_OLAT, (T, dims.n_h, dims.d_c), bf, B, tq)
    o = v3_module.region(mla.OP_DECODE, mla.BUF_O, (T, dims.n_h, dims.d_h), bf, B, tq)
    assert rel(host(qabs[rows]), ref["q_abs"]) <= TOL["bf16"]
    assert rel(host(olat[rows]), ref["o_lat"]) <= TOL["bf16"]
    assert rel(host(o[rows]), ref["o"]) <= TOL["bf16"]
    assert rel(host(u)[ref["rows"]], ref["u"]) <= TOL["bf16"]
    assert np.all(np.isfinite(host(u)))


# ---------------------------------------------------------------------------
# Device-side checks and determinism
# ---------------------------------------------------------------------------
def test_device_checks_flag_bad_cu_seqlens_and_slots(v3_module):
    dims = synth.V3
    cache = dev(np.zeros((64, dims.row)), "bf16")
    q = dev(np.zeros((2, dims.n_h, dims.d_c)), "bf16")
    qr = dev(np.zeros((2, dims.n_h, dims.d_r)), "bf16")
    bad_cu = dev_i64([0, 10, 5])          # decreasing
    v3_module.attn_decode_latent(q, qr, 2, 1, bad_cu, cache)
    s = v3_module.sync_status()
    assert mla.STATUS_NAMES[s] == "MLA_ERR_DEVICE_CHECK"
    assert mla.mla_device_error_bits(v3_module.handle) & 1
    assert v3_module.sync_status() == 0    # the word is cleared once read
    h = dev(np.zeros((2, dims.d)), "bf16")
    v3_module.cache_append(h, dev_i64([0, 1]), dev_i64([3, 64]), cache)   # slot 64 == capacity
    assert mla.STATUS_NAMES[v3_module.sync_status()] == "MLA_ERR_DEVICE_CHECK"
    assert mla.mla_device_error_bits(v3_module.handle) & 4


def test_bounded_wait_gives_up_reports_timeout_and_the_next_call_recovers(v3_module):
    # the armed launch waits for a cache tile that is never loaded; each role gives up after its
    # 20 ms limit and returns, the error word says TIMEOUT, and the same handle then runs normally
    dims = synth.V3
    lens = np.array([300, 700])
    cu = synth.cu_seqlens(lens)
    cache = synth.latent_cache(dims, int(cu[-1]), seed=70, dtype="bf16")
    q_abs = synth.normal(71, 20, (2, dims.n_h, dims.d_c), std=0.5, dtype="bf16")
    q_rope = synth.normal(71, 21, (2, dims.n_h, dims.d_r), std=1.0, dtype="bf16")
    args = (dev(q_abs, "bf16"), dev(q_rope, "bf16"), 2, 1, dev_i64(cu), dev(cache, "bf16"))
    mla.mla_test_arm_stall()
    v3_module.attn_decode_latent(*args)
    s = v3_module.sync_status()
    assert mla.STATUS_NAMES[s] == "MLA_ERR_TIMEOUT"
    assert mla.mla_device_error_bits(v3_module.handle) & (1 << 6)
    o_lat, lse = v3_module.attn_decode_latent(*args)
    _status_ok(v3_module)
    lat_ref, lse_ref = orc.attn_decode_latent(q_abs, q_rope, cache, cu, 1, dims)
    assert rel(host(o_lat), lat_ref) <= TOL["bf16"]
    assert rel(host(lse), lse_ref) <= TOL["bf16"]


def test_decode_is_deterministic(v3_module):
    dims = synth.V3
    lens = np.array([700, 3000])
    cu = synth.cu_seqlens(lens)
    cache = dev(synth.latent_cache(dims, int(cu[-1]), seed=50, dtype="bf16"), "bf16")
    h_q = dev(synth.hidden(dims, 2, seed=51, dtype="bf16"), "bf16")
    a = v3_module.decode(h_q, 2, 1, dev_i64(cu), cache).clone()
    b = v3_module.decode(h_q, 2, 1, dev_i64(cu), cache).clone()
    _status_ok(v3_module)
    assert bool((a == b).all())


# ---------------------------------------------------------------------------
# The prefill attention core alone (mla_attn_prefill): 128-row query / key tiles, ragged tails,
# a one-token sequence and a sequence that starts inside a tile of the packed layout
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("lens", [[600, 129, 1, 300], [128, 256, 127]])
def test_v3_attn_prefill_core_ragged(v3_module, lens):
    dims = synth.V3
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    x = synth.prefill_core_inputs(dims, T, seed=51)
    cache_np = synth.latent_cache(dims, T + 3, seed=52)
    d = {k: dev(v, "bf16") for k, v in x.items()}
    cache = dev(cache_np, "bf16")
    o = v3_module.torch.empty((T, dims.n_h, dims.d_h), device="cuda:0", dtype=v3_module.torch.bfloat16)
    mla.mla_attn_prefill(v3_module.handle, d["q_c"], d["q_r"], d["k_c"], d["v_c"], len(lens), dev_i64(cu), T,
                         max(lens), cache, T + 3, o, device=v3_module.device)
    _status_ok(v3_module)
    ref = np.empty((T, dims.n_h, dims.d_h))
    scale = 1.0 / np.sqrt(dims.d_h + dims.d_r)
    k_r = cache_np[:, dims.d_c:]
    for b in range(len(lens)):
        a, e = int(cu[b]), int(cu[b + 1])
        for i in range(dims.n_h):
            q = np.concatenate([x["q_c"][a:e, i], x["q_r"][a:e, i]], axis=1)
            k = np.concatenate([x["k_c"][a:e, i], k_r[a:e]], axis=1)
            ref[a:e, i], _, _, _ = orc.causal_softmax_attend(q, k, x["v_c"][a:e, i], None, np.arange(e - a), scale)
    assert rel(host(o), ref) <= TOL["bf16"]
