"""GPU parity of the FP8 (e4m3) latent cache rows: the quantizer against the oracle's
`quantize_cache_rows_fp8` (same codes, scaled k^R and scale on every row, the values compared
exactly; +0 and -0 compare equal), and the cache append writing FP8 rows against the oracle's
float64 append within the format's rounding bound. The row layout is 656 bytes: e4m3 codes [0, 512),
f16 k^R / s [512, 640), fp32 s [640, 644), zero [644, 656)."""
import numpy as np
import pytest

from mla_testlib import (E4M3, TOL, dev, dev_i64, fp8_cache, fp8_decode_rows, fp8_row_bound, host, make_module,
                         mla, orc, rel, round_bf16, synth)

pytestmark = pytest.mark.gpu

V3 = synth.V3
def stress_rows(n: int, seed: int) -> np.ndarray:
    """bf16 cache rows [n, 576] that reach every branch of the format: N(0, 1) rows at scales from
    1e-30 to 1e30, an all-zero row, rows whose k^R sets the scale (so k^R / s is at the f16 range's
    end and c^KV / s lands in e4m3 subnormals), and rows with amax(c^KV) = 448 (s = 1) whose other
    entries are exact midpoints between neighbouring e4m3 values (ties to the even code)."""
    rng = np.random.default_rng(seed)
    rows = rng.standard_normal((n, 576))
    scale = 10.0 ** rng.integers(-30, 31, size=n)
    rows *= scale[:, None]
    rows[0] = 0.0
    kr_big = np.arange(1, n, 7)
    rows[kr_big, 512:] *= 1e5
    rows[kr_big, :512] *= 1e-3
    tie_rows = np.arange(2, n, 11)
    mid = (E4M3[1:] + E4M3[:-1]) / 2          # every midpoint of the positive grid is bf16-exact
    for r in tie_rows:
        pick = rng.integers(0, len(mid), size=511)
        rows[r, 1:512] = np.where(rng.random(511) < 0.5, -1.0, 1.0) * mid[pick]
        rows[r, 0] = 448.0
        rows[r, 512:] = rng.standard_normal(64)
    return round_bf16(rows)


@pytest.fixture(scope="module")
def v3():
    W = synth.weights(V3, seed=60, dtype="bf16")
    m = make_module(V3, W, "bf16")
    yield m, W
    m.close()


@pytest.mark.parametrize("n", [1, 8, 1037])
def test_quantizer_matches_the_oracle_exactly(v3, n):
    import torch
    m, _ = v3
    rows = stress_rows(n, seed=61 + n)
    assert np.all(round_bf16(rows) == rows)
    mid = (E4M3[1:] + E4M3[:-1]) / 2
    assert np.all(round_bf16(mid) == mid)
    got = m.quantize_fp8(dev(rows, "bf16"))
    torch.cuda.synchronize()
    vals, kr, s, pad = fp8_decode_rows(got.cpu().numpy())
    codes_ref, kr_ref, s_ref = orc.quantize_cache_rows_fp8(rows, V3)
    assert np.array_equal(s, s_ref)
    assert np.array_equal(vals, codes_ref)
    assert np.array_equal(kr, kr_ref)
    assert not pad.any()


@pytest.mark.parametrize("T,cap", [(45, 64), (700, 1024)])
def test_cache_append_writes_fp8_rows(v3, T, cap):
    import torch
    m, W = v3
    h = synth.hidden(V3, T, seed=62, dtype="bf16")
    pos = np.concatenate([[0, 1, 4095, 4096, 32767], np.arange(T - 5) * 131 + 3])
    slots = np.random.default_rng(4).permutation(cap)[:T]
    ref = orc.cache_append(h, pos, W, V3)
    m.set_cache_format(mla.CACHE_FP8)
    try:
        cache8 = torch.zeros(cap, mla.FP8_ROW_BYTES, dtype=torch.uint8, device="cuda:0")
        m.cache_append(dev(h, "bf16"), dev_i64(pos), dev_i64(slots), cache8)
        assert m.sync_status() == 0
    finally:
        m.set_cache_format(mla.CACHE_BF16)
    raw = cache8.cpu().numpy()
    untouched = np.setdiff1d(np.arange(cap), slots)
    assert not raw[untouched].any()
    vals, kr, s, pad = fp8_decode_rows(raw[slots])
    assert not pad.any()
    deq = orc.dequantize_cache_rows_fp8(vals, kr, s)
    err = np.abs(deq - ref)
    assert np.all(err <= fp8_row_bound(ref, s)), float((err / fp8_row_bound(ref, s)).max())
    # the rows the bf16 format writes for the same call, put through the library's own quantizer,
    # are the same bytes (the FP8 append quantizes the very rows the bf16 append would store)
    cache16 = torch.zeros(cap, 576, dtype=torch.bfloat16, device="cuda:0")
    m.cache_append(dev(h, "bf16"), dev_i64(pos), dev_i64(slots), cache16)
    q = m.quantize_fp8(cache16[dev_i64(slots)].contiguous())
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), raw[slots])


def test_fp8_append_flags_slots_outside_the_cache(v3):
    # the projection writes the staged bf16 rows without the slots, so the quantizer is the step that
    # must report a slot outside [0, capacity) (and write nothing for it), as the bf16 append does
    import torch
    m, W = v3
    h = synth.hidden(V3, 3, seed=63, dtype="bf16")
    pos = np.array([0, 1, 2])
    ref = orc.cache_append(h, pos, W, V3)
    m.set_cache_format(mla.CACHE_FP8)
    try:
        cache8 = torch.zeros(65, mla.FP8_ROW_BYTES, dtype=torch.uint8, device="cuda:0")
        m.cache_append(dev(h, "bf16"), dev_i64(pos), dev_i64([3, 64, -1]), cache8[:64])
        assert mla.STATUS_NAMES[m.sync_status()] == "MLA_ERR_DEVICE_CHECK"
        assert mla.mla_device_error_bits(m.handle) & 4
        assert m.sync_status() == 0
        m.cache_append(dev(h[:1], "bf16"), dev_i64(pos[:1]), dev_i64([5]), cache8[:64])
        assert m.sync_status() == 0
    finally:
        m.set_cache_format(mla.CACHE_BF16)
    raw = cache8.cpu().numpy()
    assert not raw[np.setdiff1d(np.arange(65), [3, 5])].any()    # row 64 lies past the cache given
    for slot, t in ((3, 0), (5, 0)):
        vals, kr, s, pad = fp8_decode_rows(raw[slot:slot + 1])
        err = np.abs(orc.dequantize_cache_rows_fp8(vals, kr, s) - ref[t:t + 1])
        assert np.all(err <= fp8_row_bound(ref[t:t + 1], s)) and not pad.any()


# ---------------------------------------------------------------------------
# Decode over an FP8 cache: the rows the oracle quantized, packed into the 656-byte layout, against
# the oracle's attention over the rows they stand for (codes * s | (k^R / s) * s)
# ---------------------------------------------------------------------------
def test_encode_rows_round_trips_through_decode_rows():
    rows = stress_rows(50, seed=70)
    raw, deq = fp8_cache(rows)
    vals, kr, s, pad = fp8_decode_rows(raw)
    assert np.array_equal(orc.dequantize_cache_rows_fp8(vals, kr, s), deq) and not pad.any()


def _core(m, q_abs, q_rope, B, tq, cu, raw):
    import torch
    m.set_cache_format(mla.CACHE_FP8)
    try:
        cache = torch.from_numpy(raw).to("cuda:0")
        o_lat, lse = m.attn_decode_latent(dev(q_abs, "bf16"), dev(q_rope, "bf16"), B, tq, dev_i64(cu), cache)
        assert m.sync_status() == 0, hex(mla.mla_device_error_bits(m.handle))
    finally:
        m.set_cache_format(mla.CACHE_BF16)
    return host(o_lat), host(lse)


@pytest.mark.parametrize("tq,lens", [(1, [1, 63, 64, 65, 129, 1000, 4097]), (2, [2, 63, 64, 65, 129, 1000, 4097]),
                                     (1, [1, 40, 100]), (2, [33, 2, 97])])
def test_fp8_attn_core_ragged(v3, tq, lens):
    m, _ = v3
    lens = np.array(lens)
    cu = synth.cu_seqlens(lens)
    B, T = len(lens), len(lens) * tq
    raw, deq = fp8_cache(synth.latent_cache(V3, int(cu[-1]), seed=71 + tq, dtype="bf16"))
    q_abs = synth.normal(72, 20, (T, V3.n_h, V3.d_c), std=0.5, dtype="bf16")
    q_rope = synth.normal(72, 21, (T, V3.n_h, V3.d_r), std=1.0, dtype="bf16")
    lat_ref, lse_ref = orc.attn_decode_latent(q_abs, q_rope, deq, cu, tq, V3)
    o_lat, lse = _core(m, q_abs, q_rope, B, tq, cu, raw)
    assert rel(o_lat, lat_ref) <= TOL["bf16"]
    assert rel(lse, lse_ref) <= TOL["bf16"]


@pytest.mark.parametrize("tq", [1, 2])
def test_fp8_attn_core_scales_far_apart_and_rows_past_the_end(v3, tq):
    # cache rows whose scales span 2^-20 .. 2^4, so that the weights p_j s_j of the P'.C product span
    # 2^24 and more while the softmax weights p_j stay within a few units (the queries are small);
    # heads whose q~ and q^R magnitudes span 1e-2 .. 1e2 (the per-head f16 scaling of the queries:
    # near-uniform softmax on the first heads, peaked on the last); garbage (0xFF: NaN codes and a
    # NaN scale) in every row after the last sequence, which the last key tile reaches into. The
    # scores stay within a few hundred, where fp32 holds the merge's m and lse to 2^-15.
    m, _ = v3
    lens = np.array([300, 77, 129])
    cu = synth.cu_seqlens(lens)
    B, T = len(lens), len(lens) * tq
    total = int(cu[-1])
    rows = synth.latent_cache(V3, total, seed=73, dtype="bf16")
    rows *= np.exp2(np.random.default_rng(5).integers(-20, 5, size=total))[:, None]
    raw, deq = fp8_cache(rows)
    padded = np.full((total + 200, mla.FP8_ROW_BYTES), 0xFF, dtype=np.uint8)
    padded[:total] = raw
    head_scale = (10.0 ** np.linspace(-2, 2, V3.n_h))[None, :, None] * 2.0 ** -4
    q_abs = round_bf16(synth.normal(74, 20, (T, V3.n_h, V3.d_c), std=0.5, dtype="bf16") * head_scale)
    q_rope = round_bf16(synth.normal(74, 21, (T, V3.n_h, V3.d_r), std=1.0, dtype="bf16") * head_scale)
    lat_ref, lse_ref = orc.attn_decode_latent(q_abs, q_rope, deq, cu, tq, V3)
    assert np.abs(lse_ref).max() < 512
    o_lat, lse = _core(m, q_abs, q_rope, B, tq, cu, padded)
    for i in range(V3.n_h):
        assert rel(o_lat[:, i], lat_ref[:, i]) <= TOL["bf16"], i
    assert rel(lse, lse_ref) <= TOL["bf16"]


@pytest.mark.parametrize("tq", [1, 2])
def test_fp8_decode_step(v3, tq):
    import torch
    m, W = v3
    lens = np.array([1000, 4097, 65])
    cu = synth.cu_seqlens(lens)
    raw, deq = fp8_cache(synth.latent_cache(V3, int(cu[-1]), seed=75, dtype="bf16"))
    h_q = synth.hidden(V3, len(lens) * tq, seed=76, dtype="bf16")
    ref = orc.mla_decode_absorbed(h_q, deq, cu, tq, W, V3)
    m.set_cache_format(mla.CACHE_FP8)
    try:
        u = m.decode(dev(h_q, "bf16"), len(lens), tq, dev_i64(cu), torch.from_numpy(raw).to("cuda:0"))
        assert m.sync_status() == 0
    finally:
        m.set_cache_format(mla.CACHE_BF16)
    assert rel(host(u), ref["u"]) <= TOL["bf16"]


def test_fp8_append_then_decode(v3):
    # the cache rows come from the FP8 append, which quantizes the projection's rows as the bf16
    # format stores them (rounded to bf16); the reference quantizes the oracle's rows rounded the same
    # way (without that rounding the scales, and with them every code, move by up to 2^-9 and the
    # outputs by about 2 %)
    import torch
    m, W = v3
    lens = np.array([150, 333])
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    h = synth.hidden(V3, T, seed=77, dtype="bf16")
    pos = np.concatenate([np.arange(n) for n in lens])
    _, deq = fp8_cache(round_bf16(orc.cache_append(h, pos, W, V3)))
    rows = np.concatenate([np.arange(cu[b + 1] - 1, cu[b + 1]) for b in range(2)])
    ref = orc.mla_decode_absorbed(h[rows], deq, cu, 1, W, V3)
    m.set_cache_format(mla.CACHE_FP8)
    try:
        cache = torch.zeros(T, mla.FP8_ROW_BYTES, dtype=torch.uint8, device="cuda:0")
        m.cache_append(dev(h, "bf16"), dev_i64(pos), dev_i64(np.arange(T)), cache)
        u = m.decode(dev(h[rows], "bf16"), 2, 1, dev_i64(cu), cache)
        assert m.sync_status() == 0
    finally:
        m.set_cache_format(mla.CACHE_BF16)
    assert rel(host(u), ref["u"]) <= TOL["bf16"]


@pytest.mark.parametrize("tq", [1, 2])
def test_fp8_attn_core_many_short_sequences(v3, tq):
    # more sequences than clusters: each cluster walks many sequence pieces, so the converters' and
    # the scale buffers' hand-offs cross piece boundaries (q~ loads between tiles) again and again
    m, _ = v3
    lens = synth.ragged_lengths(300, tq, 70, seed=10 + tq)
    lens[:3] = tq
    cu = synth.cu_seqlens(lens)
    B, T = len(lens), len(lens) * tq
    raw, deq = fp8_cache(synth.latent_cache(V3, int(cu[-1]), seed=78 + tq, dtype="bf16"))
    q_abs = synth.normal(79, 20, (T, V3.n_h, V3.d_c), std=0.5, dtype="bf16")
    q_rope = synth.normal(79, 21, (T, V3.n_h, V3.d_r), std=1.0, dtype="bf16")
    seqs = [0, 1, 2, 57, 150, 299]
    lat_ref, lse_ref = orc.attn_decode_latent(q_abs, q_rope, deq, cu, tq, V3, seqs=seqs)
    o_lat, lse = _core(m, q_abs, q_rope, B, tq, cu, raw)
    rows = np.concatenate([np.arange(b * tq, (b + 1) * tq) for b in seqs])
    assert rel(o_lat[rows], lat_ref) <= TOL["bf16"]
    assert rel(lse[rows], lse_ref) <= TOL["bf16"]
    assert np.all(np.isfinite(o_lat))
