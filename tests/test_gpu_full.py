"""Parity at the full sizes of the DeepSeek-V3 workloads, in the launch configuration the bench
times (one mla_cache_append + one mla_decode per decode step; one mla_prefill): sampled outputs
against the oracle, computed one sequence (or query row and head) at a time, plus properties that
hold at any size (finite outputs, every appended or prefilled cache row).

The decode references use the oracle's absorbed form, which the oracle's own tests pin to the
unabsorbed definition (agreement to 1e-12); it costs O(d_c) per cached row instead of
O(n_h d_h d_c), which is what makes 32K- and 128K-row sequences checkable on the host.
"""
import numpy as np
import pytest

from mla_testlib import (TOL, dev, dev_i64, fp8_cache, fp8_decode_rows, fp8_row_bound, host, make_module, mla, orc,
                         rel, round_bf16, synth)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def w0():
    return synth.weights(synth.V3, seed=0, dtype="bf16")


@pytest.fixture(scope="module")
def mod(w0):
    m = make_module(synth.V3, w0, "bf16")
    yield m
    m.close()


def _status_ok(m):
    s = m.sync_status()
    assert s == 0, (mla.mla_status_string(s), hex(mla.mla_device_error_bits(m.handle)))


def _decode_step(mod, W, name, sample):
    """One decode step of workload `name` (seed 0): append the Tq query tokens' rows at the end of
    every sequence, then decode; u of the sampled sequences and every appended row are checked."""
    wl = synth.WORKLOADS[name]
    dims, tq = wl.dims, wl.tq
    lens = wl.lengths(0)
    cu = synth.cu_seqlens(lens)
    B, T = len(lens), len(lens) * tq
    cache = synth.latent_cache(dims, int(cu[-1]), seed=0)
    h_q = synth.hidden(dims, T, seed=0)
    # query k of sequence b sits at position len_b - Tq + k, in cache row cu[b] + position
    pos = np.concatenate([np.arange(L - tq, L) for L in lens]).astype(np.int64)
    slots = np.repeat(cu[:-1], tq) + pos
    d_cache = dev(cache, "bf16")
    d_h = dev(h_q, "bf16")
    mod.cache_append(d_h, dev_i64(pos), dev_i64(slots), d_cache)
    u = mod.decode(d_h, B, tq, dev_i64(cu), d_cache)
    _status_ok(mod)
    got_rows = host(d_cache[dev_i64(slots)])
    new_rows = orc.cache_append(h_q, pos, W, dims)
    assert rel(got_rows, new_rows) <= TOL["bf16"]
    # the oracle decodes over the cache as the step leaves it (appended rows stored as bf16)
    cache[slots] = synth.round_to(new_rows, "bf16")
    ref = orc.mla_decode_absorbed(h_q, cache, cu, tq, W, dims, seqs=sample)
    u_h = host(u)
    assert np.all(np.isfinite(u_h))
    assert rel(u_h[ref["rows"]], ref["u"]) <= TOL["bf16"]
    # the latent core's own outputs for the sampled sequences (o^lat is stored as bf16 in the
    # decode workspace, lse as fp32), before W^UV and W^O average over heads and columns
    rows = mod.torch.from_numpy(ref["rows"]).to("cuda:0")
    olat = mod.region(mla.OP_DECODE, mla.BUF_OLAT, (T, dims.n_h, dims.d_c), mod.torch.bfloat16, B, tq)
    lse = mod.region(mla.OP_DECODE, mla.BUF_LSE, (T, dims.n_h), mod.torch.float32, B, tq)
    assert rel(host(olat[rows]), ref["o_lat"]) <= TOL["bf16"]
    assert rel(host(lse[rows]), ref["lse"]) <= TOL["bf16"]


def test_decode_b16_l4096_full(mod, w0):
    _decode_step(mod, w0, "decode_b16_l4096", [0, 7, 15])


def test_decode_mtp_b64_ragged_full(mod, w0):
    lens = synth.WORKLOADS["decode_mtp_b64_ragged"].lengths(0)
    sample = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 33})
    _decode_step(mod, w0, "decode_mtp_b64_ragged", sample)


def test_decode_long_b4_l131072_full(mod, w0):
    _decode_step(mod, w0, "decode_long_b4_l131072", [0, 3])


def _decode_step_fp8(mod, W, name, sample):
    """The same step over an FP8 latent cache (656-byte rows): the seeded bf16 cache put through the
    oracle's quantizer, the query tokens' rows appended by the library as FP8 rows, then the decode.
    Every appended row is checked against the oracle's float64 append within the format's rounding
    bound; u, o^lat and lse of the sampled sequences against the oracle's absorbed decode over the
    rows the FP8 cache stands for (the appended ones quantized by the oracle from its own rows
    rounded to bf16, as the bf16 format would store them)."""
    wl = synth.WORKLOADS[name]
    dims, tq = wl.dims, wl.tq
    lens = wl.lengths(0)
    cu = synth.cu_seqlens(lens)
    B, T = len(lens), len(lens) * tq
    raw, deq = fp8_cache(synth.latent_cache(dims, int(cu[-1]), seed=0), dims)
    h_q = synth.hidden(dims, T, seed=0)
    pos = np.concatenate([np.arange(L - tq, L) for L in lens]).astype(np.int64)
    slots = np.repeat(cu[:-1], tq) + pos
    new_rows = orc.cache_append(h_q, pos, W, dims)
    _, deq[slots] = fp8_cache(round_bf16(new_rows), dims)
    ref = orc.mla_decode_absorbed(h_q, deq, cu, tq, W, dims, seqs=sample)
    torch = mod.torch
    d_cache = torch.from_numpy(raw).to("cuda:0")
    del raw
    mod.set_cache_format(mla.CACHE_FP8)
    try:
        d_h = dev(h_q, "bf16")
        mod.cache_append(d_h, dev_i64(pos), dev_i64(slots), d_cache)
        u = mod.decode(d_h, B, tq, dev_i64(cu), d_cache)
        _status_ok(mod)
        rows = torch.from_numpy(ref["rows"]).to("cuda:0")
        olat = mod.region(mla.OP_DECODE, mla.BUF_OLAT, (T, dims.n_h, dims.d_c), torch.bfloat16, B, tq)
        lse = mod.region(mla.OP_DECODE, mla.BUF_LSE, (T, dims.n_h), torch.float32, B, tq)
        olat_h, lse_h = host(olat[rows]), host(lse[rows])
    finally:
        mod.set_cache_format(mla.CACHE_BF16)
    vals, kr, s, pad = fp8_decode_rows(d_cache[dev_i64(slots)].cpu().numpy())
    assert not pad.any()
    err = np.abs(orc.dequantize_cache_rows_fp8(vals, kr, s) - new_rows)
    bound = fp8_row_bound(new_rows, s)
    assert np.all(err <= bound), float((err / bound).max())
    u_h = host(u)
    assert np.all(np.isfinite(u_h))
    assert rel(u_h[ref["rows"]], ref["u"]) <= TOL["bf16"]
    assert rel(olat_h, ref["o_lat"]) <= TOL["bf16"]
    assert rel(lse_h, ref["lse"]) <= TOL["bf16"]


def test_decode_b16_l4096_fp8_full(mod, w0):
    _decode_step_fp8(mod, w0, "decode_b16_l4096", [0, 7, 15])


def test_decode_long_b4_l131072_fp8_full(mod, w0):
    _decode_step_fp8(mod, w0, "decode_long_b4_l131072", [0, 3])


def test_prefill_l32768_full(mod, w0):
    wl = synth.WORKLOADS["prefill_l32768"]
    dims = wl.dims
    T = int(wl.length)
    cu = synth.cu_seqlens([T])
    h = synth.hidden(dims, T, seed=0)
    d_cache = mod.torch.zeros((T, dims.row), dtype=mod.torch.bfloat16, device="cuda:0")
    u = mod.prefill(dev(h, "bf16"), 1, dev_i64(cu), T, d_cache)
    _status_ok(mod)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 4095, 16383, 32766, 32767], rng.integers(0, T, 8)]))
    heads = [0, 1, 63, 127]
    ref = orc.mla_prefill(h, cu, w0, dims, query_rows=rows, heads=heads)
    assert rel(host(d_cache), ref["cache"]) <= TOL["bf16"]
    o = mod.region(mla.OP_PREFILL, mla.BUF_O, (T, dims.n_h, dims.d_h), mod.torch.bfloat16, 1, 1, T)
    got = host(o[dev_i64(ref["rows"])][:, heads])
    assert rel(got, ref["o"]) <= TOL["bf16"]
    # u = W^O [o_1; ...; o_n_h] of the sampled rows over all heads: the tile-orientation W^O launch
    # (28 weight tiles, raster groups 8/8/8/4) against the absorbed oracle on the same cache rows
    ab = orc.mla_prefill_absorbed(h, cu, w0, dims, rows, cache=ref["cache"])
    u_h = host(u)
    assert np.all(np.isfinite(u_h))
    assert rel(u_h[ab["rows"]], ab["u"]) <= TOL["bf16"]
