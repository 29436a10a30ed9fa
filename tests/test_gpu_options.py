"""GPU parity with the opt-in parts of the layer on: the RMSNorm after the latent compression
(section 三(二)1 of the DeepSeek-V3 notes) and YaRN on the decoupled RoPE (section 三(二)3:
s = 40, alpha = 1, beta = 32), against the float64 oracle with the same options."""
import numpy as np
import pytest

from mla_testlib import TOL, dev, dev_i64, host, make_module, mla, orc, rel, synth

pytestmark = pytest.mark.gpu


def _status_ok(m):
    s = m.sync_status()
    assert s == 0, (mla.mla_status_string(s), hex(mla.mla_device_error_bits(m.handle)))


def _weights(dims, seed, dtype):
    return dict(synth.weights(dims, seed=seed, dtype=dtype), **synth.gains(dims, seed=seed + 1, dtype=dtype))


# ---------------------------------------------------------------------------
# FP32 tiny configuration (YaRN from a 256-token original context, so that the tiny RoPE's pairs
# fall in all three regimes of the frequency ramp)
# ---------------------------------------------------------------------------
def test_tiny_fp32_prefill_decode_and_chunk_with_rmsnorm_and_yarn():
    dims = synth.TINY_YARN
    W = _weights(dims, 50, "fp32")
    m = make_module(dims, W, "fp32")
    try:
        # prefill of two sequences
        lens = [90, 37]
        cu = synth.cu_seqlens(lens)
        T = int(cu[-1])
        h = synth.hidden(dims, T, seed=51, dtype="fp32")
        ref = orc.mla_prefill(h, cu, W, dims)
        cache = dev(np.zeros((T, dims.row)), "fp32")
        u = m.prefill(dev(h, "fp32"), 2, dev_i64(cu), max(lens), cache)
        _status_ok(m)
        assert rel(host(cache), ref["cache"]) <= TOL["fp32"]
        assert rel(host(u), ref["u"]) <= TOL["fp32"]
        # decode (Tq = 2) over that cache: the last two tokens of each sequence
        rows = np.concatenate([np.arange(cu[b + 1] - 2, cu[b + 1]) for b in range(2)])
        u_dec = m.decode(dev(h[rows], "fp32"), 2, 2, dev_i64(cu), cache)
        _status_ok(m)
        assert rel(host(u_dec), ref["u"][rows]) <= TOL["fp32"]
        # a chunk of 20 and 5 tokens after prefixes of 70 and 32 rows of the same cache
        q_lens = [20, 5]
        rows = np.concatenate([np.arange(cu[b + 1] - q_lens[b], cu[b + 1]) for b in range(2)])
        u_ch, form = m.prefill_chunk(dev(h[rows], "fp32"), 2, dev_i64(synth.cu_seqlens(q_lens)), 20, dev_i64(cu), T,
                                     cache)
        _status_ok(m)
        assert form == mla.CHUNK_UNABSORBED
        assert rel(host(u_ch), ref["u"][rows]) <= TOL["fp32"]
    finally:
        m.close()


# ---------------------------------------------------------------------------
# BF16 at the DeepSeek-V3 sizes with the DeepSeek-V3 long-context YaRN
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def v3_opts():
    W = _weights(synth.V3_YARN, 52, "bf16")
    m = make_module(synth.V3_YARN, W, "bf16")
    yield m, W
    m.close()


def test_v3_cache_append_with_rmsnorm_and_yarn_at_long_positions(v3_opts):
    m, W = v3_opts
    dims = synth.V3_YARN
    T, cap = 45, 64
    h = synth.hidden(dims, T, seed=53, dtype="bf16")
    pos = np.concatenate([[0, 1, 4095, 4096, 32767, 131071], np.arange(T - 6) * 2917 + 7])
    slots = np.random.default_rng(3).permutation(cap)[:T]
    ref = orc.cache_append(h, pos, W, dims)
    cache = dev(np.zeros((cap, dims.row)), "bf16")
    m.cache_append(dev(h, "bf16"), dev_i64(pos), dev_i64(slots), cache)
    _status_ok(m)
    got = host(cache)[slots]
    assert rel(got[:, :dims.d_c], ref[:, :dims.d_c]) <= TOL["bf16"]
    assert rel(got[:, dims.d_c:], ref[:, dims.d_c:]) <= TOL["bf16"]


@pytest.mark.parametrize("tq", [1, 2])
def test_v3_decode_with_rmsnorm_and_yarn(v3_opts, tq):
    m, W = v3_opts
    dims = synth.V3_YARN
    lens = np.array([1000, 4097, 65])
    cu = synth.cu_seqlens(lens)
    cache = synth.latent_cache(dims, int(cu[-1]), seed=54, dtype="bf16")
    h_q = synth.hidden(dims, len(lens) * tq, seed=55, dtype="bf16")
    ref = orc.mla_decode_absorbed(h_q, cache, cu, tq, W, dims)
    u = m.decode(dev(h_q, "bf16"), len(lens), tq, dev_i64(cu), dev(cache, "bf16"))
    _status_ok(m)
    assert rel(host(u), ref["u"]) <= TOL["bf16"]
    T = len(lens) * tq
    qr = m.region(mla.OP_DECODE, mla.BUF_QR, (T, dims.n_h, dims.d_r), m.torch.bfloat16, len(lens), tq)
    _, _, qr_ref = orc.query_projections(h_q, W, dims, orc.decode_positions(cu, tq))
    assert rel(host(qr), qr_ref) <= TOL["bf16"]


def test_v3_prefill_with_rmsnorm_and_yarn(v3_opts):
    m, W = v3_opts
    dims = synth.V3_YARN
    lens = [300, 129]
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    h = synth.hidden(dims, T, seed=56, dtype="bf16")
    ref = orc.mla_prefill(h, cu, W, dims)
    cache = dev(np.zeros((T, dims.row)), "bf16")
    u = m.prefill(dev(h, "bf16"), 2, dev_i64(cu), max(lens), cache)
    _status_ok(m)
    assert rel(host(cache), ref["cache"]) <= TOL["bf16"]
    assert rel(host(u), ref["u"]) <= TOL["bf16"]
