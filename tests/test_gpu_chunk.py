"""GPU parity of the chunked prefill (mla_prefill_chunk): a chunk of new tokens per sequence after a
cached prefix, in both forms, against the float64 oracle's chunked prefill on the same seeded
inputs. The prefix rows are synthetic cache rows, which both sides use as they are; the oracle's
chunked prefill is pinned on the CPU to the prefill of the whole sequence."""
import numpy as np
import pytest

from mla_testlib import TOL, dev, dev_i64, host, make_module, mla, orc, rel, synth

pytestmark = pytest.mark.gpu


def _status_ok(m):
    s = m.sync_status()
    assert s == 0, (mla.mla_status_string(s), hex(mla.mla_device_error_bits(m.handle)))


@pytest.fixture(scope="module")
def v3_weights():
    return synth.weights(synth.V3, seed=17, dtype="bf16")


@pytest.fixture(scope="module")
def v3_module(v3_weights):
    m = make_module(synth.V3, v3_weights, "bf16")
    yield m
    m.close()


def _run_chunk(m, dims, dtype, W, kv_lens, q_lens, seed, form, extra_rows=0):
    """One chunked prefill on the GPU and in the oracle; returns (gpu dict, oracle dict)."""
    kv_lens, q_lens = np.asarray(kv_lens), np.asarray(q_lens)
    B = len(kv_lens)
    cu_kv, cu_q = synth.cu_seqlens(kv_lens), synth.cu_seqlens(q_lens)
    total_kv, total_q = int(cu_kv[-1]), int(cu_q[-1])
    cache0 = synth.latent_cache(dims, total_kv + extra_rows, seed=seed, dtype=dtype)
    h = synth.hidden(dims, total_q, seed=seed + 1, dtype=dtype)
    ref = orc.mla_prefill_chunk(h, cu_q, cache0[:total_kv], cu_kv, W, dims)
    cache = dev(cache0, dtype)
    max_q = int(q_lens.max())
    u, chosen = m.prefill_chunk(dev(h, dtype), B, dev_i64(cu_q), max_q, dev_i64(cu_kv), total_kv, cache, form)
    _status_ok(m)
    tdt = m.torch.bfloat16 if dtype == "bf16" else m.torch.float32
    o = m.chunk_region(B, total_q, max_q, total_kv, chosen, mla.BUF_O, (total_q, dims.n_h, dims.d_h), tdt)
    got = {"u": host(u), "cache": host(cache), "o": host(o), "form": chosen}
    if chosen == mla.CHUNK_ABSORBED:
        olat = m.chunk_region(B, total_q, max_q, total_kv, chosen, mla.BUF_OLAT, (total_q, dims.n_h, dims.d_c), tdt)
        lse = m.chunk_region(B, total_q, max_q, total_kv, chosen, mla.BUF_LSE, (total_q, dims.n_h), m.torch.float32)
        got["o_lat"], got["lse"] = host(olat), host(lse)
    return got, ref, cache0


def _check(got, ref, cache0, total_kv, tol):
    assert rel(got["u"], ref["u"]) <= tol
    assert rel(got["o"], ref["o"]) <= tol
    # the chunk's rows written, the prefix rows and the rows past the last sequence untouched
    assert rel(got["cache"][:total_kv], ref["cache"]) <= tol
    rows = np.setdiff1d(np.arange(total_kv), np.flatnonzero(np.any(ref["cache"] != cache0[:total_kv], axis=1)))
    np.testing.assert_array_equal(got["cache"][rows], cache0[rows])
    np.testing.assert_array_equal(got["cache"][total_kv:], cache0[total_kv:])
    if "o_lat" in got:
        assert rel(got["o_lat"], ref["o_lat"]) <= tol
        assert rel(got["lse"], ref["lse"]) <= tol


# ---------------------------------------------------------------------------
# FP32 tiny configuration
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("q_lens,form", [([10, 30, 1], mla.CHUNK_UNABSORBED), ([3, 3, 3], mla.CHUNK_ABSORBED),
                                         ([3, 3, 3], mla.CHUNK_UNABSORBED)])
def test_tiny_chunk_fp32(q_lens, form):
    dims = synth.TINY
    W = synth.weights(dims, seed=30, dtype="fp32")
    m = make_module(dims, W, "fp32")
    kv = [64, 30, 17]
    got, ref, cache0 = _run_chunk(m, dims, "fp32", W, kv, q_lens, seed=31, form=form, extra_rows=5)
    assert got["form"] == form
    _check(got, ref, cache0, sum(kv), TOL["fp32"])
    m.close()


# ---------------------------------------------------------------------------
# BF16 at the DeepSeek-V3 sizes
# ---------------------------------------------------------------------------
def test_v3_chunk_unabsorbed_ragged_prefixes(v3_module, v3_weights):
    # chunks of 200, 77, 129, 1 and 0 tokens after prefixes of 500, 223, 0, 76 and 40 rows: query
    # tiles with ragged tails, prefixes that are not whole key tiles (the causal edge crosses a key
    # tile), a chunk that is its whole sequence, a one-token chunk and an empty one
    kv, q = [700, 300, 129, 77, 40], [200, 77, 129, 1, 0]
    got, ref, cache0 = _run_chunk(v3_module, synth.V3, "bf16", v3_weights, kv, q, seed=32, form=mla.CHUNK_AUTO,
                                  extra_rows=3)
    assert got["form"] == mla.CHUNK_UNABSORBED
    _check(got, ref, cache0, sum(kv), TOL["bf16"])


@pytest.mark.parametrize("tc,kv", [(4, [4097, 1000, 65]), (16, [2000, 129])])
def test_v3_chunk_absorbed_uniform(v3_module, v3_weights, tc, kv):
    # uniform chunks on long prefixes: the automatic choice is the absorbed form (the latent core
    # with Tq = Tc); the same inputs through the unabsorbed form must agree with the oracle as well
    q = [tc] * len(kv)
    got, ref, cache0 = _run_chunk(v3_module, synth.V3, "bf16", v3_weights, kv, q, seed=33 + tc,
                                  form=mla.CHUNK_AUTO)
    assert got["form"] == mla.CHUNK_ABSORBED
    _check(got, ref, cache0, sum(kv), TOL["bf16"])
    got2, ref2, cache02 = _run_chunk(v3_module, synth.V3, "bf16", v3_weights, kv, q, seed=33 + tc,
                                     form=mla.CHUNK_UNABSORBED)
    assert got2["form"] == mla.CHUNK_UNABSORBED
    _check(got2, ref2, cache02, sum(kv), TOL["bf16"])


def test_v3_chunk_after_prefill_equals_prefill_of_the_whole_sequence(v3_module, v3_weights):
    # prefill of the first 300 tokens, then the next 129 as a chunk on the cache that prefill wrote:
    # the chunk's outputs and cache rows equal the prefill of all 429 tokens
    dims = synth.V3
    n0, n1 = 300, 129
    h = synth.hidden(dims, n0 + n1, seed=40, dtype="bf16")
    ref = orc.mla_prefill(h, synth.cu_seqlens([n0 + n1]), v3_weights, dims, query_rows=np.arange(n0, n0 + n1))
    cache = dev(np.zeros((n0 + n1, dims.row)), "bf16")
    v3_module.prefill(dev(h[:n0], "bf16"), 1, dev_i64(synth.cu_seqlens([n0])), n0, cache)
    _status_ok(v3_module)
    u, chosen = v3_module.prefill_chunk(dev(h[n0:], "bf16"), 1, dev_i64(synth.cu_seqlens([n1])), n1,
                                        dev_i64(synth.cu_seqlens([n0 + n1])), n0 + n1, cache)
    _status_ok(v3_module)
    assert chosen == mla.CHUNK_UNABSORBED
    assert rel(host(u), ref["u"]) <= TOL["bf16"]
    assert rel(host(cache), ref["cache"]) <= TOL["bf16"]
