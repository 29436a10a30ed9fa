"""mla_cache_append_noalloc: the cache append for callers that cannot allocate device memory
(code inside a stream capture that forbids allocation, runtimes with their own fixed pool,
plain C callers without an allocator). It takes no workspace; its scratch is a fixed 4 MiB
array inside the library. These checks compare it with mla_cache_append, which takes a
caller-provided workspace, on two calls in a row, and check the size limit.

This file is named so that pytest collects it last; it builds its own handle and inputs, so it
also runs alone in a fresh process.
"""
import numpy as np
import pytest

from mla_testlib import TOL, dev, dev_i64, host, make_module, mla, rel, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def module():
    W = synth.weights(synth.V3, seed=91, dtype="bf16")
    m = make_module(synth.V3, W, "bf16")
    yield m
    m.close()


def _append_both(m, T, cap, seed):
    dims = synth.V3
    h = dev(synth.hidden(dims, T, seed=seed, dtype="bf16"), "bf16")
    pos = dev_i64(np.arange(T) * 7 + seed)
    slots = dev_i64(np.random.default_rng(seed).permutation(cap)[:T])
    ref = dev(np.zeros((cap, dims.row)), "bf16")
    m.cache_append(h, pos, slots, ref)                      # workspace-based entry point
    got = dev(np.zeros((cap, dims.row)), "bf16")
    mla.mla_cache_append_noalloc(m.handle, h, pos, slots, T, got, cap, device=m.device)
    assert m.sync_status() == 0
    return host(ref), host(got)


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row(module):
    # two calls back to back, different inputs: the shared array holds the first call's partials
    # when the second one runs, so a stale read would show up here
    for seed, T in ((1, 16), (2, 40)):
        ref, got = _append_both(module, T, 200, seed)
        assert np.any(ref != 0)
        assert rel(got, ref) <= TOL["bf16"]


def test_noalloc_rejects_requests_beyond_its_scratch(module):
    dims = synth.V3
    T, cap = 100, 128          # needs about 6.5 MB of split-K scratch at these sizes
    h = dev(np.zeros((T, dims.d)), "bf16")
    idx = dev_i64(np.arange(T))
    cache = dev(np.zeros((cap, dims.row)), "bf16")
    with pytest.raises(mla.MLAError) as e:
        mla.mla_cache_append_noalloc(module.handle, h, idx, idx, T, cache, cap, device=module.device)
    assert mla.STATUS_NAMES[e.value.status] == "MLA_ERR_SCRATCH_LIMIT"
    assert not bool(cache.any())
