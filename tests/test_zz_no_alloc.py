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

from mla_testlib import TOL, dev, dev_i64, host, make_module, mla, orc, rel, synth

pytestmark = pytest.mark.gpu

SEED_W = 91


@pytest.fixture(scope="module")
def module():
    W = synth.weights(synth.V3, seed=SEED_W, dtype="bf16")
    m = make_module(synth.V3, W, "bf16")
    yield m
    m.close()


def _append_both(m, T, cap, seed):
    dims = synth.V3
    h_np = synth.hidden(dims, T, seed=seed, dtype="bf16")
    pos_np = np.arange(T) * 7 + seed
    slots_np = np.random.default_rng(seed).permutation(cap)[:T]
    h, pos, slots = dev(h_np, "bf16"), dev_i64(pos_np), dev_i64(slots_np)
    ref = dev(np.zeros((cap, dims.row)), "bf16")
    m.cache_append(h, pos, slots, ref)                      # workspace-based entry point
    got = dev(np.zeros((cap, dims.row)), "bf16")
    mla.mla_cache_append_noalloc(m.handle, h, pos, slots, T, got, cap, device=m.device)
    assert m.sync_status() == 0
    return ref, got, (h_np, pos_np, slots_np)


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row(module):
    # two calls back to back, different inputs: the shared array holds the first call's partials
    # when the second one runs, so a stale read would show up here. Both entry points launch the
    # same kernels with the same split-K layout and a fixed-order reduction, so the rows they write
    # must be equal bit for bit, not just within the bf16 tolerance.
    W = synth.weights(synth.V3, seed=SEED_W, dtype="bf16")
    for seed, T in ((1, 16), (2, 40)):
        ref, got, (h_np, pos_np, slots_np) = _append_both(module, T, 200, seed)
        assert bool(ref.any())
        assert bool(module.torch.equal(got, ref))
        # and one check of the rows themselves against the oracle's steps (5) and (7)
        rows = orc.cache_append(h_np, pos_np, W, synth.V3)
        assert rel(host(got)[slots_np], rows) <= TOL["bf16"]


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
