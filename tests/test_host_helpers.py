"""Host-side helpers the tests and the benchmark rely on: the seeded generator draws the same values
however its chunks are scheduled, and the benchmark reports recorded ncu traffic only for the kernel
source it was taken from."""
import json

import numpy as np

import bench
from mla_latent_kv_31_b200 import synth


def test_threaded_draw_equals_sequential_draw():
    n = 2 * synth._CHUNK + 12345          # several chunks, so the thread pool is used
    got = synth.normal(7, synth.TID_CACHE_C, (n,), std=0.5, dtype="bf16")
    want = np.empty(n, dtype=np.float32)
    for lo in range(0, n, synth._CHUNK):
        hi = min(n, lo + synth._CHUNK)
        want[lo:hi] = synth.round_to(synth.normal_f64(7, synth.TID_CACHE_C, hi - lo, start=lo) * 0.5, "bf16")
    assert np.array_equal(got, want)


def test_draws_are_counter_based_any_window_matches():
    a = synth.normal_f64(3, synth.TID_H, 1000)
    b = synth.normal_f64(3, synth.TID_H, 100, start=450)
    assert np.array_equal(a[450:550], b)


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("// kernel\n")
    import hashlib
    rec = {"k": {"source": str(src), "source_sha256": hashlib.sha256(src.read_bytes()).hexdigest(),
                 "dram_bytes_per_launch": 1234}}
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "kernel_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k") == 1234
    assert bench.recorded_traffic("other") is None
    src.write_text("// kernel, changed\n")
    assert bench.recorded_traffic("k") is None


def test_torch_draws_equal_numpy_draws():
    # the benchmark fills its large caches with the torch form of the same generator
    for dt in ("bf16", "fp32"):
        a = synth.normal(5, synth.TID_CACHE_KR, (300, 77), std=1.5, dtype=dt)
        b = synth.normal_torch(5, synth.TID_CACHE_KR, (300, 77), std=1.5, dtype=dt).float().numpy()
        assert np.array_equal(a, b)
    c = synth.latent_cache_torch(synth.TINY, 50, seed=2).float().numpy()
    assert np.array_equal(c, synth.latent_cache(synth.TINY, 50, seed=2))
