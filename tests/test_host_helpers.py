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


def test_fp8_row_packing_of_the_parity_tests():
    """The 656-byte rows the FP8 parity tests build from the oracle's quantizer: the code bytes are
    torch's own float8_e4m3fn encoding of the code values, k^R / s and s are their f16 / fp32 bytes,
    the padding is zero, unpacking gives the values back, and quantizing in blocks changes nothing."""
    import torch
    from mla_testlib import fp8_cache, fp8_decode_rows, fp8_encode_rows, orc, round_bf16
    rng = np.random.default_rng(11)
    rows = rng.standard_normal((300, 576)) * 10.0 ** rng.integers(-6, 7, size=300)[:, None]
    rows[3] = 0.0
    rows[5, 512:] *= 1e5                        # k^R sets the scale: c^KV / s in the e4m3 subnormals
    rows = round_bf16(rows)
    codes, kr, s = orc.quantize_cache_rows_fp8(rows, synth.V3)
    raw = fp8_encode_rows(codes, kr, s)
    assert raw.shape == (300, 656)
    want = torch.from_numpy(codes.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    same_value = (raw[:, :512] == want) | ((raw[:, :512] & 0x7F) == 0) & ((want & 0x7F) == 0)
    assert np.all(same_value)                   # +0 and -0 may differ in sign only
    assert np.array_equal(raw[:, 512:640].view(np.float16).astype(np.float64), kr)
    assert np.array_equal(raw[:, 640:644].view(np.float32)[:, 0].astype(np.float64), s)
    assert not raw[:, 644:].any()
    vals, kr2, s2, pad = fp8_decode_rows(raw)
    assert np.array_equal(vals, codes) and np.array_equal(kr2, kr) and np.array_equal(s2, s) and not pad.any()
    raw_b, deq_b = fp8_cache(rows, synth.V3, chunk=37)
    assert np.array_equal(raw_b, raw)
    assert np.array_equal(deq_b, orc.dequantize_cache_rows_fp8(codes, kr, s))


def test_algorithmic_costs_the_rooflines_divide_by():
    """The per-unit costs behind every roofline fraction of the bench line, against their closed forms
    at the DeepSeek-V3 sizes: a cached row is 576 bf16 (1152 B) or one 656-byte FP8 row; the latent
    core spends n_h * 2 * (576 + 512) flops per (query token, visible row); the unabsorbed prefill
    attention 2 * (192 + 128) flops per causal pair and head (43.98 TFLOP at 32768 tokens) and its
    five projection GEMMs 2 flops per MAC (12.26 TFLOP at 32768 tokens)."""
    d = synth.V3
    assert bench.ROW_BYTES == (d.d_c + d.d_r) * 2 == 1152
    assert bench.FP8_ROW_BYTES == d.d_c + 2 * d.d_r + 4 + 12 == 656
    assert bench.CORE_FLOP_PER_ROW == d.n_h * 2 * ((d.d_c + d.d_r) + d.d_c) == 278528
    # decode_b16_l4096: one query token per sequence sees all 4096 rows
    assert bench.core_flops([4096] * 16, 1) == 16 * 4096 * 278528 == 18_253_611_008
    # two query tokens: the first sees L - 1 rows, the second all L
    lens = [5, 2, 33]
    assert bench.core_flops(lens, 2) == sum((L - 1) + L for L in lens) * 278528
    attn, proj = bench.prefill_flops(d, [32768])
    assert attn == 32768 * 32769 // 2 * d.n_h * 2 * (2 * d.d_h + d.d_r)
    assert abs(attn / 1e12 - 43.98) < 0.005
    hd = d.n_h * d.d_h
    macs_per_token = (d.d * (d.d_c + d.d_r) + d.d * d.d_cq + d.d_cq * (hd + d.n_h * d.d_r) + 2 * d.d_c * hd
                      + hd * d.d)
    assert proj == 2 * 32768 * macs_per_token
    assert abs(proj / 1e12 - 12.26) < 0.005
    # two sequences: pairs add per sequence, projections per token
    a2, p2 = bench.prefill_flops(d, [3, 4])
    assert a2 == (6 + 10) * d.n_h * 2 * (2 * d.d_h + d.d_r) and p2 == 2 * 7 * macs_per_token


def test_clock_sampler_reads_the_nvidia_smi_fallback(tmp_path):
    """Without NVML the sampler reads nvidia-smi's CSV: the median SM clock under load, the maximum,
    and the union of the clock-event reasons it names (0x40 | 0x4: thermal slowdown and power cap);
    malformed lines are skipped."""
    import threading
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.device, s.samples, s.smax, s.nvml, s.thread = 0, [], None, None, None
    s.stop_ev = threading.Event()
    path = tmp_path / "clocks.csv"
    path.write_text("1965, 1965, 0x0000000000000000\n1800, 1965, 0x0000000000000004\nnot a sample\n"
                    "1327, 1965, 0x0000000000000044\n")

    class Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    s.proc, s.path = Proc(), str(path)
    out = s.stop()
    assert out["samples"] == 3 and out["sm_mhz"] == 1800.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert out["source"] == "nvidia-smi 200 ms"
    assert not path.exists()
