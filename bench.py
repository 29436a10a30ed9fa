#!/usr/bin/env python
"""Benchmark of the MLA latent-cache hot path on B200; prints one JSON line on rank 0.

A step is one pass of the decode hot path over one batch: mla_cache_append of the batch's
new tokens (down-projection, RoPE on k^R, cache write) followed by mla_decode (query
projections, W^UK folded into the query, the split-KV latent core with its log-sum-exp
merge, W^UV after attention, W^O). The workload is the DeepSeek-V3-shaped decode batch of
16 sequences with 4096 cached rows each (synthetic, seeded; weights ~ N(0, 1/fan_in)).

Timing: each step is replayed from a CUDA graph and bracketed by CUDA events on the
launching stream, with a 2x-L2 write between steps (outside the events) so the cache is
read from HBM. Under torchrun every rank runs its own batch (weak scaling, no collective on
the data path); the reported time is the max over ranks.

--impl reference times the CPU float64 oracle (the unabsorbed definition) on a bounded
sample of the same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mla_latent_kv_31_b200 import synth  # noqa: E402

METRIC = "MLA decode latent-cache GB/s & tokens/s; prefill TFLOP/s; % of B200 roofline"
WORKLOAD = synth.WORKLOADS["decode_b16_l4096"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CORE_FLOP_PER_ROW = 128 * 2 * (576 + 512)   # per cached row and query token: n_h * 2 * (d_c + d_R + d_c)
ROW_BYTES = 576 * 2
PREFILL = synth.WORKLOADS["prefill_l32768"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--oracle-seconds", type=float, default=12.0, help="CPU time budget of the oracle sample")
    ap.add_argument("--prefill-iters", type=int, default=5, help="timed prefill calls (0: no prefill leg)")
    ap.add_argument("--prefill-seq-len", type=int, default=PREFILL.length,
                    help="prefill sequence length (default: the 32K-token workload; smaller for profiling)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def recorded_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu record (profiles/kernel_traffic.json),
    or None when there is none or the kernel's source has changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "kernel_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != rec["source_sha256"]:
                return None
        return int(rec["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity on one rank). Every rank must call
    it at the same point. device: where the reduction tensor lives (the rank's GPU for NCCL, CPU for
    gloo)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(world: int, units_per_rank: float, seconds_max: float) -> float:
    """Units all ranks processed per second of the slowest rank (weak scaling: every rank does the
    same amount of work on its own inputs)."""
    return world * units_per_rank / seconds_max


def workload_config():
    d = WORKLOAD.dims
    return {"workload": WORKLOAD.name, "batch": WORKLOAD.batch, "query_tokens_per_seq": WORKLOAD.tq,
            "cache_len": WORKLOAD.length, "d": d.d, "n_h": d.n_h, "d_h": d.d_h, "d_c": d.d_c, "d_cq": d.d_cq,
            "d_r": d.d_r, "seed": 0}


# ---------------------------------------------------------------------------------------------
# CPU baseline: the float64 oracle on a bounded sample of the workload
# ---------------------------------------------------------------------------------------------
def oracle_sample(seconds: float):
    from threadpoolctl import threadpool_info

    from oracle import mla_oracle as orc
    dims, L, tq = WORKLOAD.dims, WORKLOAD.length, WORKLOAD.tq
    W = synth.weights(dims, seed=0, dtype="bf16")
    n_seq = WORKLOAD.batch
    cu = synth.cu_seqlens(np.full(n_seq, L))
    cache = synth.latent_cache(dims, int(cu[-1]), seed=0, dtype="bf16")
    h_q = synth.hidden(dims, n_seq * tq, seed=0, dtype="bf16")
    done = 0
    t0 = time.perf_counter()
    while done < n_seq:
        orc.mla_decode(h_q, cache, cu, tq, W, dims, seqs=[done])
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    gbs = done * L * ROW_BYTES / dt / 1e9
    return {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} of {n_seq} sequences (all {dims.n_h} heads, u included), float64 unabsorbed "
                      f"definition, {dt:.1f} s", "tokens_per_s": done * tq / dt, "seconds": dt}


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device), f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1].split()[0]))
                    smax.append(float(parts[2].split()[0]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------------------------
def kernel_only_ms(fn, which, iters, warm, flush, world):
    """Average duration of the library's attention-core launch inside fn() (CUDA events the library
    records right around that launch, on its stream), each call after an L2 flush; max over ranks."""
    import torch
    from mla_latent_kv_31_b200 import mla
    mla.mla_set_kernel_timing(True)
    try:
        for _ in range(warm):
            flush.zero_()
            fn()
        tot = 0.0
        for _ in range(iters):
            flush.zero_()
            fn()
            tot += mla.mla_kernel_time_ms(which)
    finally:
        torch.cuda.synchronize()
        mla.mla_set_kernel_timing(False)
    return max_over_ranks([tot / iters], flush.device)[0]


def prefill_flops(dims, lens):
    """FLOPs of one prefill: the unabsorbed attention minimum 2 (d_h + d_R + d_h) n_h per causal (q, k)
    pair, and the projection GEMMs (W^DKV|W^KR, W^DQ, W^UQ|W^QR, W^UK|W^UV, W^O) at 2 flops per MAC."""
    pairs = sum(L * (L + 1) // 2 for L in lens)
    attn = pairs * dims.n_h * 2 * (dims.d_h + dims.d_r + dims.d_h)
    T = sum(lens)
    hd = dims.n_h * dims.d_h
    proj = 2 * T * (dims.d * (dims.d_c + dims.d_r) + dims.d * dims.d_cq +
                    dims.d_cq * (hd + dims.n_h * dims.d_r) + dims.d_c * 2 * hd + hd * dims.d)
    return attn, proj


def run_prefill(args, m, dev, rank, world, flush, timed, peaks, peak_src):
    """Prefill of one 32K-token sequence (B = 1): the whole mla_prefill and the attention core alone
    (mla_attn_prefill on the q^C, q^R, k^C, v^C that mla_prefill left in its workspace)."""
    import torch
    from mla_latent_kv_31_b200 import mla
    L = args.prefill_seq_len
    dims, T = PREFILL.dims, PREFILL.batch * L
    lens = [L] * PREFILL.batch
    h = m.handle
    hid = torch.from_numpy(synth.hidden(dims, T, seed=rank)).to(dev, torch.bfloat16)
    cu = torch.from_numpy(synth.cu_seqlens(lens)).to(dev)
    cache = torch.zeros(T, dims.row, dtype=torch.bfloat16, device=dev)
    u = torch.empty(T, dims.d, dtype=torch.bfloat16, device=dev)
    n = mla.mla_workspace_size(h, mla.OP_PREFILL, PREFILL.batch, 1, T)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    assert mla.mla_uses_tensor_cores(h, mla.OP_PREFILL)
    reg = lambda which: ws.data_ptr() + mla.mla_workspace_offset(h, mla.OP_PREFILL, which, PREFILL.batch, 1, T)  # noqa
    o = torch.empty(T, dims.n_h, dims.d_h, dtype=torch.bfloat16, device=dev)

    def full():
        mla.mla_prefill(h, hid, PREFILL.batch, cu, T, L, cache, T, u, ws, n, device=dev.index)

    def core():
        mla.mla_attn_prefill(h, reg(mla.BUF_QC), reg(mla.BUF_QR), reg(mla.BUF_KC), reg(mla.BUF_VC), PREFILL.batch, cu,
                             T, L, cache, T, o, device=dev.index)

    full()
    core()
    torch.cuda.synchronize()
    st = mla.mla_sync_status(h, device=dev.index)
    if st != 0:
        raise RuntimeError(f"device check failed in prefill: {mla.mla_status_string(st)}")
    l0 = mla.mla_kernel_launches()
    full()
    launches = mla.mla_kernel_launches() - l0
    clock = ClockSampler(dev.index)
    clock.start()
    ms_full = timed(full, args.prefill_iters, 3)
    ms_core = timed(core, args.prefill_iters, 3)
    ms_kernel = kernel_only_ms(core, mla.TIMED_PREFILL_CORE, args.prefill_iters, 1, flush, world)
    clocks = clock.stop()
    st = mla.mla_sync_status(h, device=dev.index)
    if st != 0:
        raise RuntimeError(f"device check failed after prefill timing: {mla.mla_status_string(st)}")
    ms_full, ms_core = max_over_ranks([ms_full, ms_core], dev)
    attn, proj = prefill_flops(dims, lens)
    sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    core_tf = attn / (ms_core * 1e-3) / 1e12
    kern_tf = attn / (ms_kernel * 1e-3) / 1e12
    full_tf = (attn + proj) / (ms_full * 1e-3) / 1e12
    return {
        "workload": PREFILL.name if L == PREFILL.length else f"prefill_l{L}", "batch": PREFILL.batch, "seq_len": L,
        "call": "mla_prefill (cache append, query projections, k^C/v^C up-projection, causal attention, W^O)",
        "ms": round(ms_full, 3), "tflops": round(world * full_tf, 1), "tokens_per_s": round(world * T / (ms_full * 1e-3), 1),
        "flops_per_call": attn + proj, "gpu_launches_per_call": int(launches), "clocks": clocks,
        "step_roofline": {"bound": "tensor", "achieved": round(full_tf, 1), "peak": sus, "unit": "TFLOP/s",
                          "frac": round(full_tf / sus, 4), "peak_source": f"{peak_src} sustained"},
        "core": {"call": "mla_attn_prefill", "ms": round(ms_core, 3), "tflops": round(core_tf, 1), "flops": attn,
                 "kernel_ms": round(ms_kernel, 3),
                 "roofline": {"bound": "tensor", "achieved": round(kern_tf, 1), "peak": sus, "unit": "TFLOP/s",
                              "frac": round(kern_tf / sus, 4), "frac_of_burst_peak": round(kern_tf / burst, 4),
                              "traffic": recorded_traffic("prefill_attn_kernel") if L == PREFILL.length else None,
                              "kernel": "prefill_attn_kernel",
                              "peak_source": f"{peak_src} sustained (the call runs for tens of ms)"}},
    }


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from mla_latent_kv_31_b200 import mla
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dims, B, L, tq = WORKLOAD.dims, WORKLOAD.batch, WORKLOAD.length, WORKLOAD.tq
    T = B * tq
    W = {k: torch.from_numpy(v).to(dev, torch.bfloat16) for k, v in synth.weights(dims, seed=0).items()}
    m = mla.MLA(dims, W, mla.MLA_BF16, device=local_rank)
    h = m.handle
    lens = np.full(B, L, dtype=np.int64)
    cu_np = synth.cu_seqlens(lens)
    rows = int(cu_np[-1])
    cache = torch.from_numpy(synth.latent_cache(dims, rows, seed=rank)).to(dev, torch.bfloat16)
    h_np = synth.hidden(dims, T, seed=rank)
    pos_np = np.concatenate([np.arange(L - tq, L) for _ in range(B)]).astype(np.int64)
    slots_np = np.concatenate([cu_np[b] + np.arange(L - tq, L) for b in range(B)]).astype(np.int64)
    # device inputs
    h_dev = torch.from_numpy(h_np).to(dev, torch.bfloat16)
    cu_dev = torch.from_numpy(cu_np).to(dev)
    pos_dev = torch.from_numpy(pos_np).to(dev)
    slots_dev = torch.from_numpy(slots_np).to(dev)
    u_dev = torch.empty(T, dims.d, dtype=torch.bfloat16, device=dev)
    ws_app_n = mla.mla_workspace_size(h, mla.OP_CACHE_APPEND, 0, 1, T)
    ws_dec_n = mla.mla_workspace_size(h, mla.OP_DECODE, B, tq, 0)
    ws_core_n = mla.mla_workspace_size(h, mla.OP_ATTN_DECODE_LATENT, B, tq, 0)
    ws_app = torch.empty(max(ws_app_n, 1024), dtype=torch.uint8, device=dev)
    ws_dec = torch.empty(ws_dec_n, dtype=torch.uint8, device=dev)
    ws_core = torch.empty(ws_core_n, dtype=torch.uint8, device=dev)
    assert mla.mla_uses_tensor_cores(h, mla.OP_DECODE) and mla.mla_uses_tensor_cores(h, mla.OP_ATTN_DECODE_LATENT)

    def step():
        mla.mla_cache_append(h, h_dev, pos_dev, slots_dev, T, cache, rows, ws_app, ws_app_n, device=local_rank)
        mla.mla_decode(h, h_dev, B, tq, cu_dev, cache, rows, u_dev, ws_dec, ws_dec_n, device=local_rank)

    # the latent core alone, on the q~ / q^R the decode step produced
    off_qabs = mla.mla_workspace_offset(h, mla.OP_DECODE, mla.BUF_QABS, B, tq, 0)
    off_qr = mla.mla_workspace_offset(h, mla.OP_DECODE, mla.BUF_QR, B, tq, 0)
    q_abs = ws_dec[off_qabs:off_qabs + T * dims.n_h * dims.d_c * 2]
    q_rope = ws_dec[off_qr:off_qr + T * dims.n_h * dims.d_r * 2]
    o_lat = torch.empty(T, dims.n_h, dims.d_c, dtype=torch.float32, device=dev)
    lse = torch.empty(T, dims.n_h, dtype=torch.float32, device=dev)

    def core():
        mla.mla_attn_decode_latent(h, q_abs.data_ptr(), q_rope.data_ptr(), B, tq, cu_dev, cache, rows, o_lat, lse,
                                   ws_core, ws_core_n, device=local_rank)

    # warm-up eagerly once (first-use attribute setup), check status, then capture graphs
    step()
    core()
    torch.cuda.synchronize()
    st = mla.mla_sync_status(h, device=local_rank)
    if st != 0:
        raise RuntimeError(f"device check failed: {mla.mla_status_string(st)}")
    g_step, g_core = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, capture_error_mode="relaxed"):
        step()
    with torch.cuda.graph(g_core, capture_error_mode="relaxed"):
        core()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, iters, warm, pre=None):
        for _ in range(warm):
            flush.zero_()
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        for a, b in ev:
            flush.zero_()
            if pre:
                pre()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return sum(a.elapsed_time(b) for a, b in ev) / iters

    launches0 = mla.mla_kernel_launches()
    step()
    per_step_launches = mla.mla_kernel_launches() - launches0
    clock = ClockSampler(local_rank)
    clock.start()
    t_wall = time.perf_counter()
    ms_step = timed(g_step.replay, args.steps, args.warmup)
    wall = time.perf_counter() - t_wall
    clocks = clock.stop()
    ms_core = timed(g_core.replay, max(200, args.steps // 4), args.warmup)
    # end to end: pinned host inputs in, u out, every step
    h_host = torch.from_numpy(h_np).to(torch.bfloat16).pin_memory()
    pos_host, slots_host, cu_host = (torch.from_numpy(x).pin_memory() for x in (pos_np, slots_np, cu_np))
    u_host = torch.empty(T, dims.d, dtype=torch.bfloat16).pin_memory()

    def e2e():
        h_dev.copy_(h_host, non_blocking=True)
        pos_dev.copy_(pos_host, non_blocking=True)
        slots_dev.copy_(slots_host, non_blocking=True)
        cu_dev.copy_(cu_host, non_blocking=True)
        g_step.replay()
        u_host.copy_(u_dev, non_blocking=True)

    ms_e2e = timed(e2e, max(200, args.steps // 4), args.warmup)
    del g_step, g_core
    ms_kernel = kernel_only_ms(core, mla.TIMED_LATENT_CORE, max(200, args.steps // 4), args.warmup, flush, world)
    peaks, peak_src = load_peaks()
    prefill = (run_prefill(args, m, dev, rank, world, flush, timed, peaks, peak_src) if args.prefill_iters > 0
               else {"status": "skipped (--prefill-iters 0)"})
    st = mla.mla_sync_status(h, device=local_rank)
    if st != 0:
        raise RuntimeError(f"device check failed after timing: {mla.mla_status_string(st)}")
    ms_step_max, ms_core_max, ms_e2e_max = max_over_ranks([ms_step, ms_core, ms_e2e], dev)
    if rank != 0:
        return None
    cache_bytes = rows * ROW_BYTES
    weight_bytes = sum(v.numel() * 2 for v in W.values())
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    core_gbs = cache_bytes / (ms_core_max * 1e-3) / 1e9
    kern_gbs = cache_bytes / (ms_kernel * 1e-3) / 1e9
    core_tflops = rows * tq * CORE_FLOP_PER_ROW / (ms_core_max * 1e-3) / 1e12
    step_bytes = cache_bytes + weight_bytes
    value = whole_job_rate(world, cache_bytes, ms_step_max * 1e-3) / 1e9
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step_max, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) cache and hidden states, "
        "N(0,1/fan_in) weights, DeepSeek-V3 sizes)",
        "config": dict(workload_config(), parallelism=f"replicas{world}", l2="flushed between steps (2x L2 write)",
                       step="mla_cache_append + mla_decode, CUDA-graph replay"),
        "tokens_per_s": round(whole_job_rate(world, T, ms_step_max * 1e-3), 1),
        "step_hbm_bytes": step_bytes,
        "step_roofline": {"bound": "hbm", "achieved": round(step_bytes / (ms_step_max * 1e-3) / 1e9, 1),
                          "peak": hbm, "unit": "GB/s", "frac": round(step_bytes / (ms_step_max * 1e-3) / 1e9 / hbm, 4),
                          "note": f"cache {cache_bytes} B + weights {weight_bytes} B per step, {peak_src} peak"},
        "latent_core": {"ms": round(ms_core_max, 5), "gbs": round(core_gbs, 1), "tflops": round(core_tflops, 1),
                        "call": "mla_attn_decode_latent (device check + plan + core + combine), CUDA-graph replay"},
        "roofline": {"bound": "hbm", "achieved": round(kern_gbs, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(kern_gbs / hbm, 4), "traffic": recorded_traffic("latent_core_kernel"),
                     "kernel": "latent_core_kernel", "kernel_ms": round(ms_kernel, 5),
                     "timing": "CUDA events recorded by the library right around the kernel launch, L2 flushed",
                     "algorithmic_bytes": cache_bytes, "peak_source": peak_src},
        "e2e": {"value": round(whole_job_rate(world, cache_bytes, ms_e2e_max * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(ms_e2e_max, 5),
                "h2d_bytes_per_step": int(h_np.size * 2 + pos_np.nbytes + slots_np.nbytes + cu_np.nbytes),
                "d2h_bytes_per_step": int(T * dims.d * 2)},
        "gpu_launches": int(per_step_launches * args.steps),
        "gpu_launches_per_step": int(per_step_launches),
        "clocks": clocks,
        "timed_wall_s": round(wall, 3),
        "prefill": prefill,
    }
    return out


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        cpu = oracle_sample(args.oracle_seconds)
        line = {"impl": "reference", "metric": METRIC, "value": round(cpu["value"], 4), "unit": "GB/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": dict(workload_config(), parallelism="cpu"),
                "cpu_baseline": cpu,
                "e2e": {"value": round(cpu["value"], 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    out = run_ours(args, rank, world, local_rank)
    if rank == 0:
        cpu = oracle_sample(args.oracle_seconds) if world == 1 else None
        if cpu:
            out["cpu_baseline"] = cpu
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    del torch
    return 0


if __name__ == "__main__":
    sys.exit(main())
