"""Seeded synthetic inputs for the MLA latent-cache path.

This module holds no part of the attention arithmetic: it only draws
numbers. Both the CUDA path's tests/bench and the CPU oracle consume what it
returns, so the two sides see bit-identical inputs.

Generator (counter based, so any element can be drawn on its own):
  * SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): state_n = key + (n + 1) * 0x9E3779B97F4A7C15,
    output = mix64(state_n) with the published finaliser constants.
  * key(seed, tensor_id) = mix64((seed << 32) + tensor_id), one independent
    stream per tensor.
  * uniform(n) = (u64(n) >> 11) * 2^-53 in [0, 1).
  * normal(i) by Box-Muller on the pair of uniforms (2i, 2i+1):
    sqrt(-2 ln(1 - a)) * cos(2 pi b), in float64, then scaled by std.
  * Rounding to the input dtype: float64 -> float32 (round to nearest even),
    then for bf16 float32 -> bf16 (round to nearest even). Values are
    returned as float32 arrays that hold the rounded values exactly.

Workload recipes follow the DeepSeek-V3 model hyper-parameters (the notes
"【论文解读】DeepSeek-V3", section 三(二)1 "model hyper-parameters": d = 7168,
n_h = 128, d_h = 128, d_c = 512, d_c' = 1536, d_h^R = 64) and the decode /
prefill shapes listed in WORKLOADS below.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Tensor ids: one stream per named input.
TID_H, TID_WDQ, TID_WUQ, TID_WQR, TID_WDKV, TID_WKR, TID_WUK, TID_WUV, TID_WO = range(9)
TID_CACHE_C, TID_CACHE_KR, TID_LENGTHS = 9, 10, 11
TID_POSITIONS, TID_SLOTS = 12, 13
TID_QC, TID_QR, TID_KC, TID_VC = 14, 15, 16, 17   # inputs of the prefill attention core alone
TID_GQ, TID_GKV = 18, 19                          # RMSNorm gains of c^Q and c^KV

_CHUNK = 1 << 22


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> np.uint64:
    with np.errstate(over="ignore"):
        base = np.array([(int(seed) << 32) + int(tensor_id)], dtype=np.uint64)
        return _mix64(base + _GAMMA)[0]


def u64(seed: int, tensor_id: int, counters: np.ndarray) -> np.ndarray:
    """Raw 64-bit draws for the given counters of stream (seed, tensor_id)."""
    key = stream_key(seed, tensor_id)
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + (c + np.uint64(1)) * _GAMMA)


def _uniform(seed, tensor_id, counters):
    return (u64(seed, tensor_id, counters) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal_f64(seed: int, tensor_id: int, n: int, start: int = 0) -> np.ndarray:
    """N(0,1) draws for element indices [start, start+n), float64."""
    out = np.empty(n, dtype=np.float64)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        idx = np.arange(start + lo, start + hi, dtype=np.uint64)
        a = _uniform(seed, tensor_id, idx * np.uint64(2))
        b = _uniform(seed, tensor_id, idx * np.uint64(2) + np.uint64(1))
        out[lo:hi] = np.sqrt(-2.0 * np.log1p(-a)) * np.cos(2.0 * np.pi * b)
    return out


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to 'fp32' or 'bf16'; returns float32 holding them."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    if dtype == "fp32":
        return f
    if dtype != "bf16":
        raise ValueError(f"unknown dtype {dtype!r}")
    bits = f.view(np.uint32).astype(np.uint64)
    rounded = (bits + np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return (rounded.astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal(seed: int, tensor_id: int, shape, std: float = 1.0, dtype: str = "bf16", mean: float = 0.0) -> np.ndarray:
    """N(mean, std^2) draws rounded to dtype. Chunks are independent (counter based), so they are drawn
    on a thread pool; the values do not depend on the number of threads."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)

    def fill(lo):
        hi = min(n, lo + _CHUNK)
        out[lo:hi] = round_to(normal_f64(seed, tensor_id, hi - lo, start=lo) * std + mean, dtype)

    starts = range(0, n, _CHUNK)
    if n <= _CHUNK:
        for lo in starts:
            fill(lo)
    else:
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    return out.reshape(shape)


def _signed(x: int) -> int:
    return x - (1 << 64) if x >= (1 << 63) else x


def normal_torch(seed: int, tensor_id: int, shape, std: float = 1.0, dtype: str = "bf16", device="cpu"):
    """The same draws as normal(), computed with torch on `device` (a GPU fills large synthetic caches in
    milliseconds). uint64 arithmetic is done on int64 tensors: two's-complement products and sums wrap
    exactly like uint64, and a logical right shift is an arithmetic shift with the sign bits masked off.
    Returns a torch tensor of the dtype ('bf16' -> bfloat16, 'fp32' -> float32)."""
    import torch
    n = int(np.prod(shape))
    key = torch.tensor(_signed(int(stream_key(seed, tensor_id))), dtype=torch.int64, device=device)
    gamma = _signed(int(_GAMMA))
    m1, m2 = _signed(int(_M1)), _signed(int(_M2))

    def shr(z, k):
        return (z >> k) & ((1 << (64 - k)) - 1)

    def mix(z):
        z = (z ^ shr(z, 30)) * m1
        z = (z ^ shr(z, 27)) * m2
        return z ^ shr(z, 31)

    def uniform(c):
        return shr(mix(key + (c + 1) * gamma), 11).to(torch.float64) * (2.0 ** -53)

    out = torch.empty(n, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device=device)
    step = 1 << 24
    for lo in range(0, n, step):
        hi = min(n, lo + step)
        idx = torch.arange(lo, hi, dtype=torch.int64, device=device)
        a = uniform(2 * idx)
        b = uniform(2 * idx + 1)
        x = torch.sqrt(-2.0 * torch.log1p(-a)) * torch.cos(2.0 * np.pi * b) * std
        out[lo:hi] = x.to(torch.float32).to(out.dtype)
    return out.reshape(shape)


def latent_cache_torch(dims: "Dims", rows: int, seed: int = 0, dtype: str = "bf16", device="cpu"):
    """latent_cache() drawn with torch on `device`: [rows, d_c + d_r], c^KV then k^R, each ~ N(0,1)."""
    import torch
    c = normal_torch(seed, TID_CACHE_C, (rows, dims.d_c), dtype=dtype, device=device)
    kr = normal_torch(seed, TID_CACHE_KR, (rows, dims.d_r), dtype=dtype, device=device)
    return torch.cat([c, kr], dim=1)


@dataclass(frozen=True)
class Dims:
    """MLA dimensions in the notes' symbols: d, n_h, d_h, d_c, d_c' (d_cq), d_h^R (d_r)."""
    d: int
    n_h: int
    d_h: int
    d_c: int
    d_cq: int
    d_r: int
    rope_base: float = 10000.0
    # YaRN context extension of the decoupled RoPE (s = 1: plain RoPE) and its original context
    yarn_s: float = 1.0
    yarn_alpha: float = 1.0
    yarn_beta: float = 32.0
    yarn_l0: int = 4096
    rms_eps: float = 1e-6       # RMSNorm epsilon (the norm is on when the weights carry its gains)

    @property
    def row(self) -> int:
        """Elements per latent-cache row: [c^KV (d_c) | k^R (d_r)]."""
        return self.d_c + self.d_r


TINY = Dims(d=256, n_h=4, d_h=32, d_c=64, d_cq=96, d_r=16)
V3 = Dims(d=7168, n_h=128, d_h=128, d_c=512, d_cq=1536, d_r=64)
# the DeepSeek-V3 long-context settings: YaRN with s = 40, alpha = 1, beta = 32 from a 4K context
V3_YARN = Dims(d=7168, n_h=128, d_h=128, d_c=512, d_cq=1536, d_r=64, yarn_s=40.0, yarn_alpha=1.0, yarn_beta=32.0,
               yarn_l0=4096)
TINY_YARN = Dims(d=256, n_h=4, d_h=32, d_c=64, d_cq=96, d_r=16, yarn_s=40.0, yarn_alpha=1.0, yarn_beta=32.0,
                 yarn_l0=256)   # pair turns over L0: 40.7, 12.9, 4.1, 1.3, 0.41, ...: all three regimes

# Weight name -> (tensor id, shape(dims) [out, in]); std = 1/sqrt(fan_in) with fan_in = in.
WEIGHT_SPECS = {
    "w_dq": (TID_WDQ, lambda m: (m.d_cq, m.d)),
    "w_uq": (TID_WUQ, lambda m: (m.n_h * m.d_h, m.d_cq)),
    "w_qr": (TID_WQR, lambda m: (m.n_h * m.d_r, m.d_cq)),
    "w_dkv": (TID_WDKV, lambda m: (m.d_c, m.d)),
    "w_kr": (TID_WKR, lambda m: (m.d_r, m.d)),
    "w_uk": (TID_WUK, lambda m: (m.n_h * m.d_h, m.d_c)),
    "w_uv": (TID_WUV, lambda m: (m.n_h * m.d_h, m.d_c)),
    "w_o": (TID_WO, lambda m: (m.d, m.n_h * m.d_h)),
}


def weights(dims: Dims, seed: int = 0, dtype: str = "bf16", names=None) -> dict:
    out = {}
    for name, (tid, shape_fn) in WEIGHT_SPECS.items():
        if names is not None and name not in names:
            continue
        shape = shape_fn(dims)
        out[name] = normal(seed, tid, shape, std=1.0 / np.sqrt(shape[1]), dtype=dtype)
    return out


def gains(dims: Dims, seed: int = 0, dtype: str = "bf16") -> dict:
    """Synthetic RMSNorm gains g_q [d_cq] and g_kv [d_c]: 1 + 0.25 N(0,1) each."""
    return {"g_q": normal(seed, TID_GQ, (dims.d_cq,), std=0.25, dtype=dtype, mean=1.0),
            "g_kv": normal(seed, TID_GKV, (dims.d_c,), std=0.25, dtype=dtype, mean=1.0)}


def hidden(dims: Dims, tokens: int, seed: int = 0, dtype: str = "bf16") -> np.ndarray:
    return normal(seed, TID_H, (tokens, dims.d), dtype=dtype)


def latent_cache(dims: Dims, rows: int, seed: int = 0, dtype: str = "bf16") -> np.ndarray:
    """Synthetic latent cache rows [rows, d_c + d_r]: c^KV ~ N(0,1) then k^R ~ N(0,1)."""
    c = normal(seed, TID_CACHE_C, (rows, dims.d_c), dtype=dtype)
    kr = normal(seed, TID_CACHE_KR, (rows, dims.d_r), dtype=dtype)
    return np.concatenate([c, kr], axis=1)


def prefill_core_inputs(dims: Dims, tokens: int, seed: int = 0, dtype: str = "bf16") -> dict:
    """Inputs of the prefill attention core alone, all ~ N(0,1): q_c, k_c, v_c [tokens, n_h, d_h] and
    q_r [tokens, n_h, d_r] (k^R comes from latent_cache rows)."""
    hd = (tokens, dims.n_h, dims.d_h)
    return {"q_c": normal(seed, TID_QC, hd, dtype=dtype),
            "q_r": normal(seed, TID_QR, (tokens, dims.n_h, dims.d_r), dtype=dtype),
            "k_c": normal(seed, TID_KC, hd, dtype=dtype),
            "v_c": normal(seed, TID_VC, hd, dtype=dtype)}


def ragged_lengths(batch: int, lo: int, hi: int, seed: int = 0) -> np.ndarray:
    """Lengths uniform on [lo, hi] (inclusive) from the seed's length stream."""
    span = np.uint64(hi - lo + 1)
    draws = u64(seed, TID_LENGTHS, np.arange(batch, dtype=np.uint64))
    return (draws % span).astype(np.int64) + lo


def cu_seqlens(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    dims: Dims
    dtype: str
    batch: int
    tq: int = 1          # query tokens per sequence (decode)
    length: int = 0      # fixed cache/sequence length
    ragged: tuple = field(default=())  # (lo, hi) for ragged lengths

    def lengths(self, seed: int = 0) -> np.ndarray:
        if self.ragged:
            return ragged_lengths(self.batch, self.ragged[0], self.ragged[1], seed)
        return np.full(self.batch, self.length, dtype=np.int64)


WORKLOADS = {
    "tiny_prefill_fp32": Workload("tiny_prefill_fp32", "prefill", TINY, "fp32", batch=1, length=64),
    "decode_b16_l4096": Workload("decode_b16_l4096", "decode", V3, "bf16", batch=16, tq=1, length=4096),
    "decode_mtp_b64_ragged": Workload("decode_mtp_b64_ragged", "decode", V3, "bf16", batch=64, tq=2,
                                      ragged=(1024, 32768)),
    "prefill_l32768": Workload("prefill_l32768", "prefill", V3, "bf16", batch=1, length=32768),
    "decode_long_b4_l131072": Workload("decode_long_b4_l131072", "decode", V3, "bf16", batch=4, tq=1,
                                       length=131072),
}
