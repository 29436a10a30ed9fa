"""Shared helpers for the GPU parity tests: seeded inputs, device upload, the error metric."""
import numpy as np

from mla_latent_kv_31_b200 import mla, synth
from oracle import mla_oracle as orc

TOL = {"bf16": 1e-2, "fp32": 1e-5}


def rel(gpu, ref) -> float:
    """max_i |gpu_i - ref_i| / max_i |ref_i| over the whole tensor."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    return float(np.max(np.abs(g - r)) / max(float(np.max(np.abs(r))), 1e-300))


def dev(x, dtype: str, device="cuda:0"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(device=device, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)


def dev_i64(x, device="cuda:0"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int64)).to(device)


def host(t):
    return t.float().cpu().numpy()


def mla_dtype(dtype: str) -> int:
    return mla.MLA_BF16 if dtype == "bf16" else mla.MLA_FP32


def make_module(dims, W_np, dtype, device="cuda:0"):
    W_dev = {k: dev(v, dtype, device) for k, v in W_np.items()}
    return mla.MLA(dims, W_dev, mla_dtype(dtype), device=int(str(device).split(":")[-1]))


# ---- FP8 cache rows (656 bytes: e4m3 codes [0, 512), f16 k^R / s [512, 640), fp32 s [640, 644), zero
# [644, 656)) ------------------------------------------------------------------------------------
E4M3 = orc.e4m3_positive_values()


def round_bf16(x) -> np.ndarray:
    """x rounded to bf16 (round to nearest even), as float64."""
    import torch
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def fp8_decode_rows(raw: np.ndarray):
    """(codes as values [n, 512], k^R' [n, 64], s [n], padding bytes [n, 12]) of FP8 rows [n, 656]."""
    raw = np.ascontiguousarray(raw, dtype=np.uint8)
    codes = raw[:, :512]
    assert not np.any((codes & 0x7F) == 0x7F), "NaN code"
    vals = np.where(codes & 0x80, -1.0, 1.0) * E4M3[codes & 0x7F]
    kr = raw[:, 512:640].copy().view(np.float16).astype(np.float64)
    s = raw[:, 640:644].copy().view(np.float32)[:, 0].astype(np.float64)
    return vals, kr, s, raw[:, 644:656]


def fp8_encode_rows(codes, kr, s) -> np.ndarray:
    """FP8 rows [n, 656] from the oracle's (e4m3 values, f16 k^R / s, s)."""
    codes = np.asarray(codes, dtype=np.float64)
    mag = np.abs(codes)
    idx = np.searchsorted(E4M3, mag)
    assert np.all(E4M3[np.minimum(idx, len(E4M3) - 1)] == mag), "not an e4m3 value"
    byte = idx.astype(np.uint8) | np.where(np.signbit(codes), 0x80, 0).astype(np.uint8)
    n = codes.shape[0]
    out = np.zeros((n, mla.FP8_ROW_BYTES), dtype=np.uint8)
    out[:, :512] = byte
    out[:, 512:640] = np.ascontiguousarray(np.asarray(kr, dtype=np.float16)).view(np.uint8)
    out[:, 640:644] = np.ascontiguousarray(np.asarray(s, dtype=np.float32)[:, None]).view(np.uint8)
    return out


def fp8_cache(rows_bf16, dims=synth.V3, chunk: int = 65536):
    """(FP8 bytes [n, 656], the float64 rows they stand for [n, 576]) of bf16 cache rows, by the
    oracle's quantizer, a chunk of rows at a time (the quantizer's temporaries grow with the rows)."""
    n = rows_bf16.shape[0]
    raw = np.empty((n, mla.FP8_ROW_BYTES), dtype=np.uint8)
    deq = np.empty((n, dims.d_c + dims.d_r), dtype=np.float64)
    for r0 in range(0, n, chunk):
        codes, kr, s = orc.quantize_cache_rows_fp8(rows_bf16[r0:r0 + chunk], dims)
        raw[r0:r0 + chunk] = fp8_encode_rows(codes, kr, s)
        deq[r0:r0 + chunk] = orc.dequantize_cache_rows_fp8(codes, kr, s)
    return raw, deq


def fp8_row_bound(ref, s):
    """Per-element bound of |dequantized - ref| for rows that went fp64 -> bf16 -> FP8: bf16 rounding
    (2^-8 relative) then e4m3 rounding (2^-4 relative; s 2^-10 absolute in the subnormals) of the
    c^KV part, f16 rounding (2^-11 relative) of the k^R part, and the projection's fp32 accumulation."""
    b = np.empty_like(ref)
    b[:, :512] = (2.0 ** -4 + 2.0 ** -7) * np.abs(ref[:, :512]) + s[:, None] * 2.0 ** -9
    b[:, 512:] = 2.0 ** -7 * np.abs(ref[:, 512:]) + s[:, None] * 2.0 ** -20
    return b + 1e-5 * np.abs(ref).max(axis=1, keepdims=True)


__all__ = ["rel", "dev", "dev_i64", "host", "make_module", "TOL", "orc", "synth", "mla", "E4M3", "round_bf16",
           "fp8_decode_rows", "fp8_encode_rows", "fp8_cache", "fp8_row_bound"]
