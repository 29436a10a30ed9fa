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


__all__ = ["rel", "dev", "dev_i64", "host", "make_module", "TOL", "orc", "synth", "mla"]
