"""ctypes binding to libmla.so (include/mla.h). Argument marshalling only: every step of the
MLA path runs in the library's CUDA kernels; torch provides device memory and streams.

The functions keep the C names. Tensor arguments are torch CUDA tensors (or raw integer
device pointers); the stream defaults to torch's current stream of the handle's device.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_int, c_int32, c_int64, c_size_t, c_uint32, c_void_p

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla.so")

MLA_BF16, MLA_FP32 = 0, 1
OP_CACHE_APPEND, OP_DECODE, OP_PREFILL, OP_ATTN_DECODE_LATENT = 0, 1, 2, 3
BUF_CQ, BUF_QC, BUF_QR, BUF_QABS, BUF_OLAT, BUF_O, BUF_KC, BUF_VC, BUF_LSE = range(9)
CHUNK_AUTO, CHUNK_ABSORBED, CHUNK_UNABSORBED = 0, 1, 2
STATUS_NAMES = ["MLA_OK", "MLA_ERR_INVALID_ARG", "MLA_ERR_ALIGNMENT", "MLA_ERR_UNSUPPORTED", "MLA_ERR_WORKSPACE",
                "MLA_ERR_CUDA", "MLA_ERR_TIMEOUT", "MLA_ERR_DEVICE_CHECK", "MLA_ERR_NO_WEIGHTS",
                "MLA_ERR_SCRATCH_LIMIT"]
WEIGHT_NAMES = ["w_dq", "w_uq", "w_qr", "w_dkv", "w_kr", "w_uk", "w_uv", "w_o"]


class MlaDims(ctypes.Structure):
    _fields_ = [("d", c_int32), ("n_h", c_int32), ("d_h", c_int32), ("d_c", c_int32), ("d_cq", c_int32),
                ("d_r", c_int32), ("rope_base", c_double)]


class MlaWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in WEIGHT_NAMES]


class MLAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().mla_status_string(status).decode()}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmla.so; raises if it has not been built (there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m mla_latent_kv_31_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        H = c_void_p
        sigs = {
            "mla_create": (c_int, [POINTER(MlaDims), c_int, c_int, POINTER(H)]),
            "mla_set_weights": (c_int, [H, POINTER(MlaWeights)]),
            "mla_workspace_size": (c_int, [H, c_int, c_int64, c_int32, c_int64, POINTER(c_size_t)]),
            "mla_workspace_offset": (c_int, [H, c_int, c_int64, c_int32, c_int64, c_int, POINTER(c_size_t)]),
            "mla_cache_append": (c_int, [H, c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_int64, c_void_p,
                                         c_size_t, c_void_p]),
            "mla_cache_append_noalloc": (c_int, [H, c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_int64,
                                                 c_void_p]),
            "mla_decode": (c_int, [H, c_void_p, c_int64, c_int32, c_void_p, c_void_p, c_int64, c_void_p, c_void_p,
                                   c_size_t, c_void_p]),
            "mla_prefill": (c_int, [H, c_void_p, c_int64, c_void_p, c_int64, c_int64, c_void_p, c_int64, c_void_p,
                                    c_void_p, c_size_t, c_void_p]),
            "mla_prefill_chunk": (c_int, [H, c_void_p, c_int64, c_void_p, c_int64, c_int64, c_void_p, c_int64,
                                          c_void_p, c_int64, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
            "mla_prefill_chunk_workspace": (c_int, [H, c_int64, c_int64, c_int64, c_int64, c_int, POINTER(c_int),
                                                    POINTER(c_size_t)]),
            "mla_prefill_chunk_offset": (c_int, [H, c_int64, c_int64, c_int64, c_int64, c_int, c_int,
                                                 POINTER(c_size_t)]),
            "mla_attn_decode_latent": (c_int, [H, c_void_p, c_void_p, c_int64, c_int32, c_void_p, c_void_p, c_int64,
                                               c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
            "mla_attn_prefill": (c_int, [H, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_int64,
                                         c_int64, c_void_p, c_int64, c_void_p, c_void_p]),
            "mla_set_rmsnorm": (c_int, [H, c_void_p, c_void_p, c_double]),
            "mla_set_yarn": (c_int, [H, c_double, c_double, c_double, c_double]),
            "mla_set_cache_format": (c_int, [H, c_int]),
            "mla_cache_quantize_fp8": (c_int, [H, c_void_p, c_int64, c_void_p, c_void_p]),
            "mla_sync_status": (c_int, [H, c_void_p]),
            "mla_device_error_bits": (c_uint32, [H]),
            "mla_uses_tensor_cores": (c_int, [H, c_int]),
            "mla_kernel_launches": (ctypes.c_uint64, []),
            "mla_set_kernel_timing": (c_int, [c_int]),
            "mla_kernel_time_ms": (c_int, [c_int, POINTER(ctypes.c_float)]),
            "mla_status_string": (c_char_p, [c_int]),
            "mla_test_arm_stall": (None, []),
            "mla_destroy": (None, [H]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream, device: int):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def _check(status: int, what: str):
    if status != 0:
        raise MLAError(status, what)


# --- the C calls, same names -------------------------------------------------------------------
def mla_create(dims, dtype: int = MLA_BF16, device: int = 0) -> int:
    d = MlaDims(dims.d, dims.n_h, dims.d_h, dims.d_c, dims.d_cq, dims.d_r, float(dims.rope_base))
    h = c_void_p()
    _check(lib().mla_create(ctypes.byref(d), dtype, device, ctypes.byref(h)), "mla_create")
    return h.value


def mla_set_weights(handle: int, weights: dict):
    w = MlaWeights(*[_ptr(weights[n]) for n in WEIGHT_NAMES])
    _check(lib().mla_set_weights(handle, ctypes.byref(w)), "mla_set_weights")


def mla_workspace_size(handle: int, op: int, num_seqs: int = 0, tq: int = 1, total_tokens: int = 0) -> int:
    n = c_size_t()
    _check(lib().mla_workspace_size(handle, op, num_seqs, tq, total_tokens, ctypes.byref(n)), "mla_workspace_size")
    return n.value


def mla_workspace_offset(handle: int, op: int, which: int, num_seqs: int = 0, tq: int = 1,
                         total_tokens: int = 0) -> int:
    n = c_size_t()
    _check(lib().mla_workspace_offset(handle, op, num_seqs, tq, total_tokens, which, ctypes.byref(n)),
           "mla_workspace_offset")
    return n.value


def mla_cache_append(handle, hidden, positions, slots, T, cache, capacity, ws=None, ws_bytes=0, stream=None,
                     device=0):
    _check(lib().mla_cache_append(handle, _ptr(hidden), _ptr(positions), _ptr(slots), T, _ptr(cache), capacity,
                                  _ptr(ws), ws_bytes, _stream(stream, device)), "mla_cache_append")


def mla_cache_append_noalloc(handle, hidden, positions, slots, T, cache, capacity, stream=None, device=0):
    """mla_cache_append without a workspace: its scratch is a fixed 4 MiB array in the library."""
    _check(lib().mla_cache_append_noalloc(handle, _ptr(hidden), _ptr(positions), _ptr(slots), T, _ptr(cache),
                                          capacity, _stream(stream, device)), "mla_cache_append_noalloc")


def mla_decode(handle, h_q, B, Tq, cu_seqlens, cache, capacity, u_out, ws, ws_bytes, stream=None, device=0):
    _check(lib().mla_decode(handle, _ptr(h_q), B, Tq, _ptr(cu_seqlens), _ptr(cache), capacity, _ptr(u_out),
                            _ptr(ws), ws_bytes, _stream(stream, device)), "mla_decode")


def mla_prefill(handle, hidden, B, cu_seqlens, total_tokens, max_seqlen, cache, capacity, u_out, ws, ws_bytes,
                stream=None, device=0):
    _check(lib().mla_prefill(handle, _ptr(hidden), B, _ptr(cu_seqlens), total_tokens, max_seqlen, _ptr(cache),
                             capacity, _ptr(u_out), _ptr(ws), ws_bytes, _stream(stream, device)), "mla_prefill")


def mla_prefill_chunk(handle, hidden, B, cu_q, total_q, max_q, cu_kv, total_kv, cache, capacity, form, u_out, ws,
                      ws_bytes, stream=None, device=0):
    _check(lib().mla_prefill_chunk(handle, _ptr(hidden), B, _ptr(cu_q), total_q, max_q, _ptr(cu_kv), total_kv,
                                   _ptr(cache), capacity, form, _ptr(u_out), _ptr(ws), ws_bytes,
                                   _stream(stream, device)), "mla_prefill_chunk")


def mla_prefill_chunk_workspace(handle, B, total_q, max_q, total_kv, form=CHUNK_AUTO) -> tuple[int, int]:
    """(bytes, the form the call takes) for these arguments."""
    n, f = c_size_t(), c_int()
    _check(lib().mla_prefill_chunk_workspace(handle, B, total_q, max_q, total_kv, form, ctypes.byref(f),
                                             ctypes.byref(n)), "mla_prefill_chunk_workspace")
    return n.value, f.value


def mla_prefill_chunk_offset(handle, B, total_q, max_q, total_kv, form, which) -> int:
    n = c_size_t()
    _check(lib().mla_prefill_chunk_offset(handle, B, total_q, max_q, total_kv, form, which, ctypes.byref(n)),
           "mla_prefill_chunk_offset")
    return n.value


def mla_attn_decode_latent(handle, q_abs, q_rope, B, Tq, cu_seqlens, cache, capacity, o_lat, lse, ws, ws_bytes,
                           stream=None, device=0):
    _check(lib().mla_attn_decode_latent(handle, _ptr(q_abs), _ptr(q_rope), B, Tq, _ptr(cu_seqlens), _ptr(cache),
                                        capacity, _ptr(o_lat), _ptr(lse), _ptr(ws), ws_bytes,
                                        _stream(stream, device)), "mla_attn_decode_latent")


def mla_attn_prefill(handle, q_c, q_rope, k_c, v_c, B, cu_seqlens, total_tokens, max_seqlen, cache, capacity, o,
                     stream=None, device=0):
    _check(lib().mla_attn_prefill(handle, _ptr(q_c), _ptr(q_rope), _ptr(k_c), _ptr(v_c), B, _ptr(cu_seqlens),
                                  total_tokens, max_seqlen, _ptr(cache), capacity, _ptr(o), _stream(stream, device)),
           "mla_attn_prefill")


def mla_set_rmsnorm(handle, g_q, g_kv, eps: float = 1e-6):
    """RMSNorm gains of c^Q and c^KV (device tensors in the handle dtype), or None, None to turn it off."""
    _check(lib().mla_set_rmsnorm(handle, _ptr(g_q), _ptr(g_kv), eps), "mla_set_rmsnorm")


def mla_set_yarn(handle, s: float, alpha: float = 1.0, beta: float = 32.0, original_len: float = 4096.0):
    _check(lib().mla_set_yarn(handle, s, alpha, beta, original_len), "mla_set_yarn")


CACHE_BF16, CACHE_FP8 = 0, 1
FP8_ROW_BYTES = 656   # e4m3 codes [512] | f16 k^R / s [64] | fp32 s | zero padding


def mla_set_cache_format(handle, fmt: int):
    _check(lib().mla_set_cache_format(handle, fmt), "mla_set_cache_format")


def mla_cache_quantize_fp8(handle, rows, n, out, stream=None, device=0):
    _check(lib().mla_cache_quantize_fp8(handle, _ptr(rows), n, _ptr(out), _stream(stream, device)),
           "mla_cache_quantize_fp8")


def mla_sync_status(handle, stream=None, device=0) -> int:
    return lib().mla_sync_status(handle, _stream(stream, device))


def mla_device_error_bits(handle) -> int:
    return lib().mla_device_error_bits(handle)


def mla_uses_tensor_cores(handle, op: int) -> bool:
    return bool(lib().mla_uses_tensor_cores(handle, op))


TIMED_LATENT_CORE, TIMED_PREFILL_CORE = 0, 1


def mla_set_kernel_timing(enabled: bool):
    _check(lib().mla_set_kernel_timing(1 if enabled else 0), "mla_set_kernel_timing")


def mla_kernel_time_ms(which: int) -> float:
    ms = ctypes.c_float(0.0)
    _check(lib().mla_kernel_time_ms(which, ctypes.byref(ms)), "mla_kernel_time_ms")
    return float(ms.value)


def mla_test_arm_stall():
    """Arms the next decode latent-core launch to give up on a wait nothing signals (20 ms limit)."""
    lib().mla_test_arm_stall()


def mla_kernel_launches() -> int:
    return lib().mla_kernel_launches()


def mla_status_string(status: int) -> str:
    return lib().mla_status_string(status).decode()


def mla_destroy(handle):
    lib().mla_destroy(handle)


# --- convenience owner of a handle, its weights and workspaces -----------------------------
class MLA:
    """Owns one handle plus torch allocations (weights kept alive, workspaces reused)."""

    def __init__(self, dims, weights: dict, dtype: int = MLA_BF16, device: int = 0):
        import torch
        self.torch = torch
        self.dims, self.dtype, self.device = dims, dtype, device
        self.tdtype = torch.bfloat16 if dtype == MLA_BF16 else torch.float32
        self.handle = mla_create(dims, dtype, device)
        self.weights = {n: weights[n] for n in WEIGHT_NAMES}
        mla_set_weights(self.handle, self.weights)
        # opt-in parts of the layer: RMSNorm gains among the weights, YaRN settings in the dims
        if "g_q" in weights or "g_kv" in weights:
            self.gains = (weights["g_q"], weights["g_kv"])
            mla_set_rmsnorm(self.handle, *self.gains, getattr(dims, "rms_eps", 1e-6))
        if getattr(dims, "yarn_s", 1.0) > 1.0:
            mla_set_yarn(self.handle, dims.yarn_s, dims.yarn_alpha, dims.yarn_beta, dims.yarn_l0)
        self._ws = None

    def close(self):
        if self.handle:
            mla_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace(self, nbytes: int):
        torch = self.torch
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(max(nbytes, 1024), dtype=torch.uint8, device=f"cuda:{self.device}")
        return self._ws

    def region(self, op, which, shape, dtype, num_seqs=0, tq=1, total_tokens=0):
        """A view of a named workspace region after a call (for step-level inspection)."""
        torch = self.torch
        off = mla_workspace_offset(self.handle, op, which, num_seqs, tq, total_tokens)
        n = 1
        for s in shape:
            n *= s
        es = torch.tensor([], dtype=dtype).element_size()
        return self._ws[off:off + n * es].view(dtype).view(*shape)

    def set_cache_format(self, fmt: int):
        mla_set_cache_format(self.handle, fmt)

    def quantize_fp8(self, rows):
        """FP8 rows [n, 656] (uint8) of bf16 cache rows [n, 576]."""
        out = self.torch.empty(rows.shape[0], FP8_ROW_BYTES, dtype=self.torch.uint8, device=rows.device)
        mla_cache_quantize_fp8(self.handle, rows, rows.shape[0], out, device=self.device)
        return out

    def cache_append(self, hidden, positions, slots, cache):
        T = hidden.shape[0]
        n = mla_workspace_size(self.handle, OP_CACHE_APPEND, 0, 1, T)
        ws = self.workspace(n) if n else None
        mla_cache_append(self.handle, hidden, positions, slots, T, cache, cache.shape[0], ws, n if n else 0,
                         device=self.device)

    def decode(self, h_q, B, Tq, cu_seqlens, cache, u_out=None):
        torch = self.torch
        if u_out is None:
            u_out = torch.empty(B * Tq, self.dims.d, dtype=self.tdtype, device=h_q.device)
        n = mla_workspace_size(self.handle, OP_DECODE, B, Tq, 0)
        ws = self.workspace(n)
        mla_decode(self.handle, h_q, B, Tq, cu_seqlens, cache, cache.shape[0], u_out, ws, ws.numel(),
                   device=self.device)
        return u_out

    def prefill(self, hidden, B, cu_seqlens, max_seqlen, cache, u_out=None):
        torch = self.torch
        T = hidden.shape[0]
        if u_out is None:
            u_out = torch.empty(T, self.dims.d, dtype=self.tdtype, device=hidden.device)
        n = mla_workspace_size(self.handle, OP_PREFILL, B, 1, T)
        ws = self.workspace(n)
        mla_prefill(self.handle, hidden, B, cu_seqlens, T, max_seqlen, cache, cache.shape[0], u_out, ws, ws.numel(),
                    device=self.device)
        return u_out

    def prefill_chunk(self, hidden, B, cu_q, max_q, cu_kv, total_kv, cache, form=CHUNK_AUTO, u_out=None):
        """Chunked prefill; returns (u, the form taken)."""
        torch = self.torch
        T = hidden.shape[0]
        if u_out is None:
            u_out = torch.empty(T, self.dims.d, dtype=self.tdtype, device=hidden.device)
        n, chosen = mla_prefill_chunk_workspace(self.handle, B, T, max_q, total_kv, form)
        ws = self.workspace(n)
        mla_prefill_chunk(self.handle, hidden, B, cu_q, T, max_q, cu_kv, total_kv, cache, cache.shape[0], form, u_out,
                          ws, ws.numel(), device=self.device)
        return u_out, chosen

    def chunk_region(self, B, total_q, max_q, total_kv, form, which, shape, dtype):
        """A view of a named workspace region after a prefill_chunk call."""
        torch = self.torch
        off = mla_prefill_chunk_offset(self.handle, B, total_q, max_q, total_kv, form, which)
        n = 1
        for s in shape:
            n *= s
        es = torch.tensor([], dtype=dtype).element_size()
        return self._ws[off:off + n * es].view(dtype).view(*shape)

    def attn_decode_latent(self, q_abs, q_rope, B, Tq, cu_seqlens, cache, o_lat=None, lse=None):
        torch = self.torch
        T = B * Tq
        dev = q_abs.device
        if o_lat is None:
            o_lat = torch.empty(T, self.dims.n_h, self.dims.d_c, dtype=torch.float32, device=dev)
        if lse is None:
            lse = torch.empty(T, self.dims.n_h, dtype=torch.float32, device=dev)
        n = mla_workspace_size(self.handle, OP_ATTN_DECODE_LATENT, B, Tq, 0)
        ws = self.workspace(n)
        mla_attn_decode_latent(self.handle, q_abs, q_rope, B, Tq, cu_seqlens, cache, cache.shape[0], o_lat, lse, ws,
                               ws.numel(), device=self.device)
        return o_lat, lse

    def sync_status(self) -> int:
        return mla_sync_status(self.handle, device=self.device)
