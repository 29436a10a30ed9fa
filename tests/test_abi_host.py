"""Host-side checks of the C ABI: the library loads, exports every declared symbol, and rejects
bad arguments before any CUDA call (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

from mla_latent_kv_31_b200 import build as mla_build
from mla_latent_kv_31_b200 import mla, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    mla_build.build()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "mla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 12
    L = ctypes.CDLL(mla._LIB_PATH)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    for i, name in enumerate(mla.STATUS_NAMES):
        assert mla.mla_status_string(i).startswith(name)


def test_create_validates_dims():
    with pytest.raises(mla.MLAError) as e:
        mla.mla_create(synth.Dims(d=0, n_h=1, d_h=1, d_c=1, d_cq=1, d_r=2))
    assert e.value.status == 1
    with pytest.raises(mla.MLAError):
        mla.mla_create(synth.Dims(d=8, n_h=1, d_h=4, d_c=4, d_cq=4, d_r=3))  # odd d_r
    with pytest.raises(mla.MLAError) as e:
        mla.mla_create(synth.Dims(d=8, n_h=1, d_h=4, d_c=1024, d_cq=4, d_r=2))
    assert e.value.status == 3
    h = mla.mla_create(synth.V3)
    assert h
    mla.mla_destroy(h)


def test_workspace_sizes_and_offsets():
    h = mla.mla_create(synth.V3, mla.MLA_BF16)
    try:
        n = mla.mla_workspace_size(h, mla.OP_DECODE, 16, 1, 0)
        T = 16
        d = synth.V3
        # c^Q, q^C, q^R, o, q~, o^lat, lse, positions at least
        floor = T * (d.d_cq + 2 * d.n_h * d.d_h + d.n_h * d.d_r + 2 * d.n_h * d.d_c) * 2 + T * d.n_h * 4
        assert n >= floor
        offs = [mla.mla_workspace_offset(h, mla.OP_DECODE, b, 16, 1, 0)
                for b in (mla.BUF_CQ, mla.BUF_QC, mla.BUF_QR, mla.BUF_O, mla.BUF_QABS, mla.BUF_OLAT, mla.BUF_LSE)]
        assert offs == sorted(offs) and len(set(offs)) == len(offs)
        assert all(o % 1024 == 0 and o < n for o in offs)
        with pytest.raises(mla.MLAError):
            mla.mla_workspace_offset(h, mla.OP_DECODE, mla.BUF_KC, 16, 1, 0)  # prefill-only region
        # cache append: split-K partials of the [W^DKV; W^KR] projection at small T only
        small = mla.mla_workspace_size(h, mla.OP_CACHE_APPEND, 0, 1, 10)
        assert small >= 2 * 10 * (d.d_c + d.d_r) * 4 and small % 1024 == 0
        assert mla.mla_workspace_size(h, mla.OP_CACHE_APPEND, 0, 1, 4096) == 0
        p = mla.mla_workspace_size(h, mla.OP_PREFILL, 1, 1, 4096)
        assert p > 4096 * d.n_h * d.d_h * 2 * 3
        with pytest.raises(mla.MLAError):
            mla.mla_workspace_size(h, mla.OP_DECODE, 4, 3, 0)   # Tq must be 1 or 2
        with pytest.raises(mla.MLAError):
            mla.mla_workspace_size(h, 7, 4, 1, 0)
    finally:
        mla.mla_destroy(h)


def test_calls_reject_bad_arguments_before_any_launch():
    h = mla.mla_create(synth.TINY, mla.MLA_FP32)
    A = 0x10000  # aligned fake device address: never dereferenced, validation fails first
    try:
        with pytest.raises(mla.MLAError) as e:   # null h_q
            mla.mla_decode(h, None, 2, 1, A, A, 10, A, A, 1 << 20, stream=0)
        assert e.value.status == 1
        with pytest.raises(mla.MLAError) as e:   # Tq = 3
            mla.mla_decode(h, A, 2, 3, A, A, 10, A, A, 1 << 20, stream=0)
        assert e.value.status == 1
        with pytest.raises(mla.MLAError) as e:   # misaligned cache
            mla.mla_decode(h, A, 2, 1, A, A + 2, 10, A, A, 1 << 20, stream=0)
        assert e.value.status == 2
        with pytest.raises(mla.MLAError) as e:   # workspace too small
            mla.mla_decode(h, A, 2, 1, A, A, 10, A, A, 16, stream=0)
        assert e.value.status == 4
        with pytest.raises(mla.MLAError) as e:   # no weights given yet
            mla.mla_decode(h, A, 2, 1, A, A, 10, A, A, 1 << 30, stream=0)
        assert e.value.status == 8
        with pytest.raises(mla.MLAError) as e:   # prefill: capacity below the token count
            mla.mla_prefill(h, A, 1, A, 64, 64, A, 32, A, A, 1 << 30, stream=0)
        assert e.value.status == 1
        with pytest.raises(mla.MLAError) as e:   # cache append: misaligned slots
            mla.mla_cache_append(h, A, A, A + 8, 4, A, 10, stream=0)
        assert e.value.status == 2
        with pytest.raises(mla.MLAError) as e:   # core: workspace too small
            mla.mla_attn_decode_latent(h, A, A, 2, 1, A, A, 10, A, A, A, 0, stream=0)
        assert e.value.status in (1, 4)
        with pytest.raises(mla.MLAError) as e:   # weights: misaligned pointer
            mla.mla_set_weights(h, {n: A + (2 if n == "w_o" else 0) for n in mla.WEIGHT_NAMES})
        assert e.value.status == 2
        # prefill core alone: null k^C, capacity below the token count, max_seqlen 0, misaligned o
        with pytest.raises(mla.MLAError) as e:
            mla.mla_attn_prefill(h, A, A, None, A, 1, A, 64, 64, A, 64, A, stream=0)
        assert e.value.status == 1
        with pytest.raises(mla.MLAError) as e:
            mla.mla_attn_prefill(h, A, A, A, A, 1, A, 64, 64, A, 63, A, stream=0)
        assert e.value.status == 1
        with pytest.raises(mla.MLAError) as e:
            mla.mla_attn_prefill(h, A, A, A, A, 1, A, 64, 0, A, 64, A, stream=0)
        assert e.value.status == 1
        with pytest.raises(mla.MLAError) as e:
            mla.mla_attn_prefill(h, A, A, A, A, 1, A, 64, 64, A, 64, A + 4, stream=0)
        assert e.value.status == 2
    finally:
        mla.mla_destroy(h)


def test_kernel_timing_calls_validate_without_a_launch():
    mla.mla_set_kernel_timing(False)
    for which in (-1, 2):
        with pytest.raises(mla.MLAError) as e:
            mla.mla_kernel_time_ms(which)
        assert e.value.status == 1
    # nothing has been bracketed in this process: no time to report
    with pytest.raises(mla.MLAError) as e:
        mla.mla_kernel_time_ms(mla.TIMED_PREFILL_CORE)
    assert e.value.status == 1


def test_tensor_core_routing_is_declared():
    bf = mla.mla_create(synth.V3, mla.MLA_BF16)
    f32 = mla.mla_create(synth.TINY, mla.MLA_FP32)
    try:
        for op in range(4):
            assert mla.mla_uses_tensor_cores(f32, op) is False
            assert isinstance(mla.mla_uses_tensor_cores(bf, op), bool)
    finally:
        mla.mla_destroy(bf)
        mla.mla_destroy(f32)


def test_chunked_prefill_form_choice_workspace_and_validation():
    h = mla.mla_create(synth.V3, mla.MLA_BF16)
    d = synth.V3
    try:
        ws = mla.mla_prefill_chunk_workspace
        # uniform short chunks on long prefixes: absorbed; ragged, long or prefix-light: unabsorbed
        assert ws(h, 4, 16, 4, 4000)[1] == mla.CHUNK_ABSORBED
        assert ws(h, 4, 15, 4, 4000)[1] == mla.CHUNK_UNABSORBED
        assert ws(h, 2, 200, 100, 40000)[1] == mla.CHUNK_UNABSORBED
        assert ws(h, 4, 16, 4, 31)[1] == mla.CHUNK_UNABSORBED
        assert ws(h, 4, 16, 4, 32)[1] == mla.CHUNK_ABSORBED
        assert ws(h, 4, 16, 4, 4000, mla.CHUNK_UNABSORBED)[1] == mla.CHUNK_UNABSORBED
        with pytest.raises(mla.MLAError) as e:          # forced absorbed on ragged chunks
            ws(h, 4, 15, 4, 4000, mla.CHUNK_ABSORBED)
        assert e.value.status == 1
        with pytest.raises(mla.MLAError) as e:          # fewer key rows than chunk tokens
            ws(h, 1, 16, 16, 15)
        assert e.value.status == 1
        # regions: the absorbed form has q~ and no k^C; the unabsorbed form's k^C spans every key row
        off = mla.mla_prefill_chunk_offset
        assert off(h, 4, 16, 4, 4000, mla.CHUNK_ABSORBED, mla.BUF_QABS) >= 0
        with pytest.raises(mla.MLAError):
            off(h, 4, 16, 4, 4000, mla.CHUNK_ABSORBED, mla.BUF_KC)
        with pytest.raises(mla.MLAError):
            off(h, 4, 15, 4, 4000, mla.CHUNK_AUTO, mla.BUF_QABS)
        kc = off(h, 4, 15, 4, 4000, mla.CHUNK_AUTO, mla.BUF_KC)
        vc = off(h, 4, 15, 4, 4000, mla.CHUNK_AUTO, mla.BUF_VC)
        assert vc - kc >= 4000 * d.n_h * d.d_h * 2
        assert ws(h, 4, 15, 4, 4000)[0] >= vc + 4000 * d.n_h * d.d_h * 2
        A = 1 << 20
        call = mla.mla_prefill_chunk
        with pytest.raises(mla.MLAError) as e:          # capacity below the key rows
            call(h, A, 2, A, 8, 4, A, 100, A, 99, mla.CHUNK_AUTO, A, A, 1 << 40, stream=0)
        assert e.value.status == 1
        with pytest.raises(mla.MLAError) as e:          # misaligned cu_kv
            call(h, A, 2, A, 8, 4, A + 8, 100, A, 100, mla.CHUNK_AUTO, A, A, 1 << 40, stream=0)
        assert e.value.status == 2
        with pytest.raises(mla.MLAError) as e:          # workspace too small
            call(h, A, 2, A, 8, 4, A, 100, A, 100, mla.CHUNK_AUTO, A, A, 1024, stream=0)
        assert e.value.status == 4
        with pytest.raises(mla.MLAError) as e:          # no weights given yet
            call(h, A, 2, A, 8, 4, A, 100, A, 100, mla.CHUNK_AUTO, A, A, 1 << 40, stream=0)
        assert e.value.status == 8
        with pytest.raises(mla.MLAError) as e:          # unknown form
            call(h, A, 2, A, 8, 4, A, 100, A, 100, 7, A, A, 1 << 40, stream=0)
        assert e.value.status == 1
    finally:
        mla.mla_destroy(h)


def test_option_setters_validate_on_the_host():
    h = mla.mla_create(synth.V3, mla.MLA_BF16)
    A = 1 << 20
    try:
        mla.mla_set_rmsnorm(h, A, A + 1024, 1e-6)
        mla.mla_set_rmsnorm(h, None, None, 1e-6)            # off again
        for args, status in (((A, None, 1e-6), 1), ((A, A, -1.0), 1), ((A + 8, A, 1e-6), 2)):
            with pytest.raises(mla.MLAError) as e:
                mla.mla_set_rmsnorm(h, *args)
            assert e.value.status == status
        mla.mla_set_yarn(h, 40.0, 1.0, 32.0, 4096.0)
        mla.mla_set_yarn(h, 1.0)                             # plain RoPE again
        for args in ((0.5,), (40.0, 32.0, 1.0), (40.0, 1.0, 32.0, 0.0)):
            with pytest.raises(mla.MLAError) as e:
                mla.mla_set_yarn(h, *args)
            assert e.value.status == 1
    finally:
        mla.mla_destroy(h)


def test_cache_format_setter_and_fp8_guards():
    A = 1 << 20
    h32 = mla.mla_create(synth.TINY, mla.MLA_FP32)
    try:
        with pytest.raises(mla.MLAError) as e:   # FP8 rows are laid out for the DeepSeek-V3 sizes in bf16
            mla.mla_set_cache_format(h32, mla.CACHE_FP8)
        assert e.value.status == 3
        mla.mla_set_cache_format(h32, mla.CACHE_BF16)
    finally:
        mla.mla_destroy(h32)
    h = mla.mla_create(synth.V3, mla.MLA_BF16)
    try:
        with pytest.raises(mla.MLAError) as e:
            mla.mla_set_cache_format(h, 2)
        assert e.value.status == 1
        mla.mla_set_cache_format(h, mla.CACHE_FP8)
        # the calls that read the cache as bf16 rows refuse an FP8 handle before any launch
        with pytest.raises(mla.MLAError) as e:
            mla.mla_prefill(h, A, 1, A, 64, 64, A, 64, A, A, 1 << 30, stream=0)
        assert e.value.status == 3
        with pytest.raises(mla.MLAError) as e:
            mla.mla_cache_append_noalloc(h, A, A, A, 4, A, 10, stream=0)
        assert e.value.status == 3
        with pytest.raises(mla.MLAError) as e:
            mla.mla_attn_prefill(h, A, A, A, A, 1, A, 64, 64, A, 64, A, stream=0)
        assert e.value.status == 3
        with pytest.raises(mla.MLAError) as e:
            mla.mla_prefill_chunk(h, A, 1, A, 4, 4, A, 64, A, 64, mla.CHUNK_AUTO, A, A, 1 << 30, stream=0)
        assert e.value.status == 3
        # the FP8 append stages its T bf16 rows (576 columns) in the workspace before quantizing them
        for T in (1, 45, 700):
            ws8 = mla.mla_workspace_size(h, mla.OP_CACHE_APPEND, 0, 1, T)
            mla.mla_set_cache_format(h, mla.CACHE_BF16)
            ws16 = mla.mla_workspace_size(h, mla.OP_CACHE_APPEND, 0, 1, T)
            mla.mla_set_cache_format(h, mla.CACHE_FP8)
            assert ws8 >= ws16 + T * 576 * 2, (T, ws8, ws16)
        # the quantizer validates its arguments on the host
        with pytest.raises(mla.MLAError) as e:
            mla.mla_cache_quantize_fp8(h, A, 0, A, stream=0)
        assert e.value.status == 1
        with pytest.raises(mla.MLAError) as e:
            mla.mla_cache_quantize_fp8(h, A + 8, 4, A, stream=0)
        assert e.value.status == 2
        mla.mla_set_cache_format(h, mla.CACHE_BF16)
    finally:
        mla.mla_destroy(h)


def test_a_plain_c_caller_compiles_links_and_runs(tmp_path):
    """include/mla.h as C99 (-Wall -Werror) and libmla.so linked like any C library: a C program makes
    the host-side calls (handle, workspace arithmetic, validation before any launch, the FP8 format's
    guards, status strings) and checks every status."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(mla._LIB_PATH)
    exe = tmp_path / "abi_c_client"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "abi_c_client.c"), "-o", str(exe), mla._LIB_PATH,
                    f"-Wl,-rpath,{libdir}"], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
