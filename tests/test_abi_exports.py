"""The C-ABI library loads and exports every symbol include/i4rt.h declares (no GPU needed).

Also checks host-side argument validation: invalid calls return their
negative status before any CUDA call is made.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "i4rt.h")).read()
    return sorted(set(re.findall(r"^I4_API\s+[\w\s\*]*?\b(\w+)\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ["int4_gemv", "int4_gemm", "paged_gqa_decode", "paged_gqa_decode_ws_bytes", "rmsnorm_rope", "silu_mul",
                     "decode_step_graph_create", "decode_step_graph_replay", "decode_step_graph_destroy",
                     "decode_step_eager", "i4_int4_unpack", "i4_paged_gather", "i4_last_error"]:
        assert required in names


def test_library_exports_every_declared_symbol(i4lib):
    raw = ctypes.CDLL(i4lib.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(raw, name), name
    assert sorted(i4lib.exported_symbols()) == declared_symbols()


def test_version_and_empty_error(i4lib):
    assert b"sm_100a" in i4lib.lib().i4_version()


def test_host_validation_without_gpu(i4lib):
    L = i4lib.lib()
    assert L.int4_gemv(None, None, None, None, None, 0, 1, 16, 128, 128, None) == i4lib.I4_EINVAL
    assert b"null" in L.i4_last_error()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    assert L.int4_gemv(fake, fake, fake, None, fake, 0, 1, 16, 128, 64, None) == i4lib.I4_EUNSUPPORTED
    assert L.int4_gemv(fake, fake, fake, None, fake, 0, 1, 16, 100, 128, None) == i4lib.I4_EINVAL
    # more than 8 rows go to the tcgen05 GEMM, which validates the same way before any launch
    assert L.int4_gemv(fake, fake, fake, None, fake, 0, 9, 16, 128, 64, None) == i4lib.I4_EUNSUPPORTED
    assert L.int4_gemm(fake, fake, fake, None, fake, 0, 512, 16, 100, 128, None, 0, None) == i4lib.I4_EINVAL
    assert L.int4_gemm(ctypes.c_void_p((1 << 20) + 8), fake, fake, None, fake, 0, 512, 16, 128, 128, None, 0,
                       None) == i4lib.I4_EALIGN
    assert L.int4_gemm(None, fake, fake, None, fake, 0, 512, 16, 128, 128, None, 0, None) == i4lib.I4_EINVAL
    assert L.int4_gemm(fake, fake, fake, None, fake, 0, 512, 16, 128, 128, ctypes.c_void_p((1 << 20) + 16), 1 << 20,
                       None) == i4lib.I4_EALIGN
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert L.int4_gemv(odd, fake, fake, None, fake, 0, 1, 16, 128, 128, None) == i4lib.I4_EALIGN
    assert L.paged_gqa_decode(fake, fake, fake, fake, fake, fake, 1, 28, 4, 64, 16, 4, 1.0, fake, 1 << 20,
                              None) == i4lib.I4_EUNSUPPORTED
    assert L.paged_gqa_decode(fake, fake, fake, fake, fake, fake, 1, 28, 4, 128, 12, 4, 1.0, fake, 1 << 20,
                              None) == i4lib.I4_EUNSUPPORTED
    assert L.paged_gqa_decode(fake, fake, fake, fake, fake, fake, 1, 28, 4, 128, 16, 4, 1.0, fake, 16,
                              None) == i4lib.I4_EINVAL
    assert L.silu_mul(None, fake, 1, 4, None) == i4lib.I4_EINVAL
    assert L.paged_gqa_decode_ws_bytes(1, 28, 4, 128, 16, 256) > 0
    assert L.paged_gqa_decode_ws_bytes(1, 28, 4, 64, 16, 256) == 0
    assert L.decode_step_graph_replay(None, None) == i4lib.I4_EINVAL
    assert L.i4_set_option(b"nonsense", 1) == i4lib.I4_EINVAL
    # option ranges (host-side settings, no GPU involved); defaults restored afterwards
    assert L.i4_set_option(b"gemv_prex", 9) == i4lib.I4_EINVAL
    assert L.i4_set_option(b"gemv_prex", -1) == i4lib.I4_EINVAL
    assert L.i4_set_option(b"gemv_prex", 2) == i4lib.I4_OK
    assert L.i4_set_option(b"gemv_prex", 1) == i4lib.I4_OK
    assert L.i4_set_option(b"gemv_ctas_per_sm", 3) == i4lib.I4_EINVAL
    assert L.i4_set_option(b"stream_smem_kb", 8) == i4lib.I4_EINVAL
    assert L.i4_set_option(b"unpack", 9) == i4lib.I4_EINVAL
    assert L.i4_set_option(b"test_stall", 0) == i4lib.I4_OK


def test_batched_decode_entries_validate_without_gpu(i4lib):
    L = i4lib.lib()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    # q rows closer than Hq * D, or not a multiple of 8 elements apart
    assert L.i4_paged_gqa_decode_strided(fake, 28 * 128 - 8, fake, fake, fake, fake, fake, 2, 28, 4, 128, 16, 4,
                                         1.0, fake, 1 << 20, None) == i4lib.I4_EINVAL
    assert L.i4_paged_gqa_decode_strided(fake, 4608 + 4, fake, fake, fake, fake, fake, 2, 28, 4, 128, 16, 4,
                                         1.0, fake, 1 << 20, None) == i4lib.I4_EINVAL
    assert b"q_stride" in L.i4_last_error()
    # the strided entry applies paged_gqa_decode's checks too
    assert L.i4_paged_gqa_decode_strided(fake, 4608, fake, fake, fake, fake, fake, 2, 28, 4, 128, 12, 4,
                                         1.0, fake, 1 << 20, None) == i4lib.I4_EUNSUPPORTED
    assert L.i4_embed_gather(None, fake, fake, 2, 64, 10, None) == i4lib.I4_EINVAL
    assert L.i4_embed_gather(fake, fake, fake, 2, 60, 10, None) == i4lib.I4_EINVAL       # H % 8
    assert L.i4_embed_gather(ctypes.c_void_p((1 << 20) + 2), fake, fake, 2, 64, 10, None) == i4lib.I4_EALIGN
    assert L.i4_argmax_rows(fake, fake, None, None, 0, 10, None) == i4lib.I4_EINVAL
    assert L.i4_argmax_rows(None, fake, None, None, 1, 10, None) == i4lib.I4_EINVAL


def test_graph_create_validation_without_gpu(i4lib):
    desc = i4lib.ModelDesc(28, 3584, 18944, 28, 4, 64, 152064, 128, 16, 4096, 1e6, 1e-6)
    handle = ctypes.c_void_p()
    w = i4lib.ModelWeights()
    s = i4lib.SeqState()
    st = i4lib.lib().decode_step_graph_create(ctypes.byref(desc), ctypes.byref(w), ctypes.byref(s),
                                              ctypes.byref(handle))
    assert st == i4lib.I4_EUNSUPPORTED  # head_dim 64
    desc.head_dim = 128
    desc.group = 64
    assert i4lib.lib().decode_step_graph_create(ctypes.byref(desc), ctypes.byref(w), ctypes.byref(s),
                                                ctypes.byref(handle)) == i4lib.I4_EUNSUPPORTED
    desc.group = 128
    assert i4lib.lib().decode_step_graph_create(ctypes.byref(desc), ctypes.byref(w), ctypes.byref(s),
                                                ctypes.byref(handle)) == i4lib.I4_EINVAL  # null weights
    assert not handle.value
