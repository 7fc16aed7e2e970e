"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/qmv.h declares, and rejects bad arguments on the
host before enqueueing anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qmv.h")


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_qmv_b200 import _build
    _build.build()
    import weight_only_quantized_qmv_b200 as q
    return q.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qmv_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("qmv_encode_fp4", "qmv_encode_int4", "qmv_encode_int8", "qmv_matvec_fp4", "qmv_matvec_int4",
                 "qmv_matvec_int4km", "qmv_matvec_int8", "qmv_gather_matvec", "qmv_dequant", "qmv_status_fetch",
                 "qmv_last_error", "qmv_version"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    import weight_only_quantized_qmv_b200 as q
    assert set(q.SIGNATURES) == set(declared_functions())


def test_version(L):
    assert L.qmv_version().decode().count(".") == 2


FAKE = ctypes.c_void_p(0x10000)  # aligned, never dereferenced: every call below fails on the host
MIS = ctypes.c_void_p(0x10008)


def _err(L):
    return L.qmv_last_error().decode()


def test_matvec_argument_checks(L):
    q = pytest.importorskip("weight_only_quantized_qmv_b200")
    for fn in (L.qmv_matvec_fp4, L.qmv_matvec_int4, L.qmv_matvec_int4km, L.qmv_matvec_int8):
        assert fn(None, FAKE, FAKE, 1, 64, 64, FAKE, None) == q.ERR_ARG
        assert fn(FAKE, FAKE, None, 1, 64, 64, FAKE, None) == q.ERR_ARG
        assert fn(FAKE, FAKE, FAKE, 1, 64, 64, None, None) == q.ERR_ARG
        assert fn(MIS, FAKE, FAKE, 1, 64, 64, FAKE, None) == q.ERR_ARG
        assert fn(FAKE, FAKE, MIS, 1, 64, 64, FAKE, None) == q.ERR_ARG
        # K not a multiple of the block (the pages' silent-skip pitfall is an error here)
        assert fn(FAKE, FAKE, FAKE, 1, 64, 48, FAKE, None) == q.ERR_SHAPE
        assert "multiple of the 32-element block" in _err(L)
        assert fn(FAKE, FAKE, FAKE, 1, 64, 0, FAKE, None) == q.ERR_SHAPE
        assert fn(FAKE, FAKE, FAKE, 1, 0, 64, FAKE, None) == q.ERR_SHAPE
        assert fn(FAKE, FAKE, FAKE, 0, 64, 64, FAKE, None) == q.ERR_UNSUPPORTED
        assert fn(FAKE, FAKE, FAKE, 17, 64, 64, FAKE, None) == q.ERR_UNSUPPORTED
    # the palette must be 16-byte aligned, fp16 scales 2-byte aligned
    assert L.qmv_matvec_int4km(FAKE, MIS, FAKE, 1, 64, 64, FAKE, None) == q.ERR_ARG
    assert L.qmv_matvec_int4(FAKE, ctypes.c_void_p(0x10001), FAKE, 1, 64, 64, FAKE, None) == q.ERR_ARG


def test_gather_argument_checks(L):
    q = pytest.importorskip("weight_only_quantized_qmv_b200")
    g = L.qmv_gather_matvec
    assert g(9, FAKE, FAKE, 8, 64, 64, FAKE, 2, 2, FAKE, 0, FAKE, None) == q.ERR_ARG
    assert g(q.FMT_INT4KM, FAKE, FAKE, 0, 64, 64, FAKE, 2, 2, FAKE, 0, FAKE, None) == q.ERR_SHAPE
    assert g(q.FMT_INT4KM, FAKE, FAKE, 8, 64, 64, None, 2, 2, FAKE, 0, FAKE, None) == q.ERR_ARG
    assert g(q.FMT_INT4KM, FAKE, FAKE, 8, 64, 64, FAKE, 2, 17, FAKE, 0, FAKE, None) == q.ERR_UNSUPPORTED
    assert g(q.FMT_INT4KM, FAKE, FAKE, 8, 64, 64, FAKE, 17, 2, FAKE, 0, FAKE, None) == q.ERR_UNSUPPORTED
    assert g(q.FMT_INT4KM, FAKE, FAKE, 8, 64, 64, FAKE, 2, 2, FAKE, 2, FAKE, None) == q.ERR_ARG
    assert g(q.FMT_INT4KM, FAKE, FAKE, 8, 64, 33, FAKE, 2, 2, FAKE, 0, FAKE, None) == q.ERR_SHAPE


def test_encoder_argument_checks(L):
    q = pytest.importorskip("weight_only_quantized_qmv_b200")
    clips = (ctypes.c_float * 2)(1.0, 0.9)
    bad = (ctypes.c_float * 1)(-1.0)
    assert L.qmv_encode_fp4(None, 4, 64, FAKE, FAKE, None) == q.ERR_ARG
    assert L.qmv_encode_fp4(FAKE, 4, 40, FAKE, FAKE, None) == q.ERR_SHAPE
    for fn in (L.qmv_encode_int4, L.qmv_encode_int8):
        assert fn(FAKE, 4, 64, None, 1, FAKE, FAKE, None) == q.ERR_ARG
        assert fn(FAKE, 4, 64, clips, 0, FAKE, FAKE, None) == q.ERR_ARG
        assert fn(FAKE, 4, 64, clips, 17, FAKE, FAKE, None) == q.ERR_ARG
        assert fn(FAKE, 4, 64, bad, 1, FAKE, FAKE, None) == q.ERR_ARG
        assert fn(FAKE, 4, 96 + 1, clips, 2, FAKE, FAKE, None) == q.ERR_SHAPE
    assert L.qmv_dequant(7, FAKE, FAKE, 4, 64, FAKE, None) == q.ERR_ARG
    assert L.qmv_dequant(q.FMT_FP4, FAKE, FAKE, 4, 64, MIS, None) == q.ERR_ARG
    assert L.qmv_status_fetch(None, None) == q.ERR_ARG


def test_weight_prefetch_option(L):
    import weight_only_quantized_qmv_b200 as q
    assert L.qmv_set_weight_prefetch(2) == q.ERR_ARG
    assert L.qmv_set_weight_prefetch(-1) == q.ERR_ARG
    assert L.qmv_set_weight_prefetch(1) == q.OK
    assert L.qmv_set_weight_prefetch(0) == q.OK


def test_encode_int8km_argument_checks(L):
    import weight_only_quantized_qmv_b200 as q
    nb = L.qmv_int8km_encode_workspace_bytes(100, 2048)
    # 4 groups in flight, next_pow2(32 * 2048) keys of 4 bytes each
    assert nb == 4 * 65536 * 4
    assert L.qmv_int8km_encode_workspace_bytes(1000000, 96) == 160 * 4096 * 4
    assert L.qmv_int8km_encode_workspace_bytes(5, 96) == 1 * 512 * 4
    assert L.qmv_int8km_encode_workspace_bytes(0, 96) == 0
    fn = L.qmv_encode_int8km
    assert fn(None, 100, 2048, 20, FAKE, FAKE, FAKE, nb, None) == q.ERR_ARG
    assert fn(FAKE, 100, 2048, 20, None, FAKE, FAKE, nb, None) == q.ERR_ARG
    assert fn(FAKE, 100, 2048, 20, ctypes.c_void_p(0x10001), FAKE, FAKE, nb, None) == q.ERR_ARG
    assert fn(FAKE, 100, 2048, 20, FAKE, None, FAKE, nb, None) == q.ERR_ARG
    assert fn(FAKE, 100, 2048, -1, FAKE, FAKE, FAKE, nb, None) == q.ERR_ARG
    assert fn(FAKE, 100, 2048, 1001, FAKE, FAKE, FAKE, nb, None) == q.ERR_ARG
    assert fn(FAKE, 100, 2048, 20, FAKE, FAKE, None, nb, None) == q.ERR_ARG
    assert fn(FAKE, 100, 2048, 20, FAKE, FAKE, FAKE, nb - 1, None) == q.ERR_ARG
    assert "workspace" in _err(L)
    assert fn(FAKE, 100, 2040, 20, FAKE, FAKE, FAKE, nb, None) == q.ERR_SHAPE
    assert fn(FAKE, 0, 2048, 20, FAKE, FAKE, FAKE, nb, None) == q.ERR_SHAPE
    assert fn(FAKE, 10, 16416, 20, FAKE, FAKE, FAKE, 1 << 30, None) == q.ERR_UNSUPPORTED


def test_fp4_tensor_core_option(L):
    import weight_only_quantized_qmv_b200 as q
    assert L.qmv_set_fp4_tensor_cores(2) == q.ERR_ARG
    assert L.qmv_set_fp4_tensor_cores(-1) == q.ERR_ARG
    assert L.qmv_set_fp4_tensor_cores(1) == q.OK
    assert L.qmv_set_fp4_tensor_cores(0) == q.OK


def test_binding_rejects_cpu_tensors():
    import torch
    import weight_only_quantized_qmv_b200 as q
    with pytest.raises(ValueError):
        q.encode_fp4(torch.zeros(4, 64))
    with pytest.raises(ValueError):
        q.matvec_fp4(torch.zeros(4, 32, dtype=torch.uint8), torch.zeros(4, 2, dtype=torch.uint8),
                     torch.zeros(64, dtype=torch.float16))
