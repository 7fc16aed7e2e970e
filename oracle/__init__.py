"""CPU oracle for weight-only block-quantized matvec -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
leg may import this package.  The product path (the CUDA library and its
Python binding) never does, and this package imports nothing from it.

numpy in, numpy out.  fp16 values travel as numpy float16 arrays (their bit
patterns are what the C code reads).  The C source (qmv_oracle.c) cites the
passages of the pages each function follows; its parity status is stated in
its header.
"""
import ctypes
import os

import numpy as np

from . import build as _build

FMT_FP4, FMT_INT4, FMT_INT4KM, FMT_INT8, FMT_INT4AFF, FMT_INT8KM = 0, 1, 2, 3, 4, 5
KM8_GROUP = 32  # int8km: output rows sharing one 256-entry LUT
FLAG_NONFINITE, FLAG_SCALE_OVERFLOW, FLAG_BAD_EXPERT = 1, 2, 4

# Clip lists: the int4 list of the int4 lm_head workload (1.00 down to 0.50
# in steps of 0.05, as float32 literals) and plain symmetric int8 ({1.0}).
INT4_CLIPS = np.array([1.0 - 0.05 * i for i in range(11)], dtype=np.float32)
INT8_CLIPS = np.array([1.0], dtype=np.float32)
KMEANS_ITERS = 20

_lib = None


def lib():
    global _lib
    if _lib is None:
        # QMV_ORACLE_LIB: load another build of the same source (the mutation
        # tests point it at deliberately broken copies)
        path = os.environ.get("QMV_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P, I64, I32, U32P = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_uint32)
        L.oracle_f32_to_f16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_f16.restype = ctypes.c_uint16
        L.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_f32.restype = ctypes.c_float
        L.oracle_e2m1_code.argtypes = [ctypes.c_float]
        L.oracle_e2m1_code.restype = I32
        L.oracle_e8m0_byte.argtypes = [ctypes.c_float]
        L.oracle_e8m0_byte.restype = I32
        L.oracle_encode_fp4.argtypes = [P, I64, I64, P, P, U32P]
        L.oracle_encode_int_sym.argtypes = [P, I64, I64, I32, P, I32, P, P, U32P]
        L.oracle_kmeans_int4km.argtypes = [P, I64, I64, I32, P, P, P, U32P]
        L.oracle_encode_int4aff.argtypes = [P, I64, I64, P, P, U32P]
        L.oracle_int4aff_aux_row_bytes.argtypes = [I64]
        L.oracle_int4aff_aux_row_bytes.restype = I64
        L.oracle_kmeans_int8km.argtypes = [P, I64, I64, I32, P, P, P, U32P]
        L.oracle_outlier_columns.argtypes = [P, I64, I64, I64, P]
        L.oracle_encode_int4km_o8.argtypes = [P, I64, I64, I64, I32, P, P, P, P, P, U32P]
        L.oracle_dequant_int4km_o8.argtypes = [P, P, P, P, P, I64, I64, I64, P]
        L.oracle_matvec_int4km_o8.argtypes = [P, P, P, P, P, P, I32, I64, I64, I64, P]
        L.oracle_int8km_groups.argtypes = [I64]
        L.oracle_int8km_groups.restype = I64
        L.oracle_dequant.argtypes = [I32, P, P, I64, I64, P]
        L.oracle_matvec_rows.argtypes = [I32, P, P, P, I32, I64, I64, P, I64, P]
        L.oracle_gather_matvec.argtypes = [I32, P, P, I32, I64, I64, P, I32, I32, P, I32, P, U32P]
        L.oracle_num_threads.restype = I32
        L.oracle_set_num_threads.argtypes = [I32]
        for f in ("oracle_encode_fp4", "oracle_encode_int_sym", "oracle_kmeans_int4km", "oracle_encode_int4aff",
                  "oracle_kmeans_int8km", "oracle_outlier_columns", "oracle_encode_int4km_o8",
                  "oracle_dequant_int4km_o8", "oracle_matvec_int4km_o8",
                  "oracle_dequant",
                  "oracle_matvec_rows", "oracle_gather_matvec"):
            getattr(L, f).restype = I32
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with {rc}")


def num_threads():
    return lib().oracle_num_threads()


def set_num_threads(n):
    lib().oracle_set_num_threads(int(n))


def f32_to_f16_bits(v: float) -> int:
    return int(lib().oracle_f32_to_f16(float(v)))


def f16_bits_to_f32(h: int) -> float:
    return float(lib().oracle_f16_to_f32(int(h)))


def e2m1_code(v: float) -> int:
    return int(lib().oracle_e2m1_code(float(v)))


def e8m0_byte(amax: float) -> int:
    return int(lib().oracle_e8m0_byte(float(amax)))


def encode_fp4(W):
    """W float32 [N, K] -> (codes uint8 [N, K/2], scales uint8 [N, K/32], flags)."""
    W = _c(W, np.float32)
    N, K = W.shape
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // 32), np.uint8)
    fl = ctypes.c_uint32(0)
    _check(lib().oracle_encode_fp4(_p(W), N, K, _p(codes), _p(scales), ctypes.byref(fl)), "encode_fp4")
    return codes, scales, fl.value


def _encode_sym(W, qmax, clips):
    W = _c(W, np.float32)
    clips = _c(clips, np.float32)
    N, K = W.shape
    codes = np.zeros((N, K // 2) if qmax == 7 else (N, K), np.uint8 if qmax == 7 else np.int8)
    scales = np.zeros((N, K // 32), np.float16)
    fl = ctypes.c_uint32(0)
    _check(lib().oracle_encode_int_sym(_p(W), N, K, qmax, _p(clips), len(clips), _p(codes), _p(scales),
                                       ctypes.byref(fl)), "encode_int_sym")
    return codes, scales, fl.value


def encode_int4(W, clips=INT4_CLIPS):
    """-> (codes uint8 [N, K/2] holding q+8 nibbles, scales float16 [N, K/32], flags)."""
    return _encode_sym(W, 7, clips)


def encode_int8(W, clips=INT8_CLIPS):
    """-> (codes int8 [N, K], scales float16 [N, K/32], flags)."""
    return _encode_sym(W, 127, clips)


def int4aff_aux_row_bytes(K):
    return int(lib().oracle_int4aff_aux_row_bytes(int(K)))


def encode_int4aff(W):
    """-> (codes uint8 [N, K/2] (q nibbles), aux uint8 [N, row bytes] (fp16
    scales [K/32] then zero-point nibbles), flags)."""
    W = _c(W, np.float32)
    N, K = W.shape
    codes = np.zeros((N, K // 2), np.uint8)
    aux = np.zeros((N, int4aff_aux_row_bytes(K)), np.uint8)
    fl = ctypes.c_uint32(0)
    _check(lib().oracle_encode_int4aff(_p(W), N, K, _p(codes), _p(aux), ctypes.byref(fl)), "encode_int4aff")
    return codes, aux, fl.value


def kmeans_int4km(W, iters=KMEANS_ITERS, want_sse=False):
    """-> (lut float16 [N, 16], idx uint8 [N, K/2], flags[, sse double [N, iters+1]])."""
    W = _c(W, np.float32)
    N, K = W.shape
    lut = np.zeros((N, 16), np.float16)
    idx = np.zeros((N, K // 2), np.uint8)
    sse = np.zeros((N, iters + 1), np.float64) if want_sse else None
    fl = ctypes.c_uint32(0)
    _check(lib().oracle_kmeans_int4km(_p(W), N, K, iters, _p(lut), _p(idx),
                                      _p(sse) if want_sse else None, ctypes.byref(fl)), "kmeans")
    return (lut, idx, fl.value, sse) if want_sse else (lut, idx, fl.value)


def int8km_groups(N):
    return int(lib().oracle_int8km_groups(int(N)))


def kmeans_int8km(W, iters=KMEANS_ITERS, want_sse=False):
    """-> (lut float16 [ceil(N/32), 256], idx uint8 [N, K], flags[, sse double [ceil(N/32), iters+1]])."""
    W = _c(W, np.float32)
    N, K = W.shape
    G = int8km_groups(N)
    lut = np.zeros((G, 256), np.float16)
    idx = np.zeros((N, K), np.uint8)
    sse = np.zeros((G, iters + 1), np.float64) if want_sse else None
    fl = ctypes.c_uint32(0)
    _check(lib().oracle_kmeans_int8km(_p(W), N, K, iters, _p(lut), _p(idx),
                                      _p(sse) if want_sse else None, ctypes.byref(fl)), "kmeans8")
    return (lut, idx, fl.value, sse) if want_sse else (lut, idx, fl.value)


def outlier_columns(W, C):
    """The C columns (ascending, int32) with the largest max |w| (ties: lower index)."""
    W = _c(W, np.float32)
    N, K = W.shape
    cols = np.zeros(C, np.int32)
    _check(lib().oracle_outlier_columns(_p(W), N, K, int(C), _p(cols)), "outlier_columns")
    return cols


def encode_int4km_o8(W, C, iters=KMEANS_ITERS, cols=None):
    """Mixed int4km + int8 outlier columns.  -> (cols int32 [C], lut float16 [N, 16],
    idx uint8 [N, (K-C)/2], ocodes int8 [N, C], oscales float16 [N, C/32], flags)."""
    W = _c(W, np.float32)
    N, K = W.shape
    cols = outlier_columns(W, C) if cols is None else _c(cols, np.int32)
    lut = np.zeros((N, 16), np.float16)
    idx = np.zeros((N, (K - C) // 2), np.uint8)
    oc = np.zeros((N, C), np.int8)
    osc = np.zeros((N, C // 32), np.float16)
    fl = ctypes.c_uint32(0)
    _check(lib().oracle_encode_int4km_o8(_p(W), N, K, int(C), int(iters), _p(cols), _p(lut), _p(idx), _p(oc),
                                         _p(osc), ctypes.byref(fl)), "encode_int4km_o8")
    return cols, lut, idx, oc, osc, fl.value


def dequant_int4km_o8(cols, lut, idx, oc, osc, N, K):
    C = len(cols)
    out = np.zeros((N, K), np.float32)
    args = [_c(a, t) for a, t in ((lut, np.float16), (idx, np.uint8), (oc, np.int8), (osc, np.float16),
                                  (cols, np.int32))]
    _check(lib().oracle_dequant_int4km_o8(*[_p(a) for a in args], N, K, C, _p(out)), "dequant_int4km_o8")
    return out


def matvec_int4km_o8(cols, lut, idx, oc, osc, x, N, K):
    """fp64 r = x Wdq^T for the mixed format.  x float16 [B, K] -> float64 [B, N]."""
    C = len(cols)
    x = _c(x, np.float16)
    if x.ndim == 1:
        x = x[None]
    B = x.shape[0]
    out = np.zeros((B, N), np.float64)
    args = [_c(a, t) for a, t in ((lut, np.float16), (idx, np.uint8), (oc, np.int8), (osc, np.float16),
                                  (cols, np.int32))]
    _check(lib().oracle_matvec_int4km_o8(*[_p(a) for a in args], _p(x), B, N, K, C, _p(out)), "matvec_int4km_o8")
    return out


def dequant(fmt, codes, aux, N, K):
    """Exact float32 [N, K] dequantized weights."""
    codes = np.ascontiguousarray(codes)
    aux = np.ascontiguousarray(aux)
    out = np.zeros((N, K), np.float32)
    _check(lib().oracle_dequant(fmt, _p(codes), _p(aux), N, K, _p(out)), "dequant")
    return out


def matvec(fmt, codes, aux, x, N, K, rows=None):
    """fp64 r = x Wdq^T.  x float16 [B, K].  Returns float64 [B, N] (or [B, len(rows)])."""
    codes = np.ascontiguousarray(codes)
    aux = np.ascontiguousarray(aux)
    x = _c(x, np.float16)
    if x.ndim == 1:
        x = x[None]
    B = x.shape[0]
    if rows is None:
        R, rp = N, None
    else:
        rows = _c(rows, np.int64)
        R, rp = len(rows), rows
    out = np.zeros((B, R), np.float64)
    _check(lib().oracle_matvec_rows(fmt, _p(codes), _p(aux), _p(x), B, N, K,
                                    _p(rp) if rp is not None else None, R, _p(out)), "matvec")
    return out


def gather_matvec(fmt, codes_stack, aux_stack, E, N, K, ids, x, x_per_slot):
    """ids int32 [B, topk]; x float16 [B, K] or [B, topk, K].  -> (float64 [B, topk, N], flags)."""
    codes_stack = np.ascontiguousarray(codes_stack)
    aux_stack = np.ascontiguousarray(aux_stack)
    ids = _c(ids, np.int32)
    x = _c(x, np.float16)
    B, topk = ids.shape
    out = np.zeros((B, topk, N), np.float64)
    fl = ctypes.c_uint32(0)
    _check(lib().oracle_gather_matvec(fmt, _p(codes_stack), _p(aux_stack), E, N, K, _p(ids), B, topk, _p(x),
                                      int(x_per_slot), _p(out), ctypes.byref(fl)), "gather")
    return out, fl.value
