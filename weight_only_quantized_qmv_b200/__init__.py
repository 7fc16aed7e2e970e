"""weight_only_quantized_qmv_b200 -- Python binding of libqmv (B200, sm_100a).

Argument marshalling only: every step of encode / matvec / gather runs in the
library's CUDA kernels (libqmv.so, next to this file, built by _build.py).
PyTorch supplies device memory and the current stream.  There is no CPU or
library fallback: importing the binding without libqmv.so raises.

The functions mirror the C ABI in include/qmv.h (same names without the
``qmv_`` prefix).  Packed layouts: 4-bit codes uint8 [N, K/2] (element 2j in
the low nibble), fp4 scales uint8 [N, K/32] (e8m0), int4/int8 scales float16
[N, K/32], int4km palette float16 [N, 16]; activations float16 [B, K];
outputs float32 [B, N].
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqmv.so")

FMT_FP4, FMT_INT4, FMT_INT4KM, FMT_INT8, FMT_INT4AFF, FMT_INT8KM = 0, 1, 2, 3, 4, 5
FMT_NAMES = {FMT_FP4: "fp4", FMT_INT4: "int4", FMT_INT4KM: "int4km", FMT_INT8: "int8", FMT_INT4AFF: "int4aff",
             FMT_INT8KM: "int8km"}
KM8_GROUP = 32  # int8km: output rows sharing one 256-entry LUT
FLAG_NONFINITE, FLAG_SCALE_OVERFLOW, FLAG_BAD_EXPERT, FLAG_TIMEOUT = 1, 2, 4, 8
OK, ERR_ARG, ERR_SHAPE, ERR_UNSUPPORTED, ERR_DATA, ERR_CUDA = 0, -1, -2, -3, -4, -5

# Clip lists of the workloads: int4 searches 1.00, 0.95, ..., 0.50 (float32
# literals); int8 is plain symmetric absmax.
INT4_CLIPS = [1.0 - 0.05 * i for i in range(11)]
INT8_CLIPS = [1.0]


class QmvError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"libqmv status {status}: {msg}")
        self.status = status


_lib = None

# (name, argtypes) of every exported entry point
_P, _I64, _I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
SIGNATURES = {
    "qmv_encode_fp4": [_P, _I64, _I64, _P, _P, _P],
    "qmv_encode_int4": [_P, _I64, _I64, _P, _I32, _P, _P, _P],
    "qmv_encode_int8": [_P, _I64, _I64, _P, _I32, _P, _P, _P],
    "qmv_encode_int4km": [_P, _I64, _I64, _I32, _P, _P, _P],
    "qmv_encode_int4aff": [_P, _I64, _I64, _P, _P, _P],
    "qmv_int4aff_aux_row_bytes": [_I64],
    "qmv_matvec_fp4": [_P, _P, _P, _I32, _I64, _I64, _P, _P],
    "qmv_matvec_int4": [_P, _P, _P, _I32, _I64, _I64, _P, _P],
    "qmv_matvec_int4km": [_P, _P, _P, _I32, _I64, _I64, _P, _P],
    "qmv_matvec_int8": [_P, _P, _P, _I32, _I64, _I64, _P, _P],
    "qmv_matvec_int4aff": [_P, _P, _P, _I32, _I64, _I64, _P, _P],
    "qmv_matvec_int8km": [_P, _P, _P, _I32, _I64, _I64, _P, _P],
    "qmv_int4km_o8_encode_workspace_bytes": [_I64, _I64, _I64],
    "qmv_outlier_columns": [_P, _I64, _I64, _I64, _P, _P, ctypes.c_size_t, _P],
    "qmv_encode_int4km_o8": [_P, _I64, _I64, _I64, _I32, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "qmv_matvec_int4km_o8": [_P, _P, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _P, _P],
    "qmv_gather_matvec": [_I32, _P, _P, _I32, _I64, _I64, _P, _I32, _I32, _P, _I32, _P, _P],
    "qmv_matvec_argmax": [_I32, _P, _P, _P, _I32, _I64, _I64, _P, ctypes.c_size_t, _P, _P, _P],
    "qmv_argmax_workspace_bytes": [ctypes.POINTER(ctypes.c_size_t)],
    "qmv_matvec_argmax_static": [_I32, _P, _P, _P, _I32, _I64, _I64, _P, _P, _P],
    "qmv_dequant": [_I32, _P, _P, _I64, _I64, _P, _P],
    "qmv_status_fetch": [_P, ctypes.POINTER(ctypes.c_uint32)],
    "qmv_set_weight_prefetch": [_I32],
    "qmv_set_fp4_tensor_cores": [_I32],
    "qmv_encode_int8km": [_P, _I64, _I64, _I32, _P, _P, _P, ctypes.c_size_t, _P],
    "qmv_int8km_encode_workspace_bytes": [_I64, _I64],
    "qmv_last_error": [],
    "qmv_version": [],
}


def lib() -> ctypes.CDLL:
    """The loaded libqmv.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libqmv.so not found at {LIB_PATH}: build it with "
                              "`python -m weight_only_quantized_qmv_b200._build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in SIGNATURES.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = (ctypes.c_char_p if name in ("qmv_last_error", "qmv_version")
                         else ctypes.c_int64 if name.endswith("_bytes") and name != "qmv_argmax_workspace_bytes"
                         else ctypes.c_int)
        _lib = L
    return _lib


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _call(name, *args):
    rc = getattr(lib(), name)(*args)
    if rc != OK:
        raise QmvError(rc, lib().qmv_last_error().decode())
    return rc


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def version() -> str:
    return lib().qmv_version().decode()


# ---------------------------------------------------------------- encoders

def encode_fp4(W: torch.Tensor, stream=None):
    """W float32 [N, K] -> (codes uint8 [N, K/2], scales uint8 [N, K/32])."""
    _need(W, "W", torch.float32)
    N, K = W.shape
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N, K // 32), dtype=torch.uint8, device=W.device)
    _call("qmv_encode_fp4", _ptr(W), N, K, _ptr(codes), _ptr(scales), _stream(stream))
    return codes, scales


def _encode_int(name, W, clips, bits, stream):
    _need(W, "W", torch.float32)
    N, K = W.shape
    c = (ctypes.c_float * len(clips))(*[float(v) for v in clips])
    codes = torch.empty((N, K * bits // 8), dtype=torch.uint8 if bits == 4 else torch.int8, device=W.device)
    scales = torch.empty((N, K // 32), dtype=torch.float16, device=W.device)
    _call(name, _ptr(W), N, K, c, len(clips), _ptr(codes), _ptr(scales), _stream(stream))
    return codes, scales


def encode_int4(W: torch.Tensor, clips=INT4_CLIPS, stream=None):
    """-> (codes uint8 [N, K/2] (q + 8 nibbles), scales float16 [N, K/32])."""
    return _encode_int("qmv_encode_int4", W, clips, 4, stream)


def encode_int8(W: torch.Tensor, clips=INT8_CLIPS, stream=None):
    """-> (codes int8 [N, K], scales float16 [N, K/32])."""
    return _encode_int("qmv_encode_int8", W, clips, 8, stream)


KMEANS_ITERS = 20  # Lloyd steps of the int4km workloads


def encode_int4km(W: torch.Tensor, iters: int = KMEANS_ITERS, stream=None):
    """W float32 [N, K] -> (idx uint8 [N, K/2], lut float16 [N, 16]): per-row
    16-entry k-means palette and packed indices."""
    _need(W, "W", torch.float32)
    N, K = W.shape
    idx = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    lut = torch.empty((N, 16), dtype=torch.float16, device=W.device)
    _call("qmv_encode_int4km", _ptr(W), N, K, int(iters), _ptr(lut), _ptr(idx), _stream(stream))
    return idx, lut


def int4aff_aux_row_bytes(K: int) -> int:
    """Bytes of one int4aff aux row: fp16 scales [K/32], then zero points two per byte."""
    return int(lib().qmv_int4aff_aux_row_bytes(int(K)))


def encode_int4aff(W: torch.Tensor, stream=None):
    """W float32 [N, K] -> (codes uint8 [N, K/2] (q nibbles), aux uint8 [N,
    int4aff_aux_row_bytes(K)]): affine int4 per block of 32."""
    _need(W, "W", torch.float32)
    N, K = W.shape
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    aux = torch.empty((N, int4aff_aux_row_bytes(K)), dtype=torch.uint8, device=W.device)
    _call("qmv_encode_int4aff", _ptr(W), N, K, _ptr(codes), _ptr(aux), _stream(stream))
    return codes, aux


# ---------------------------------------------------------------- matvec

_AUX = {FMT_FP4: torch.uint8, FMT_INT4: torch.float16, FMT_INT4KM: torch.float16, FMT_INT8: torch.float16,
        FMT_INT4AFF: torch.uint8, FMT_INT8KM: torch.float16}
_CODES = {FMT_FP4: torch.uint8, FMT_INT4: torch.uint8, FMT_INT4KM: torch.uint8, FMT_INT8: torch.int8,
          FMT_INT4AFF: torch.uint8, FMT_INT8KM: torch.uint8}
_ENTRY = {FMT_FP4: "qmv_matvec_fp4", FMT_INT4: "qmv_matvec_int4", FMT_INT4KM: "qmv_matvec_int4km",
          FMT_INT8: "qmv_matvec_int8", FMT_INT4AFF: "qmv_matvec_int4aff", FMT_INT8KM: "qmv_matvec_int8km"}


def encode_int8km(W: torch.Tensor, iters: int = KMEANS_ITERS, stream=None):
    """W float32 [N, K] -> (idx uint8 [N, K], lut float16 [ceil(N/32), 256]):
    a 256-entry k-means palette per 32 rows and one index per weight."""
    _need(W, "W", torch.float32)
    N, K = W.shape
    idx = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    lut = torch.empty((int8km_groups(N), 256), dtype=torch.float16, device=W.device)
    nb = int(lib().qmv_int8km_encode_workspace_bytes(N, K))
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=W.device)
    _call("qmv_encode_int8km", _ptr(W), N, K, int(iters), _ptr(lut), _ptr(idx), _ptr(ws), ws.numel(),
          _stream(stream))
    return idx, lut


def int8km_groups(N: int) -> int:
    """LUT groups of an int8km matrix of N rows: ceil(N / 32)."""
    return (int(N) + KM8_GROUP - 1) // KM8_GROUP


def _nk(fmt, codes):
    N = codes.shape[-2]
    K = codes.shape[-1] * (1 if fmt in (FMT_INT8, FMT_INT8KM) else 2)
    return N, K


def aux_shape(fmt: int, N: int, K: int):
    """Shape of one matrix's scales / palette / aux rows in format fmt."""
    if fmt in (FMT_FP4, FMT_INT4, FMT_INT8):
        return (N, K // 32)
    if fmt == FMT_INT4KM:
        return (N, 16)
    if fmt == FMT_INT4AFF:
        return (N, int4aff_aux_row_bytes(K))
    if fmt == FMT_INT8KM:
        return (int8km_groups(N), 256)
    raise ValueError(f"unknown format {fmt}")


def _need_aux(fmt, aux, N, K, lead=()):
    want = tuple(lead) + aux_shape(fmt, N, K)
    if tuple(aux.shape) != want:
        raise ValueError(f"{FMT_NAMES[fmt]} aux must have shape {want}, got {tuple(aux.shape)}")


def matvec(fmt: int, codes: torch.Tensor, aux: torch.Tensor, x: torch.Tensor, out=None, stream=None):
    """y float32 [B, N] = x Wdq^T for x float16 [B, K] (or [K] -> [N])."""
    _need(codes, "codes", _CODES[fmt])
    _need(aux, "scales/lut", _AUX[fmt])
    N, K = _nk(fmt, codes)
    _need_aux(fmt, aux, N, K)
    squeeze = x.dim() == 1
    xx = x.unsqueeze(0) if squeeze else x
    _need(xx, "x", torch.float16)
    B = xx.shape[0]
    if xx.shape[1] != K:
        raise ValueError(f"x has {xx.shape[1]} features, weights have {K}")
    if out is None:
        out = torch.empty((B, N), dtype=torch.float32, device=codes.device)
    _need(out, "out", torch.float32, (B, N))
    _call(_ENTRY[fmt], _ptr(codes), _ptr(aux), _ptr(xx), B, N, K, _ptr(out), _stream(stream))
    return out[0] if squeeze else out


def matvec_fp4(codes, scales, x, out=None, stream=None):
    return matvec(FMT_FP4, codes, scales, x, out, stream)


def matvec_int4(codes, scales, x, out=None, stream=None):
    return matvec(FMT_INT4, codes, scales, x, out, stream)


def matvec_int4km(idx, lut, x, out=None, stream=None):
    return matvec(FMT_INT4KM, idx, lut, x, out, stream)


def matvec_int8(codes, scales, x, out=None, stream=None):
    return matvec(FMT_INT8, codes, scales, x, out, stream)


def matvec_int4aff(codes, aux, x, out=None, stream=None):
    return matvec(FMT_INT4AFF, codes, aux, x, out, stream)


def matvec_int8km(idx, lut, x, out=None, stream=None):
    """idx uint8 [N, K], lut float16 [ceil(N/32), 256] -> y float32 [B, N]."""
    return matvec(FMT_INT8KM, idx, lut, x, out, stream)


def argmax_workspace_bytes() -> int:
    """Workspace bytes matvec_argmax needs on the current device."""
    n = ctypes.c_size_t(0)
    _call("qmv_argmax_workspace_bytes", ctypes.byref(n))
    return int(n.value)


def argmax_workspace(device=None) -> torch.Tensor:
    """A zero-filled workspace for matvec_argmax (reusable, one call at a time)."""
    return torch.zeros(argmax_workspace_bytes(), dtype=torch.uint8, device=device or "cuda")


def matvec_argmax(fmt: int, codes: torch.Tensor, aux: torch.Tensor, x: torch.Tensor, workspace: torch.Tensor,
                  idx=None, val=None, stream=None):
    """Per activation row b: (idx int32 [B], val float32 [B]) = the lowest n
    with y[b, n] maximal and that maximum, y = x Wdq^T (not materialised)."""
    _need(codes, "codes", _CODES[fmt])
    _need(aux, "scales/lut", _AUX[fmt])
    _need(workspace, "workspace", torch.uint8)
    N, K = _nk(fmt, codes)
    _need_aux(fmt, aux, N, K)
    xx = x.unsqueeze(0) if x.dim() == 1 else x
    _need(xx, "x", torch.float16)
    B = xx.shape[0]
    if xx.shape[1] != K:
        raise ValueError(f"x has {xx.shape[1]} features, weights have {K}")
    if idx is None:
        idx = torch.empty(B, dtype=torch.int32, device=codes.device)
    if val is None:
        val = torch.empty(B, dtype=torch.float32, device=codes.device)
    _need(idx, "idx", torch.int32, (B,))
    _need(val, "val", torch.float32, (B,))
    _call("qmv_matvec_argmax", fmt, _ptr(codes), _ptr(aux), _ptr(xx), B, N, K, _ptr(workspace),
          workspace.numel(), _ptr(idx), _ptr(val), _stream(stream))
    return idx, val


def matvec_argmax_static(fmt: int, codes: torch.Tensor, aux: torch.Tensor, x: torch.Tensor, idx=None, val=None,
                         stream=None):
    """matvec_argmax on the library's own static scratch (no workspace, no
    allocation; one call at a time per device)."""
    _need(codes, "codes", _CODES[fmt])
    _need(aux, "scales/lut", _AUX[fmt])
    N, K = _nk(fmt, codes)
    _need_aux(fmt, aux, N, K)
    xx = x.unsqueeze(0) if x.dim() == 1 else x
    _need(xx, "x", torch.float16)
    B = xx.shape[0]
    if xx.shape[1] != K:
        raise ValueError(f"x has {xx.shape[1]} features, weights have {K}")
    if idx is None:
        idx = torch.empty(B, dtype=torch.int32, device=codes.device)
    if val is None:
        val = torch.empty(B, dtype=torch.float32, device=codes.device)
    _need(idx, "idx", torch.int32, (B,))
    _need(val, "val", torch.float32, (B,))
    _call("qmv_matvec_argmax_static", fmt, _ptr(codes), _ptr(aux), _ptr(xx), B, N, K, _ptr(idx), _ptr(val),
          _stream(stream))
    return idx, val


def gather_matvec(fmt: int, codes_stack: torch.Tensor, aux_stack: torch.Tensor, expert_ids: torch.Tensor,
                  x: torch.Tensor, x_per_slot: bool = False, out=None, stream=None):
    """y float32 [B, topk, N]; codes_stack [E, N, ...], aux_stack [E, N, ...],
    expert_ids int32 [B, topk], x float16 [B, K] or [B, topk, K]."""
    _need(codes_stack, "codes_stack", _CODES[fmt])
    _need(aux_stack, "aux_stack", _AUX[fmt])
    _need(expert_ids, "expert_ids", torch.int32)
    _need(x, "x", torch.float16)
    E = codes_stack.shape[0]
    N, K = _nk(fmt, codes_stack)
    if codes_stack.dim() != 3:
        raise ValueError("codes_stack must be [E, N, ...]")
    _need_aux(fmt, aux_stack, N, K, lead=(E,))
    B, topk = expert_ids.shape
    want = (B, topk, K) if x_per_slot else (B, K)
    if tuple(x.shape) != want:
        raise ValueError(f"x must have shape {want}, got {tuple(x.shape)}")
    if out is None:
        out = torch.empty((B, topk, N), dtype=torch.float32, device=codes_stack.device)
    _need(out, "out", torch.float32, (B, topk, N))
    _call("qmv_gather_matvec", fmt, _ptr(codes_stack), _ptr(aux_stack), E, N, K, _ptr(expert_ids), B, topk,
          _ptr(x), int(bool(x_per_slot)), _ptr(out), _stream(stream))
    return out


def dequant(fmt: int, codes: torch.Tensor, aux: torch.Tensor, stream=None) -> torch.Tensor:
    """Exact float32 [N, K] dequantized weights (test support)."""
    _need(codes, "codes", _CODES[fmt])
    _need(aux, "aux", _AUX[fmt])
    N, K = _nk(fmt, codes)
    _need_aux(fmt, aux, N, K)
    out = torch.empty((N, K), dtype=torch.float32, device=codes.device)
    _call("qmv_dequant", fmt, _ptr(codes), _ptr(aux), N, K, _ptr(out), _stream(stream))
    return out


# ---------------------------------------------------------------- mixed int4km + int8 outlier columns

def outlier_columns(W: torch.Tensor, C: int, stream=None) -> torch.Tensor:
    """int32 [C]: the C columns of W (float32 [N, K]) with the largest max |w|, ascending."""
    _need(W, "W", torch.float32)
    N, K = W.shape
    cols = torch.empty(C, dtype=torch.int32, device=W.device)
    ws = torch.empty(max(8 * K, 16), dtype=torch.uint8, device=W.device)
    _call("qmv_outlier_columns", _ptr(W), N, K, int(C), _ptr(cols), _ptr(ws), ws.numel(), _stream(stream))
    return cols


def encode_int4km_o8(W: torch.Tensor, C: int, iters: int = KMEANS_ITERS, stream=None):
    """W float32 [N, K] -> (cols int32 [C], lut float16 [N, 16], idx uint8 [N, (K-C)/2],
    ocodes int8 [N, C], oscales float16 [N, C/32])."""
    _need(W, "W", torch.float32)
    N, K = W.shape
    dev = W.device
    cols = torch.empty(C, dtype=torch.int32, device=dev)
    lut = torch.empty((N, 16), dtype=torch.float16, device=dev)
    idx = torch.empty((N, (K - C) // 2), dtype=torch.uint8, device=dev)
    oc = torch.empty((N, C), dtype=torch.int8, device=dev)
    osc = torch.empty((N, C // 32), dtype=torch.float16, device=dev)
    nb = int(lib().qmv_int4km_o8_encode_workspace_bytes(N, K, int(C)))
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
    _call("qmv_encode_int4km_o8", _ptr(W), N, K, int(C), int(iters), _ptr(cols), _ptr(lut), _ptr(idx), _ptr(oc),
          _ptr(osc), _ptr(ws), ws.numel(), _stream(stream))
    return cols, lut, idx, oc, osc


def matvec_int4km_o8(cols, lut, idx, oc, osc, x, out=None, stream=None):
    """y float32 [B, N] = x Wdq^T for the mixed format; x float16 [B, K] (or [K])."""
    _need(idx, "idx", torch.uint8)
    _need(lut, "lut", torch.float16)
    _need(oc, "ocodes", torch.int8)
    _need(osc, "oscales", torch.float16)
    _need(cols, "cols", torch.int32)
    N = idx.shape[0]
    C = cols.numel()
    K = 2 * idx.shape[1] + C
    if tuple(lut.shape) != (N, 16) or tuple(oc.shape) != (N, C) or tuple(osc.shape) != (N, C // 32):
        raise ValueError("lut / ocodes / oscales shapes do not match idx and cols")
    squeeze = x.dim() == 1
    xx = x.unsqueeze(0) if squeeze else x
    _need(xx, "x", torch.float16)
    B = xx.shape[0]
    if xx.shape[1] != K:
        raise ValueError(f"x has {xx.shape[1]} features, weights have {K}")
    if out is None:
        out = torch.empty((B, N), dtype=torch.float32, device=idx.device)
    _need(out, "out", torch.float32, (B, N))
    _call("qmv_matvec_int4km_o8", _ptr(idx), _ptr(lut), _ptr(oc), _ptr(osc), _ptr(cols), _ptr(xx), B, N, K, C,
          _ptr(out), _stream(stream))
    return out[0] if squeeze else out


def set_weight_prefetch(enable: bool) -> None:
    """Let dense matvec launches start streaming weights before the preceding
    work in their stream completes (only while nothing in flight writes the
    weights; see qmv_set_weight_prefetch in include/qmv.h)."""
    _call("qmv_set_weight_prefetch", int(bool(enable)))


def set_fp4_tensor_cores(enable: bool) -> None:
    """Run dense fp4 matvecs at 2..16 activation columns on the tcgen05
    tensor-memory kernel where their shape allows (see
    qmv_set_fp4_tensor_cores in include/qmv.h); off: the mma.sync kernel."""
    _call("qmv_set_fp4_tensor_cores", int(bool(enable)))


def status_fetch(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device status flags."""
    flags = ctypes.c_uint32(0)
    rc = lib().qmv_status_fetch(_stream(stream), ctypes.byref(flags))
    if rc not in (OK, ERR_DATA):
        raise QmvError(rc, lib().qmv_last_error().decode())
    return int(flags.value)
