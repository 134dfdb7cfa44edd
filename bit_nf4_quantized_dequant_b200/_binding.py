"""ctypes binding of libqlora: argument marshalling only.

Every call maps one-to-one onto a C entry point of ``include/qlora.h``; torch
supplies device memory (output tensors are allocated with torch when the
caller passes none) and the current CUDA stream. No step of the computation
runs here. If the shared library is missing or cannot be loaded, every call
raises ``QloraUnavailable``; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

__all__ = [
    "QloraError", "QloraUnavailable", "NF4Matrix", "library", "library_path", "SYMBOLS",
    "nf4_sizes", "nf4_codebook", "nf4_quantize", "nf4_dequantize",
    "linear_workspace", "linear_fwd", "linear_bwd", "status_string", "STATUS",
    "lora_xa", "fused_fwd", "lora_dyb", "fused_dx", "lora_grads", "linear_fwd_noalloc",
    "fused_workspace", "swiglu_fwd", "swiglu_bwd", "swiglu_pack_b", "swiglu_unpack_db", "swiglu_interleave",
    "nf4_merge", "codec_levels", "codec_quantize", "codec_dequantize", "CODEBOOK_NF4", "CODEBOOK_INT4",
    "adamw8_step", "AdamW8State", "set_gemm_schedule", "gemm_schedule",
    "SCHEDULE_AUTO", "SCHEDULE_SINGLE", "SCHEDULE_PAIR", "dqfp8_sizes", "dqfp8_quantize", "dqfp8_dequantize",
    "lora_grads_adamw8", "selftest_bounded_wait", "linear_fwd_group", "linear_fwd_group_workspace",
    "LinearProblem", "FWD_OVERLAP_PREVIOUS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libqlora.so")

STATUS = {
    0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_UNSUPPORTED_SHAPE",
    3: "QLORA_ERR_MISALIGNED", 4: "QLORA_ERR_WORKSPACE", 5: "QLORA_ERR_NONFINITE",
    6: "QLORA_ERR_TIMEOUT", 7: "QLORA_ERR_CUDA",
}

# every symbol include/qlora.h declares
SYMBOLS = [
    "qlora_nf4_sizes", "qlora_nf4_codebook", "qlora_nf4_quantize", "qlora_nf4_dequantize",
    "qlora_linear_workspace", "qlora_linear_fwd", "qlora_linear_bwd", "qlora_status_string",
    "qlora_lora_xa", "qlora_fused_fwd", "qlora_lora_dyb", "qlora_fused_dx", "qlora_lora_grads",
    "qlora_linear_fwd_noalloc", "qlora_fused_workspace",
    "qlora_swiglu_fwd", "qlora_swiglu_bwd", "qlora_swiglu_pack_b", "qlora_swiglu_unpack_db",
    "qlora_nf4_merge", "qlora_codec_levels", "qlora_codec_quantize", "qlora_codec_dequantize",
    "qlora_adamw8_step", "qlora_set_gemm_schedule",
    "qlora_dqfp8_sizes", "qlora_dqfp8_quantize", "qlora_dqfp8_dequantize",
    "qlora_lora_grads_adamw8", "qlora_selftest_bounded_wait",
    "qlora_linear_fwd_group_workspace", "qlora_linear_fwd_group",
]


class _Adam8(ctypes.Structure):
    _fields_ = [("p", ctypes.c_void_p), ("p_bf16", ctypes.c_void_p), ("m_q", ctypes.c_void_p),
                ("v_q", ctypes.c_void_p), ("m_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p)]


class QloraUnavailable(RuntimeError):
    """libqlora.so is missing or failed to load."""


class QloraError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call} returned {STATUS.get(status, status)}")


class _NF4(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("scale8", ctypes.c_void_p), ("scale2", ctypes.c_void_p)]


class _Problem(ctypes.Structure):
    _fields_ = [("W", _NF4), ("X", ctypes.c_void_p), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p),
                ("r", ctypes.c_int32), ("s", ctypes.c_float), ("Y", ctypes.c_void_p), ("sU_out", ctypes.c_void_p)]


FWD_OVERLAP_PREVIOUS = 1

_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t


def library():
    """The loaded shared library (loaded once)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise QloraUnavailable(f"{library_path} not built (run bit_nf4_quantized_dequant_b200._build)")
    try:
        lib = ctypes.CDLL(library_path)
    except OSError as e:  # pragma: no cover - depends on the machine
        raise QloraUnavailable(f"cannot load {library_path}: {e}") from e
    st = ctypes.c_int
    lib.qlora_nf4_sizes.argtypes = [_I64, _I64, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)]
    lib.qlora_nf4_sizes.restype = st
    lib.qlora_nf4_codebook.argtypes = [ctypes.POINTER(ctypes.c_float)]
    lib.qlora_nf4_codebook.restype = st
    lib.qlora_nf4_quantize.argtypes = [_P, ctypes.POINTER(_NF4), _P, _P]
    lib.qlora_nf4_quantize.restype = st
    lib.qlora_nf4_dequantize.argtypes = [ctypes.POINTER(_NF4), _P, _P]
    lib.qlora_nf4_dequantize.restype = st
    lib.qlora_linear_workspace.argtypes = [_I64, _I64, _I64, ctypes.c_int32, ctypes.POINTER(_SZ)]
    lib.qlora_linear_workspace.restype = st
    lib.qlora_linear_fwd.argtypes = [ctypes.POINTER(_NF4), _P, _I64, _P, _P, ctypes.c_int32, ctypes.c_float,
                                     _P, _P, _P, _SZ, _P, _P]
    lib.qlora_linear_fwd.restype = st
    lib.qlora_linear_bwd.argtypes = [ctypes.POINTER(_NF4), _P, _I64, _P, _P, ctypes.c_int32, ctypes.c_float,
                                     _P, _P, _P, _P, _P, _P, _SZ, _P, _P]
    lib.qlora_linear_bwd.restype = st
    lib.qlora_lora_xa.argtypes = [_P, _I64, _I64, _P, ctypes.c_int32, ctypes.c_float, _P, _P, _SZ, _P]
    lib.qlora_lora_xa.restype = st
    lib.qlora_lora_dyb.argtypes = [_P, _I64, _I64, _P, ctypes.c_int32, ctypes.c_float, _P, _P, _SZ, _P]
    lib.qlora_lora_dyb.restype = st
    lib.qlora_swiglu_fwd.argtypes = [ctypes.POINTER(_NF4), _P, _I64, _P, ctypes.c_int32, _P, _P, _P, _P]
    lib.qlora_swiglu_fwd.restype = st
    lib.qlora_swiglu_bwd.argtypes = [ctypes.POINTER(_NF4), _P, _I64, _P, ctypes.c_int32, _P, _P, _P, _P, _P]
    lib.qlora_swiglu_bwd.restype = st
    lib.qlora_swiglu_pack_b.argtypes = [_P, _P, _I64, ctypes.c_int32, _P, _P]
    lib.qlora_swiglu_pack_b.restype = st
    lib.qlora_swiglu_unpack_db.argtypes = [_P, _I64, ctypes.c_int32, _P, _P, _P]
    lib.qlora_swiglu_unpack_db.restype = st
    lib.qlora_adamw8_step.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I64, ctypes.c_int32, ctypes.c_float,
                                      ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_float, _P]
    lib.qlora_adamw8_step.restype = st
    lib.qlora_set_gemm_schedule.argtypes = [ctypes.c_int32]
    lib.qlora_set_gemm_schedule.restype = st
    lib.qlora_dqfp8_sizes.argtypes = [_I64, _I64, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)]
    lib.qlora_dqfp8_sizes.restype = st
    lib.qlora_dqfp8_quantize.argtypes = [_P, ctypes.POINTER(_NF4), _P, _P]
    lib.qlora_dqfp8_quantize.restype = st
    lib.qlora_dqfp8_dequantize.argtypes = [ctypes.POINTER(_NF4), _P, _P]
    lib.qlora_dqfp8_dequantize.restype = st
    lib.qlora_lora_grads_adamw8.argtypes = [_P, _P, _I64, _I64, _I64, _P, _P, ctypes.c_int32, _P, _P,
                                            ctypes.POINTER(_Adam8), ctypes.POINTER(_Adam8), ctypes.c_int32,
                                            ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                            ctypes.c_float, _P]
    lib.qlora_lora_grads_adamw8.restype = st
    lib.qlora_selftest_bounded_wait.argtypes = [_P, _P]
    lib.qlora_selftest_bounded_wait.restype = st
    lib.qlora_codec_levels.argtypes = [ctypes.c_int32, ctypes.POINTER(ctypes.c_float)]
    lib.qlora_codec_levels.restype = st
    lib.qlora_codec_quantize.argtypes = [_P, ctypes.POINTER(_NF4), ctypes.c_int32, _P, _P]
    lib.qlora_codec_quantize.restype = st
    lib.qlora_codec_dequantize.argtypes = [ctypes.POINTER(_NF4), ctypes.c_int32, _P, _P]
    lib.qlora_codec_dequantize.restype = st
    lib.qlora_nf4_merge.argtypes = [ctypes.POINTER(_NF4), _P, _P, ctypes.c_int32, ctypes.c_float, _P, ctypes.c_int32,
                                    _P]
    lib.qlora_nf4_merge.restype = st
    lib.qlora_fused_workspace.argtypes = [_I64, ctypes.POINTER(_SZ)]
    lib.qlora_fused_workspace.restype = st
    lib.qlora_fused_fwd.argtypes = [ctypes.POINTER(_NF4), _P, _I64, _P, ctypes.c_int32, _P, _P, _P, _SZ, _P, _P]
    lib.qlora_fused_fwd.restype = st
    lib.qlora_fused_dx.argtypes = [ctypes.POINTER(_NF4), _P, _I64, _P, ctypes.c_int32, _P, _P, _P, _SZ, _P, _P]
    lib.qlora_fused_dx.restype = st
    lib.qlora_lora_grads.argtypes = [_P, _P, _I64, _I64, _I64, _P, _P, ctypes.c_int32, _P, _P, _P, _SZ, _P]
    lib.qlora_lora_grads.restype = st
    lib.qlora_linear_fwd_noalloc.argtypes = [ctypes.POINTER(_NF4), _P, _I64, _P, _P, ctypes.c_int32,
                                             ctypes.c_float, _P, _P, _P, _P]
    lib.qlora_linear_fwd_noalloc.restype = st
    lib.qlora_linear_fwd_group_workspace.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int32, _I64,
                                                     ctypes.POINTER(_SZ)]
    lib.qlora_linear_fwd_group_workspace.restype = st
    lib.qlora_linear_fwd_group.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int32, _I64, ctypes.c_int32, _P, _SZ,
                                           _P, _P]
    lib.qlora_linear_fwd_group.restype = st
    lib.qlora_status_string.argtypes = [ctypes.c_int]
    lib.qlora_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(status: int, call: str):
    if status != 0:
        raise QloraError(status, call)


def status_string(status: int) -> str:
    return library().qlora_status_string(status).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def nf4_sizes(rows: int, cols: int):
    """(code bytes, scale8 bytes, scale2 bytes) of a [rows, cols] NF4 matrix."""
    a, b, c = _SZ(), _SZ(), _SZ()
    _check(library().qlora_nf4_sizes(rows, cols, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "qlora_nf4_sizes")
    return a.value, b.value, c.value


def nf4_codebook():
    import numpy as np
    out = (ctypes.c_float * 16)()
    _check(library().qlora_nf4_codebook(out), "qlora_nf4_codebook")
    return np.frombuffer(bytes(out), dtype=np.float32).copy()


@dataclass
class NF4Matrix:
    """Device buffers of one NF4 matrix (torch uint8/uint8/float32 tensors)."""
    rows: int
    cols: int
    codes: object
    scale8: object
    scale2: object

    def c_struct(self) -> _NF4:
        return _NF4(self.rows, self.cols, self.codes.data_ptr(), self.scale8.data_ptr(), self.scale2.data_ptr())

    @classmethod
    def empty(cls, rows: int, cols: int, device="cuda"):
        import torch
        cb, sb, s2b = nf4_sizes(rows, cols)
        return cls(rows, cols, torch.empty(cb, dtype=torch.uint8, device=device),
                   torch.empty(sb, dtype=torch.uint8, device=device),
                   torch.empty(s2b // 4, dtype=torch.float32, device=device))


def nf4_quantize(W, out: NF4Matrix | None = None, status=None, stream=None) -> NF4Matrix:
    """Quantise a contiguous float32 CUDA tensor W[N, K] (K % 64 == 0)."""
    rows, cols = W.shape
    q = out if out is not None else NF4Matrix.empty(rows, cols, W.device)
    s = q.c_struct()
    _check(library().qlora_nf4_quantize(_ptr(W), ctypes.byref(s), _ptr(status), _stream(stream)),
           "qlora_nf4_quantize")
    return q


def nf4_dequantize(q: NF4Matrix, out=None, stream=None):
    import torch
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=torch.bfloat16, device=q.codes.device)
    s = q.c_struct()
    _check(library().qlora_nf4_dequantize(ctypes.byref(s), _ptr(out), _stream(stream)), "qlora_nf4_dequantize")
    return out


def linear_workspace(M: int, N: int, K: int, r: int) -> int:
    b = _SZ()
    _check(library().qlora_linear_workspace(M, N, K, r, ctypes.byref(b)), "qlora_linear_workspace")
    return b.value


def _ws(ws, M, N, K, r, device):
    import torch
    need = linear_workspace(M, N, K, r)
    if ws is None:   # the first bytes (a counter page) must be zero before first use
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
    return ws


def linear_fwd(q: NF4Matrix, X, A, B, s: float, Y=None, sU=None, ws=None, status=None, stream=None,
               want_sU: bool = True):
    """Y = X W'^T + s (X A^T) B^T. Returns (Y, sU) with sU = bf16(s X A^T) (or None)."""
    import torch
    M, K = X.shape
    r = A.shape[0]
    N = q.rows
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    if sU is None and want_sU:
        sU = torch.empty((M, r), dtype=torch.bfloat16, device=X.device)
    ws = _ws(ws, M, N, K, r, X.device)
    st = q.c_struct()
    _check(library().qlora_linear_fwd(ctypes.byref(st), _ptr(X), M, _ptr(A), _ptr(B), r, s, _ptr(Y), _ptr(sU),
                                      _ptr(ws), ws.numel(), _ptr(status), _stream(stream)), "qlora_linear_fwd")
    return Y, sU


def linear_bwd(q: NF4Matrix, X, A, B, s: float, dY, sU=None, dX=None, dA=None, dB=None, ws=None,
               status=None, stream=None, want_dX: bool = True):
    """(dX, dA, dB) of the QLoRA linear; dW is never formed."""
    import torch
    M, K = X.shape
    r = A.shape[0]
    N = q.rows
    if dX is None and want_dX:
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=X.device)
    if dA is None:
        dA = torch.empty((r, K), dtype=torch.float32, device=X.device)
    if dB is None:
        dB = torch.empty((N, r), dtype=torch.float32, device=X.device)
    ws = _ws(ws, M, N, K, r, X.device)
    st = q.c_struct()
    _check(library().qlora_linear_bwd(ctypes.byref(st), _ptr(X), M, _ptr(A), _ptr(B), r, s, _ptr(dY), _ptr(sU),
                                      _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), _ptr(status),
                                      _stream(stream)), "qlora_linear_bwd")
    return dX, dA, dB


@dataclass
class LinearProblem:
    """One linear of a grouped few-token forward: Y = X W'^T + s (X A^T) B^T."""
    q: NF4Matrix
    X: object
    A: object
    B: object
    s: float
    Y: object
    sU: object = None

    def c_struct(self) -> _Problem:
        return _Problem(self.q.c_struct(), self.X.data_ptr(), self.A.data_ptr(), self.B.data_ptr(),
                        self.A.shape[0], self.s, self.Y.data_ptr(), None if self.sU is None else self.sU.data_ptr())


def _problem_array(problems):
    arr = (_Problem * len(problems))()
    for i, p in enumerate(problems):
        arr[i] = p.c_struct()
    return arr


def linear_fwd_group_workspace(problems, M: int) -> int:
    b = _SZ()
    _check(library().qlora_linear_fwd_group_workspace(_problem_array(problems), len(problems), M, ctypes.byref(b)),
           "qlora_linear_fwd_group_workspace")
    return b.value


def linear_fwd_group(problems, ws=None, flags: int = 0, status=None, stream=None, arr=None):
    """Few-token forward (M <= 16) of several linears in one launch. `arr` may
    hold a prebuilt ctypes problem array (e.g. for repeated calls)."""
    import torch
    M = problems[0].X.shape[0]
    if arr is None:
        arr = _problem_array(problems)
    if ws is None:
        ws = torch.zeros(linear_fwd_group_workspace(problems, M), dtype=torch.uint8, device=problems[0].X.device)
    _check(library().qlora_linear_fwd_group(arr, len(problems), M, flags, _ptr(ws), ws.numel(), _ptr(status),
                                            _stream(stream)), "qlora_linear_fwd_group")
    return [p.Y for p in problems]


# ---- the individual steps of the layer ---------------------------------------

def lora_xa(X, A, s: float, sU, ws, stream=None):
    """sU = bf16(s X A^T)."""
    M, K = X.shape
    _check(library().qlora_lora_xa(_ptr(X), M, K, _ptr(A), A.shape[0], s, _ptr(sU), _ptr(ws), ws.numel(),
                                   _stream(stream)), "qlora_lora_xa")
    return sU


def lora_dyb(dY, B, s: float, sT, ws, stream=None):
    """sT = bf16(s dY B)."""
    M, N = dY.shape
    _check(library().qlora_lora_dyb(_ptr(dY), M, N, _ptr(B), B.shape[1], s, _ptr(sT), _ptr(ws), ws.numel(),
                                    _stream(stream)), "qlora_lora_dyb")
    return sT


def fused_workspace(M: int) -> int:
    """Bytes of the optional stream-K workspace of fused_fwd / fused_dx."""
    b = _SZ(0)
    _check(library().qlora_fused_workspace(M, ctypes.byref(b)), "qlora_fused_workspace")
    return b.value


def _ws_args(ws):
    return (None, 0) if ws is None else (_ptr(ws), ws.numel() * ws.element_size())


def fused_fwd(q: NF4Matrix, X, B, sU, Y, status=None, stream=None, ws=None):
    """Y = X W'^T + sU B^T (dequantisation fused into the tensor-core GEMM).
    With `ws` (fused_workspace(M) bytes) the work is split stream-K over all SMs."""
    st = q.c_struct()
    _check(library().qlora_fused_fwd(ctypes.byref(st), _ptr(X), X.shape[0], _ptr(B), B.shape[1], _ptr(sU),
                                     _ptr(Y), *_ws_args(ws), _ptr(status), _stream(stream)), "qlora_fused_fwd")
    return Y


def fused_dx(q: NF4Matrix, dY, A, sT, dX, status=None, stream=None, ws=None):
    """dX = dY W' + sT A (dequantisation fused into the tensor-core GEMM); `ws` as in fused_fwd."""
    st = q.c_struct()
    _check(library().qlora_fused_dx(ctypes.byref(st), _ptr(dY), dY.shape[0], _ptr(A), A.shape[0], _ptr(sT),
                                    _ptr(dX), *_ws_args(ws), _ptr(status), _stream(stream)), "qlora_fused_dx")
    return dX


def lora_grads(X, dY, sU, sT, dA, dB, ws, stream=None):
    """dA = sT^T X, dB = dY^T sU (fp32, overwritten)."""
    M, K = X.shape
    N = dY.shape[1]
    r = sU.shape[1]
    _check(library().qlora_lora_grads(_ptr(X), _ptr(dY), M, N, K, _ptr(sU), _ptr(sT), r, _ptr(dA), _ptr(dB),
                                      _ptr(ws), ws.numel(), _stream(stream)), "qlora_lora_grads")
    return dA, dB


def linear_fwd_noalloc(q: NF4Matrix, X, A, B, s: float, Y=None, sU=None, status=None, stream=None):
    """Y = X W'^T + s (X A^T) B^T without a workspace: the library takes its
    scratch from a fixed device array (see qlora_linear_fwd_noalloc)."""
    import torch
    M = X.shape[0]
    r = A.shape[0]
    if Y is None:
        Y = torch.empty((M, q.rows), dtype=torch.bfloat16, device=X.device)
    st = q.c_struct()
    _check(library().qlora_linear_fwd_noalloc(ctypes.byref(st), _ptr(X), M, _ptr(A), _ptr(B), r, s, _ptr(Y),
                                              _ptr(sU), _ptr(status), _stream(stream)), "qlora_linear_fwd_noalloc")
    return Y, sU


# ---------------------------------------------------------------------------
# Fused SwiGLU projection (gate and up in one GEMM over the row-interleaved
# weight; see include/qlora.h)
# ---------------------------------------------------------------------------
def swiglu_interleave(Wg, Wu):
    """[Wg; Wu] with rows interleaved in chunks of 64 (a torch tensor op on the
    float32 weights before quantisation; F % 64 == 0)."""
    import torch
    F, K = Wg.shape
    return torch.stack([Wg.reshape(F // 64, 64, K), Wu.reshape(F // 64, 64, K)], 1).reshape(2 * F, K).contiguous()


def swiglu_pack_b(Bg, Bu, out=None, stream=None):
    """Block-diagonal [2F, 2r] up-projection of the fused product."""
    import torch
    F, r = Bg.shape
    if out is None:
        out = torch.empty((2 * F, 2 * r), dtype=torch.bfloat16, device=Bg.device)
    _check(library().qlora_swiglu_pack_b(_ptr(Bg), _ptr(Bu), F, r, _ptr(out), _stream(stream)), "qlora_swiglu_pack_b")
    return out


def swiglu_unpack_db(dBgu, dBg=None, dBu=None, stream=None):
    import torch
    F2, r2 = dBgu.shape
    F, r = F2 // 2, r2 // 2
    if dBg is None:
        dBg = torch.empty((F, r), dtype=torch.float32, device=dBgu.device)
    if dBu is None:
        dBu = torch.empty((F, r), dtype=torch.float32, device=dBgu.device)
    _check(library().qlora_swiglu_unpack_db(_ptr(dBgu), F, r, _ptr(dBg), _ptr(dBu), _stream(stream)),
           "qlora_swiglu_unpack_db")
    return dBg, dBu


def swiglu_fwd(q: NF4Matrix, X, Bgu, sUgu, H=None, status=None, stream=None):
    """H = bf16(silu(g) u) for the interleaved gate/up weight q [2F, K]."""
    import torch
    M = X.shape[0]
    if H is None:
        H = torch.empty((M, q.rows // 2), dtype=torch.bfloat16, device=X.device)
    st = q.c_struct()
    _check(library().qlora_swiglu_fwd(ctypes.byref(st), _ptr(X), M, _ptr(Bgu), Bgu.shape[1], _ptr(sUgu), _ptr(H),
                                      _ptr(status), _stream(stream)), "qlora_swiglu_fwd")
    return H


def swiglu_bwd(q: NF4Matrix, X, Bgu, sUgu, dH, dGU=None, status=None, stream=None):
    """dGU [M, 2F] (dg in gate rows, du in up rows) with g, u recomputed."""
    import torch
    M = X.shape[0]
    if dGU is None:
        dGU = torch.empty((M, q.rows), dtype=torch.bfloat16, device=X.device)
    st = q.c_struct()
    _check(library().qlora_swiglu_bwd(ctypes.byref(st), _ptr(X), M, _ptr(Bgu), Bgu.shape[1], _ptr(sUgu), _ptr(dH),
                                      _ptr(dGU), _ptr(status), _stream(stream)), "qlora_swiglu_bwd")
    return dGU


def nf4_merge(q: NF4Matrix, A, B, s: float, out=None, f32: bool = False, stream=None):
    """W' + s B A as bf16 (or fp32 with f32=True) [rows, cols]."""
    import torch
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=torch.float32 if f32 else torch.bfloat16, device=A.device)
    st = q.c_struct()
    _check(library().qlora_nf4_merge(ctypes.byref(st), _ptr(A), _ptr(B), A.shape[0], s, _ptr(out), 1 if f32 else 0,
                                     _stream(stream)), "qlora_nf4_merge")
    return out


CODEBOOK_NF4, CODEBOOK_INT4 = 0, 1


def codec_levels(codebook: int):
    out = (ctypes.c_float * 16)()
    _check(library().qlora_codec_levels(codebook, out), "qlora_codec_levels")
    return list(out)


def codec_quantize(W, codebook: int, out: NF4Matrix | None = None, status=None, stream=None) -> NF4Matrix:
    """Quantise with NF4 or the evenly spaced int4 comparison codebook (same format)."""
    rows, cols = W.shape
    q = out if out is not None else NF4Matrix.empty(rows, cols, W.device)
    s = q.c_struct()
    _check(library().qlora_codec_quantize(_ptr(W), ctypes.byref(s), codebook, _ptr(status), _stream(stream)),
           "qlora_codec_quantize")
    return q


def codec_dequantize(q: NF4Matrix, codebook: int, out=None, stream=None):
    import torch
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=torch.bfloat16, device=q.codes.device)
    s = q.c_struct()
    _check(library().qlora_codec_dequantize(ctypes.byref(s), codebook, _ptr(out), _stream(stream)),
           "qlora_codec_dequantize")
    return out


class AdamW8State:
    """8-bit AdamW states of one parameter tensor (zero-initialised)."""

    def __init__(self, numel: int, device="cuda"):
        import torch
        blocks = -(-numel // 256)
        self.m_q = torch.zeros(numel, dtype=torch.int8, device=device)
        self.v_q = torch.zeros(numel, dtype=torch.uint8, device=device)
        self.m_scale = torch.zeros(blocks, dtype=torch.float32, device=device)
        self.v_scale = torch.zeros(blocks, dtype=torch.float32, device=device)
        self.step = 0


def adamw8_step(p, grad, state: AdamW8State, lr: float, beta1: float = 0.9, beta2: float = 0.999,
                eps: float = 1e-8, weight_decay: float = 0.0, p_bf16=None, stream=None):
    """One AdamW step on fp32 p (in place) with 8-bit states; optional bf16 copy."""
    state.step += 1
    _check(library().qlora_adamw8_step(_ptr(p), _ptr(p_bf16), _ptr(grad), _ptr(state.m_q), _ptr(state.v_q),
                                       _ptr(state.m_scale), _ptr(state.v_scale), p.numel(), state.step, lr, beta1,
                                       beta2, eps, weight_decay, _stream(stream)), "qlora_adamw8_step")
    return p


# ---------------------------------------------------------------------------
# fused-GEMM tile schedule (process-wide)
# ---------------------------------------------------------------------------
SCHEDULE_AUTO, SCHEDULE_SINGLE, SCHEDULE_PAIR = 0, 1, 2


class gemm_schedule:
    """Context manager that selects the fused GEMM's tile schedule
    (qlora_set_gemm_schedule) and restores the automatic one on exit."""

    def __init__(self, schedule: int):
        self.schedule = schedule

    def __enter__(self):
        set_gemm_schedule(self.schedule)
        return self

    def __exit__(self, *exc):
        set_gemm_schedule(SCHEDULE_AUTO)
        return False


def set_gemm_schedule(schedule: int) -> None:
    _check(library().qlora_set_gemm_schedule(int(schedule)), "qlora_set_gemm_schedule")


# ---------------------------------------------------------------------------
# comparison second level: E4M3 codes of mean-centred block constants
# ---------------------------------------------------------------------------
def dqfp8_sizes(rows: int, cols: int):
    a, b, c = _SZ(), _SZ(), _SZ()
    _check(library().qlora_dqfp8_sizes(rows, cols, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "qlora_dqfp8_sizes")
    return a.value, b.value, c.value


def dqfp8_quantize(W, status=None, stream=None) -> NF4Matrix:
    """NF4 codes with the fp8 mean-centred second level; scale2 holds (d, mu)
    per group of 256 blocks."""
    import torch
    rows, cols = W.shape
    cb, sb, s2b = dqfp8_sizes(rows, cols)
    q = NF4Matrix(rows, cols, torch.empty(cb, dtype=torch.uint8, device=W.device),
                  torch.empty(sb, dtype=torch.uint8, device=W.device),
                  torch.empty(s2b // 4, dtype=torch.float32, device=W.device))
    s = q.c_struct()
    _check(library().qlora_dqfp8_quantize(_ptr(W), ctypes.byref(s), _ptr(status), _stream(stream)),
           "qlora_dqfp8_quantize")
    return q


def dqfp8_dequantize(q: NF4Matrix, out=None, stream=None):
    import torch
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=torch.bfloat16, device=q.codes.device)
    s = q.c_struct()
    _check(library().qlora_dqfp8_dequantize(ctypes.byref(s), _ptr(out), _stream(stream)), "qlora_dqfp8_dequantize")
    return out


def lora_grads_adamw8(X, dY, sU, sT, A_master, B_master, A_state: AdamW8State, B_state: AdamW8State, lr: float,
                      beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
                      A_bf16=None, B_bf16=None, dA=None, dB=None, stream=None):
    """Adapter gradients and one 8-bit AdamW step of both adapters in one
    launch (qlora_lora_grads_adamw8). A_master is the fp32 master copy of A^T
    ([K, r]), B_master that of B ([N, r]); A_bf16 [r, K] and B_bf16 [N, r]
    receive the bf16 operands; dA [r, K] / dB [N, r] the fp32 gradients when
    given. Both states advance one step (they share the step count)."""
    M, K = X.shape
    N = dY.shape[1]
    r = sU.shape[1]
    A_state.step += 1
    B_state.step = A_state.step
    ptr = lambda t: None if t is None else t.data_ptr()
    a = _Adam8(A_master.data_ptr(), ptr(A_bf16), A_state.m_q.data_ptr(), A_state.v_q.data_ptr(),
               A_state.m_scale.data_ptr(), A_state.v_scale.data_ptr())
    b = _Adam8(B_master.data_ptr(), ptr(B_bf16), B_state.m_q.data_ptr(), B_state.v_q.data_ptr(),
               B_state.m_scale.data_ptr(), B_state.v_scale.data_ptr())
    _check(library().qlora_lora_grads_adamw8(_ptr(X), _ptr(dY), M, N, K, _ptr(sU), _ptr(sT), r, _ptr(dA), _ptr(dB),
                                             ctypes.byref(a), ctypes.byref(b), A_state.step, lr, beta1, beta2, eps,
                                             weight_decay, _stream(stream)), "qlora_lora_grads_adamw8")


def selftest_bounded_wait(status, stream=None) -> None:
    """Launch one CTA whose bounded wait runs out (qlora_selftest_bounded_wait);
    after a synchronise, status (int32 CUDA tensor) holds QLORA_ERR_TIMEOUT."""
    _check(library().qlora_selftest_bounded_wait(_ptr(status), _stream(stream)), "qlora_selftest_bounded_wait")
