"""Thin ctypes binding of ``libqlin.so`` (the C ABI in include/qlin.h).

Argument marshalling only: every step of the layer runs in the CUDA
library.  Tensors are torch CUDA tensors (PyTorch provides device memory and
streams); each function passes their raw pointers and the current CUDA
stream and raises :class:`QlinError` on a non-OK status.  There is no CPU or
PyTorch fallback: if the library is missing, importing it fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlin.so")

QLIN_W4_PERCHANNEL = 0
QLIN_W4_G128 = 1
QLIN_W8_PERCHANNEL = 2

STATUS = {0: "QLIN_OK", 1: "QLIN_ERR_ARG", 2: "QLIN_ERR_SHAPE", 3: "QLIN_ERR_ALIGN",
          4: "QLIN_ERR_WORKSPACE", 5: "QLIN_ERR_CUDA", 6: "QLIN_ERR_TIMEOUT"}

EXPORTED = [
    "qlin_status_string", "qlin_last_error", "qlin_weights_bytes", "qlin_weights_bind",
    "qlin_pack_weights", "qlin_quant_act_workspace", "qlin_quant_act", "qlin_outlier_colmax",
    "qlin_momentum_update", "qlin_gemm_workspace", "qlin_gemm", "qlin_forward_workspace",
    "qlin_forward", "qlin_poll_device_status", "qlin_quant_act_noalloc", "qlin_backward_dx",
    "qlin_backward_dx_workspace", "qlin_debug_set", "qlin_debug_get", "qlin_forward_grouped_workspace",
    "qlin_forward_grouped", "qlin_gptq_workspace", "qlin_gptq_quantize", "qlin_smooth_search_workspace",
    "qlin_smooth_search", "qlin_offq_codes_bytes", "qlin_offq_rotate_weights", "qlin_offq_pack",
    "qlin_offq_quant_act", "qlin_offq_gemm_workspace", "qlin_offq_gemm", "qlin_offq_forward_workspace",
    "qlin_offq_forward",
]

# test / measurement knobs (qlin_debug_set, include/qlin.h)
QLIN_KNOB_PDL = 0
QLIN_KNOB_CLUSTER = 1
QLIN_KNOB_CLUSTER_SIZE = 2
QLIN_KNOB_MAX_CTAS = 3
QLIN_KNOB_MAX_TOKEN_TILE = 4
QLIN_KNOB_WIDEN_MIN_M = 5
QLIN_KNOB_FUSED_MOMENTUM_MAX_M = 6
QLIN_KNOB_WAIT_NS = 7
QLIN_KNOB_PAIR_MMA = 8
QLIN_KNOB_CONVERT_MAX_M = 9
QLIN_KNOB_PAIR_SPLIT = 10


class QlinError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")
        self.status = status


class qlin_weights(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int32), ("N", ctypes.c_int32), ("fmt", ctypes.c_int32),
        ("group", ctypes.c_int32), ("n_outlier", ctypes.c_int32), ("n_outlier_pad", ctypes.c_int32),
        ("codes", ctypes.c_void_p), ("chan_scale", ctypes.c_void_p), ("group_scale", ctypes.c_void_p),
        ("fold_ratio", ctypes.c_void_p), ("outlier_idx", ctypes.c_void_p), ("W_Ot", ctypes.c_void_p),
        ("wmax_O", ctypes.c_void_p),
    ]


_lib = None
P = ctypes.c_void_p
I32 = ctypes.c_int32
SZ = ctypes.c_size_t
F32 = ctypes.c_float


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m quantized_linear_layers_token_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.qlin_status_string.argtypes = [ctypes.c_int]
        L.qlin_status_string.restype = ctypes.c_char_p
        L.qlin_last_error.argtypes = []
        L.qlin_last_error.restype = ctypes.c_char_p
        W = ctypes.POINTER(qlin_weights)
        sigs = {
            "qlin_weights_bytes": [I32, I32, I32, I32, ctypes.POINTER(SZ)],
            "qlin_weights_bind": [W, I32, I32, I32, I32, P, SZ],
            "qlin_pack_weights": [P, P, W, P],
            "qlin_quant_act_workspace": [I32, W, ctypes.POINTER(SZ)],
            "qlin_quant_act": [P, I32, W, P, F32, I32, P, P, P, P, SZ, P],
            "qlin_outlier_colmax": [P, I32, W, P, P],
            "qlin_momentum_update": [W, P, P, F32, P],
            "qlin_gemm_workspace": [I32, W, ctypes.POINTER(SZ)],
            "qlin_gemm": [W, P, P, P, P, I32, P, P, P, SZ, P],
            "qlin_forward_workspace": [I32, W, ctypes.POINTER(SZ)],
            "qlin_forward": [P, I32, W, P, F32, I32, P, P, SZ, P],
            "qlin_poll_device_status": [P],
            "qlin_quant_act_noalloc": [P, I32, W, P, F32, I32, P, P, P, P],
            "qlin_backward_dx": [W, P, I32, P, P, P, SZ, P],
            "qlin_backward_dx_workspace": [I32, W, ctypes.POINTER(SZ)],
            "qlin_debug_set": [I32, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)],
            "qlin_forward_grouped_workspace": [I32, P, I32, ctypes.POINTER(SZ)],
            "qlin_forward_grouped": [I32, P, P, P, P, I32, F32, I32, P, SZ, P],
            "qlin_gptq_workspace": [I32, I32, ctypes.POINTER(SZ)],
            "qlin_gptq_quantize": [P, I32, I32, I32, P, P, I32, P, P, P, P, SZ, P],
            "qlin_smooth_search_workspace": [I32, I32, I32, I32, ctypes.POINTER(SZ)],
            "qlin_smooth_search": [P, I32, I32, P, I32, I32, P, P, P, P, SZ, P],
            "qlin_debug_get": [I32, ctypes.POINTER(ctypes.c_int64)],
            "qlin_offq_codes_bytes": [I32, I32, ctypes.POINTER(SZ)],
            "qlin_offq_rotate_weights": [P, I32, I32, P, P, P],
            "qlin_offq_pack": [P, I32, I32, P, P, P, P, P, P],
            "qlin_offq_quant_act": [P, I32, I32, P, P, P, P, P],
            "qlin_offq_gemm_workspace": [I32, I32, I32, ctypes.POINTER(SZ)],
            "qlin_offq_gemm": [P, P, P, I32, I32, I32, P, P, P, P, P, SZ, P],
            "qlin_offq_forward_workspace": [I32, I32, I32, ctypes.POINTER(SZ)],
            "qlin_offq_forward": [P, I32, I32, I32, P, P, P, P, P, P, SZ, P],
        }
        for name, argt in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = argt
            fn.restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise QlinError(status, where, lib().qlin_last_error().decode(errors="replace"))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _size(fn, *args) -> int:
    out = SZ(0)
    _check(fn(*args, ctypes.byref(out)), fn.__name__)
    return int(out.value)


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def qlin_weights_bytes(K: int, N: int, fmt: int, n_outlier: int) -> int:
    return _size(lib().qlin_weights_bytes, K, N, fmt, n_outlier)


def qlin_weights_bind(K: int, N: int, fmt: int, n_outlier: int, base: int, nbytes: int) -> qlin_weights:
    w = qlin_weights()
    _check(lib().qlin_weights_bind(ctypes.byref(w), K, N, fmt, n_outlier, base, nbytes), "qlin_weights_bind")
    return w


def qlin_pack_weights(W: torch.Tensor, O_host: np.ndarray, w: qlin_weights, stream=None):
    O_host = np.ascontiguousarray(O_host, dtype=np.int32)
    optr = O_host.ctypes.data if len(O_host) else None
    _check(lib().qlin_pack_weights(_ptr(W), optr, ctypes.byref(w), _stream(stream)), "qlin_pack_weights")


def qlin_quant_act_workspace(M: int, w: qlin_weights) -> int:
    return _size(lib().qlin_quant_act_workspace, M, ctypes.byref(w))


def qlin_quant_act(X, M: int, w: qlin_weights, s, gamma: float, update_momentum: bool, Xq, a, XqO,
                   workspace, ws_bytes: int, stream=None):
    _check(lib().qlin_quant_act(_ptr(X), M, ctypes.byref(w), _ptr(s), float(gamma), int(bool(update_momentum)),
                                _ptr(Xq), _ptr(a), _ptr(XqO), _ptr(workspace), ws_bytes, _stream(stream)),
           "qlin_quant_act")


def qlin_quant_act_noalloc(X, M: int, w: qlin_weights, s, gamma: float, update_momentum: bool, Xq, a, XqO,
                           stream=None):
    """qlin_quant_act with the library's fixed internal scratch instead of a
    caller workspace (for callers that cannot allocate device memory; at most
    1024 outlier channels; calls that overlap on the GPU race)."""
    _check(lib().qlin_quant_act_noalloc(_ptr(X), M, ctypes.byref(w), _ptr(s), float(gamma),
                                        int(bool(update_momentum)), _ptr(Xq), _ptr(a), _ptr(XqO), _stream(stream)),
           "qlin_quant_act_noalloc")


def qlin_outlier_colmax(X, M: int, w: qlin_weights, cmax, stream=None):
    _check(lib().qlin_outlier_colmax(_ptr(X), M, ctypes.byref(w), _ptr(cmax), _stream(stream)),
           "qlin_outlier_colmax")


def qlin_momentum_update(w: qlin_weights, cmax, s, gamma: float, stream=None):
    _check(lib().qlin_momentum_update(ctypes.byref(w), _ptr(cmax), _ptr(s), float(gamma), _stream(stream)),
           "qlin_momentum_update")


def qlin_gemm_workspace(M: int, w: qlin_weights) -> int:
    return _size(lib().qlin_gemm_workspace, M, ctypes.byref(w))


def qlin_gemm(w: qlin_weights, Xq, a, XqO, s, M: int, Y, acc_debug, workspace, ws_bytes: int, stream=None):
    _check(lib().qlin_gemm(ctypes.byref(w), _ptr(Xq), _ptr(a), _ptr(XqO), _ptr(s), M, _ptr(Y), _ptr(acc_debug),
                           _ptr(workspace), ws_bytes, _stream(stream)), "qlin_gemm")


def qlin_forward_workspace(M: int, w: qlin_weights) -> int:
    return _size(lib().qlin_forward_workspace, M, ctypes.byref(w))


def qlin_forward(X, M: int, w: qlin_weights, s, gamma: float, update_momentum: bool, Y, workspace,
                 ws_bytes: int, stream=None):
    _check(lib().qlin_forward(_ptr(X), M, ctypes.byref(w), _ptr(s), float(gamma), int(bool(update_momentum)),
                              _ptr(Y), _ptr(workspace), ws_bytes, _stream(stream)), "qlin_forward")


def _weights_array(ws):
    arr = (ctypes.POINTER(qlin_weights) * len(ws))(*[ctypes.pointer(w) for w in ws])
    return arr


def _ptr_array(ts):
    return (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])


def qlin_forward_grouped_workspace(ws, M: int) -> int:
    arr = _weights_array(ws)
    return _size(lib().qlin_forward_grouped_workspace, len(ws), ctypes.cast(arr, P), M)


def qlin_forward_grouped(ws, Xs, ss, Ys, M: int, gamma: float, update_momentum: bool, workspace, ws_bytes: int,
                         stream=None):
    """Independent forwards of len(ws) layers at the same token count in one
    quantization launch and one GEMM launch (C ABI qlin_forward_grouped)."""
    n = len(ws)
    assert len(Xs) == n and len(ss) == n and len(Ys) == n
    arr = _weights_array(ws)
    xa, sa, ya = _ptr_array(Xs), _ptr_array(ss), _ptr_array(Ys)
    _check(lib().qlin_forward_grouped(n, ctypes.cast(arr, P), ctypes.cast(xa, P), ctypes.cast(sa, P),
                                      ctypes.cast(ya, P), M, float(gamma), int(bool(update_momentum)),
                                      _ptr(workspace), ws_bytes, _stream(stream)), "qlin_forward_grouped")


def qlin_gptq_workspace(K: int, N: int) -> int:
    return _size(lib().qlin_gptq_workspace, K, N)


def qlin_gptq_quantize(X, ns: int, K: int, N: int, W, scale, qmax: int, codes, Hinv, singular, workspace,
                       ws_bytes: int, stream=None):
    _check(lib().qlin_gptq_quantize(_ptr(X), ns, K, N, _ptr(W), _ptr(scale), qmax, _ptr(codes), _ptr(Hinv),
                                    _ptr(singular), _ptr(workspace), ws_bytes, _stream(stream)),
           "qlin_gptq_quantize")


def qlin_smooth_search_workspace(M: int, K: int, N: int, G: int) -> int:
    return _size(lib().qlin_smooth_search_workspace, M, K, N, G)


def qlin_smooth_search(X, M: int, K: int, W, N: int, G: int, loss, best, s_best, workspace, ws_bytes: int,
                       stream=None):
    _check(lib().qlin_smooth_search(_ptr(X), M, K, _ptr(W), N, G, _ptr(loss), _ptr(best), _ptr(s_best),
                                    _ptr(workspace), ws_bytes, _stream(stream)), "qlin_smooth_search")


def _signs(signs) -> tuple:
    """Host int8 [128] copy of the OffQ signs d (kept alive by the caller's frame)."""
    arr = np.ascontiguousarray(np.asarray(signs, dtype=np.int8))
    if arr.shape != (128,):
        raise ValueError(f"signs must have 128 entries, got shape {arr.shape}")
    return arr, arr.ctypes.data


def qlin_offq_codes_bytes(K: int, N: int) -> int:
    return _size(lib().qlin_offq_codes_bytes, K, N)


def qlin_offq_rotate_weights(W, K: int, N: int, signs, Wr, stream=None):
    arr, sp = _signs(signs)
    _check(lib().qlin_offq_rotate_weights(_ptr(W), K, N, sp, _ptr(Wr), _stream(stream)),
           "qlin_offq_rotate_weights")


def qlin_offq_pack(W, K: int, N: int, signs, codes, chan_scale, colsum, Wr, stream=None):
    arr, sp = _signs(signs)
    _check(lib().qlin_offq_pack(_ptr(W), K, N, sp, _ptr(codes), _ptr(chan_scale), _ptr(colsum), _ptr(Wr),
                                _stream(stream)), "qlin_offq_pack")


def qlin_offq_quant_act(X, M: int, K: int, signs, Xq, scale, offset, stream=None):
    arr, sp = _signs(signs)
    _check(lib().qlin_offq_quant_act(_ptr(X), M, K, sp, _ptr(Xq), _ptr(scale), _ptr(offset), _stream(stream)),
           "qlin_offq_quant_act")


def qlin_offq_gemm_workspace(M: int, K: int, N: int) -> int:
    return _size(lib().qlin_offq_gemm_workspace, M, K, N)


def qlin_offq_gemm(Xq, scale, offset, M: int, K: int, N: int, codes, chan_scale, colsum, Y, workspace,
                   ws_bytes: int, stream=None):
    _check(lib().qlin_offq_gemm(_ptr(Xq), _ptr(scale), _ptr(offset), M, K, N, _ptr(codes), _ptr(chan_scale),
                                _ptr(colsum), _ptr(Y), _ptr(workspace), ws_bytes, _stream(stream)),
           "qlin_offq_gemm")


def qlin_offq_forward_workspace(M: int, K: int, N: int) -> int:
    return _size(lib().qlin_offq_forward_workspace, M, K, N)


def qlin_offq_forward(X, M: int, K: int, N: int, signs, codes, chan_scale, colsum, Y, workspace, ws_bytes: int,
                      stream=None):
    arr, sp = _signs(signs)
    _check(lib().qlin_offq_forward(_ptr(X), M, K, N, sp, _ptr(codes), _ptr(chan_scale), _ptr(colsum), _ptr(Y),
                                   _ptr(workspace), ws_bytes, _stream(stream)), "qlin_offq_forward")


def qlin_backward_dx_workspace(M: int, w: qlin_weights) -> int:
    return _size(lib().qlin_backward_dx_workspace, M, ctypes.byref(w))


def qlin_backward_dx(w: qlin_weights, dY, M: int, s, dX, workspace=None, ws_bytes: int = 0, stream=None):
    _check(lib().qlin_backward_dx(ctypes.byref(w), _ptr(dY), M, _ptr(s), _ptr(dX), _ptr(workspace), ws_bytes,
                                  _stream(stream)), "qlin_backward_dx")


def qlin_debug_set(knob: int, value: int) -> int:
    """Set a test/measurement knob; returns its previous value."""
    prev = ctypes.c_int64(0)
    _check(lib().qlin_debug_set(knob, int(value), ctypes.byref(prev)), "qlin_debug_set")
    return int(prev.value)


def qlin_debug_get(knob: int) -> int:
    v = ctypes.c_int64(0)
    _check(lib().qlin_debug_get(knob, ctypes.byref(v)), "qlin_debug_get")
    return int(v.value)


class knobs:
    """Context manager: set knobs for the duration of a block, then restore."""

    def __init__(self, **settings):
        self.settings = {globals()["QLIN_KNOB_" + k.upper()]: v for k, v in settings.items()}
        self.saved = {}

    def __enter__(self):
        for k, v in self.settings.items():
            self.saved[k] = qlin_debug_set(k, v)
        return self

    def __exit__(self, *exc):
        for k, v in self.saved.items():
            qlin_debug_set(k, v)
        return False


def qlin_poll_device_status(stream=None):
    _check(lib().qlin_poll_device_status(_stream(stream)), "qlin_poll_device_status")


# ---------------------------------------------------------------------------
# small conveniences over the entry points (allocation via torch only)
# ---------------------------------------------------------------------------

def empty_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Zero-filled device buffer, 256-byte aligned (torch's allocator aligns
    to 512 bytes), usable as any workspace."""
    return torch.zeros(max(int(nbytes), 1), dtype=torch.uint8, device=device)


class PackedLayer:
    """One layer's packed weights in a single device buffer."""

    def __init__(self, K: int, N: int, fmt: int, n_outlier: int, device="cuda"):
        self.K, self.N, self.fmt, self.n_outlier = K, N, fmt, n_outlier
        self.nbytes = qlin_weights_bytes(K, N, fmt, n_outlier)
        self.buffer = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)
        self.w = qlin_weights_bind(K, N, fmt, n_outlier, self.buffer.data_ptr(), self.nbytes)

    @classmethod
    def pack(cls, W: torch.Tensor, O: np.ndarray, fmt: int, stream=None) -> "PackedLayer":
        K, N = W.shape
        layer = cls(K, N, fmt, len(O), device=W.device)
        qlin_pack_weights(W, O, layer.w, stream)
        return layer

    def clone(self) -> "PackedLayer":
        """A copy at a distinct device address (same packed bytes)."""
        other = PackedLayer(self.K, self.N, self.fmt, self.n_outlier, device=self.buffer.device)
        other.buffer.copy_(self.buffer)
        return other

    def view(self, name: str) -> torch.Tensor:
        """Typed view of one packed sub-buffer (for parity checks)."""
        w = self.w
        base = self.buffer.data_ptr()
        K, N, nO = w.K, w.N, w.n_outlier
        TN, KB, IB = -(-N // 128), -(-K // 128), -(-nO // 64)
        block = 16384 if self.fmt == QLIN_W8_PERCHANNEL else 8192
        spec = {
            "codes": (w.codes, torch.uint8, (TN * KB * block,)),       # tile-major (include/qlin.h)
            "chan_scale": (w.chan_scale, torch.float32, (N,)),
            "group_scale": (w.group_scale, torch.int16, (K // 128, N)),
            "fold_ratio": (w.fold_ratio, torch.int16, (K // 128, N)),
            "outlier_idx": (w.outlier_idx, torch.int32, (nO,)),
            "W_Ot": (w.W_Ot, torch.int16, (TN * IB * 8192,)),           # tiled, swizzled fp16
            "wmax_O": (w.wmax_O, torch.float32, (nO,)),
        }[name]
        ptr, dtype, shape = spec
        if ptr is None:
            raise ValueError(f"{name} is not present in this format")
        off = ptr - base
        nbytes = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        return self.buffer[off:off + nbytes].view(dtype).view(*shape)
