"""ctypes binding to the CPU oracle (``qlin_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
CPU-baseline leg of ``bench.py``; never by the product library.  It is
independent of the CUDA library: it neither imports nor links anything from
the package, and the package never imports this module.

Every function takes and returns numpy arrays; fp16 values travel as their
IEEE binary16 bit patterns (``np.uint16``) so the oracle's own binary16 code
does every conversion.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qlin_oracle.c")
_LIB = os.path.join(_HERE, "liboqlin.so")

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (single-threaded, no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


P = ctypes.c_void_p
I = ctypes.c_int
F = ctypes.c_float
D = ctypes.c_double


def _declare(L):
    L.oq_half_to_double.argtypes = [ctypes.c_uint16]
    L.oq_half_to_double.restype = D
    L.oq_double_to_half.argtypes = [D]
    L.oq_double_to_half.restype = ctypes.c_uint16
    L.oq_float_to_half.argtypes = [F]
    L.oq_float_to_half.restype = ctypes.c_uint16
    L.oq_rne.argtypes = [D]
    L.oq_rne.restype = D
    L.oq_quant_weight_per_channel.argtypes = [P, I, I, I, P, P]
    L.oq_quant_weight_per_channel.restype = None
    L.oq_quant_weight_group.argtypes = [P, I, I, I, P, P, P, P, P]
    L.oq_quant_weight_group.restype = I
    L.oq_pack_nibbles.argtypes = [P, I, I, P]
    L.oq_pack_nibbles.restype = None
    L.oq_outlier_wmax.argtypes = [P, I, I, P, I, P]
    L.oq_outlier_wmax.restype = None
    L.oq_momentum_update.argtypes = [P, I, I, P, I, P, F, P]
    L.oq_momentum_update.restype = None
    L.oq_backward_dx.argtypes = [P, I, I, I, P, P, P, P, I, P, P]
    L.oq_backward_dx.restype = None
    L.oq_quant_act.argtypes = [P, I, I, P, I, P, P, P, P]
    L.oq_quant_act.restype = None
    L.oq_int_gemm.argtypes = [P, P, I, I, I, P]
    L.oq_int_gemm.restype = I
    L.oq_int_gemm_rows.argtypes = [P, P, I, I, P, I, P]
    L.oq_int_gemm_rows.restype = I
    L.oq_int_gemm_rows_nk.argtypes = [P, P, I, I, P, I, P]
    L.oq_int_gemm_rows_nk.restype = I
    L.oq_dequant.argtypes = [P, P, P, P, P, P, I, P, I, P, I, P]
    L.oq_dequant.restype = None
    L.oq_fast_fp16_to_int8_single.argtypes = [ctypes.c_uint16, P]
    L.oq_fast_fp16_to_int8_single.restype = ctypes.c_int8
    L.oq_fast_fp16_to_int8_two_add.argtypes = [ctypes.c_uint16, P]
    L.oq_fast_fp16_to_int8_two_add.restype = ctypes.c_int8
    L.oq_gptq_hessian.argtypes = [P, I, I, P]
    L.oq_gptq_hessian.restype = I
    L.oq_gptq_delta.argtypes = [P, P, I, I, D, P]
    L.oq_gptq_delta.restype = None
    L.oq_gptq_downdate.argtypes = [P, I, I]
    L.oq_gptq_downdate.restype = None
    L.oq_gptq_quantize.argtypes = [P, I, I, P, D, I, P, P]
    L.oq_gptq_quantize.restype = I
    L.oq_gptq_quantize_layer.argtypes = [P, I, I, I, P, P, I, P, P]
    L.oq_gptq_quantize_layer.restype = I
    L.oq_smooth_search.argtypes = [P, I, I, P, I, I, P]
    L.oq_smooth_search.restype = I
    L.oq_offq_transform.argtypes = [P, I, I, P, P]
    L.oq_offq_transform.restype = None
    L.oq_offq_quant_act.argtypes = [P, I, I, P, P, P, P]
    L.oq_offq_quant_act.restype = None
    L.oq_offq_rotate_weights.argtypes = [P, I, I, P, P]
    L.oq_offq_rotate_weights.restype = None
    L.oq_quant_weight_per_channel_f32.argtypes = [P, I, I, I, P, P]
    L.oq_quant_weight_per_channel_f32.restype = None
    L.oq_offq_gemm_rows.argtypes = [P, P, P, P, P, I, I, P, I, P]
    L.oq_offq_gemm_rows.restype = None
    L.oq_invert.argtypes = [P, I, P]
    L.oq_invert.restype = I


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --- binary16 ---------------------------------------------------------------

def half_to_double(bits: int) -> float:
    return lib().oq_half_to_double(int(bits))


def double_to_half(x: float) -> int:
    return lib().oq_double_to_half(float(x))


def float_to_half(x) -> int:
    return lib().oq_float_to_half(float(np.float32(x)))


def rne(x: float) -> float:
    return lib().oq_rne(float(x))


# --- weights ----------------------------------------------------------------

def quant_weight_per_channel(W_bits: np.ndarray, qmax: int):
    """W_bits: uint16 [K][N].  Returns (codes int8 [K][N], scale fp32 [N])."""
    W_bits = _c(W_bits, np.uint16)
    K, N = W_bits.shape
    codes = np.zeros((K, N), np.int8)
    scale = np.zeros(N, np.float32)
    lib().oq_quant_weight_per_channel(_p(W_bits), K, N, int(qmax), _p(codes), _p(scale))
    return codes, scale


def quant_weight_group(W_bits: np.ndarray, group: int = 128):
    """Returns (q4, q8 int8 [K][N], g_h, r_h uint16 [K/g][N], c fp32 [N], bad)."""
    W_bits = _c(W_bits, np.uint16)
    K, N = W_bits.shape
    G = K // group
    q4 = np.zeros((K, N), np.int8)
    q8 = np.zeros((K, N), np.int8)
    gh = np.zeros((G, N), np.uint16)
    rh = np.zeros((G, N), np.uint16)
    c = np.zeros(N, np.float32)
    bad = lib().oq_quant_weight_group(_p(W_bits), K, N, group, _p(q4), _p(q8), _p(gh), _p(rh), _p(c))
    return q4, q8, gh, rh, c, bad


def pack_nibbles(q: np.ndarray) -> np.ndarray:
    """q: int8 [K][N] in [-8, 7] -> uint8 [N][K/2] (layout in qlin_oracle.c)."""
    q = _c(q, np.int8)
    K, N = q.shape
    out = np.zeros((N, K // 2), np.uint8)
    lib().oq_pack_nibbles(_p(q), K, N, _p(out))
    return out


def outlier_wmax(W_bits: np.ndarray, O: np.ndarray) -> np.ndarray:
    W_bits = _c(W_bits, np.uint16)
    O = _c(O, np.int32)
    K, N = W_bits.shape
    out = np.zeros(len(O), np.float32)
    lib().oq_outlier_wmax(_p(W_bits), K, N, _p(O), len(O), _p(out))
    return out


# --- activations ------------------------------------------------------------

def momentum_update(X_bits: np.ndarray, O: np.ndarray, wmaxO: np.ndarray, gamma: float,
                    s: np.ndarray) -> np.ndarray:
    """Returns the updated momentum state (a new array)."""
    X_bits = _c(X_bits, np.uint16)
    O = _c(O, np.int32)
    wmaxO = _c(wmaxO, np.float32)
    s2 = np.array(s, dtype=np.float32, copy=True)
    M, K = X_bits.shape
    lib().oq_momentum_update(_p(X_bits), M, K, _p(O), len(O), _p(wmaxO), float(np.float32(gamma)), _p(s2))
    return s2


def quant_act(X_bits: np.ndarray, O: np.ndarray, s: np.ndarray):
    """Returns (Xq int8 [M][K], a fp32 [M], XqO int8 [M][nO])."""
    X_bits = _c(X_bits, np.uint16)
    O = _c(O, np.int32)
    s = _c(s, np.float32)
    M, K = X_bits.shape
    nO = len(O)
    Xq = np.zeros((M, K), np.int8)
    a = np.zeros(M, np.float32)
    XqO = np.zeros((M, max(nO, 0)), np.int8)
    lib().oq_quant_act(_p(X_bits), M, K, _p(O), nO, _p(s), _p(Xq), _p(a), _p(XqO))
    return Xq, a, XqO


# --- GEMM and epilogue ------------------------------------------------------

def int_gemm(Xq: np.ndarray, B: np.ndarray):
    """acc int64 [M][N] = Xq [M][K] . B [K][N]; also returns an overflow flag."""
    Xq = _c(Xq, np.int8)
    B = _c(B, np.int8)
    M, K = Xq.shape
    K2, N = B.shape
    assert K == K2
    acc = np.zeros((M, N), np.int64)
    ovf = lib().oq_int_gemm(_p(Xq), _p(B), M, K, N, _p(acc))
    return acc, ovf


def int_gemm_rows(Xq: np.ndarray, B: np.ndarray, rows: np.ndarray):
    Xq = _c(Xq, np.int8)
    B = _c(B, np.int8)
    rows = _c(rows, np.int32)
    M, K = Xq.shape
    N = B.shape[1]
    acc = np.zeros((len(rows), N), np.int64)
    ovf = lib().oq_int_gemm_rows(_p(Xq), _p(B), K, N, _p(rows), len(rows), _p(acc))
    return acc, ovf


def int_gemm_rows_nk(Xq: np.ndarray, Bt: np.ndarray, rows: np.ndarray):
    """int_gemm_rows with the operand given transposed (Bt [N][K])."""
    Xq = _c(Xq, np.int8)
    Bt = _c(Bt, np.int8)
    rows = _c(rows, np.int32)
    M, K = Xq.shape
    N = Bt.shape[0]
    assert Bt.shape[1] == K
    acc = np.zeros((len(rows), N), np.int64)
    ovf = lib().oq_int_gemm_rows_nk(_p(Xq), _p(Bt), K, N, _p(rows), len(rows), _p(acc))
    return acc, ovf


def dequant(acc: np.ndarray, a: np.ndarray, cscale: np.ndarray, XqO: np.ndarray, s: np.ndarray,
            W_bits: np.ndarray, O: np.ndarray, rows: np.ndarray | None = None) -> np.ndarray:
    """fp64 y [R][N] for the rows of acc (rows[r] indexes a / XqO)."""
    acc = _c(acc, np.int64)
    a = _c(a, np.float32)
    cscale = _c(cscale, np.float32)
    O = _c(O, np.int32)
    nO = len(O)
    XqO = _c(XqO if nO else np.zeros((len(a), 0), np.int8), np.int8)
    s = _c(s if nO else np.zeros(0, np.float32), np.float32)
    W_bits = _c(W_bits, np.uint16)
    R, N = acc.shape
    if rows is None:
        rows = np.arange(R, dtype=np.int32)
    rows = _c(rows, np.int32)
    y = np.zeros((R, N), np.float64)
    lib().oq_dequant(_p(acc), _p(a), _p(cscale), _p(XqO), _p(s), _p(W_bits), N, _p(O), nO,
                     _p(rows), R, _p(y))
    return y


# --- FastFP16toINT8 ---------------------------------------------------------

def fast_fp16_to_int8(v_bits: int, single: bool = True):
    hi = ctypes.c_uint8(0)
    f = lib().oq_fast_fp16_to_int8_single if single else lib().oq_fast_fp16_to_int8_two_add
    code = f(int(v_bits), ctypes.byref(hi))
    return int(code), int(hi.value)


# --- GPTQ -------------------------------------------------------------------

def gptq_hessian(X: np.ndarray) -> np.ndarray:
    X = _c(X, np.float64)
    ns, d = X.shape
    H = np.zeros((d, d), np.float64)
    lib().oq_gptq_hessian(_p(X), ns, d, _p(H))
    return H


def gptq_delta(w: np.ndarray, Hinv: np.ndarray, i: int, q_i: float) -> np.ndarray:
    w = _c(w, np.float64)
    Hinv = _c(Hinv, np.float64)
    d = len(w)
    out = np.zeros(d, np.float64)
    lib().oq_gptq_delta(_p(w), _p(Hinv), d, int(i), float(q_i), _p(out))
    return out


def gptq_downdate(Hinv: np.ndarray, i: int) -> np.ndarray:
    Hc = np.array(Hinv, dtype=np.float64, copy=True, order="C")
    lib().oq_gptq_downdate(_p(Hc), Hc.shape[0], int(i))
    return Hc


def gptq_quantize(X: np.ndarray, w: np.ndarray, scale: float, qmax: int):
    X = _c(X, np.float64)
    ns, d = X.shape
    w2 = np.array(w, dtype=np.float64, copy=True)
    Hinv = np.zeros((d, d), np.float64)
    deltas = np.zeros((d, d), np.float64)
    r = lib().oq_gptq_quantize(_p(X), ns, d, _p(w2), float(scale), int(qmax), _p(Hinv), _p(deltas))
    if r:
        raise ValueError("Hessian is singular")
    return w2, Hinv, deltas


def gptq_quantize_layer(X: np.ndarray, W: np.ndarray, scale: np.ndarray, qmax: int):
    """Hessian-compensated quantization of a layer W [d][N] (fp64): every
    output channel n is oq_gptq_quantize's w with grid step scale[n].
    Returns (W after compensation = the grid values, codes int8 [d][N],
    inverse Hessian)."""
    X = _c(X, np.float64)
    ns, d = X.shape
    W2 = np.array(W, dtype=np.float64, copy=True, order="C")
    assert W2.shape[0] == d
    N = W2.shape[1]
    scale = _c(scale, np.float64)
    codes = np.zeros((d, N), np.int8)
    Hinv = np.zeros((d, d), np.float64)
    r = lib().oq_gptq_quantize_layer(_p(X), ns, d, N, _p(W2), _p(scale), int(qmax), _p(codes), _p(Hinv))
    if r:
        raise ValueError("Hessian is singular")
    return W2, codes, Hinv


def smooth_search(X_bits: np.ndarray, W_bits: np.ndarray, G: int):
    """QQQ adaptive smoothing threshold search (readings in qlin_oracle.c):
    returns (loss fp64 [G], index of the least loss)."""
    X_bits = _c(X_bits, np.uint16)
    W_bits = _c(W_bits, np.uint16)
    M, K = X_bits.shape
    N = W_bits.shape[1]
    loss = np.zeros(G, np.float64)
    best = lib().oq_smooth_search(_p(X_bits), M, K, _p(W_bits), N, int(G), _p(loss))
    return loss, int(best)


def offq_transform(X_bits: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """y = x (D H) per 128-channel group, fp64 [M][K] (unnormalised)."""
    X_bits = _c(X_bits, np.uint16)
    M, K = X_bits.shape
    y = np.zeros((M, K), np.float64)
    lib().oq_offq_transform(_p(X_bits), M, K, _p(_c(signs, np.int8)), _p(y))
    return y


def offq_quant_act(X_bits: np.ndarray, signs: np.ndarray):
    """OffQ activations: (q int8 [M][K] in 0..15, scale fp32 [M][K/128], offset fp32 [M][K/128]);
    the dequantized value is q * scale + offset."""
    X_bits = _c(X_bits, np.uint16)
    M, K = X_bits.shape
    G = K // 128
    Xq = np.zeros((M, K), np.int8)
    sc = np.zeros((M, G), np.float32)
    off = np.zeros((M, G), np.float32)
    lib().oq_offq_quant_act(_p(X_bits), M, K, _p(_c(signs, np.int8)), _p(Xq), _p(sc), _p(off))
    return Xq, sc, off


def offq_pack_layer(W_bits: np.ndarray, signs: np.ndarray) -> dict:
    """OffQ weights: W' = (1/128) H D W per group (fp32), then per-channel INT4."""
    W_bits = _c(W_bits, np.uint16)
    K, N = W_bits.shape
    Wr = np.zeros((K, N), np.float32)
    lib().oq_offq_rotate_weights(_p(W_bits), K, N, _p(_c(signs, np.int8)), _p(Wr))
    q = np.zeros((K, N), np.int8)
    c = np.zeros(N, np.float32)
    lib().oq_quant_weight_per_channel_f32(_p(Wr), K, N, 7, _p(q), _p(c))
    B = (q.astype(np.int16) * 16).astype(np.int8)
    return {"K": K, "N": N, "Wr": Wr, "q": q, "c": c, "B": B, "Bt": np.ascontiguousarray(B.T),
            "cscale": (c / np.float32(16.0)).astype(np.float32), "packed": pack_nibbles(q)}


def offq_gemm_rows(Xq: np.ndarray, scale: np.ndarray, offset: np.ndarray, packed: dict,
                   rows: np.ndarray) -> np.ndarray:
    Xq = _c(Xq, np.int8)
    scale = _c(scale, np.float32)
    offset = _c(offset, np.float32)
    rows = _c(rows, np.int32)
    K, N = packed["K"], packed["N"]
    y = np.zeros((len(rows), N), np.float64)
    lib().oq_offq_gemm_rows(_p(Xq), _p(scale), _p(offset), _p(packed["Bt"]), _p(_c(packed["cscale"], np.float32)),
                            K, N, _p(rows), len(rows), _p(y))
    return y


# --- whole layer, composed from the steps above ------------------------------

FMT_W4_PERCHANNEL = 0
FMT_W4_G128 = 1
FMT_W8_PERCHANNEL = 2


def backward_dx(dY_bits: np.ndarray, W_bits: np.ndarray, packed: dict, s: np.ndarray) -> np.ndarray:
    """Input gradient under the straight-through estimator, fp64 [M][K]:
    dX = (dY W_eff^T) / s with W_eff the dequantized weights plus the
    compensation rows (s_i - 1) W[O_i, :]."""
    dY_bits = _c(dY_bits, np.uint16)
    W_bits = _c(W_bits, np.uint16)
    M, N = dY_bits.shape
    K = packed["K"]
    B = _c(packed["B"], np.int8)
    cs = _c(packed["cscale"], np.float32)
    O = _c(packed["O"], np.int32)
    s = _c(s if len(O) else np.zeros(1), np.float32)
    dX = np.zeros((M, K), np.float64)
    lib().oq_backward_dx(_p(dY_bits), M, N, K, _p(B), _p(cs), _p(W_bits), _p(O), len(O), _p(s), _p(dX))
    return dX


def pack_layer(W_bits: np.ndarray, O: np.ndarray, fmt: int) -> dict:
    """Quantize one layer's weights; returns every artefact the GPU packer
    produces, in the oracle's logical layouts, plus the INT8 MMA operand."""
    W_bits = _c(W_bits, np.uint16)
    K, N = W_bits.shape
    out = {"fmt": fmt, "K": K, "N": N, "O": _c(O, np.int32)}
    if fmt == FMT_W4_PERCHANNEL:
        q, c = quant_weight_per_channel(W_bits, 7)
        out.update(q=q, c=c, B=(q.astype(np.int16) * 16).astype(np.int8),
                   cscale=(c / np.float32(16.0)).astype(np.float32), packed=pack_nibbles(q))
    elif fmt == FMT_W4_G128:
        q4, q8, gh, rh, c, bad = quant_weight_group(W_bits, 128)
        assert not bad, "requantized code outside [-127, 127]"
        out.update(q=q4, q8=q8, g_h=gh, r_h=rh, c=c, B=q8, cscale=c, packed=pack_nibbles(q4))
    elif fmt == FMT_W8_PERCHANNEL:
        q, c = quant_weight_per_channel(W_bits, 127)
        out.update(q=q, c=c, B=q, cscale=c, packed=np.ascontiguousarray(q.T))
    else:
        raise ValueError(fmt)
    out["wmaxO"] = outlier_wmax(W_bits, out["O"])
    return out


def forward(X_bits: np.ndarray, W_bits: np.ndarray, packed: dict, s: np.ndarray, gamma: float,
            update_momentum: bool = True, rows: np.ndarray | None = None) -> dict:
    """The whole hot path: momentum update, per-token quantization, integer
    GEMM, fp64 dequant + compensation.  ``rows`` restricts the GEMM and
    epilogue to a subset of tokens (quantization always covers every row)."""
    O = packed["O"]
    s1 = momentum_update(X_bits, O, packed["wmaxO"], gamma, s) if (update_momentum and len(O)) \
        else np.array(s, np.float32, copy=True)
    Xq, a, XqO = quant_act(X_bits, O, s1)
    M = Xq.shape[0]
    if rows is None:
        rows = np.arange(M, dtype=np.int32)
    if len(rows):
        if "Bt" not in packed:  # the operand transposed once per layer (a copy, no arithmetic)
            packed["Bt"] = np.ascontiguousarray(packed["B"].T)
        acc, ovf = int_gemm_rows_nk(Xq, packed["Bt"], rows)
        assert not ovf
        y = dequant(acc, a, packed["cscale"], XqO, s1, W_bits, O, rows)
    else:
        acc = np.zeros((0, packed["N"]), np.int64)
        y = np.zeros((0, packed["N"]), np.float64)
    return {"s": s1, "Xq": Xq, "a": a, "XqO": XqO, "acc": acc, "y": y, "rows": rows}
