"""Plain CPU oracle for fine-grained FP8 W8A8 (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does: it has
no CPU path at all.

The arithmetic lives in ``oracle.c`` (plain C, fp64 for decoding and the GEMM,
IEEE fp32 for the quantizer's scale and quotient); this module compiles it with
gcc on first use and exposes numpy-facing wrappers.

Sources (page title, section):
  * "FP8 W8A8" (vLLM docs), "Two FP8 representations": E4M3 holds +-448 and NaN.
  * "Fine-grained FP8" (Transformers docs), introduction: 128x128 weight blocks,
    per-token activation groups matching the weight's input-channel block (128).
  * "Fine-grained FP8", "DeepGEMM fast path": the dynamic activation scheme.
  * "Fine-grained FP8", "UE8M0 scale format": float8_e8m0fnu scales.
  * "FP8 W8A8", "Applying quantization": the FP8_DYNAMIC scheme (per-channel
    weights, per-token activations); the OwLite FP8 page: AbsMax per-tensor
    scales (static activation scales).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

GROUP = 128
SCALE_F32 = 0
SCALE_UE8M0 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, no fast-math, no FMA
    contraction, OpenMP).  Returns the library path."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # FGFP8_ORACLE_LIB points the wrapper at another build of oracle.c
            # (the planted-mistake tests compile deliberately broken copies).
            path = os.environ.get("FGFP8_ORACLE_LIB") or build()
            lib = ctypes.CDLL(path)
            c = ctypes
            P = c.c_void_p
            i64 = c.c_int64
            lib.orc_e4m3_decode.argtypes = [c.c_uint8]
            lib.orc_e4m3_decode.restype = c.c_double
            lib.orc_e4m3_encode.argtypes = [c.c_float]
            lib.orc_e4m3_encode.restype = c.c_uint8
            lib.orc_scale_f32.argtypes = [c.c_float]
            lib.orc_scale_f32.restype = c.c_float
            lib.orc_scale_ue8m0.argtypes = [c.c_float]
            lib.orc_scale_ue8m0.restype = c.c_uint8
            lib.orc_ue8m0_decode.argtypes = [c.c_uint8]
            lib.orc_ue8m0_decode.restype = c.c_double
            lib.orc_quant_act.argtypes = [P, i64, i64, i64, P, P, i64, c.c_int]
            lib.orc_quant_act.restype = None
            lib.orc_quant_weight.argtypes = [P, i64, i64, i64, P, P, c.c_int]
            lib.orc_quant_weight.restype = None
            lib.orc_dequant_act.argtypes = [P, P, i64, i64, i64, c.c_int, P]
            lib.orc_dequant_act.restype = None
            lib.orc_dequant_weight.argtypes = [P, P, i64, i64, c.c_int, P]
            lib.orc_dequant_weight.restype = None
            lib.orc_gemm.argtypes = [P, P, i64, P, P, i64, i64, c.c_int, P, i64, P, P]
            lib.orc_gemm.restype = None
            lib.orc_grouped_gemm.argtypes = [P, P, i64, P, P, P, c.c_int32, i64, i64,
                                             c.c_int, P, i64, P, P, P]
            lib.orc_grouped_gemm.restype = c.c_int
            lib.orc_quant_rows.argtypes = [P, i64, i64, i64, P, P]
            lib.orc_quant_rows.restype = None
            lib.orc_tensor_scale.argtypes = [P, i64, i64, i64]
            lib.orc_tensor_scale.restype = c.c_float
            lib.orc_quant_static.argtypes = [P, i64, i64, i64, c.c_float, P]
            lib.orc_quant_static.restype = None
            lib.orc_gemm_rowcol.argtypes = [P, P, c.c_int, P, P, c.c_int, i64, i64, P, i64, P, P]
            lib.orc_gemm_rowcol.restype = None
            lib.orc_bf16_rne.argtypes = [c.c_double]
            lib.orc_bf16_rne.restype = c.c_uint16
            for name in ("orc_e4m3_encode_array", "orc_scale_f32_array",
                         "orc_scale_ue8m0_array", "orc_bf16_rne_array"):
                getattr(lib, name).argtypes = [P, i64, P]
                getattr(lib, name).restype = None
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _u16(x) -> np.ndarray:
    """bf16 data as raw uint16 bits (accepts a torch bf16 tensor or uint16 array)."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        x = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "expected bf16 bits as uint16"
    return x


def _scale_dtype(fmt: int):
    return np.float32 if fmt == SCALE_F32 else np.uint8


# ---------------------------------------------------------------- codecs
def e4m3_decode(codes) -> np.ndarray:
    """fp64 value of each E4M3FN code (NaN for 0x7F/0xFF)."""
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    flat = out.reshape(-1)
    for i, c in enumerate(codes.reshape(-1)):
        flat[i] = lib.orc_e4m3_decode(int(c))
    return out


def e4m3_table() -> np.ndarray:
    """The 256 code values, index = code."""
    return e4m3_decode(np.arange(256, dtype=np.uint8))


def e4m3_encode(values) -> np.ndarray:
    """Nearest E4M3FN code, RNE, saturating to +-448, NaN -> 0x7F (fp32 input)."""
    lib = _load()
    v = np.ascontiguousarray(values, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib.orc_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def scale_f32(amax_c) -> np.ndarray:
    """fp32 scale amax_c / 448 (amax_c already clamped)."""
    lib = _load()
    a = np.ascontiguousarray(amax_c, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.float32)
    lib.orc_scale_f32_array(_ptr(a), a.size, _ptr(out))
    return out


def scale_ue8m0(amax_c) -> np.ndarray:
    """UE8M0 byte of the smallest power of two >= amax_c / 448."""
    lib = _load()
    a = np.ascontiguousarray(amax_c, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint8)
    lib.orc_scale_ue8m0_array(_ptr(a), a.size, _ptr(out))
    return out


def ue8m0_decode(e) -> np.ndarray:
    lib = _load()
    e = np.asarray(e, dtype=np.uint8).reshape(-1)
    return np.array([lib.orc_ue8m0_decode(int(x)) for x in e], dtype=np.float64)


def bf16_rne(values) -> np.ndarray:
    """bf16 bits (uint16) nearest to each fp64 value, ties to even."""
    lib = _load()
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib.orc_bf16_rne_array(_ptr(v), v.size, _ptr(out))
    return out


# ---------------------------------------------------------------- quantizers
def scale_rows(M: int, fmt: int) -> int:
    """Default padded row count of the MN-major activation scale array:
    M rounded up so each scale row starts on a 16-byte boundary."""
    unit = 4 if fmt == SCALE_F32 else 16
    return max(unit, (M + unit - 1) // unit * unit)


def quant_act(X, fmt: int, ld_s: int | None = None):
    """Per-token 1x128 activation quantization.

    X: bf16 [M, K] (torch bf16 or uint16 bits).  Returns (Xq u8 [M, K],
    Xs [K/128, ld_s]) with Xs[g, m] the scale of token m, group g (MN-major);
    columns m >= M are left zero."""
    lib = _load()
    X = _u16(X)
    M, K = X.shape
    assert K % GROUP == 0
    ld_s = scale_rows(M, fmt) if ld_s is None else ld_s
    Xq = np.empty((M, K), dtype=np.uint8)
    Xs = np.zeros((K // GROUP, ld_s), dtype=_scale_dtype(fmt))
    lib.orc_quant_act(_ptr(X), M, K, K, _ptr(Xq), _ptr(Xs), ld_s, fmt)
    return Xq, Xs


def quant_weight(W, fmt: int):
    """128x128 block weight quantization.  W: bf16 [N, K].  Returns
    (Wq u8 [N, K], Ws [N/128, K/128])."""
    lib = _load()
    W = _u16(W)
    N, K = W.shape
    assert N % GROUP == 0 and K % GROUP == 0
    Wq = np.empty((N, K), dtype=np.uint8)
    Ws = np.empty((N // GROUP, K // GROUP), dtype=_scale_dtype(fmt))
    lib.orc_quant_weight(_ptr(W), N, K, K, _ptr(Wq), _ptr(Ws), fmt)
    return Wq, Ws


def dequant_act(Xq: np.ndarray, Xs: np.ndarray, fmt: int) -> np.ndarray:
    lib = _load()
    Xq = np.ascontiguousarray(Xq)
    Xs = np.ascontiguousarray(Xs)
    M, K = Xq.shape
    out = np.empty((M, K), dtype=np.float64)
    lib.orc_dequant_act(_ptr(Xq), _ptr(Xs), Xs.shape[1], M, K, fmt, _ptr(out))
    return out


def dequant_weight(Wq: np.ndarray, Ws: np.ndarray, fmt: int) -> np.ndarray:
    lib = _load()
    Wq = np.ascontiguousarray(Wq)
    Ws = np.ascontiguousarray(Ws)
    N, K = Wq.shape
    out = np.empty((N, K), dtype=np.float64)
    lib.orc_dequant_weight(_ptr(Wq), _ptr(Ws), N, K, fmt, _ptr(out))
    return out


# ---------------------------------------------------------------- GEMMs
def gemm(Xq, Xs, Wq, Ws, fmt: int, rows=None):
    """Block-scaled GEMM reference.  Returns (Y fp64 [R, N], S fp64 [R, N]) for
    the requested rows (all rows when rows is None), with
    S[m, n] = sum_k |x_hat[m,k] * w_hat[n,k]| for the tolerance."""
    lib = _load()
    Xq = np.ascontiguousarray(Xq)
    Xs = np.ascontiguousarray(Xs)
    Wq = np.ascontiguousarray(Wq)
    Ws = np.ascontiguousarray(Ws)
    M, K = Xq.shape
    N = Wq.shape[0]
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    Y = np.empty((len(rows), N), dtype=np.float64)
    S = np.empty((len(rows), N), dtype=np.float64)
    lib.orc_gemm(_ptr(Xq), _ptr(Xs), Xs.shape[1], _ptr(Wq), _ptr(Ws), N, K, fmt,
                 _ptr(rows), len(rows), _ptr(Y), _ptr(S))
    return Y, S


def grouped_gemm(Xq, Xs, Wq, Ws, group_offs, fmt: int, rows=None):
    """M-grouped GEMM reference: row m of Xq uses expert e's weights Wq[e]
    ([N, K]) and scales Ws[e] ([N/128, K/128]) when
    group_offs[e] <= m < group_offs[e+1].  Returns (Y, S) for the rows."""
    lib = _load()
    Xq = np.ascontiguousarray(Xq)
    Xs = np.ascontiguousarray(Xs)
    Wq = np.ascontiguousarray(Wq)
    Ws = np.ascontiguousarray(Ws)
    offs = np.ascontiguousarray(group_offs, dtype=np.int32)
    E, N, K = Wq.shape
    assert offs.shape == (E + 1,)
    rows = (np.arange(int(offs[-1]), dtype=np.int64) if rows is None
            else np.ascontiguousarray(rows, dtype=np.int64))
    Y = np.empty((len(rows), N), dtype=np.float64)
    S = np.empty((len(rows), N), dtype=np.float64)
    scratch = np.empty(len(rows), dtype=np.int64)
    rc = lib.orc_grouped_gemm(_ptr(Xq), _ptr(Xs), Xs.shape[1], _ptr(Wq), _ptr(Ws),
                              _ptr(offs), E, N, K, fmt, _ptr(rows), len(rows),
                              _ptr(Y), _ptr(S), _ptr(scratch))
    if rc != 0:
        raise ValueError("a requested row lies outside every expert segment")
    return Y, S


# ---------------------------------------------------------------- row / tensor scales
def quant_rows(X):
    """One fp32 scale per row over all K ("FP8 W8A8", FP8_DYNAMIC: per-token
    activations, per-output-channel weights).  X: bf16 [R, K].  Returns
    (Xq u8 [R, K], scales fp32 [R])."""
    lib = _load()
    X = _u16(X)
    R, K = X.shape
    Xq = np.empty((R, K), dtype=np.uint8)
    sc = np.empty(R, dtype=np.float32)
    lib.orc_quant_rows(_ptr(X), R, K, K, _ptr(Xq), _ptr(sc))
    return Xq, sc


def tensor_scale(X) -> np.float32:
    """Per-tensor AbsMax scale: max(amax(X), 1e-4) / 448 in fp32."""
    lib = _load()
    X = _u16(X)
    R, K = X.shape
    return np.float32(lib.orc_tensor_scale(_ptr(X), R, K, K))


def quant_static(X, scale) -> np.ndarray:
    """Codes of X / scale for a given (static) fp32 scale."""
    lib = _load()
    X = _u16(X)
    R, K = X.shape
    Xq = np.empty((R, K), dtype=np.uint8)
    lib.orc_quant_static(_ptr(X), R, K, K, float(np.float32(scale)), _ptr(Xq))
    return Xq


def gemm_rowcol(Xq, sx, Wq, sw, rows=None):
    """Row/column-scaled GEMM reference: Y[m, n] = sx[m] * sw[n] *
    sum_k x_code * w_code, with a one-element sx or sw meaning a per-tensor
    scale.  Returns (Y fp64 [R, N], S fp64 [R, N])."""
    lib = _load()
    Xq = np.ascontiguousarray(Xq)
    Wq = np.ascontiguousarray(Wq)
    sx = np.ascontiguousarray(sx, dtype=np.float32).reshape(-1)
    sw = np.ascontiguousarray(sw, dtype=np.float32).reshape(-1)
    M, K = Xq.shape
    N = Wq.shape[0]
    assert sx.size in (1, M) and sw.size in (1, N)
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    Y = np.empty((len(rows), N), dtype=np.float64)
    S = np.empty((len(rows), N), dtype=np.float64)
    lib.orc_gemm_rowcol(_ptr(Xq), _ptr(sx), int(sx.size == 1 and M != 1), _ptr(Wq), _ptr(sw),
                        int(sw.size == 1 and N != 1), N, K, _ptr(rows), len(rows), _ptr(Y), _ptr(S))
    return Y, S


# ---------------------------------------------------------------- SwiGLU MLP
def silu_mul(g, u) -> np.ndarray:
    """h = SiLU(g) * u = g / (1 + exp(-g)) * u in fp64: the input of a SwiGLU
    MLP's down projection (Llama-3-8B's MLP, whose down-projection input the
    measured configurations model as a post-SiLU heavy-tailed activation)."""
    g = np.asarray(g, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u


def gemm_within_tolerance(Y_test, Y_ref, S) -> np.ndarray:
    """Elementwise |Y_test - Y_ref| <= 2^-7 |Y_ref| + 1e-4 S (the stated GEMM
    tolerance).  Y_test may be fp32/fp64 or bf16 torch data."""
    Y_test = np.asarray(Y_test, dtype=np.float64)
    return np.abs(Y_test - Y_ref) <= (2.0 ** -7) * np.abs(Y_ref) + 1e-4 * S
