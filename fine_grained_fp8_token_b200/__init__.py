"""Python binding of libfgfp8 — fine-grained FP8 W8A8 linear layers on B200.

Argument marshalling only: every step of the computation runs in the CUDA
library (include/fgfp8.h).  PyTorch supplies device memory and streams.  There
is no CPU path: without the compiled library or without an sm_100a GPU every
compute call raises.

Raw entry points keep the C names (``fgfp8_quant_act`` ...) and take integers
(device addresses, sizes, a stream handle).  The tensor helpers
(``quant_act``, ``quant_weight``, ``gemm``, ``grouped_gemm``) allocate the
outputs with torch on the input's device and call the raw entry points on the
current stream.
"""
from __future__ import annotations

import ctypes
import os
import threading

SCALE_F32 = 0
SCALE_UE8M0 = 1

_STATUS = {
    0: "FGFP8_OK", 1: "FGFP8_ERR_INVALID_ARG", 2: "FGFP8_ERR_SHAPE", 3: "FGFP8_ERR_ALIGN",
    4: "FGFP8_ERR_UNSUPPORTED", 5: "FGFP8_ERR_CUDA", 6: "FGFP8_ERR_TIMEOUT", 7: "FGFP8_ERR_DEVICE",
}

# Every symbol include/fgfp8.h declares, with (restype, argtypes).
_P, _I64, _I32, _INT = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
SIGNATURES = {
    "fgfp8_version": (_INT, []),
    "fgfp8_last_error_string": (ctypes.c_char_p, []),
    "fgfp8_quant_weight": (_INT, [_P, _I64, _I64, _I64, _P, _P, _INT, _P]),
    "fgfp8_quant_act": (_INT, [_P, _I64, _I64, _I64, _P, _P, _I64, _INT, _P]),
    "fgfp8_gemm": (_INT, [_P, _P, _I64, _P, _P, _P, _I64, _I64, _I64, _INT, _P]),
    "fgfp8_grouped_gemm": (_INT, [_P, _P, _I64, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _INT, _P]),
    "fgfp8_linear": (_INT, [_P, _I64, _P, _P, _I64, _P, _P, _P, _I64, _I64, _I64, _INT, _P]),
    "fgfp8_grouped_linear": (_INT, [_P, _I64, _P, _P, _I64, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _INT, _P]),
    "fgfp8_linear_noalloc": (_INT, [_P, _I64, _P, _P, _P, _I64, _I64, _I64, _INT, _P]),
    "fgfp8_quant_rows": (_INT, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "fgfp8_tensor_scale": (_INT, [_P, _I64, _I64, _I64, _P, _P]),
    "fgfp8_quant_static": (_INT, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "fgfp8_gemm_rowcol": (_INT, [_P, _P, _INT, _P, _P, _INT, _P, _I64, _I64, _I64, _P]),
    "fgfp8_gemm_swiglu_quant": (_INT, [_P, _P, _I64, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P]),
    "fgfp8_masked_gemm": (_INT, [_P, _P, _I64, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _INT, _P]),
    "fgfp8_quant_act_masked": (_INT, [_P, _I64, _P, _I32, _I64, _I64, _P, _P, _I64, _INT, _P]),
    "fgfp8_masked_linear": (_INT, [_P, _I64, _P, _P, _I64, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _INT, _P]),
    "fgfp8_check_device_status": (_INT, [_P]),
    "fgfp8_gather_cols": (_INT, [_P, _I64, _I64, _I64, _P, _P]),
    "fgfp8_selftest_expired_wait": (_INT, [_P]),
    "fgfp8_selftest_gemm_timeout": (_INT, [_P, _P, _I64, _P, _P, _P, _I64, _I64, _I64, _INT, _I64, _P]),
}

_lock = threading.Lock()
_lib = None


class FGFP8Error(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {message}")


def library_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfgfp8.so")


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libfgfp8.so (building it with nvcc first when it is missing or
    older than its sources).  Raises when the library cannot be produced."""
    global _lib
    with _lock:
        if _lib is None:
            from . import build as _build
            path = library_path()
            if build_if_missing and _build.is_stale():
                _build.build()
            if not os.path.exists(path):
                raise FGFP8Error(5, "load", f"{path} is missing; run fine_grained_fp8_token_b200.build")
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _check(status: int, where: str) -> None:
    if status != 0:
        msg = load().fgfp8_last_error_string().decode(errors="replace")
        raise FGFP8Error(status, where, msg)


def _raw(name):
    def call(*args):
        return getattr(load(), name)(*args)
    call.__name__ = name
    return call


fgfp8_version = _raw("fgfp8_version")
fgfp8_quant_weight = _raw("fgfp8_quant_weight")
fgfp8_quant_act = _raw("fgfp8_quant_act")
fgfp8_gemm = _raw("fgfp8_gemm")
fgfp8_grouped_gemm = _raw("fgfp8_grouped_gemm")
fgfp8_linear = _raw("fgfp8_linear")
fgfp8_grouped_linear = _raw("fgfp8_grouped_linear")
fgfp8_linear_noalloc = _raw("fgfp8_linear_noalloc")
fgfp8_quant_rows = _raw("fgfp8_quant_rows")
fgfp8_tensor_scale = _raw("fgfp8_tensor_scale")
fgfp8_quant_static = _raw("fgfp8_quant_static")
fgfp8_gemm_rowcol = _raw("fgfp8_gemm_rowcol")
fgfp8_gemm_swiglu_quant = _raw("fgfp8_gemm_swiglu_quant")
fgfp8_masked_gemm = _raw("fgfp8_masked_gemm")
fgfp8_quant_act_masked = _raw("fgfp8_quant_act_masked")
fgfp8_masked_linear = _raw("fgfp8_masked_linear")
fgfp8_check_device_status = _raw("fgfp8_check_device_status")
fgfp8_gather_cols = _raw("fgfp8_gather_cols")
fgfp8_selftest_expired_wait = _raw("fgfp8_selftest_expired_wait")
fgfp8_selftest_gemm_timeout = _raw("fgfp8_selftest_gemm_timeout")


def fgfp8_last_error_string() -> str:
    return load().fgfp8_last_error_string().decode(errors="replace")


# ---------------------------------------------------------------- tensor helpers
def _stream(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def scale_rows(M: int, fmt: int) -> int:
    """Padded row count (ld_s) of an activation scale array for M tokens."""
    unit = 4 if fmt == SCALE_F32 else 16
    return max(unit, (M + unit - 1) // unit * unit)


def _scale_dtype(fmt: int):
    import torch
    return torch.float32 if fmt == SCALE_F32 else torch.uint8


def quant_act(X, fmt: int, Xq=None, Xs=None, ld_s: int | None = None, stream=None):
    """Per-token 1x128 quantization of X (bf16 [M, K], CUDA).  Returns
    (Xq uint8 [M, K], Xs [K/128, ld_s]) with Xs[g, m] the scale of token m."""
    import torch
    M, K = X.shape
    ld_s = scale_rows(M, fmt) if ld_s is None else ld_s
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
    if Xs is None:
        Xs = torch.empty((K // 128, ld_s), dtype=_scale_dtype(fmt), device=X.device)
    _check(fgfp8_quant_act(X.data_ptr(), M, K, X.stride(0), Xq.data_ptr(), Xs.data_ptr(), ld_s, fmt,
                           _stream(stream)), "fgfp8_quant_act")
    return Xq, Xs


def quant_weight(W, fmt: int, Wq=None, Ws=None, stream=None):
    """128x128 block quantization of W (bf16 [N, K], CUDA).  Returns
    (Wq uint8 [N, K], Ws [N/128, K/128])."""
    import torch
    N, K = W.shape
    if Wq is None:
        Wq = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    if Ws is None:
        Ws = torch.empty((N // 128, K // 128), dtype=_scale_dtype(fmt), device=W.device)
    _check(fgfp8_quant_weight(W.data_ptr(), N, K, W.stride(0), Wq.data_ptr(), Ws.data_ptr(), fmt,
                              _stream(stream)), "fgfp8_quant_weight")
    return Wq, Ws


def gemm(Xq, Xs, Wq, Ws, fmt: int, Y=None, stream=None):
    """Y = X W^T (bf16 [M, N]) from the quantized operands."""
    import torch
    M, K = Xq.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    _check(fgfp8_gemm(Xq.data_ptr(), Xs.data_ptr(), Xs.shape[1], Wq.data_ptr(), Ws.data_ptr(), Y.data_ptr(),
                      M, N, K, fmt, _stream(stream)), "fgfp8_gemm")
    return Y


def grouped_gemm(Xq, Xs, Wq, Ws, group_offs, fmt: int, Y=None, stream=None):
    """M-grouped expert GEMM: Wq [E, N, K], Ws [E, N/128, K/128], group_offs
    int32 [E+1] on the device.  Returns Y bf16 [M_total, N]."""
    import torch
    M_total, K = Xq.shape
    E, N, _ = Wq.shape
    if Y is None:
        Y = torch.empty((M_total, N), dtype=torch.bfloat16, device=Xq.device)
    _check(fgfp8_grouped_gemm(Xq.data_ptr(), Xs.data_ptr(), Xs.shape[1], Wq.data_ptr(), Ws.data_ptr(),
                              Y.data_ptr(), group_offs.data_ptr(), E, M_total, N, K, fmt, _stream(stream)),
           "fgfp8_grouped_gemm")
    return Y


def _act_buffers(X, fmt, Xq, Xs, ld_s):
    import torch
    M, K = X.shape
    ld_s = scale_rows(M, fmt) if ld_s is None else ld_s
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
    if Xs is None:
        Xs = torch.empty((K // 128, ld_s), dtype=_scale_dtype(fmt), device=X.device)
    return Xq, Xs, ld_s


def linear(X, Wq, Ws, fmt: int, Y=None, Xq=None, Xs=None, ld_s: int | None = None, stream=None):
    """The W8A8 linear layer Y = X W^T (bf16 [M, N]) from bf16 X [M, K] and the
    pre-quantized weight: one call that quantizes X into Xq / Xs (allocated
    here when not given) and runs the GEMM.  Returns Y."""
    import torch
    M, K = X.shape
    N = Wq.shape[0]
    Xq, Xs, ld_s = _act_buffers(X, fmt, Xq, Xs, ld_s)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _check(fgfp8_linear(X.data_ptr(), X.stride(0), Xq.data_ptr(), Xs.data_ptr(), ld_s, Wq.data_ptr(), Ws.data_ptr(),
                        Y.data_ptr(), M, N, K, fmt, _stream(stream)), "fgfp8_linear")
    return Y


def grouped_linear(X, Wq, Ws, group_offs, fmt: int, Y=None, Xq=None, Xs=None, ld_s: int | None = None,
                   stream=None):
    """The M-grouped expert layer from bf16 rows X [M_total, K] grouped per
    expert: quantization and grouped GEMM in one call.  Returns Y."""
    import torch
    M_total, K = X.shape
    E, N, _ = Wq.shape
    Xq, Xs, ld_s = _act_buffers(X, fmt, Xq, Xs, ld_s)
    if Y is None:
        Y = torch.empty((M_total, N), dtype=torch.bfloat16, device=X.device)
    _check(fgfp8_grouped_linear(X.data_ptr(), X.stride(0), Xq.data_ptr(), Xs.data_ptr(), ld_s, Wq.data_ptr(),
                                Ws.data_ptr(), Y.data_ptr(), group_offs.data_ptr(), E, M_total, N, K, fmt,
                                _stream(stream)), "fgfp8_grouped_linear")
    return Y


# ---------------------------------------------------------------- row / tensor scales
def quant_rows(X, Xq=None, scales=None, stream=None):
    """One fp32 scale per row of X (bf16 [R, K], CUDA): per-token
    activations or per-output-channel weights.  Returns (Xq uint8 [R, K],
    scales fp32 [R])."""
    import torch
    R, K = X.shape
    if Xq is None:
        Xq = torch.empty((R, K), dtype=torch.uint8, device=X.device)
    if scales is None:
        scales = torch.empty((R,), dtype=torch.float32, device=X.device)
    _check(fgfp8_quant_rows(X.data_ptr(), R, K, X.stride(0), Xq.data_ptr(), scales.data_ptr(), _stream(stream)),
           "fgfp8_quant_rows")
    return Xq, scales


def tensor_scale(X, scale=None, stream=None):
    """Per-tensor AbsMax scale of X (bf16 [R, K], CUDA) as a float32 [1] tensor."""
    import torch
    R, K = X.shape
    if scale is None:
        scale = torch.empty((1,), dtype=torch.float32, device=X.device)
    _check(fgfp8_tensor_scale(X.data_ptr(), R, K, X.stride(0), scale.data_ptr(), _stream(stream)),
           "fgfp8_tensor_scale")
    return scale


def quant_static(X, scale, Xq=None, stream=None):
    """Codes of X / scale for a given float32 [1] device scale.  Returns Xq."""
    import torch
    R, K = X.shape
    if Xq is None:
        Xq = torch.empty((R, K), dtype=torch.uint8, device=X.device)
    _check(fgfp8_quant_static(X.data_ptr(), R, K, X.stride(0), scale.data_ptr(), Xq.data_ptr(), _stream(stream)),
           "fgfp8_quant_static")
    return Xq


def gemm_rowcol(Xq, sx, Wq, sw, Y=None, stream=None):
    """Y = sx[m] sw[n] sum_k Xq Wq (bf16 [M, N]); a one-element sx or sw is a
    per-tensor scale."""
    import torch
    M, K = Xq.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    x_t = int(sx.numel() == 1 and M != 1)
    w_t = int(sw.numel() == 1 and N != 1)
    _check(fgfp8_gemm_rowcol(Xq.data_ptr(), sx.data_ptr(), x_t, Wq.data_ptr(), sw.data_ptr(), w_t, Y.data_ptr(),
                             M, N, K, _stream(stream)), "fgfp8_gemm_rowcol")
    return Y


def masked_gemm(Xq, Xs, Wq, Ws, counts, fmt: int, Y=None, stream=None):
    """Masked expert GEMM: Xq [E * cap, K] with expert e's tokens in rows
    [e * cap, e * cap + counts[e]), Wq [E, N, K], Ws [E, N/128, K/128],
    counts int32 [E] on the device.  Returns Y bf16 [E * cap, N] (padding
    rows are not written)."""
    import torch
    M_total, K = Xq.shape
    E, N, _ = Wq.shape
    cap = M_total // E
    if Y is None:
        Y = torch.empty((M_total, N), dtype=torch.bfloat16, device=Xq.device)
    _check(fgfp8_masked_gemm(Xq.data_ptr(), Xs.data_ptr(), Xs.shape[1], Wq.data_ptr(), Ws.data_ptr(), Y.data_ptr(),
                             counts.data_ptr(), E, cap, N, K, fmt, _stream(stream)), "fgfp8_masked_gemm")
    return Y


def quant_act_masked(X, counts, E: int, fmt: int, Xq=None, Xs=None, ld_s: int | None = None, stream=None):
    """The 1x128 quantizer over the token rows of the masked layout only
    (X bf16 [E * cap, K]; expert e's tokens in rows [e * cap, e * cap +
    counts[e]), counts int32 [E] on the device).  Padding rows of Xq / Xs
    are left as they are.  Returns (Xq, Xs)."""
    import torch
    M, K = X.shape
    cap = M // E
    ld_s = scale_rows(M, fmt) if ld_s is None else ld_s
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
    if Xs is None:
        Xs = torch.empty((K // 128, ld_s), dtype=torch.float32 if fmt == SCALE_F32 else torch.uint8, device=X.device)
    _check(fgfp8_quant_act_masked(X.data_ptr(), X.stride(0), counts.data_ptr(), E, cap, K, Xq.data_ptr(),
                                  Xs.data_ptr(), ld_s, fmt, _stream(stream)), "fgfp8_quant_act_masked")
    return Xq, Xs


def masked_linear(X, Wq, Ws, counts, fmt: int, Y=None, Xq=None, Xs=None, ld_s: int | None = None, stream=None):
    """The masked expert layer in one call (token rows quantized, then the
    masked GEMM).  Returns Y bf16 [E * cap, N] (padding rows not written)."""
    import torch
    M, K = X.shape
    E, N, _ = Wq.shape
    cap = M // E
    ld_s = scale_rows(M, fmt) if ld_s is None else ld_s
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
    if Xs is None:
        Xs = torch.empty((K // 128, ld_s), dtype=torch.float32 if fmt == SCALE_F32 else torch.uint8, device=X.device)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _check(fgfp8_masked_linear(X.data_ptr(), X.stride(0), Xq.data_ptr(), Xs.data_ptr(), ld_s, Wq.data_ptr(),
                               Ws.data_ptr(), Y.data_ptr(), counts.data_ptr(), E, cap, N, K, fmt, _stream(stream)),
           "fgfp8_masked_linear")
    return Y


# ---------------------------------------------------------------- fused SwiGLU MLP
def interleave_gate_up(gate, up, block: int = 128):
    """Stack gate and up [R, ...] into the [2R, ...] layout that
    fgfp8_gemm_swiglu_quant takes: blocks of `block` rows alternating gate,
    up.  Weights (bf16, or their E4M3 codes) use block=128; their
    [I/128, K/128] block scales use block=1.  Pure data layout (a torch stack
    and reshape)."""
    import torch
    R = gate.shape[0]
    g = gate.reshape(R // block, block, *gate.shape[1:])
    u = up.reshape(R // block, block, *up.shape[1:])
    return torch.stack([g, u], dim=1).reshape(2 * R, *gate.shape[1:]).contiguous()


def gemm_swiglu_quant(Xq, Xs, Wq_gu, Ws_gu, Hq=None, Hs=None, ld_h: int | None = None, stream=None):
    """h = SiLU(gate) * up of the interleaved gate/up projection, quantized
    per 1x128 group for the down projection (fp32 scales).  Returns (Hq uint8
    [M, I], Hs float32 [I/128, ld_h])."""
    import torch
    M, K = Xq.shape
    I = Wq_gu.shape[0] // 2
    ld_h = scale_rows(M, SCALE_F32) if ld_h is None else ld_h
    if Hq is None:
        Hq = torch.empty((M, I), dtype=torch.uint8, device=Xq.device)
    if Hs is None:
        Hs = torch.empty((I // 128, ld_h), dtype=torch.float32, device=Xq.device)
    _check(fgfp8_gemm_swiglu_quant(Xq.data_ptr(), Xs.data_ptr(), Xs.shape[1], Wq_gu.data_ptr(), Ws_gu.data_ptr(),
                                   Hq.data_ptr(), Hs.data_ptr(), ld_h, M, I, K, _stream(stream)),
           "fgfp8_gemm_swiglu_quant")
    return Hq, Hs


def selftest_expired_wait(stream=None) -> None:
    """Launch the bounded-wait self-test (a wait that nothing completes; it
    gives up after one second and records a timeout in the status word)."""
    _check(fgfp8_selftest_expired_wait(_stream(stream)), "fgfp8_selftest_expired_wait")


def gather_cols(parts, Y=None, stream=None):
    """parts bf16 [P, M, n] (an all-gather of per-rank column blocks) ->
    Y bf16 [M, P * n] with Y[m, p * n + j] = parts[p, m, j]."""
    import torch
    P, M, n = parts.shape
    if Y is None:
        Y = torch.empty((M, P * n), dtype=parts.dtype, device=parts.device)
    _check(fgfp8_gather_cols(parts.data_ptr(), P, M, n, Y.data_ptr(), _stream(stream)), "fgfp8_gather_cols")
    return Y


def selftest_gemm_timeout(Xq, Xs, Wq, Ws, fmt: int, withhold_kb: int, Y=None, stream=None):
    """Run the dense GEMM with work item 0's K block withhold_kb never
    requested (the GEMM self-test of its bounded waits).  Returns Y; the
    status word then holds a timeout."""
    import torch
    M, K = Xq.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    _check(fgfp8_selftest_gemm_timeout(Xq.data_ptr(), Xs.data_ptr(), Xs.shape[1], Wq.data_ptr(), Ws.data_ptr(),
                                       Y.data_ptr(), M, N, K, fmt, withhold_kb, _stream(stream)),
           "fgfp8_selftest_gemm_timeout")
    return Y


def check_device_status(stream=None) -> None:
    """Synchronize and raise if a kernel recorded a timeout or bad input."""
    _check(fgfp8_check_device_status(_stream(stream)), "fgfp8_check_device_status")
