"""Shared helpers for the GPU parity tests: move seeded inputs between torch
and the oracle, and compare results (bit-exact for codes and scales, the
stated tolerance for GEMM outputs)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle

F32, UE8M0 = 0, 1


def require_gpu() -> torch.device:
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    major, minor = torch.cuda.get_device_capability(0)
    if (major, minor) != (10, 0):
        pytest.fail(f"sm_100a (B200) required, found sm_{major}{minor}")
    return torch.device("cuda:0")


def bits16(x: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> uint16 numpy bits."""
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def scale_bits(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint32) if a.dtype == np.float32 else a


def assert_codes_equal(gpu: np.ndarray, ref: np.ndarray, what: str):
    if not np.array_equal(gpu, ref):
        bad = np.argwhere(gpu != ref)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatching entries, first at {i}: gpu={gpu[i]:#x} "
                             f"oracle={ref[i]:#x}")


def assert_scales_equal(gpu: np.ndarray, ref: np.ndarray, what: str):
    assert_codes_equal(scale_bits(np.ascontiguousarray(gpu)), scale_bits(np.ascontiguousarray(ref)), what)


def y_to_f64(Y: torch.Tensor) -> np.ndarray:
    return Y.detach().float().cpu().double().numpy()


def assert_gemm_close(Y_gpu: np.ndarray, Y_ref: np.ndarray, S: np.ndarray, what: str):
    ok = oracle.gemm_within_tolerance(Y_gpu, Y_ref, S)
    if not ok.all():
        bad = np.argwhere(~ok)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} of {ok.size} outside |d| <= 2^-7|ref| + 1e-4 S; first at {i}: "
                             f"gpu={Y_gpu[i]!r} ref={Y_ref[i]!r} S={S[i]!r}")
    assert np.isfinite(Y_gpu).all()


class Guarded:
    """A device output buffer with canary bytes on both sides: a stand-in for
    a memory checker that finds writes outside an output (a wrong tile
    index, row limit or leading dimension).  The inner tensor starts at a
    256-byte boundary, so every alignment rule of the library holds."""

    PAD = 4096
    CANARY = 0xA5

    def __init__(self, shape, dtype, device, fill=None):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((self.PAD + n + self.PAD,), self.CANARY, dtype=torch.uint8, device=device)
        self.t = self.raw[self.PAD:self.PAD + n].view(dtype).view(*shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, what="output"):
        lo = self.raw[:self.PAD]
        hi = self.raw[-self.PAD:]
        assert bool((lo == self.CANARY).all()), f"{what}: bytes written before the buffer"
        assert bool((hi == self.CANARY).all()), f"{what}: bytes written after the buffer"
