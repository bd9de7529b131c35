"""The C ABI on the host (CPU only, no compute): the library loads, exports
every symbol include/fgfp8.h declares, validates arguments before touching
the GPU, and fails loudly (FGFP8_ERR_CUDA) instead of computing on the CPU
when no usable GPU is present."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import fine_grained_fp8_token_b200 as fg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fgfp8.h")

OK, INVALID, SHAPE, ALIGN, UNSUP, CUDA = 0, 1, 2, 3, 4, 5
A = 1 << 20          # a fake, 16-byte aligned "device" address; never dereferenced on these paths


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:fgfp8_status|int|const char\*)\s+(fgfp8_\w+)\s*\(", text, re.M)))


def test_library_builds_and_loads():
    lib = fg.load()
    assert lib.fgfp8_version() == 1


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 7
    assert set(names) == set(fg.SIGNATURES), "binding signatures and header disagree"
    out = subprocess.run(["nm", "-D", "--defined-only", fg.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (fgfp8_\w+)$", out, re.M))
    missing = set(names) - exported
    assert not missing, f"declared but not exported: {missing}"


def test_no_cpu_library_on_product_path():
    """The product library links no oracle code and the package imports none."""
    out = subprocess.run(["nm", "-D", fg.library_path()], capture_output=True, text=True, check=True).stdout
    assert "orc_" not in out
    src = open(os.path.join(ROOT, "fine_grained_fp8_token_b200", "__init__.py")).read()
    assert "oracle" not in src.replace("# oracle", "")


def st(code):
    return code


def test_quant_act_validation():
    f = fg.fgfp8_quant_act
    assert f(A, 4, 100, 100, A, A, 4, 0, None) == SHAPE                 # K % 128
    assert f(A, 4, 256, 128, A, A, 4, 0, None) == SHAPE                 # ldx < K
    assert f(A, 4, 256, 256, A, A, 2, 0, None) == SHAPE                 # ld_s < M
    assert f(A, 4, 256, 256, A, A, 6, 0, None) == ALIGN                 # ld_s % 4 (fp32)
    assert f(A, 4, 256, 256, A, A, 8, 1, None) == ALIGN                 # ld_s % 16 (ue8m0)
    assert f(A, 4, 256, 256, A, A, 4, 2, None) == INVALID               # fmt
    assert f(0, 4, 256, 256, A, A, 4, 0, None) == INVALID               # NULL X
    assert f(A + 2, 4, 256, 256, A, A, 4, 0, None) == ALIGN             # X alignment
    assert f(A, 4, 256, 260, A, A, 4, 0, None) == ALIGN                 # ldx % 8
    assert f(A, 4, 256, 256, A + 8, A, 4, 0, None) == ALIGN             # Xq alignment
    assert f(A, -1, 256, 256, A, A, 4, 0, None) == INVALID              # negative
    assert f(A, 0, 256, 256, A, A, 4, 0, None) == OK                    # empty: no-op
    assert "ld" in fg.fgfp8_last_error_string() or fg.fgfp8_last_error_string() == ""


def test_quant_weight_validation():
    f = fg.fgfp8_quant_weight
    assert f(A, 100, 256, 256, A, A, 0, None) == SHAPE                  # N % 128
    assert f(A, 128, 200, 256, A, A, 0, None) == SHAPE                  # K % 128
    assert f(A, 128, 256, 128, A, A, 0, None) == SHAPE                  # ldw < K
    assert f(A, 128, 256, 256, A, A + 2, 0, None) == ALIGN              # fp32 Ws alignment
    assert f(A, 128, 256, 256, A, 0, 1, None) == INVALID                # NULL Ws
    assert f(A, 0, 256, 256, A, A, 0, None) == OK


def test_gemm_validation():
    f = fg.fgfp8_gemm
    assert f(A, A, 4, A, A, A, 4, 256, 100, 0, None) == SHAPE           # K
    assert f(A, A, 4, A, A, A, 4, 200, 256, 0, None) == SHAPE           # N
    assert f(A, A, 2, A, A, A, 4, 256, 256, 0, None) == SHAPE           # ld_s < M
    assert f(A, A, 4, A, A, A + 8, 4, 256, 256, 0, None) == ALIGN       # Y
    assert f(A, A + 4, 4, A, A, A, 4, 256, 256, 0, None) == ALIGN       # Xs 16-byte
    assert f(A, A, 4, 0, A, A, 4, 256, 256, 0, None) == INVALID         # NULL Wq
    assert f(A, A, 4, A, A, A, 4, 256, 256, 7, None) == INVALID         # fmt
    assert f(A, A, 4, A, A, A, 1 << 31, 256, 256, 0, None) == SHAPE     # M too large (ld_s < M first)
    assert f(A, A, 4, A, A, A, 0, 256, 256, 0, None) == OK              # empty


def test_grouped_gemm_validation():
    f = fg.fgfp8_grouped_gemm
    assert f(A, A, 256, A, A, A, A, 0, 256, 256, 256, 1, None) == INVALID     # E
    assert f(A, A, 256, A, A, A, A, 4, 200, 256, 256, 1, None) == SHAPE       # M_total % 128
    assert f(A, A, 256, A, A, A, 0, 4, 256, 256, 256, 1, None) == INVALID     # NULL offsets
    assert f(A, A, 256, A, A, A, A + 2, 4, 256, 256, 256, 1, None) == ALIGN   # offsets alignment
    assert f(A, A, 256, A, A, A, A, 4, 0, 256, 256, 1, None) == OK            # empty


def test_linear_validates_both_halves_first():
    """fgfp8_linear checks the quantizer's and the GEMM's arguments before it
    launches anything: a bad GEMM argument is reported even though the
    quantizer's arguments are valid (so no kernel has written Xq / Xs)."""
    f = fg.fgfp8_linear
    # X, ldx, Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, fmt, stream
    assert f(A, 256, A, A, 4, A, A, A, 4, 256, 100, 0, None) == SHAPE      # K % 128 (both)
    assert f(A, 128, A, A, 4, A, A, A, 4, 256, 256, 0, None) == SHAPE      # ldx < K (quantizer)
    assert f(A, 256, A, A, 4, A, A, A, 4, 200, 256, 0, None) == SHAPE      # N % 128 (GEMM only)
    assert f(A, 256, A, A, 4, A, A, A + 8, 4, 256, 256, 0, None) == ALIGN  # Y (GEMM only)
    assert f(A, 256, A, A, 4, 0, A, A, 4, 256, 256, 0, None) == INVALID    # NULL Wq (GEMM only)
    assert f(A, 256, A, A, 4, A, A, A, 4, 256, 256, 3, None) == INVALID    # fmt
    assert f(A, 256, A, A, 4, A, A, A, 0, 256, 256, 0, None) == OK         # empty
    g = fg.fgfp8_grouped_linear
    # X, ldx, Xq, Xs, ld_s, Wq, Ws, Y, offs, E, M_total, N, K, fmt, stream
    assert g(A, 256, A, A, 256, A, A, A, A, 0, 256, 256, 256, 1, None) == INVALID   # E
    assert g(A, 256, A, A, 256, A, A, A, A, 4, 200, 256, 256, 1, None) == SHAPE     # M_total % 128
    assert g(A, 256, A, A, 256, A, A, A, 0, 4, 256, 256, 256, 1, None) == INVALID   # NULL offsets
    assert g(A, 256, A, A, 256, A, A, A, A, 4, 0, 256, 256, 1, None) == OK          # empty


def test_row_and_tensor_scale_validation():
    q, t, st = fg.fgfp8_quant_rows, fg.fgfp8_tensor_scale, fg.fgfp8_quant_static
    # X, R, K, ldx, Xq, scales, stream
    assert q(A, 4, 100, 100, A, A, None) == SHAPE                    # K % 128
    assert q(A, 4, 256, 128, A, A, None) == SHAPE                    # ldx < K
    assert q(A, 4, 256, 260, A, A, None) == ALIGN                    # ldx % 8
    assert q(A, 4, 256, 256, A + 8, A, None) == ALIGN                # Xq alignment
    assert q(A, 4, 256, 256, A, 0, None) == INVALID                  # NULL scales
    assert q(A, 4, 256, 256, A, A + 2, None) == ALIGN                # scales alignment
    assert q(A, 0, 256, 256, A, A, None) == OK                       # empty
    assert t(A, 4, 256, 256, 0, None) == INVALID                     # NULL scale
    assert t(A + 4, 4, 256, 256, A, None) == ALIGN                   # X alignment
    assert st(A, 4, 256, 256, 0, A, None) == INVALID                 # NULL scale
    assert st(A, 4, 256, 256, A, 0, None) == INVALID                 # NULL Xq
    assert st(A, 0, 256, 256, A, A, None) == OK                      # empty


def test_gemm_rowcol_validation():
    g = fg.fgfp8_gemm_rowcol
    # Xq, sx, x_per_tensor, Wq, sw, w_per_tensor, Y, M, N, K, stream
    assert g(A, A, 0, A, A, 0, A, 4, 256, 100, None) == SHAPE        # K
    assert g(A, A, 0, A, A, 0, A, 4, 200, 256, None) == SHAPE        # N
    assert g(A, A, 2, A, A, 0, A, 4, 256, 256, None) == INVALID      # flag
    assert g(A, A, 0, A, A + 4, 0, A, 4, 256, 256, None) == ALIGN    # per-channel sw must be 16-byte aligned
    assert g(A, A + 2, 0, A, A, 0, A, 4, 256, 256, None) == ALIGN    # sx alignment
    assert g(A, A, 0, A, 0, 1, A, 4, 256, 256, None) == INVALID      # NULL sw
    assert g(A, A, 0, A, A, 0, A + 8, 4, 256, 256, None) == ALIGN    # Y
    assert g(A, A, 0, A, A, 0, A, 0, 256, 256, None) == OK           # empty


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_valid_call_without_gpu_fails_loudly():
    """No CPU fallback: a well-formed request on a machine without an
    sm_100a GPU returns FGFP8_ERR_CUDA and launches nothing."""
    assert fg.fgfp8_quant_act(A, 4, 256, 256, A, A, 4, 0, None) == CUDA
    assert "cuda" in fg.fgfp8_last_error_string().lower()
    assert fg.fgfp8_gemm(A, A, 4, A, A, A, 4, 256, 256, 0, None) == CUDA
    assert fg.fgfp8_linear(A, 256, A, A, 4, A, A, A, 4, 256, 256, 0, None) == CUDA
    assert fg.fgfp8_quant_rows(A, 4, 256, 256, A, A, None) == CUDA
    assert fg.fgfp8_gemm_rowcol(A, A, 0, A, A, 0, A, 4, 256, 256, None) == CUDA
    assert fg.fgfp8_selftest_expired_wait(None) == CUDA
    assert fg.fgfp8_quant_act_masked(A, 256, A, 2, 128, 256, A, A, 256, 0, None) == CUDA
    assert fg.fgfp8_masked_linear(A, 256, A, A, 256, A, A, A, A, 2, 128, 256, 256, 0, None) == CUDA
    with pytest.raises(fg.FGFP8Error):
        fg._check(fg.fgfp8_quant_weight(A, 128, 256, 256, A, A, 0, None), "quant_weight")


def test_masked_quant_and_linear_validation():
    """The masked quantizer and the one-call masked layer check their
    arguments on the host before any launch."""
    f = fg.fgfp8_quant_act_masked     # X, ldx, counts, E, cap, K, Xq, Xs, ld_s, fmt, stream
    assert f(A, 256, A, 0, 128, 256, A, A, 256, 0, None) == INVALID          # E < 1
    assert f(A, 256, A, 2, 100, 256, A, A, 256, 0, None) == SHAPE            # cap % 128
    assert f(A, 256, A, 70000, 128, 256, A, A, 70000 * 128, 0, None) == SHAPE   # E > 65535
    assert f(A, 256, 0, 2, 128, 256, A, A, 256, 0, None) == INVALID          # NULL counts
    assert f(A, 256, A + 2, 2, 128, 256, A, A, 256, 0, None) == ALIGN        # counts alignment
    assert f(A, 256, A, 2, 128, 200, A, A, 256, 0, None) == SHAPE            # K % 128
    assert f(A, 256, A, 2, 128, 256, A, A, 128, 0, None) == SHAPE            # ld_s < E * cap
    assert f(A + 2, 256, A, 2, 128, 256, A, A, 256, 0, None) == ALIGN        # X alignment
    g = fg.fgfp8_masked_linear        # X, ldx, Xq, Xs, ld_s, Wq, Ws, Y, counts, E, cap, N, K, fmt, stream
    assert g(A, 256, A, A, 256, A, A, A, A, 2, 128, 200, 256, 0, None) == SHAPE    # N % 128
    assert g(A, 256, A, A, 256, A, A, A, 0, 2, 128, 256, 256, 0, None) == INVALID  # NULL counts
    assert g(A, 256, A, A, 256, A, A, A, A, 2, 128, 256, 256, 3, None) == INVALID  # fmt



def test_gather_cols_validation():
    f = fg.fgfp8_gather_cols
    assert f(A, 2, 4, 12, A, None) == SHAPE                             # n % 8
    assert f(A, -1, 4, 16, A, None) == INVALID                          # negative
    assert f(0, 2, 4, 16, A, None) == INVALID                           # NULL parts
    assert f(A, 2, 4, 16, 0, None) == INVALID                           # NULL Y
    assert f(A + 8, 2, 4, 16, A, None) == ALIGN                         # parts alignment
    assert f(A, 2, 4, 16, A + 4, None) == ALIGN                         # Y alignment
    assert f(A, 1 << 16, 1 << 16, 1 << 10, A, None) == SHAPE            # P * M * n / 8 >= 2^32
    assert f(A, 0, 4, 16, A, None) == OK                                # empty: no-op
    assert f(A, 2, 0, 16, A, None) == OK


def test_selftest_gemm_timeout_validation():
    f = fg.fgfp8_selftest_gemm_timeout
    assert f(A, A, 256, A, A, A, 256, 512, 1024, 0, 8, None) == INVALID    # withhold_kb >= K/128
    assert f(A, A, 256, A, A, A, 256, 512, 1024, 0, -1, None) == INVALID   # negative
    assert f(A, A, 64, A, A, A, 64, 512, 1024, 0, 1, None) == SHAPE        # M <= 64: not the persistent kernel
    assert f(A, A, 256, A, A, A, 256, 384, 1024, 0, 1, None) == SHAPE      # N % 256
    assert f(A, A, 256, A, A, A, 256, 512, 1000, 0, 1, None) == SHAPE      # K % 128
    assert f(A, A, 256, A, A, A, 256, 512, 1024, 3, 1, None) == INVALID    # fmt


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_new_entry_points_without_gpu_fail_loudly():
    assert fg.fgfp8_gather_cols(A, 2, 4, 16, A, None) == CUDA
    assert fg.fgfp8_selftest_gemm_timeout(A, A, 256, A, A, A, 256, 512, 1024, 0, 1, None) == CUDA
