"""fgfp8_linear_noalloc: the linear layer for callers that cannot allocate
device memory (a plugin handed only its input and output buffers, a loop
that must not call cudaMalloc, a fixed-size memory pool).  It keeps the
quantized activations in the library's static per-device scratch array
instead of caller buffers.

The GPU test calls the entry point through the C ABI several times in a row
on one stream (each call overwrites the shared scratch) and compares every
output with fgfp8_linear's for the same inputs, within the GEMM tolerance
|d| <= 2^-7 |ref| + 1e-4 sum_k |x_hat w_hat| (sum from the oracle), and with
the oracle itself.  This file is collected last on purpose."""
import pytest
import torch

import fine_grained_fp8_token_b200 as fg
import oracle
import workloads
from parity import F32, UE8M0, assert_gemm_close, bits16, require_gpu, y_to_f64

OK, INVALID, SHAPE, CUDA = 0, 1, 2, 5
A = 1 << 20          # a fake, aligned "device" address; never dereferenced on these paths
LIMIT = 32 << 20     # FGFP8_NOALLOC_SCRATCH_BYTES


def scratch_bytes(M, K, fmt):
    codes = (M * K + 255) // 256 * 256
    return codes + (K // 128) * ((M + 15) // 16 * 16) * (4 if fmt == F32 else 1)


def test_noalloc_rejects_requests_beyond_the_static_scratch():
    """Checked on the host before any CUDA call, so this runs without a GPU."""
    f = fg.fgfp8_linear_noalloc
    # X, ldx, Wq, Ws, Y, M, N, K, fmt, stream
    assert scratch_bytes(8192, 4096, F32) > LIMIT
    assert f(A, 4096, A, A, A, 8192, 256, 4096, F32, None) == SHAPE
    assert "static scratch" in fg.fgfp8_last_error_string()
    assert f(A, 4096, A, A, A, 1 << 40, 256, 4096, UE8M0, None) == SHAPE
    assert f(A, 256, A, A, A, 4, 256, 100, F32, None) == SHAPE           # K % 128
    assert f(A, 256, A, A, A, 4, 200, 256, F32, None) == SHAPE           # N % 128
    assert f(A, 256, A, A, A, 4, 256, 256, 5, None) == INVALID           # fmt
    assert f(0, 256, A, A, A, 4, 256, 256, F32, None) == INVALID         # NULL X
    assert f(A, 256, A, A, A, 0, 256, 256, F32, None) == OK              # empty: no-op


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_noalloc_without_gpu_fails_loudly():
    assert scratch_bytes(4096, 4096, F32) <= LIMIT
    assert fg.fgfp8_linear_noalloc(A, 4096, A, A, A, 4096, 256, 4096, F32, None) == CUDA


# (M, N, K, fmt): the M > 64 persistent GEMM (both formats) and the few-token kernel
CASES = [(300, 640, 2048, F32), (40, 1280, 7168, UE8M0), (129, 384, 1024, UE8M0), (7, 256, 384, F32)]


@pytest.mark.gpu
def test_noalloc_matches_linear_on_consecutive_calls():
    dev = require_gpu()
    fg.load()
    stream = torch.cuda.current_stream(dev)
    inputs = []
    for M, N, K, fmt in CASES:
        cfg = workloads.scaled_linear(workloads.TINY, M=M, N=N, K=K, seed=13 * M + N + K)
        X, W = workloads.linear_inputs(cfg)
        Wq, Ws = fg.quant_weight(W.to(dev), fmt)
        inputs.append((X, W, X.to(dev), Wq, Ws))

    # two rounds of back-to-back calls on one stream, no host sync in between:
    # each call overwrites the scratch the previous one used
    outs = []
    for _ in range(2):
        for (M, N, K, fmt), (_, _, Xd, Wq, Ws) in zip(CASES, inputs):
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            st = fg.fgfp8_linear_noalloc(Xd.data_ptr(), Xd.stride(0), Wq.data_ptr(), Ws.data_ptr(), Y.data_ptr(),
                                         M, N, K, fmt, stream.cuda_stream)
            assert st == OK, fg.fgfp8_last_error_string()
            outs.append(Y)
    fg.check_device_status()

    for i, ((M, N, K, fmt), (X, W, Xd, Wq, Ws)) in enumerate(zip(CASES * 2, inputs * 2)):
        Y_lin = fg.linear(Xd, Wq, Ws, fmt)
        fg.check_device_status()
        Wq_r, Ws_r = oracle.quant_weight(bits16(W), fmt)
        Xq_r, Xs_r = oracle.quant_act(bits16(X), fmt)
        Y_ref, S = oracle.gemm(Xq_r, Xs_r, Wq_r, Ws_r, fmt)
        what = f"call {i}: noalloc {M}x{N}x{K} fmt {fmt}"
        # against the existing entry point: the same kernels on the same inputs
        # (only the scale rows' stride differs), so the same bits, which also
        # lies within the GEMM tolerance around its output
        assert torch.equal(outs[i], Y_lin), what + " differs from fgfp8_linear"
        assert_gemm_close(y_to_f64(outs[i]), y_to_f64(Y_lin), S, what + " vs fgfp8_linear")
        # and against the oracle
        assert_gemm_close(y_to_f64(outs[i]), Y_ref, S, what + " vs oracle")
