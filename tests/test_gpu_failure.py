"""Failure detection on the GPU without a fault: a barrier wait that nothing
completes gives up after its one-second limit, the device status word
reports FGFP8_ERR_TIMEOUT to the host, the word is cleared by the read, and
the same context then runs work correctly."""
import time

import numpy as np
import pytest

import fine_grained_fp8_token_b200 as fg
import oracle
import workloads
from parity import F32, assert_gemm_close, bits16, require_gpu, y_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    d = require_gpu()
    fg.load()
    return d


def test_expired_wait_reported_and_context_usable(dev):
    fg.check_device_status()                            # clean start
    t0 = time.monotonic()
    fg.selftest_expired_wait()
    with pytest.raises(fg.FGFP8Error) as ei:
        fg.check_device_status()
    waited = time.monotonic() - t0
    assert ei.value.status == 6                         # FGFP8_ERR_TIMEOUT
    assert 0.9 < waited < 30.0, waited                  # the one-second limit, not an endless wait
    fg.check_device_status()                            # the read cleared the word
    cfg = workloads.scaled_linear(workloads.TINY, M=200, N=256, K=512, seed=13)
    X, W = workloads.linear_inputs(cfg)
    Xq, Xs = fg.quant_act(X.to(dev), F32)
    Wq, Ws = fg.quant_weight(W.to(dev), F32)
    Y = fg.gemm(Xq, Xs, Wq, Ws, F32)
    fg.check_device_status()
    Wq_r, Ws_r = oracle.quant_weight(bits16(W), F32)
    Xq_r, Xs_r = oracle.quant_act(bits16(X), F32)
    Y_ref, S = oracle.gemm(Xq_r, Xs_r, Wq_r, Ws_r, F32)
    assert_gemm_close(y_to_f64(Y), Y_ref, S, "GEMM after the expired wait")


@pytest.mark.parametrize("fmt", [0, 1], ids=["fp32_promotion", "ue8m0_block_scaled"])
def test_gemm_withheld_tile_unwinds(dev, fmt):
    """The dense GEMM with one K block of work item 0 never requested: the
    MMA issuer's wait expires, the producer, scale and epilogue waits follow,
    every role unwinds (bounded waits for its own copies and MMAs, TMEM
    freed) and the launch ends within seconds with FGFP8_ERR_TIMEOUT.  The
    other CTAs' tiles are still correct, and the next GEMM on the same
    context matches the oracle everywhere."""
    M, N, K = 1024, 512, 1024
    cfg = workloads.scaled_linear(workloads.TINY, M=M, N=N, K=K, seed=29 + fmt)
    X, W = workloads.linear_inputs(cfg)
    Xq, Xs = fg.quant_act(X.to(dev), fmt)
    Wq, Ws = fg.quant_weight(W.to(dev), fmt)
    fg.check_device_status()                            # clean start
    t0 = time.monotonic()
    Y = fg.selftest_gemm_timeout(Xq, Xs, Wq, Ws, fmt, withhold_kb=3)
    with pytest.raises(fg.FGFP8Error) as ei:
        fg.check_device_status()
    waited = time.monotonic() - t0
    assert ei.value.status == 6                         # FGFP8_ERR_TIMEOUT
    assert 0.9 < waited < 30.0, waited
    fg.check_device_status()                            # cleared
    Wq_r, Ws_r = oracle.quant_weight(bits16(W), fmt)
    Xq_r, Xs_r = oracle.quant_act(bits16(X), fmt)
    Y_ref, S = oracle.gemm(Xq_r, Xs_r, Wq_r, Ws_r, fmt)
    Yf = y_to_f64(Y)
    # work item 0 is the 128 x 256 tile at rows 0..127, columns 0..255
    assert_gemm_close(Yf[128:], Y_ref[128:], S[128:], "tiles of the other CTAs")
    assert_gemm_close(Yf[:128, 256:], Y_ref[:128, 256:], S[:128, 256:], "tiles of the other CTAs")
    Y2 = fg.gemm(Xq, Xs, Wq, Ws, fmt)
    fg.check_device_status()
    assert_gemm_close(y_to_f64(Y2), Y_ref, S, "GEMM after the unwound launch")
