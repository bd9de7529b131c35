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
