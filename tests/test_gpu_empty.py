"""Empty inputs through the binding and the C ABI on the GPU: every entry
point with zero tokens (or zero rows) returns without launching work,
leaves its outputs untouched and leaves the device status word clear.  A
zero-size torch tensor may hand the library a NULL pointer; the header
specifies these calls as no-ops."""
import numpy as np
import pytest
import torch

import fine_grained_fp8_token_b200 as fg
import oracle
import workloads
from parity import F32, UE8M0, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    d = require_gpu()
    fg.load()
    return d


def weights(dev, N, K, fmt, E=None):
    if E is None:
        return fg.quant_weight(workloads.weights((N, K), seed=5, device=dev), fmt)
    Wq = torch.empty((E, N, K), dtype=torch.uint8, device=dev)
    Ws = torch.empty((E, N // 128, K // 128), dtype=torch.float32 if fmt == F32 else torch.uint8, device=dev)
    for e in range(E):
        fg.quant_weight(workloads.weights((N, K), seed=6 + e, device=dev), fmt, Wq=Wq[e], Ws=Ws[e])
    return Wq, Ws


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_zero_tokens_quant_gemm_linear(dev, fmt):
    N, K = 256, 512
    Wq, Ws = weights(dev, N, K, fmt)
    X = torch.empty((0, K), dtype=torch.bfloat16, device=dev)
    Xq, Xs = fg.quant_act(X, fmt)
    assert Xq.shape == (0, K)
    Y = fg.gemm(Xq, Xs, Wq, Ws, fmt)
    assert Y.shape == (0, N)
    Y = fg.linear(X, Wq, Ws, fmt)
    assert Y.shape == (0, N)
    torch.cuda.synchronize()
    fg.check_device_status()


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_zero_rows_grouped_and_masked(dev, fmt):
    E, N, K = 3, 256, 256
    Wq, Ws = weights(dev, N, K, fmt, E=E)
    # grouped: every expert empty, M_total = 0
    Xq = torch.empty((0, K), dtype=torch.uint8, device=dev)
    Xs = torch.empty((K // 128, fg.scale_rows(0, fmt)), dtype=torch.float32 if fmt == F32 else torch.uint8,
                     device=dev)
    offs = torch.zeros(E + 1, dtype=torch.int32, device=dev)
    Y = fg.grouped_gemm(Xq, Xs, Wq, Ws, offs, fmt)
    assert Y.shape == (0, N)
    # masked: every expert block of padding only (all counts 0): nothing written
    cap = 128
    X = workloads.activations((E * cap, K), "normal", seed=3, device=dev)
    Xq, Xs = fg.quant_act(X, fmt)
    cnt = torch.zeros(E, dtype=torch.int32, device=dev)
    Y = torch.full((E * cap, N), 7.0, dtype=torch.bfloat16, device=dev)
    fg.masked_gemm(Xq, Xs, Wq, Ws, cnt, fmt, Y=Y)
    torch.cuda.synchronize()
    fg.check_device_status()
    assert (Y.float() == 7.0).all()


def test_zero_rows_row_and_tensor_scales(dev):
    K, N = 256, 384
    X = torch.empty((0, K), dtype=torch.bfloat16, device=dev)
    Xq, s = fg.quant_rows(X)
    assert Xq.shape == (0, K) and s.shape == (0,)
    # the scale of an empty tensor is the 1e-4 floor's, as for an all-zero one
    st = fg.tensor_scale(X)
    assert float(st) == float(np.float32(1e-4) / np.float32(448.0))
    assert float(st) == float(oracle.tensor_scale(np.zeros((0, K), dtype=np.uint16)))
    assert fg.quant_static(X, st).shape == (0, K)
    Wq, sw = fg.quant_rows(workloads.weights((N, K), seed=2, device=dev))
    Y = fg.gemm_rowcol(Xq, s, Wq, sw)
    assert Y.shape == (0, N)
    torch.cuda.synchronize()
    fg.check_device_status()


def test_zero_tokens_fused_swiglu(dev):
    I, K = 256, 512
    W_gu = fg.interleave_gate_up(workloads.weights((I, K), seed=8), workloads.weights((I, K), seed=9))
    Wq, Ws = fg.quant_weight(W_gu.to(dev), F32)
    Xq, Xs = fg.quant_act(torch.empty((0, K), dtype=torch.bfloat16, device=dev), F32)
    Hq, Hs = fg.gemm_swiglu_quant(Xq, Xs, Wq, Ws)
    assert Hq.shape == (0, I)
    torch.cuda.synchronize()
    fg.check_device_status()
