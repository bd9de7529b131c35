"""GPU side of the tensor-parallel column split on one B200: the output
layout kernel against its definition, and a P-way split whose shards run in
sequence on this GPU (each rank's quantized weight rows, its fgfp8_linear,
the stacked parts as the all-gather leaves them, fgfp8_gather_cols) against
the oracle of the unsplit layer.  A world of one NCCL rank runs the
ColumnParallelLinear path itself.  Splits over several GPUs are not run here
(one GPU per test run)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import fine_grained_fp8_token_b200 as fg
import oracle
import workloads
from fine_grained_fp8_token_b200 import tp
from parity import F32, UE8M0, Guarded, assert_gemm_close, bits16, require_gpu, y_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    d = require_gpu()
    fg.load()
    return d


@pytest.mark.parametrize("P,M,n", [(1, 7, 128), (2, 300, 256), (3, 129, 384), (8, 64, 2304), (4, 8192, 7168)])
def test_gather_cols_layout(dev, P, M, n):
    parts = torch.randn((P, M, n), device=dev).to(torch.bfloat16)
    gY = Guarded((M, P * n), torch.bfloat16, dev)
    Y = fg.gather_cols(parts, Y=gY.t)
    fg.check_device_status()
    gY.check("Y")
    assert torch.equal(Y, parts.permute(1, 0, 2).reshape(M, P * n))


@pytest.mark.parametrize("fmt", [F32, UE8M0])
@pytest.mark.parametrize("world", [2, 4])
def test_split_layer_shards_in_sequence(dev, fmt, world):
    M, N, K = 300, 1024, 512
    cfg = workloads.scaled_linear(workloads.TINY, M=M, N=N, K=K, seed=71 + world + fmt)
    X, W = workloads.linear_inputs(cfg)
    Xd, Wd = X.to(dev), W.to(dev)
    Wq_full, Ws_full = fg.quant_weight(Wd, fmt)
    parts = []
    for r in range(world):
        n0, n1 = tp.shard_range(N, world, r)
        Wq_r, Ws_r = fg.quant_weight(Wd[n0:n1], fmt)
        q, s = tp.shard_weight(Wq_full, Ws_full, world, r)
        assert torch.equal(Wq_r, q) and torch.equal(Ws_r.view(torch.uint8), s.view(torch.uint8))
        parts.append(fg.linear(Xd, Wq_r, Ws_r, fmt))
    Y = fg.gather_cols(torch.stack(parts))
    fg.check_device_status()
    Wq_o, Ws_o = oracle.quant_weight(bits16(W), fmt)
    Xq_o, Xs_o = oracle.quant_act(bits16(X), fmt)
    Y_ref, S = oracle.gemm(Xq_o, Xs_o, Wq_o, Ws_o, fmt)
    assert_gemm_close(y_to_f64(Y), Y_ref, S, f"{world}-way column split, fmt {fmt}")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_column_parallel_linear_nccl_world_one(dev):
    """ColumnParallelLinear over a one-rank NCCL group: quantize the rank's
    rows, fgfp8_linear, NCCL all-gather, fgfp8_gather_cols; the output equals
    the unsplit layer bit for bit."""
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=dev)
    try:
        cfg = workloads.scaled_linear(workloads.TINY, M=257, N=768, K=1024, seed=5)
        X, W = workloads.linear_inputs(cfg, device=dev)
        layer = tp.ColumnParallelLinear.from_weight(W, F32)
        Y = layer.forward(X)
        torch.cuda.synchronize(dev)
        Wq, Ws = fg.quant_weight(W, F32)
        Y_full = fg.linear(X, Wq, Ws, F32)
        fg.check_device_status()
        assert torch.equal(Y, Y_full)
    finally:
        dist.destroy_process_group()
