"""Host logic of the tensor-parallel column split (CPU, gloo ranks): the
shard plan, the per-rank weight rows, the all-gather of the parts and the
layout of the gathered output.  The GPU side (each shard's GEMM against the
oracle, the layout kernel) is in test_gpu_tp.py."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from fine_grained_fp8_token_b200 import tp  # noqa: E402


@pytest.mark.parametrize("N,world", [(4096, 1), (4096, 2), (28672, 8), (18432, 4), (1024, 8)])
def test_shard_range_partitions_whole_blocks(N, world):
    ranges = [tp.shard_range(N, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == N
    for (a0, a1), (b0, _) in zip(ranges, ranges[1:]):
        assert a1 == b0                              # contiguous, disjoint
    assert len({b - a for a, b in ranges}) == 1      # equal parts for the all-gather
    assert all(a % 128 == 0 and b % 128 == 0 for a, b in ranges)


@pytest.mark.parametrize("N,world,rank", [(4096, 3, 0), (1000, 1, 0), (1024, 16, 0), (4096, 2, 2), (4096, 2, -1)])
def test_shard_range_rejects(N, world, rank):
    with pytest.raises(ValueError):
        tp.shard_range(N, world, rank)


def test_shard_weight_rows_equal_quantized_slice(orc):
    """Quantizing a rank's rows of W gives exactly the full layer's codes and
    block scales for those rows (the oracle as the quantizer), in both scale
    formats: splitting in whole 128-row blocks keeps every block intact."""
    import workloads
    W = workloads.weights((512, 384), seed=3)
    wb = W.contiguous().view(torch.int16).numpy().view(np.uint16)
    for fmt in (0, 1):
        Wq, Ws = orc.quant_weight(wb, fmt)
        for world in (1, 2, 4):
            for r in range(world):
                q, s = tp.shard_weight(torch.from_numpy(Wq), torch.from_numpy(Ws), world, r)
                n0, n1 = tp.shard_range(512, world, r)
                q_r, s_r = orc.quant_weight(np.ascontiguousarray(wb[n0:n1]), fmt)
                assert np.array_equal(q.numpy(), q_r)
                assert np.array_equal(s.numpy().view(np.uint8), s_r.view(np.uint8))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


M, N = 5, 512


def _full_output():
    return torch.arange(M * N, dtype=torch.float32).reshape(M, N).to(torch.bfloat16)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        n0, n1 = tp.shard_range(N, world, rank)
        Y_local = _full_output()[:, n0:n1].contiguous()     # this rank's columns of the layer output
        parts = tp.all_gather_parts(Y_local)
        out[rank] = parts.float().numpy()
    finally:
        dist.destroy_process_group()


def test_all_gather_parts_and_layout_gloo_world2():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    full = _full_output().float().numpy()
    n = N // world
    for rank in range(world):
        parts = res[rank]
        assert parts.shape == (world, M, n)
        for p in range(world):
            assert np.array_equal(parts[p], full[:, p * n:(p + 1) * n])
        # the layout fgfp8_gather_cols writes: Y[m, p * n + j] = parts[p, m, j]
        Y = np.transpose(parts, (1, 0, 2)).reshape(M, world * n)
        assert np.array_equal(Y, full)
