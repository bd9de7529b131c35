"""GPU parity of the quantizers against the oracle: E4M3 codes and scales
must match bit for bit (finite inputs), for the small ragged cases and for
every activation / weight tensor of the five workloads at full size."""
import numpy as np
import pytest
import torch

import fine_grained_fp8_token_b200 as fg
import oracle
import workloads
from parity import (F32, UE8M0, assert_codes_equal, assert_scales_equal, bits16, require_gpu, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    d = require_gpu()
    fg.load()
    return d


def gpu_quant_act(X_dev, fmt, ld_s=None, sentinel=True):
    M, K = X_dev.shape
    ld_s = fg.scale_rows(M, fmt) if ld_s is None else ld_s
    Xs = torch.empty((K // 128, ld_s), dtype=torch.float32 if fmt == F32 else torch.uint8, device=X_dev.device)
    if sentinel:
        Xs.view(torch.uint8).fill_(0xAB)
    Xq, Xs = fg.quant_act(X_dev, fmt, Xs=Xs, ld_s=ld_s)
    torch.cuda.synchronize()
    fg.check_device_status()
    return to_np(Xq), to_np(Xs)


def check_act(X_cpu_bits: np.ndarray, Xq_gpu, Xs_gpu, fmt, M, what):
    Xq_ref, Xs_ref = oracle.quant_act(X_cpu_bits, fmt, ld_s=Xs_gpu.shape[1])
    assert_codes_equal(Xq_gpu, Xq_ref, what + " codes")
    assert_scales_equal(Xs_gpu[:, :M], Xs_ref[:, :M], what + " scales")


SMALL = [(128, 512, "normal_outliers"), (1, 128, "normal"), (7, 384, "normal_outliers"),
         (129, 1024, "heavy_tail"), (300, 4096, "normal_outliers"), (33, 7168, "normal"),
         (2, 14336, "heavy_tail"), (1000, 256, "normal_outliers")]


@pytest.mark.parametrize("fmt", [F32, UE8M0])
@pytest.mark.parametrize("M,K,kind", SMALL)
def test_quant_act_small(dev, fmt, M, K, kind):
    X = workloads.activations((M, K), kind, seed=M * 7 + K)
    Xq, Xs = gpu_quant_act(X.to(dev), fmt)
    check_act(bits16(X), Xq, Xs, fmt, M, f"act {M}x{K}")
    # scale padding beyond M is untouched
    pad = Xs[:, M:].view(np.uint8)
    assert (pad == 0xAB).all()


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_quant_act_strided_input_and_wide_ld_s(dev, fmt):
    M, K = 77, 640
    X = workloads.activations((M, K), "normal_outliers", seed=5)
    buf = torch.zeros((M, K + 136), dtype=torch.bfloat16, device=dev)   # ldx = K + 136 (multiple of 8)
    buf[:, 64:64 + K] = X.to(dev)
    Xv = buf[:, 64:64 + K]
    assert Xv.stride(0) == K + 136
    Xq, Xs = gpu_quant_act(Xv, fmt, ld_s=fg.scale_rows(M, fmt) + 32)
    check_act(bits16(X), Xq, Xs, fmt, M, "strided act")


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_quant_act_random_bit_patterns(dev, fmt):
    """Uniformly random finite bf16 bit patterns: groups mix subnormals, huge
    values and everything between (the quotient meets every exponent)."""
    g = torch.Generator().manual_seed(17)
    raw = torch.randint(0, 1 << 16, (512, 1024), generator=g, dtype=torch.int32)
    exp = (raw >> 7) & 0xFF
    raw = torch.where(exp == 0xFF, raw & ~(1 << 14), raw)        # drop Inf/NaN patterns
    X = raw.to(torch.int16).view(torch.bfloat16)
    Xq, Xs = gpu_quant_act(X.to(dev), fmt)
    check_act(bits16(X), Xq, Xs, fmt, 512, "random bits")


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_quant_act_special_values(dev, fmt):
    rows = []
    z = torch.zeros(128)
    rows.append(z.clone())                                      # all zero -> floor scale
    r = z.clone(); r[3] = -0.0; rows.append(r)                  # negative zero keeps its sign
    r = z.clone(); r[0] = 448; r[1] = 17; r[2] = 19; r[3] = 1.0625; r[4] = -17; rows.append(r)   # ties
    r = z.clone(); r[0] = 3.3895e38; r[1] = -1e38; r[2] = 1.0; rows.append(r)   # near bf16 max
    r = torch.full((128,), 9.1835e-41); r[5] = -9.1835e-41; rows.append(r)      # bf16 subnormals
    r = z.clone(); r[0] = 5e-5; r[1] = -2.5e-5; rows.append(r)                 # below the amax floor
    r = torch.linspace(-1, 1, 128); rows.append(r)
    X = torch.stack(rows).to(torch.bfloat16)
    X = torch.cat([X, -X], dim=0)
    Xq, Xs = gpu_quant_act(X.to(dev), fmt)
    check_act(bits16(X), Xq, Xs, fmt, X.shape[0], "special values")
    assert Xq[1, 3] == 0x80


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_quant_act_nonfinite_groups(dev, fmt):
    """Finite groups stay bit-exact next to groups holding NaN or Inf, whose
    scale is non-finite (codes of such a group are unspecified)."""
    X = workloads.activations((4, 512), "normal", seed=1)
    X[0, 5] = float("nan")
    X[1, 300] = float("inf")
    X[2, 140] = float("-inf")
    Xq, Xs = gpu_quant_act(X.to(dev), fmt)
    Xq_ref, Xs_ref = oracle.quant_act(bits16(X), fmt, ld_s=Xs.shape[1])
    bad = {(0, 0), (2, 1), (1, 2)}               # (group, row) with a non-finite element
    for g in range(4):
        for m in range(4):
            if (g, m) in bad:
                if fmt == F32:
                    assert not np.isfinite(Xs[g, m])
                else:
                    assert Xs[g, m] == 0xFF
            else:
                assert_codes_equal(Xq[m, g * 128:(g + 1) * 128], Xq_ref[m, g * 128:(g + 1) * 128], "finite group")
                assert_scales_equal(Xs[g:g + 1, m], Xs_ref[g:g + 1, m], "finite group scale")


FULL_ACT = [(workloads.LLAMA_ATTN, None), (workloads.LLAMA_GATE_UP, None), (workloads.LLAMA_DOWN, None)] + \
           [(workloads.DS_DECODE[m], None) for m in (1, 8, 32, 64)]


@pytest.mark.parametrize("cfg", [c for c, _ in FULL_ACT], ids=lambda c: c.name)
def test_quant_act_full_size(dev, cfg):
    X = workloads.activations((cfg.M, cfg.K), cfg.x_kind, cfg.seed, device=dev)
    Xq, Xs = gpu_quant_act(X, cfg.fmt)
    check_act(bits16(X), Xq, Xs, cfg.fmt, cfg.M, cfg.name)


def test_quant_act_moe_rows(dev):
    cfg = workloads.MOE
    r = workloads.moe_routing(cfg)
    X = workloads.moe_grouped_rows(workloads.moe_tokens(cfg, device=dev), r)
    Xq, Xs = gpu_quant_act(X, cfg.fmt)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([rng.integers(0, r.M_total, 400), r.group_offs[:-1][:64],
                                     [r.M_total - 1]]))
    Xq_ref, Xs_ref = oracle.quant_act(bits16(X[torch.as_tensor(rows, device=dev)]), cfg.fmt)
    assert_codes_equal(Xq[rows], Xq_ref, "moe rows codes")
    assert_scales_equal(Xs[:, rows], Xs_ref[:, :len(rows)], "moe rows scales")


# ---------------------------------------------------------------- weights
@pytest.mark.parametrize("fmt", [F32, UE8M0])
@pytest.mark.parametrize("N,K", [(128, 128), (384, 256), (256, 1152), (1280, 7168)])
def test_quant_weight_small(dev, fmt, N, K):
    W = workloads.weights((N, K), seed=N + K)
    W[N // 2, K - 1] = 0.9                              # one outlier block
    Wq, Ws = fg.quant_weight(W.to(dev), fmt)
    Wq_ref, Ws_ref = oracle.quant_weight(bits16(W), fmt)
    assert_codes_equal(to_np(Wq), Wq_ref, "weight codes")
    assert_scales_equal(to_np(Ws), Ws_ref, "weight scales")


def special_blocks():
    """A [256, 512] bf16 weight whose eight 128x128 blocks each hold one
    degenerate pattern: all zero, negative zero, rounding ties, near the bf16
    maximum, bf16 subnormals, below the amax floor, a ramp, and a single
    nonzero element."""
    W = torch.zeros((256, 512))
    blocks = [(r, c) for r in range(2) for c in range(4)]
    def blk(i):
        r, c = blocks[i]
        return W[r * 128:(r + 1) * 128, c * 128:(c + 1) * 128]
    blk(1)[5, 7] = -0.0
    b = blk(2); b[0, 0] = 448; b[0, 1] = 17; b[0, 2] = 19; b[1, 0] = 1.0625; b[1, 1] = -17
    b = blk(3); b[0, 0] = 3.3895e38; b[0, 1] = -1e38; b[2, 2] = 1.0
    blk(4).fill_(9.1835e-41); blk(4)[3, 3] = -9.1835e-41
    b = blk(5); b[0, 0] = 5e-5; b[9, 9] = -2.5e-5
    blk(6).copy_(torch.linspace(-1, 1, 128 * 128).reshape(128, 128))
    blk(7)[64, 64] = -0.75
    return W.to(torch.bfloat16)


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_quant_weight_special_blocks(dev, fmt):
    W = special_blocks()
    W = torch.cat([W, -W], dim=0)
    Wq, Ws = fg.quant_weight(W.to(dev), fmt)
    Wq_ref, Ws_ref = oracle.quant_weight(bits16(W), fmt)
    assert_codes_equal(to_np(Wq), Wq_ref, "special weight codes")
    assert_scales_equal(to_np(Ws), Ws_ref, "special weight scales")
    assert to_np(Wq)[5, 128 + 7] == 0x80                 # negative zero keeps its sign


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_quant_weight_nonfinite_blocks(dev, fmt):
    """Finite blocks stay bit-exact next to blocks holding NaN or Inf, whose
    scale is non-finite (their codes are unspecified)."""
    W = workloads.weights((256, 384), seed=4)
    W[3, 5] = float("nan")                               # block (0, 0)
    W[200, 300] = float("inf")                           # block (1, 2)
    W[130, 140] = float("-inf")                          # block (1, 1)
    Wq, Ws = fg.quant_weight(W.to(dev), fmt)
    Wq_ref, Ws_ref = oracle.quant_weight(bits16(W), fmt)
    Wq, Ws = to_np(Wq), to_np(Ws)
    bad = {(0, 0), (1, 2), (1, 1)}
    for nb in range(2):
        for kb in range(3):
            rows, cols = slice(nb * 128, nb * 128 + 128), slice(kb * 128, kb * 128 + 128)
            if (nb, kb) in bad:
                if fmt == F32:
                    assert not np.isfinite(Ws[nb, kb])
                else:
                    assert Ws[nb, kb] == 0xFF
            else:
                assert_codes_equal(Wq[rows, cols], Wq_ref[rows, cols], "finite block")
                assert_scales_equal(Ws[nb:nb + 1, kb:kb + 1], Ws_ref[nb:nb + 1, kb:kb + 1], "finite block scale")


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_quant_weight_strided(dev, fmt):
    N, K = 256, 384
    W = workloads.weights((N, K), seed=3)
    buf = torch.zeros((N, K + 256), dtype=torch.bfloat16, device=dev)
    buf[:, 128:128 + K] = W.to(dev)
    Wq, Ws = fg.quant_weight(buf[:, 128:128 + K], fmt)
    Wq_ref, Ws_ref = oracle.quant_weight(bits16(W), fmt)
    assert_codes_equal(to_np(Wq), Wq_ref, "strided weight codes")
    assert_scales_equal(to_np(Ws), Ws_ref, "strided weight scales")


@pytest.mark.parametrize("cfg", [workloads.LLAMA_ATTN, workloads.LLAMA_GATE_UP, workloads.LLAMA_DOWN,
                                 workloads.DS_DECODE[1]], ids=lambda c: c.name)
def test_quant_weight_full_size(dev, cfg):
    W = workloads.weights((cfg.N, cfg.K), cfg.seed + 1, device=dev)
    Wq, Ws = fg.quant_weight(W, cfg.fmt)
    Wq_ref, Ws_ref = oracle.quant_weight(bits16(W), cfg.fmt)
    assert_codes_equal(to_np(Wq), Wq_ref, cfg.name + " weight codes")
    assert_scales_equal(to_np(Ws), Ws_ref, cfg.name + " weight scales")


def test_quant_weight_moe_expert_stack(dev):
    """Three experts quantized as one [3*N, K] stack equal three separate
    oracle quantizations (blocks never straddle experts)."""
    cfg = workloads.MOE
    experts = [0, 117, 255]
    W = torch.cat([workloads.moe_expert_weight(cfg, e, device=dev) for e in experts])
    Wq, Ws = fg.quant_weight(W, cfg.fmt)
    Wq, Ws = to_np(Wq), to_np(Ws)
    for i, e in enumerate(experts):
        Wq_ref, Ws_ref = oracle.quant_weight(bits16(W[i * cfg.N:(i + 1) * cfg.N]), cfg.fmt)
        assert_codes_equal(Wq[i * cfg.N:(i + 1) * cfg.N], Wq_ref, f"expert {e} codes")
        assert_scales_equal(Ws[i * cfg.N // 128:(i + 1) * cfg.N // 128], Ws_ref, f"expert {e} scales")
