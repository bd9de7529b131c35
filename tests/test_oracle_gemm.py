"""Pins for the oracle's block-scaled GEMM and M-grouped GEMM (CPU only).

Pinned by: an fp64 brute-force product of the dequantized operands through
numpy's matmul (a library routine) on tiny shapes, special cases with exact
closed-form results, the hand-derived example in tests/golden/gemm_tiny.json,
and the M-grouped GEMM checked row by row against brute force with each row's
own expert weights.
"""
import json
import os

import numpy as np
import pytest
import torch

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32, UE8M0 = 0, 1


def bits(x):
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def brute(orc, Xq, Xs, Wq, Ws, fmt):
    xh = orc.dequant_act(Xq, Xs, fmt)
    wh = orc.dequant_weight(Wq, Ws, fmt)
    return xh @ wh.T, np.abs(xh) @ np.abs(wh).T


SHAPES = [(128, 256, 512)] + [(m, n, k) for m in (128, 256) for n in (128, 256) for k in (128, 256, 384)] + [(7, 384, 640)]


@pytest.mark.parametrize("fmt", [F32, UE8M0])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_vs_fp64_brute_force(orc, fmt, M, N, K):
    cfg = workloads.scaled_linear(workloads.TINY, M=M, N=N, K=K, fmt=fmt, seed=M + N + K)
    X, W = workloads.linear_inputs(cfg)
    Xq, Xs = orc.quant_act(bits(X), fmt)
    Wq, Ws = orc.quant_weight(bits(W), fmt)
    Y, S = orc.gemm(Xq, Xs, Wq, Ws, fmt)
    Yb, Sb = brute(orc, Xq, Xs, Wq, Ws, fmt)
    # the block sums are exact; only the scaling and the cross-block fp64 sum round
    assert (np.abs(Y - Yb) <= 1e-12 * Sb).all()
    assert (np.abs(S - Sb) <= 1e-12 * Sb).all()
    assert orc.gemm_within_tolerance(Y, Y, S).all()


def test_gemm_row_subset_is_consistent(orc):
    cfg = workloads.scaled_linear(workloads.TINY, M=64, N=256, K=256)
    X, W = workloads.linear_inputs(cfg)
    Xq, Xs = orc.quant_act(bits(X), F32)
    Wq, Ws = orc.quant_weight(bits(W), F32)
    Y, S = orc.gemm(Xq, Xs, Wq, Ws, F32)
    rows = np.array([63, 0, 17, 17])
    Yr, Sr = orc.gemm(Xq, Xs, Wq, Ws, F32, rows=rows)
    assert (Yr == Y[rows]).all() and (Sr == S[rows]).all()


def test_gemm_all_ones_unit_scales(orc):
    """Codes 0x38 (= 1.0) with unit scales: every output equals K."""
    M, N, K = 4, 128, 384
    Xq = np.full((M, K), 0x38, np.uint8)
    Wq = np.full((N, K), 0x38, np.uint8)
    Xs = np.ones((K // 128, 4), np.float32)
    Ws = np.ones((N // 128, K // 128), np.float32)
    Y, S = orc.gemm(Xq, Xs, Wq, Ws, F32)
    assert (Y == K).all() and (S == K).all()
    # UE8M0 byte 127 is the unit scale; byte 128 doubles one operand
    Xs8 = np.full((K // 128, 16), 127, np.uint8)
    Ws8 = np.full((N // 128, K // 128), 127, np.uint8)
    Ws8[0, 1] = 128
    Y8, _ = orc.gemm(Xq, Xs8, Wq, Ws8, UE8M0)
    assert (Y8 == K + 128).all()


def test_gemm_identity_like_weight_exact(orc):
    """W = 0.5 * I (K = N): with UE8M0 the diagonal 0.5 quantizes exactly
    (0.5 / 2^-9 = 256), so Y = 0.5 * x_hat exactly."""
    K = N = 256
    X = workloads.activations((16, K), "normal_outliers", seed=9)
    W = (torch.eye(N) * 0.5).to(torch.bfloat16)
    Xq, Xs = orc.quant_act(bits(X), UE8M0)
    Wq, Ws = orc.quant_weight(bits(W), UE8M0)
    Y, _ = orc.gemm(Xq, Xs, Wq, Ws, UE8M0)
    xh = orc.dequant_act(Xq, Xs, UE8M0)
    assert (Y == 0.5 * xh).all()


def test_gemm_sign_and_operand_order(orc):
    """A single nonzero weight picks one input column with its sign: a
    transposed operand or a wrong scale index breaks this."""
    M, N, K = 8, 256, 384
    X = workloads.activations((M, K), "normal", seed=4)
    W = torch.zeros((N, K), dtype=torch.bfloat16)
    W[200, 300] = -0.25
    Xq, Xs = orc.quant_act(bits(X), UE8M0)
    Wq, Ws = orc.quant_weight(bits(W), UE8M0)
    Y, _ = orc.gemm(Xq, Xs, Wq, Ws, UE8M0)
    xh = orc.dequant_act(Xq, Xs, UE8M0)
    expect = np.zeros((M, N))
    expect[:, 200] = -0.25 * xh[:, 300]
    assert (Y == expect).all()


def test_gemm_golden_tiny(orc):
    g = json.load(open(os.path.join(GOLDEN, "gemm_tiny.json")))
    X = torch.zeros((g["M"], g["K"]), dtype=torch.float32)
    for k, v in g["x"].items():
        X[0, int(k)] = v
    W = torch.zeros((g["N"], g["K"]), dtype=torch.float32)
    for nk, v in g["w"].items():
        n, k = map(int, nk.split(","))
        W[n, k] = v
    Xb, Wb = X.to(torch.bfloat16), W.to(torch.bfloat16)
    Xq, Xs = orc.quant_act(bits(Xb), UE8M0)
    Wq, Ws = orc.quant_weight(bits(Wb), UE8M0)
    assert Xs[0, 0] == g["x_scale_byte"] and Ws[0, 0] == g["w_scale_byte"]
    for k, v in g["x_codes"].items():
        assert Xq[0, int(k)] == v
    for nk, v in g["w_codes"].items():
        n, k = map(int, nk.split(","))
        assert Wq[n, k] == v
    Y, _ = orc.gemm(Xq, Xs, Wq, Ws, UE8M0)
    expect = np.zeros(g["N"])
    for n, v in g["y"].items():
        expect[int(n)] = v
    assert (Y[0] == expect).all()


@pytest.mark.parametrize("fmt", [UE8M0, F32])
def test_grouped_gemm_rows_vs_brute_force(orc, fmt):
    cfg = workloads.scaled_moe(workloads.MOE, E=6, N=256, K=384, tokens=40, topk=2)
    r = workloads.moe_routing(cfg)
    X = workloads.moe_grouped_rows(workloads.moe_tokens(cfg), r)
    Ws_l, Wq_l = [], []
    for e in range(cfg.E):
        q, s = orc.quant_weight(bits(workloads.moe_expert_weight(cfg, e)), fmt)
        Wq_l.append(q)
        Ws_l.append(s)
    Wq, Ws = np.stack(Wq_l), np.stack(Ws_l)
    Xq, Xs = orc.quant_act(bits(X), fmt)
    Y, S = orc.grouped_gemm(Xq, Xs, Wq, Ws, r.group_offs, fmt)
    offs = r.group_offs
    for e in range(cfg.E):
        lo, hi = offs[e], offs[e + 1]
        if hi == lo:
            continue
        Yb, Sb = brute(orc, Xq[lo:hi], _rows_scale(Xs, lo, hi, fmt), Wq[e], Ws[e], fmt)
        assert (np.abs(Y[lo:hi] - Yb) <= 1e-12 * Sb + 1e-300).all()
    # padding rows are all-zero inputs and give zero outputs
    pad = r.row_token < 0
    assert (Y[pad] == 0).all()
    with pytest.raises(ValueError):
        orc.grouped_gemm(Xq, Xs, Wq, Ws, r.group_offs, fmt, rows=[int(offs[-1])])


def _rows_scale(Xs, lo, hi, fmt):
    """MN-major scales of rows lo..hi as a fresh [KB, ld] array."""
    n = hi - lo
    unit = 4 if fmt == F32 else 16
    ld = max(unit, (n + unit - 1) // unit * unit)
    out = np.zeros((Xs.shape[0], ld), dtype=Xs.dtype)
    out[:, :n] = Xs[:, lo:hi]
    return out


def test_tolerance_accepts_bf16_rounding(orc):
    cfg = workloads.scaled_linear(workloads.TINY, M=32, N=128, K=256)
    X, W = workloads.linear_inputs(cfg)
    Xq, Xs = orc.quant_act(bits(X), F32)
    Wq, Ws = orc.quant_weight(bits(W), F32)
    Y, S = orc.gemm(Xq, Xs, Wq, Ws, F32)
    yb = torch.from_numpy(orc.bf16_rne(Y).view(np.int16)).view(torch.bfloat16).double().numpy()
    assert orc.gemm_within_tolerance(yb, Y, S).all()
    # an error of 2^-6 relative on a large output is rejected
    big = np.abs(Y) > 200 * 1e-4 * S       # then 2^-7|Y| > 1e-4 S
    assert big.any()
    assert not orc.gemm_within_tolerance(Y * (1 + 2.0 ** -6), Y, S)[big].any()
