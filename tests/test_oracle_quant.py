"""Pins for the oracle's activation and weight quantizers (CPU only).

Pinned by: hand-derived golden groups (tests/golden/quant_groups.json), an
independent restatement through torch library routines (amax, IEEE fp32
division, torch's float8_e4m3fn conversion), the quantize/dequantize error
bound that follows from E4M3's 3 mantissa bits, and layout invariants.
"""
import json
import os

import numpy as np
import pytest
import torch

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32, UE8M0 = 0, 1


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def torch_quant_groups(x: torch.Tensor, fmt: int):
    """Quantize rows of 128-element groups with torch ops only.
    x: bf16 [G, 128] -> (codes u8 [G, 128], scale fp32 [G] or e8m0 byte [G])."""
    xf = x.float()
    amax = xf.abs().amax(dim=1)
    amax = torch.where(amax < torch.tensor(1e-4, dtype=torch.float32),
                       torch.tensor(1e-4, dtype=torch.float32), amax)
    t = amax / torch.tensor(448.0, dtype=torch.float32)
    if fmt == F32:
        s = t
        stored = t
    else:
        mant, ex = torch.frexp(t)
        p = torch.where(mant == 0.5, ex - 1, ex)
        s = torch.ldexp(torch.ones_like(t), p)
        stored = (p + 127).to(torch.uint8)
    q = (xf / s[:, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    return q.numpy(), stored.numpy()


def group_from_case(case):
    x = torch.zeros(128, dtype=torch.float32)
    for k, v in case["x"].items():
        x[int(k)] = v
    xb = x.to(torch.bfloat16)
    assert (xb.float() == x).all(), "golden inputs must be bf16-exact"
    return xb


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "quant_groups.json")))["cases"],
                         ids=lambda c: c["name"])
def test_golden_groups(orc, case):
    fmt = F32 if case["fmt"] == "f32" else UE8M0
    xb = group_from_case(case)
    # as one token's single group (activation) ...
    Xq, Xs = orc.quant_act(bf16_bits(xb[None, :]), fmt)
    codes = np.zeros(128, dtype=np.uint8)
    for k, v in case["codes"].items():
        codes[int(k)] = v
    assert (Xq[0] == codes).all()
    if fmt == F32:
        assert Xs[0, 0] == np.float32(case["scale"])
    else:
        assert Xs[0, 0] == case["scale_byte"]
    # ... and as row 0 of a 128x128 weight block (other rows zero)
    W = torch.zeros((128, 128), dtype=torch.bfloat16)
    W[0] = xb
    Wq, Ws = orc.quant_weight(bf16_bits(W), fmt)
    assert (Wq[0] == codes).all() and (Wq[1:] == 0).all()
    assert Ws[0, 0] == Xs[0, 0]


def test_all_zero_group_scale_floor(orc):
    Xq, Xs = orc.quant_act(np.zeros((1, 128), dtype=np.uint16), F32)
    assert (Xq == 0).all()
    assert Xs[0, 0] == np.float32(1e-4) / np.float32(448.0)
    Xq, Xs = orc.quant_act(np.zeros((1, 128), dtype=np.uint16), UE8M0)
    assert (Xq == 0).all() and Xs[0, 0] == 105
    # negative zeros keep their sign
    negz = np.full((1, 128), 0x8000, dtype=np.uint16)
    Xq, _ = orc.quant_act(negz, F32)
    assert (Xq == 0x80).all()


@pytest.mark.parametrize("fmt", [F32, UE8M0])
@pytest.mark.parametrize("shape,kind", [((37, 384), "normal_outliers"), ((130, 256), "heavy_tail"),
                                        ((5, 1024), "normal")])
def test_quant_act_matches_torch_restatement(orc, fmt, shape, kind):
    X = workloads.activations(shape, kind, seed=11)
    M, K = shape
    Xq, Xs = orc.quant_act(bf16_bits(X), fmt)
    q_ref, s_ref = torch_quant_groups(X.reshape(M * K // 128, 128), fmt)
    assert (Xq.reshape(-1, 128) == q_ref).all()
    # MN-major scales: Xs[g, m]
    s_ref = s_ref.reshape(M, K // 128).T
    if fmt == F32:
        assert (Xs[:, :M].view(np.uint32) == s_ref.view(np.uint32)).all()
    else:
        assert (Xs[:, :M] == s_ref).all()
    assert (Xs[:, M:] == 0).all()


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_quant_weight_matches_torch_restatement(orc, fmt):
    N, K = 384, 256           # non-square block grid catches a transposed layout
    W = workloads.weights((N, K), seed=5)
    W[5, 200] = 0.75          # a distinct outlier in block (0, 1)
    Wq, Ws = orc.quant_weight(bf16_bits(W), fmt)
    blocks = W.reshape(N // 128, 128, K // 128, 128).permute(0, 2, 1, 3).reshape(-1, 128 * 128)
    # a block is one group of 16384 values for the amax; quantize it in one go
    xf = blocks.float()
    amax = xf.abs().amax(dim=1).clamp_min(1e-4)
    t = amax / torch.tensor(448.0)
    if fmt == F32:
        s, stored = t, t
    else:
        mant, ex = torch.frexp(t)
        p = torch.where(mant == 0.5, ex - 1, ex)
        s, stored = torch.ldexp(torch.ones_like(t), p), (p + 127).to(torch.uint8)
    q = (xf / s[:, None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    q = q.reshape(N // 128, K // 128, 128, 128).permute(0, 2, 1, 3).reshape(N, K)
    assert (Wq == q.numpy()).all()
    stored = stored.reshape(N // 128, K // 128).numpy()
    if fmt == F32:
        assert (Ws.view(np.uint32) == stored.view(np.uint32)).all()
    else:
        assert (Ws == stored).all()
    # the outlier's block has the largest scale in block row 0
    assert Ws[0, 1] > Ws[0, 0]


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_quant_dequant_error_bound(orc, fmt):
    """E4M3 keeps 3 mantissa bits: a normal code is within 2^-4 relative of
    x/s, a subnormal one within 2^-10 absolute (in units of s); the fp32
    quotient adds at most 2^-24 relative, covered by the (1 + 2^-20) slack."""
    X = workloads.activations((64, 2048), "normal_outliers", seed=3)
    Xq, Xs = orc.quant_act(bf16_bits(X), fmt)
    xhat = orc.dequant_act(Xq, Xs, fmt)
    x = X.double().numpy()
    per_group = Xs[:, :64].T.astype(np.float64)            # [M, K/128]
    if fmt == UE8M0:
        per_group = np.ldexp(1.0, Xs[:, :64].T.astype(np.int64) - 127)
    scale = np.repeat(per_group, 128, axis=1)
    r = np.abs(x) / scale
    err = np.abs(xhat - x)
    normal = r >= 2.0 ** -6
    assert (err[normal] <= 2.0 ** -4 * np.abs(x[normal]) * (1 + 2.0 ** -20)).all()
    assert (err[~normal] <= 2.0 ** -10 * scale[~normal] * (1 + 2.0 ** -20)).all()
    # the largest element of each group lands on the top binade
    g = np.abs(Xq.reshape(64, 16, 128).astype(np.int64) & 0x7F).max(axis=2)
    if fmt == F32:
        assert (g == 0x7E).all()
    else:
        assert (g >= 0x76).all()      # amax/s in (224, 448]


def test_ld_s_padding_and_stride(orc):
    X = workloads.activations((6, 256), "normal", seed=2)
    Xq_a, Xs_a = orc.quant_act(bf16_bits(X), F32)
    Xq_b, Xs_b = orc.quant_act(bf16_bits(X), F32, ld_s=20)
    assert Xs_a.shape == (2, 8) and Xs_b.shape == (2, 20)
    assert (Xq_a == Xq_b).all() and (Xs_a[:, :6] == Xs_b[:, :6]).all()
    assert (Xs_b[:, 6:] == 0).all()


def test_nonfinite_groups_have_nonfinite_scales(orc):
    X = torch.zeros((3, 128), dtype=torch.bfloat16)
    X[0, 4] = float("nan")
    X[1, 9] = float("inf")
    X[2, 0] = 1.0
    _, Xs = orc.quant_act(bf16_bits(X), F32)
    assert np.isnan(Xs[0, 0]) and np.isinf(Xs[0, 1]) and np.isfinite(Xs[0, 2])
    _, Xs = orc.quant_act(bf16_bits(X), UE8M0)
    assert Xs[0, 0] == 0xFF and Xs[0, 1] == 0xFF and Xs[0, 2] != 0xFF
