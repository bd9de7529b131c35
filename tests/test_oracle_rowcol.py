"""Pins for the oracle's row- and tensor-granularity scales and the
row/column-scaled GEMM (CPU only): the FP8_DYNAMIC scheme of the "FP8 W8A8"
page ("Applying quantization": per-channel weights, per-token activations)
and per-tensor AbsMax scales (static activation scales).

Pinned by: the special case K = 128, where a row is one 1x128 group and the
row quantizer must reproduce the (separately pinned) group quantizer; numpy's
IEEE fp32 division for the scales; torch's float8_e4m3fn conversion for the
codes; the quantize/dequantize error bound; an fp64 brute-force GEMM of the
dequantized operands; the special case where per-channel scales are uniform
over 128-channel blocks and K = 128, which must equal the block-scaled GEMM;
and an all-ones product that must equal K exactly.
"""
import numpy as np
import pytest
import torch

import workloads

F32 = 0


def bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def inputs(R, K, seed, kind="normal_outliers"):
    return workloads.activations((R, K), kind, seed)


def numpy_scale(x_rows: np.ndarray) -> np.ndarray:
    """max(amax, 1e-4) / 448 per row, fp32 division by numpy."""
    a = np.abs(x_rows.astype(np.float32)).max(axis=1)
    a = np.maximum(a, np.float32(1e-4)).astype(np.float32)
    return (a / np.float32(448.0)).astype(np.float32)


def torch_codes(x: np.ndarray, s) -> np.ndarray:
    """E4M3 codes of x / s (fp32 quotient), clamped to +-448, through torch's conversion."""
    q = torch.from_numpy((x.astype(np.float32) / np.asarray(s, dtype=np.float32)).astype(np.float32))
    return q.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@pytest.mark.parametrize("R", [1, 7, 64])
def test_quant_rows_equals_group_quantizer_at_k128(orc, R):
    X = inputs(R, 128, seed=R)
    q_rows, s_rows = orc.quant_rows(bits(X))
    q_grp, s_grp = orc.quant_act(bits(X), F32)
    assert np.array_equal(q_rows, q_grp)
    assert np.array_equal(s_rows.view(np.uint32), s_grp[0, :R].view(np.uint32))


@pytest.mark.parametrize("R,K,kind", [(33, 4096, "normal_outliers"), (5, 14336, "heavy_tail"),
                                      (16, 384, "normal")])
def test_quant_rows_against_numpy_and_torch(orc, R, K, kind):
    X = inputs(R, K, seed=K + R, kind=kind)
    xf = X.float().numpy()
    q, s = orc.quant_rows(bits(X))
    s_ref = numpy_scale(xf)
    assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q, torch_codes(xf, s_ref[:, None]))


def test_quant_rows_error_bound(orc):
    X = inputs(12, 2048, seed=3)
    x = X.float().numpy().astype(np.float64)
    q, s = orc.quant_rows(bits(X))
    xh = orc.e4m3_decode(q) * s[:, None].astype(np.float64)
    r = np.abs(x) / s[:, None]
    big = r >= 2.0 ** -6
    err = np.abs(xh - x)
    assert (err[big] <= 2.0 ** -4 * np.abs(x[big]) * (1 + 2.0 ** -20)).all()
    sb = np.broadcast_to(s[:, None].astype(np.float64), x.shape)
    assert (err[~big] <= 2.0 ** -10 * sb[~big] * (1 + 2.0 ** -20)).all()
    # each row's largest element reaches the top codes
    top = (q & 0x7F).max(axis=1)
    assert (top >= 0x7D).all()


def test_tensor_scale_and_static_codes(orc):
    X = inputs(40, 1024, seed=11)
    xf = X.float().numpy()
    s = orc.tensor_scale(bits(X))
    s_ref = numpy_scale(xf.reshape(1, -1))[0]
    assert np.float32(s).view(np.uint32) == s_ref.view(np.uint32)
    q = orc.quant_static(bits(X), s)
    assert np.array_equal(q, torch_codes(xf, s_ref))
    # a given (calibrated) scale other than the tensor's own
    q2 = orc.quant_static(bits(X), np.float32(0.0031))
    assert np.array_equal(q2, torch_codes(xf, np.float32(0.0031)))
    # all-zero tensor: the 1e-4 floor
    Z = torch.zeros((3, 256), dtype=torch.bfloat16)
    assert np.float32(orc.tensor_scale(bits(Z))) == np.float32(1e-4) / np.float32(448.0)


def test_static_equals_rows_for_one_row(orc):
    X = inputs(1, 512, seed=5)
    q_rows, s_rows = orc.quant_rows(bits(X))
    assert np.array_equal(orc.quant_static(bits(X), s_rows[0]), q_rows)


def brute_force(orc, Xq, sx, Wq, sw):
    xh = orc.e4m3_decode(Xq) * np.asarray(sx, dtype=np.float64).reshape(-1, 1)
    wh = orc.e4m3_decode(Wq) * np.asarray(sw, dtype=np.float64).reshape(-1, 1)
    return xh @ wh.T, np.abs(xh) @ np.abs(wh).T


@pytest.mark.parametrize("M,N,K", [(8, 128, 128), (33, 256, 640), (130, 384, 1024)])
@pytest.mark.parametrize("x_tensor,w_tensor", [(0, 0), (1, 0), (0, 1), (1, 1)])
def test_gemm_rowcol_brute_force(orc, M, N, K, x_tensor, w_tensor):
    X = inputs(M, K, seed=M + K)
    W = workloads.weights((N, K), seed=N + K)
    if x_tensor:
        sx = np.array([orc.tensor_scale(bits(X))], dtype=np.float32)
        Xq = orc.quant_static(bits(X), sx[0])
    else:
        Xq, sx = orc.quant_rows(bits(X))
    if w_tensor:
        sw = np.array([orc.tensor_scale(bits(W))], dtype=np.float32)
        Wq = orc.quant_static(bits(W), sw[0])
    else:
        Wq, sw = orc.quant_rows(bits(W))
    Y, S = orc.gemm_rowcol(Xq, sx, Wq, sw)
    sxb = np.broadcast_to(sx, (M,)) if sx.size == 1 else sx
    swb = np.broadcast_to(sw, (N,)) if sw.size == 1 else sw
    Yb, Sb = brute_force(orc, Xq, sxb, Wq, swb)
    assert np.allclose(Y, Yb, rtol=1e-12, atol=1e-12 * np.abs(Sb).max())
    assert np.allclose(S, Sb, rtol=1e-12)
    rows = np.array([0, M - 1, M // 2])
    Yr, Sr = orc.gemm_rowcol(Xq, sx, Wq, sw, rows=rows)
    assert np.array_equal(Yr, Y[rows]) and np.array_equal(Sr, S[rows])


def test_gemm_rowcol_equals_block_gemm_when_scales_agree(orc):
    """K = 128 and per-channel scales constant over each 128-channel block:
    the row/column-scaled GEMM and the block-scaled GEMM compute the same
    sum."""
    M, N, K = 40, 256, 128
    rng = np.random.default_rng(1)
    Xq = rng.integers(0, 0x7E, size=(M, K), dtype=np.uint8) | (rng.integers(0, 2, size=(M, K)) * 0x80).astype(np.uint8)
    Wq = rng.integers(0, 0x7E, size=(N, K), dtype=np.uint8)
    sx = rng.uniform(0.01, 0.1, size=M).astype(np.float32)
    sw_blk = np.array([0.003, 0.0005], dtype=np.float32)
    sw = np.repeat(sw_blk, 128)
    Y, S = orc.gemm_rowcol(Xq, sx, Wq, sw)
    ld_s = 40
    Xs = sx.reshape(1, ld_s).copy()
    Ws = sw_blk.reshape(2, 1).copy()
    Yb, Sb = orc.gemm(Xq, Xs, Wq, Ws, F32)
    assert np.allclose(Y, Yb, rtol=1e-15, atol=0) and np.allclose(S, Sb, rtol=1e-15)


def test_gemm_rowcol_all_ones():
    import oracle as orc
    M, N, K = 4, 128, 2048
    Xq = np.full((M, K), 0x38, dtype=np.uint8)      # E4M3 1.0
    Wq = np.full((N, K), 0x38, dtype=np.uint8)
    Y, S = orc.gemm_rowcol(Xq, np.ones(1, np.float32), Wq, np.ones(1, np.float32))
    assert (Y == K).all() and (S == K).all()
    Wq[:, ::2] = 0xB8                               # -1.0 on even k: the sum cancels
    Y, S = orc.gemm_rowcol(Xq, np.ones(M, np.float32), Wq, np.full(N, 2.0, np.float32))
    assert (Y == 0).all() and (S == 2 * K).all()


def test_silu_mul_against_torch_and_limits():
    """SiLU(g) * u against torch's silu in float64 (a library routine), and the
    closed forms SiLU(0) = 0, SiLU(g) -> g for large g, SiLU(g) -> 0 for very
    negative g."""
    import oracle as orc
    rng = np.random.default_rng(2)
    g = np.concatenate([rng.normal(0, 3, 5000), [0.0, 40.0, -40.0, 1e-8, -1e-8, 700.0, -745.0]])
    u = rng.normal(0, 1, g.size)
    h = orc.silu_mul(g, u)
    ref = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    assert np.allclose(h, ref, rtol=1e-15, atol=0)
    assert orc.silu_mul(0.0, 5.0) == 0.0
    assert abs(orc.silu_mul(40.0, 1.0) - 40.0) < 1e-15 * 40
    assert abs(orc.silu_mul(-745.0, 1.0)) < 1e-300
