"""GPU checks of the gate/up projection fused with the down projection's
activation quantizer (fgfp8_gemm_swiglu_quant): h = SiLU(gate) * up of the
block-scaled gate/up GEMM, quantized per 1x128 group with fp32 scales.

The GEMM outputs are rounded in fp32 and bf16 on the GPU and exact in the
oracle, so h cannot match bit for bit; the checks are
  * against the oracle: every dequantized element within a bound derived from
    the GEMM tolerance (|d| <= 2^-7 |ref| + 1e-4 S on g and u), the Lipschitz
    constant of SiLU (<= 1.1), the bf16 rounding of h and E4M3's half step;
    every scale within the bound implied for the group's amax;
  * exactly: every group's largest code is 0x7E (the amax element maps to
    448), as for any activation group;
  * against the unfused GPU path (the same GEMM kernel writing bf16 gate/up
    outputs, SiLU * up and the 1x128 quantizer on the host in fp32 / bf16):
    codes equal except where h lands within one bf16 step of a rounding
    boundary, and those differ by one E4M3 step at most."""
import numpy as np
import pytest
import torch

import fine_grained_fp8_token_b200 as fg
import oracle
import workloads
from parity import bits16, require_gpu, to_np

pytestmark = pytest.mark.gpu
F32 = 0


@pytest.fixture(scope="module")
def dev():
    d = require_gpu()
    fg.load()
    return d


def build(dev, M, I, K, seed):
    X = workloads.activations((M, K), "normal_outliers", seed=seed)
    Wg = workloads.weights((I, K), seed=seed + 1)
    Wu = workloads.weights((I, K), seed=seed + 2)
    W_gu = fg.interleave_gate_up(Wg, Wu)
    Xq, Xs = fg.quant_act(X.to(dev), F32)
    Wq, Ws = fg.quant_weight(W_gu.to(dev), F32)
    return X, Wg, Wu, W_gu, Xq, Xs, Wq, Ws


def oracle_h(X, W_gu, I):
    Xq_r, Xs_r = oracle.quant_act(bits16(X), F32)
    Wq_r, Ws_r = oracle.quant_weight(bits16(W_gu), F32)
    Y, S = oracle.gemm(Xq_r, Xs_r, Wq_r, Ws_r, F32)
    M = Y.shape[0]
    Yb = Y.reshape(M, I // 128, 2, 128)
    Sb = S.reshape(M, I // 128, 2, 128)
    g, u = Yb[:, :, 0, :].reshape(M, I), Yb[:, :, 1, :].reshape(M, I)
    Sg, Su = Sb[:, :, 0, :].reshape(M, I), Sb[:, :, 1, :].reshape(M, I)
    return g, u, Sg, Su


def check_against_oracle(Hq, Hs, g, u, Sg, Su, M, I):
    dg = 2.0 ** -7 * np.abs(g) + 1e-4 * Sg
    du = 2.0 ** -7 * np.abs(u) + 1e-4 * Su
    h = oracle.silu_mul(g, u)
    silu_g = oracle.silu_mul(g, np.ones_like(g))
    dh = 1.1 * (1.1 * dg * (np.abs(u) + du) + np.abs(silu_g) * du + 2.0 ** -8 * np.abs(h))
    hs = np.asarray(Hs, dtype=np.float64)[:, :M].T                   # [M, I/128]
    scale = np.repeat(hs, 128, axis=1)
    deq = oracle.e4m3_decode(Hq) * scale
    tol = dh + 2.0 ** -4 * (np.abs(h) + dh) + 2.0 ** -10 * scale
    bad = np.abs(deq - h) > tol
    assert not bad.any(), f"{bad.sum()} elements outside the bound, first at {np.argwhere(bad)[0]}"
    # scales: amax of h within the group's largest element bound
    amax_ref = np.abs(h).reshape(M, I // 128, 128).max(axis=2)
    damax = dh.reshape(M, I // 128, 128).max(axis=2)
    s_ref = np.maximum(amax_ref, 1e-4) / 448.0
    assert (np.abs(hs - s_ref) <= damax / 448.0 + 2.0 ** -22 * s_ref).all()
    # the amax element of every group reaches the top code
    top = (Hq & 0x7F).reshape(M, I // 128, 128).max(axis=2)
    assert (top == 0x7E).all()


@pytest.mark.parametrize("M,I,K", [(128, 128, 512), (300, 512, 1024), (1, 256, 768), (700, 1280, 2048)])
def test_swiglu_quant_against_oracle(dev, M, I, K):
    X, Wg, Wu, W_gu, Xq, Xs, Wq, Ws = build(dev, M, I, K, seed=M + I + K)
    Hq, Hs = fg.gemm_swiglu_quant(Xq, Xs, Wq, Ws)
    fg.check_device_status()
    g, u, Sg, Su = oracle_h(X, W_gu, I)
    check_against_oracle(to_np(Hq), to_np(Hs), g, u, Sg, Su, M, I)


def test_swiglu_quant_full_mlp_sampled_rows(dev):
    """The Llama-3-8B MLP's gate/up projection at full size (8192 tokens,
    K = 4096, I = 14336, the inputs the MLP benchmark builds): every M tile's
    first and last row plus random rows against the oracle, with the same
    bounds as above."""
    c = workloads.LLAMA_GATE_UP
    M, K, I = 8192, 4096, 14336
    X = workloads.activations((M, K), c.x_kind, c.seed, device=dev)
    Wg = workloads.weights((I, K), c.seed + 1, device=dev)
    Wu = workloads.weights((I, K), c.seed + 2, device=dev)
    W_gu = fg.interleave_gate_up(Wg, Wu)
    del Wg, Wu
    Xq, Xs = fg.quant_act(X, F32)
    Wq, Ws = fg.quant_weight(W_gu, F32)
    Hq, Hs = fg.gemm_swiglu_quant(Xq, Xs, Wq, Ws)
    fg.check_device_status()
    rng = np.random.default_rng(1)
    tiles = np.arange(0, M, 128)
    rows = np.unique(np.concatenate([tiles[::4], tiles[::4] + 127, rng.integers(0, M, 8)]))
    idx = torch.as_tensor(rows, device=dev)
    g, u, Sg, Su = oracle_h(X[idx], W_gu, I)
    check_against_oracle(to_np(Hq[idx]), to_np(Hs[:, idx]), g, u, Sg, Su, len(rows), I)


def host_swiglu_quant(Y_gu: torch.Tensor, I: int):
    """The unfused path's last two steps on the host: SiLU(g) * u in fp32 from
    the bf16 GEMM output, rounded to bf16, then the 1x128 quantizer."""
    M = Y_gu.shape[0]
    Yb = Y_gu.float().cpu().reshape(M, I // 128, 2, 128)
    g = Yb[:, :, 0, :].reshape(M, I).numpy().astype(np.float32)
    u = Yb[:, :, 1, :].reshape(M, I).numpy().astype(np.float32)
    with np.errstate(over="ignore"):
        sig = (np.float32(1.0) / (np.float32(1.0) + np.exp(-g, dtype=np.float32))).astype(np.float32)
    h = ((g * sig).astype(np.float32) * u).astype(np.float32)
    hb = torch.from_numpy(h).to(torch.bfloat16)
    return oracle.quant_act(bits16(hb), F32)


@pytest.mark.parametrize("M,I,K", [(300, 512, 1024), (1024, 1024, 4096)])
def test_swiglu_quant_against_unfused_path(dev, M, I, K):
    X, Wg, Wu, W_gu, Xq, Xs, Wq, Ws = build(dev, M, I, K, seed=3 * M + I)
    Hq, Hs = fg.gemm_swiglu_quant(Xq, Xs, Wq, Ws)
    Y = fg.gemm(Xq, Xs, Wq, Ws, F32)                  # the same kernel, bf16 gate/up output
    fg.check_device_status()
    Hq_u, Hs_u = host_swiglu_quant(Y, I)
    a, b = to_np(Hq), Hq_u
    diff = a != b
    assert diff.mean() < 2e-3, f"{diff.mean():.2e} of the codes differ from the unfused path"
    if diff.any():
        da = (a[diff] & 0x7F).astype(int)
        db = (b[diff] & 0x7F).astype(int)
        assert (np.abs(da - db) <= 1).all() and ((a[diff] & 0x80) == (b[diff] & 0x80)).all()
    sa, sb = to_np(Hs)[:, :M], Hs_u[:, :M]
    rel = np.abs(sa.astype(np.float64) - sb) / sb
    assert (rel <= 2.0 ** -7).all()


def test_swiglu_quant_feeds_down_projection(dev):
    """The fused output is a valid input of the block-scaled GEMM: the down
    projection from Hq / Hs agrees with the down projection of the unfused
    path's quantized h within the GEMM tolerance of their difference."""
    M, I, K, N = 256, 512, 1024, 384
    X, Wg, Wu, W_gu, Xq, Xs, Wq, Ws = build(dev, M, I, K, seed=17)
    Hq, Hs = fg.gemm_swiglu_quant(Xq, Xs, Wq, Ws)
    Wd = workloads.weights((N, I), seed=19).to(dev)
    Wdq, Wds = fg.quant_weight(Wd, F32)
    Yd = fg.gemm(Hq, Hs, Wdq, Wds, F32)
    fg.check_device_status()
    Y_ref, S = oracle.gemm(to_np(Hq), to_np(Hs), to_np(Wdq), to_np(Wds), F32)
    assert oracle.gemm_within_tolerance(Yd.float().cpu().double().numpy(), Y_ref, S).all()
