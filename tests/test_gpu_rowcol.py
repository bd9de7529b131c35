"""GPU parity of the row / tensor scale granularity against the oracle: the
FP8_DYNAMIC scheme ("FP8 W8A8", "Applying quantization": per-output-channel
weights, per-token activations) and static per-tensor scales.

Codes and scales bit-exact; GEMM outputs within |gpu - ref| <= 2^-7 |ref| +
1e-4 sum_k |x_hat w_hat|.  The GPU path and the oracle quantize the same
seeded bf16 inputs each on their own; the oracle's GEMM inputs are its own
codes."""
import numpy as np
import pytest
import torch

import fine_grained_fp8_token_b200 as fg
import oracle
import workloads
from parity import assert_codes_equal, assert_gemm_close, assert_scales_equal, bits16, require_gpu, to_np, y_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    d = require_gpu()
    fg.load()
    return d


@pytest.mark.parametrize("R,K,kind", [(1, 128, "normal"), (7, 4096, "normal_outliers"), (33, 14336, "heavy_tail"),
                                      (130, 384, "normal"), (3, 20480, "normal_outliers"), (300, 1024, "heavy_tail")])
def test_quant_rows(dev, R, K, kind):
    X = workloads.activations((R, K), kind, seed=R + K)
    Xq, s = fg.quant_rows(X.to(dev))
    fg.check_device_status()
    Xq_r, s_r = oracle.quant_rows(bits16(X))
    assert_codes_equal(to_np(Xq), Xq_r, f"row codes {R}x{K}")
    assert_scales_equal(to_np(s), s_r, f"row scales {R}x{K}")


@pytest.mark.parametrize("K", [256, 8192])
def test_quant_rows_special_values(dev, K):
    """Degenerate rows (all zero, negative zero, ties, near the bf16 maximum,
    subnormals, below the amax floor) bit-exact, for both row kernels (one
    warp per row up to 4096 elements, one CTA per row above); rows holding
    NaN or Inf get a non-finite scale while the other rows stay exact."""
    z = torch.zeros(K)
    rows = [z.clone()]
    r = z.clone(); r[3] = -0.0; rows.append(r)
    r = z.clone(); r[0] = 448; r[1] = 17; r[2] = 19; r[K - 1] = 1.0625; r[K // 2] = -17; rows.append(r)
    r = z.clone(); r[0] = 3.3895e38; r[K - 2] = -1e38; r[2] = 1.0; rows.append(r)
    r = torch.full((K,), 9.1835e-41); r[5] = -9.1835e-41; rows.append(r)
    r = z.clone(); r[0] = 5e-5; r[K - 1] = -2.5e-5; rows.append(r)
    r = torch.linspace(-1, 1, K); rows.append(r)
    X = torch.stack(rows).to(torch.bfloat16)
    X = torch.cat([X, -X], dim=0)
    Xq, s = fg.quant_rows(X.to(dev))
    fg.check_device_status()
    Xq_r, s_r = oracle.quant_rows(bits16(X))
    assert_codes_equal(to_np(Xq), Xq_r, f"special rows K={K}")
    assert_scales_equal(to_np(s), s_r, f"special row scales K={K}")
    assert to_np(Xq)[1, 3] == 0x80
    Y = X.clone()
    Y[2, K - 1] = float("nan")
    Y[5, 0] = float("inf")
    Yq, sy = fg.quant_rows(Y.to(dev))
    sy = to_np(sy)
    assert not np.isfinite(sy[2]) and not np.isfinite(sy[5])
    ok = [i for i in range(Y.shape[0]) if i not in (2, 5)]
    assert_codes_equal(to_np(Yq)[ok], Xq_r[ok], "finite rows next to non-finite ones")
    assert_scales_equal(sy[ok], s_r[ok], "finite row scales")


def test_quant_rows_strided_input(dev):
    R, K, ldx = 20, 1024, 1536
    big = workloads.activations((R, ldx), "normal_outliers", seed=9).to(dev)
    X = big[:, :K]
    Xq, s = fg.quant_rows(X)
    Xq_r, s_r = oracle.quant_rows(bits16(X))
    assert_codes_equal(to_np(Xq), Xq_r, "strided row codes")
    assert_scales_equal(to_np(s), s_r, "strided row scales")


@pytest.mark.parametrize("R,K", [(1, 128), (64, 7168), (4096, 4096), (513, 640)])
def test_tensor_scale_and_static_quant(dev, R, K):
    X = workloads.activations((R, K), "normal_outliers", seed=3 * R + K)
    Xd = X.to(dev)
    s = fg.tensor_scale(Xd)
    Xq = fg.quant_static(Xd, s)
    fg.check_device_status()
    s_r = oracle.tensor_scale(bits16(X))
    assert to_np(s).view(np.uint32)[0] == np.float32(s_r).view(np.uint32), (float(s), float(s_r))
    assert_codes_equal(to_np(Xq), oracle.quant_static(bits16(X), s_r), f"static codes {R}x{K}")
    # a calibrated scale that is not the tensor's own: saturation and small codes
    for given in (np.float32(0.0031), np.float32(1.7e-5)):
        Xq2 = fg.quant_static(Xd, torch.tensor([given], device=dev))
        assert_codes_equal(to_np(Xq2), oracle.quant_static(bits16(X), given), f"static codes, scale {given}")


def all_bf16_rows(K=128):
    """Every finite bf16 value of both signs (65,280 of them, +-0 included),
    as rows of K elements: the full range a static quotient x / s can meet."""
    pos = np.arange(0, 0x7F80, dtype=np.uint16)
    bits = np.concatenate([pos, pos | np.uint16(0x8000)])
    rng = np.random.default_rng(11)
    rng.shuffle(bits)
    return torch.from_numpy(bits.view(np.int16).reshape(-1, K).copy()).view(torch.bfloat16)


F32_MAX = float(np.finfo(np.float32).max)
TINY_SUB = float(np.float32(2.0) ** -149)
STATIC_EDGE_SCALES = [0.5, 1.0, 1e-39, 2.0 ** -126, 2.0 ** -127, 2.9387359e-39, TINY_SUB, 2.0 ** -92,
                      float(np.nextafter(np.float32(2.0 ** -92), np.float32(0))), 2.0 ** 126,
                      float(np.nextafter(np.float32(2.0 ** 126), np.float32(np.inf))), 2.0 ** 127, F32_MAX,
                      float("inf"), 0.0031, 3.7e-12, 1.5e20]


@pytest.mark.parametrize("scale", STATIC_EDGE_SCALES, ids=lambda v: f"{v:.6g}")
def test_quant_static_every_bf16_value_at_edge_scales(dev, scale):
    """A caller-given static scale meets every finite bf16 value: the codes
    equal the oracle's E4M3(x / s) with the IEEE fp32 quotient bit for bit,
    also where x / s overflows fp32 (|x| near the bf16 maximum over s = 0.5
    saturates to 448, not NaN), for subnormal scales (1 / s overflows), at
    the ends of the kernel's FMA window and for s = +inf."""
    X = all_bf16_rows()
    s = np.float32(scale)
    Xq = fg.quant_static(X.to(dev), torch.tensor([s], dtype=torch.float32, device=dev))
    fg.check_device_status()
    assert_codes_equal(to_np(Xq), oracle.quant_static(bits16(X), s), f"static codes, scale {scale!r}")


def test_quant_static_overflowing_quotient_saturates(dev):
    """Rows holding +-3.0e38 and the bf16 maximum +-3.3895e38 over scale 0.5:
    the quotient overflows fp32 and the code saturates to 0x7E / 0xFE."""
    X = torch.zeros((2, 256), dtype=torch.bfloat16)
    X[0, 0], X[0, 1], X[0, 2], X[0, 3] = 3.0e38, -3.0e38, 3.3895e38, -3.3895e38
    X[1, 5], X[1, 6] = 1.0, -224.0
    Xq = to_np(fg.quant_static(X.to(dev), torch.tensor([0.5], dtype=torch.float32, device=dev)))
    fg.check_device_status()
    assert list(Xq[0, :4]) == [0x7E, 0xFE, 0x7E, 0xFE]
    assert_codes_equal(Xq, oracle.quant_static(bits16(X), np.float32(0.5)), "overflowing quotients")


@pytest.mark.parametrize("bad", [0.0, -0.0, -1.0, float("nan"), -float("inf")])
def test_quant_static_rejects_non_positive_scale(dev, bad):
    """A scale <= 0 or NaN is reported through the device status word and
    no code is written."""
    X = workloads.activations((4, 256), "normal", seed=5).to(dev)
    Xq = torch.full((4, 256), 0x5A, dtype=torch.uint8, device=dev)
    fg.quant_static(X, torch.tensor([bad], dtype=torch.float32, device=dev), Xq=Xq)
    with pytest.raises(fg.FGFP8Error) as e:
        fg.check_device_status()
    assert e.value.status == 7                     # FGFP8_ERR_DEVICE
    assert bool((Xq == 0x5A).all())
    fg.check_device_status()                      # the word was cleared


def test_tensor_scale_zero_and_nan(dev):
    Z = torch.zeros((3, 256), dtype=torch.bfloat16, device=dev)
    assert float(fg.tensor_scale(Z)) == float(np.float32(1e-4) / np.float32(448.0))
    X = torch.ones((5, 256), dtype=torch.bfloat16, device=dev)
    X[4, 17] = float("nan")
    assert torch.isnan(fg.tensor_scale(X)).all()


def make_operands(dev, M, N, K, x_tensor, w_tensor, seed):
    X = workloads.activations((M, K), "normal_outliers", seed=seed)
    W = workloads.weights((N, K), seed=seed + 1)
    Xd, Wd = X.to(dev), W.to(dev)
    if x_tensor:
        sx = fg.tensor_scale(Xd)
        Xq = fg.quant_static(Xd, sx)
        sx_r = np.array([oracle.tensor_scale(bits16(X))], dtype=np.float32)
        Xq_r = oracle.quant_static(bits16(X), sx_r[0])
    else:
        Xq, sx = fg.quant_rows(Xd)
        Xq_r, sx_r = oracle.quant_rows(bits16(X))
    if w_tensor:
        sw = fg.tensor_scale(Wd)
        Wq = fg.quant_static(Wd, sw)
        sw_r = np.array([oracle.tensor_scale(bits16(W))], dtype=np.float32)
        Wq_r = oracle.quant_static(bits16(W), sw_r[0])
    else:
        Wq, sw = fg.quant_rows(Wd)
        Wq_r, sw_r = oracle.quant_rows(bits16(W))
    return (Xq, sx, Wq, sw), (Xq_r, sx_r, Wq_r, sw_r)


@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (300, 640, 2048), (1, 1280, 7168), (513, 384, 1024),
                                   (64, 2304, 4096), (1200, 4096, 256)])
@pytest.mark.parametrize("x_tensor,w_tensor", [(0, 0), (1, 0), (0, 1), (1, 1)])
def test_gemm_rowcol(dev, M, N, K, x_tensor, w_tensor):
    (Xq, sx, Wq, sw), (Xq_r, sx_r, Wq_r, sw_r) = make_operands(dev, M, N, K, x_tensor, w_tensor, seed=M + 7 * N + K)
    Y = fg.gemm_rowcol(Xq, sx, Wq, sw)
    fg.check_device_status()
    Y_ref, S = oracle.gemm_rowcol(Xq_r, sx_r, Wq_r, sw_r)
    assert_gemm_close(y_to_f64(Y), Y_ref, S, f"rowcol {M}x{N}x{K} x_tensor={x_tensor} w_tensor={w_tensor}")


@pytest.mark.parametrize("cfg", [workloads.LLAMA_ATTN, workloads.LLAMA_GATE_UP, workloads.LLAMA_DOWN],
                         ids=lambda c: c.name)
def test_gemm_rowcol_full_size_sampled_rows(dev, cfg):
    """The Llama-3-8B shapes the benchmark times in the FP8_DYNAMIC scheme:
    M tiles' first and last rows plus random rows against the oracle (every
    tile for the attention projection, every fourth for the larger ones)."""
    X = workloads.activations((cfg.M, cfg.K), cfg.x_kind, cfg.seed, device=dev)
    W = workloads.weights((cfg.N, cfg.K), cfg.seed + 1, device=dev)
    Xq, sx = fg.quant_rows(X)
    Wq, sw = fg.quant_rows(W)
    Y = fg.gemm_rowcol(Xq, sx, Wq, sw)
    fg.check_device_status()
    rng = np.random.default_rng(0)
    tiles = np.arange(0, cfg.M, 128)
    if cfg.M * cfg.N > 4096 * 4096:
        tiles = tiles[::4]
    rows = np.unique(np.concatenate([tiles, tiles + 127, rng.integers(0, cfg.M, 16)]))
    Xq_r, sx_r = oracle.quant_rows(bits16(X[torch.as_tensor(rows, device=dev)]))
    Wq_r, sw_r = oracle.quant_rows(bits16(W))
    Y_ref, S = oracle.gemm_rowcol(Xq_r, sx_r, Wq_r, sw_r)
    assert_gemm_close(y_to_f64(Y[torch.as_tensor(rows, device=dev)]), Y_ref, S, f"FP8_DYNAMIC {cfg.name}")


def test_gemm_rowcol_static_activation_scale_full_size(dev):
    """The attention projection with a static per-tensor activation scale
    (the benchmark's static workload: the scale calibrated on the layer's
    input, then the static quantizer) x per-channel weights, sampled rows."""
    cfg = workloads.LLAMA_ATTN
    X = workloads.activations((cfg.M, cfg.K), cfg.x_kind, cfg.seed, device=dev)
    W = workloads.weights((cfg.N, cfg.K), cfg.seed + 1, device=dev)
    sx = fg.tensor_scale(X)
    Xq = fg.quant_static(X, sx)
    Wq, sw = fg.quant_rows(W)
    Y = fg.gemm_rowcol(Xq, sx, Wq, sw)
    fg.check_device_status()
    rng = np.random.default_rng(2)
    tiles = np.arange(0, cfg.M, 128)
    rows = np.unique(np.concatenate([tiles[::2], tiles[1::2] + 127, rng.integers(0, cfg.M, 16)]))
    Xb = bits16(X)
    sx_r = np.array([oracle.tensor_scale(Xb)], dtype=np.float32)
    assert to_np(sx).view(np.uint32)[0] == sx_r.view(np.uint32)[0]
    Xq_r = oracle.quant_static(Xb[rows], sx_r[0])
    Wq_r, sw_r = oracle.quant_rows(bits16(W))
    Y_ref, S = oracle.gemm_rowcol(Xq_r, sx_r, Wq_r, sw_r)
    assert_gemm_close(y_to_f64(Y[torch.as_tensor(rows, device=dev)]), Y_ref, S, "static per-tensor 4096^3")


def test_gemm_rowcol_empty_and_repeatable(dev):
    (Xq, sx, Wq, sw), _ = make_operands(dev, 200, 512, 1024, 0, 0, seed=1)
    Y1 = fg.gemm_rowcol(Xq, sx, Wq, sw)
    Y2 = fg.gemm_rowcol(Xq, sx, Wq, sw)
    assert torch.equal(Y1, Y2)
    Y0 = fg.gemm_rowcol(Xq[:0], sx[:0], Wq, sw)
    assert Y0.shape == (0, 512)
