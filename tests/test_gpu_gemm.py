"""GPU parity of the block-scaled GEMM and the M-grouped GEMM against the
oracle: every output within |gpu - ref| <= 2^-7 |ref| + 1e-4 sum_k |x_hat w_hat|.

The GPU path and the oracle each quantize the same seeded bf16 inputs on
their own (their codes are bit-identical, checked in test_gpu_quant.py), then
multiply; no oracle input comes from the GPU."""
import numpy as np
import pytest
import torch

import fine_grained_fp8_token_b200 as fg
import oracle
import workloads
from parity import F32, UE8M0, Guarded, assert_gemm_close, bits16, require_gpu, to_np, y_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    d = require_gpu()
    fg.load()
    return d


def gpu_linear(X_dev, W_dev, fmt):
    """Quantizer, weight quantizer and GEMM, every output inside canary bytes."""
    M, K = X_dev.shape
    N = W_dev.shape[0]
    sdt = torch.float32 if fmt == F32 else torch.uint8
    gXq = Guarded((M, K), torch.uint8, X_dev.device)
    gXs = Guarded((K // 128, fg.scale_rows(M, fmt)), sdt, X_dev.device, fill=0)
    gY = Guarded((M, N), torch.bfloat16, X_dev.device)
    Xq, Xs = fg.quant_act(X_dev, fmt, Xq=gXq.t, Xs=gXs.t)
    Wq, Ws = fg.quant_weight(W_dev, fmt)
    Y = fg.gemm(Xq, Xs, Wq, Ws, fmt, Y=gY.t)
    fg.check_device_status()
    gXq.check("Xq")
    gXs.check("Xs")
    gY.check("Y")
    return Y


def oracle_linear(X_bits, W_bits, fmt, rows=None):
    Wq, Ws = oracle.quant_weight(W_bits, fmt)
    if rows is not None:
        X_bits = X_bits[rows]
    Xq, Xs = oracle.quant_act(X_bits, fmt)
    return oracle.gemm(Xq, Xs, Wq, Ws, fmt)


SMALL = [(128, 256, 512), (1, 128, 128), (7, 256, 384), (129, 384, 1024), (300, 640, 2048),
         (513, 512, 4096), (64, 1280, 7168), (256, 2304, 256), (17, 128, 14336)]


@pytest.mark.parametrize("fmt", [F32, UE8M0])
@pytest.mark.parametrize("M,N,K", SMALL)
def test_gemm_small(dev, fmt, M, N, K):
    cfg = workloads.scaled_linear(workloads.TINY, M=M, N=N, K=K, seed=M + 3 * N + 7 * K)
    X, W = workloads.linear_inputs(cfg)
    Y = gpu_linear(X.to(dev), W.to(dev), fmt)
    Y_ref, S = oracle_linear(bits16(X), bits16(W), fmt)
    assert_gemm_close(y_to_f64(Y), Y_ref, S, f"gemm {M}x{N}x{K}")


def test_gemm_tiny_config_exact_shape(dev):
    """The tiny parity configuration, every output element."""
    cfg = workloads.TINY
    X, W = workloads.linear_inputs(cfg)
    Y = gpu_linear(X.to(dev), W.to(dev), cfg.fmt)
    Y_ref, S = oracle_linear(bits16(X), bits16(W), cfg.fmt)
    assert_gemm_close(y_to_f64(Y), Y_ref, S, cfg.name)


def test_gemm_repeatable(dev):
    cfg = workloads.scaled_linear(workloads.TINY, M=300, N=512, K=1024)
    X, W = workloads.linear_inputs(cfg)
    Y1 = gpu_linear(X.to(dev), W.to(dev), F32)
    Y2 = gpu_linear(X.to(dev), W.to(dev), F32)
    assert torch.equal(Y1, Y2)


def test_gemm_zero_and_unit_codes(dev):
    """All codes 1.0 with unit scales gives K exactly; zero codes give 0."""
    M, N, K = 130, 256, 1024
    Xq = torch.full((M, K), 0x38, dtype=torch.uint8, device=dev)
    Wq = torch.full((N, K), 0x38, dtype=torch.uint8, device=dev)
    Xs = torch.ones((K // 128, fg.scale_rows(M, F32)), dtype=torch.float32, device=dev)
    Ws = torch.ones((N // 128, K // 128), dtype=torch.float32, device=dev)
    Y = fg.gemm(Xq, Xs, Wq, Ws, F32)
    assert (Y.float() == K).all()
    Y = fg.gemm(torch.zeros_like(Xq), Xs, Wq, Ws, F32)
    assert (Y.float() == 0).all()


@pytest.mark.parametrize("fmt", [F32, UE8M0])
@pytest.mark.parametrize("M,N,K", [(1200, 4096, 256), (2560, 2304, 384), (1200, 4096, 1152)])
def test_gemm_half_tile_tail(dev, M, N, K, fmt):
    """Shapes whose last partial wave of 128x256 tiles runs as 128x128 half
    tiles on a 148-SM B200 (1200x4096: 160 tiles = 148 + 12, ragged last
    M tile; 2560x2304: 180 tiles = 148 + 32), in both scale formats (the
    UE8M0 kernel's scale groups of four K blocks: K = 1152 ends in a group
    of one): every output against the oracle."""
    cfg = workloads.scaled_linear(workloads.TINY, M=M, N=N, K=K, seed=M + N + K)
    X, W = workloads.linear_inputs(cfg)
    Y = gpu_linear(X.to(dev), W.to(dev), fmt)
    Y_ref, S = oracle_linear(bits16(X), bits16(W), fmt)
    assert_gemm_close(y_to_f64(Y), Y_ref, S, f"half-tile tail {M}x{N}x{K} fmt {fmt}")


def sample_rows(M, n_random=48, seed=0):
    rng = np.random.default_rng(seed)
    tiles = np.arange(0, M, 128)
    rows = np.concatenate([tiles, np.minimum(tiles + 127, M - 1), rng.integers(0, M, n_random)])
    return np.unique(rows)


@pytest.mark.parametrize("cfg", [workloads.LLAMA_ATTN, workloads.LLAMA_GATE_UP, workloads.LLAMA_DOWN,
                                 *workloads.LLAMA_UE8M0.values()], ids=lambda c: c.name)
def test_gemm_full_size_sampled_rows(dev, cfg):
    """The full-size dense shapes the benchmark times: the first and last row
    of every 128-row M tile plus random rows, every output column, against
    the oracle."""
    X = workloads.activations((cfg.M, cfg.K), cfg.x_kind, cfg.seed, device=dev)
    W = workloads.weights((cfg.N, cfg.K), cfg.seed + 1, device=dev)
    Y = gpu_linear(X, W, cfg.fmt)
    rows = sample_rows(cfg.M, n_random=16 if cfg.N > 8192 else 48)
    tiles = np.arange(0, cfg.M, 128)
    assert np.isin(tiles, rows).all() and np.isin(np.minimum(tiles + 127, cfg.M - 1), rows).all()
    Y_ref, S = oracle_linear(bits16(X), bits16(W), cfg.fmt, rows=rows)
    assert_gemm_close(y_to_f64(Y[torch.as_tensor(rows, device=dev)]), Y_ref, S, cfg.name)


@pytest.mark.parametrize("m", [1, 8, 32, 64])
def test_gemm_decode_ue8m0(dev, m):
    cfg = workloads.DS_DECODE[m]
    X = workloads.activations((cfg.M, cfg.K), cfg.x_kind, cfg.seed, device=dev)
    W = workloads.weights((cfg.N, cfg.K), cfg.seed + 1, device=dev)
    Y = gpu_linear(X, W, cfg.fmt)
    rows = np.arange(cfg.M) if cfg.M <= 8 else np.unique(np.r_[0, cfg.M - 1, np.arange(1, cfg.M, 5)])
    Y_ref, S = oracle_linear(bits16(X), bits16(W), cfg.fmt, rows=rows)
    assert_gemm_close(y_to_f64(Y[torch.as_tensor(rows, device=dev)]), Y_ref, S, cfg.name)


# ---------------------------------------------------------------- grouped
def build_moe(cfg, dev):
    r = workloads.moe_routing(cfg)
    X = workloads.moe_grouped_rows(workloads.moe_tokens(cfg, device=dev), r)
    Wq = torch.empty((cfg.E, cfg.N, cfg.K), dtype=torch.uint8, device=dev)
    Ws = torch.empty((cfg.E, cfg.N // 128, cfg.K // 128), dtype=torch.float32 if cfg.fmt == F32 else torch.uint8,
                     device=dev)
    for e in range(cfg.E):
        fg.quant_weight(workloads.moe_expert_weight(cfg, e, device=dev), cfg.fmt, Wq=Wq[e], Ws=Ws[e])
    Xq, Xs = fg.quant_act(X, cfg.fmt)
    offs = torch.as_tensor(r.group_offs, device=dev)
    Y = fg.grouped_gemm(Xq, Xs, Wq, Ws, offs, cfg.fmt)
    fg.check_device_status()
    return r, X, Y


def oracle_moe_rows(cfg, r, X, rows, dev):
    Y_ref = np.empty((len(rows), cfg.N))
    S = np.empty((len(rows), cfg.N))
    expert_of = np.searchsorted(r.group_offs, rows, side="right") - 1
    X_rows = bits16(X[torch.as_tensor(rows, device=dev)])
    for e in np.unique(expert_of):
        sel = np.where(expert_of == e)[0]
        W = workloads.moe_expert_weight(cfg, int(e), device=dev)
        y, s = oracle_linear(X_rows, bits16(W), cfg.fmt, rows=sel)
        Y_ref[sel], S[sel] = y, s
    return Y_ref, S


@pytest.mark.parametrize("fmt", [UE8M0, F32])
def test_grouped_gemm_small(dev, fmt):
    cfg = workloads.scaled_moe(workloads.MOE, E=9, N=256, K=512, tokens=300, topk=3, fmt=fmt)
    r, X, Y = build_moe(cfg, dev)
    valid = np.where(r.row_token >= 0)[0]
    Y_ref, S = oracle_moe_rows(cfg, r, X, valid, dev)
    assert_gemm_close(y_to_f64(Y[torch.as_tensor(valid, device=dev)]), Y_ref, S, "grouped small")
    pad = torch.as_tensor(np.where(r.row_token < 0)[0], device=dev)
    assert (Y[pad].float() == 0).all()


@pytest.mark.parametrize("fmt", [UE8M0, F32])
def test_grouped_gemm_every_row_mixed_experts(dev, fmt):
    """Zipf-routed experts with many row tiles and experts with one (the
    UE8M0 kernel interleaves the two kinds of row tiles in its schedule):
    every token row against the oracle, every padding row zero."""
    cfg = workloads.scaled_moe(workloads.MOE, E=48, N=256, K=512, tokens=1024, topk=6, fmt=fmt)
    r, X, Y = build_moe(cfg, dev)
    tiles = np.diff(r.group_offs) // 128
    assert (tiles >= 2).any() and (tiles == 1).any()
    valid = np.where(r.row_token >= 0)[0]
    Y_ref, S = oracle_moe_rows(cfg, r, X, valid, dev)
    assert_gemm_close(y_to_f64(Y[torch.as_tensor(valid, device=dev)]), Y_ref, S, "grouped mixed experts")
    pad = torch.as_tensor(np.where(r.row_token < 0)[0], device=dev)
    assert (Y[pad].float() == 0).all()


def test_grouped_gemm_empty_experts(dev):
    """Experts with no rows (zero-length segments) are skipped."""
    cfg = workloads.scaled_moe(workloads.MOE, E=40, N=128, K=256, tokens=20, topk=1, zipf=3.0)
    r, X, Y = build_moe(cfg, dev)
    assert (r.counts == 0).any()
    valid = np.where(r.row_token >= 0)[0]
    Y_ref, S = oracle_moe_rows(cfg, r, X, valid, dev)
    assert_gemm_close(y_to_f64(Y[torch.as_tensor(valid, device=dev)]), Y_ref, S, "grouped empty experts")


@pytest.mark.parametrize("cfg", [workloads.MOE, workloads.MOE_F32], ids=lambda c: c.name)
def test_grouped_gemm_full_moe_every_expert(dev, cfg):
    """The full 256-expert layer the benchmark times (4096 tokens top-8,
    Zipf-routed, 128-row padding), in both scale formats: the first and the
    last token row of every expert segment, plus a middle row of the three
    busiest experts, against the oracle with that expert's weights; every
    padding row zero."""
    r, X, Y = build_moe(cfg, dev)
    starts = r.group_offs[:-1]
    rows = []
    for e in range(cfg.E):
        lo, n = int(starts[e]), int(r.counts[e])
        if n:
            rows += [lo, lo + n - 1]
    for e in np.argsort(-r.counts)[:3]:
        rows.append(int(starts[e]) + int(r.counts[e]) // 2)
    rows = np.unique(np.array(rows))
    assert len(rows) >= 2 * int((r.counts > 0).sum())
    Y_ref, S = oracle_moe_rows(cfg, r, X, rows, dev)
    assert_gemm_close(y_to_f64(Y[torch.as_tensor(rows, device=dev)]), Y_ref, S, cfg.name)
    pad = torch.as_tensor(np.where(r.row_token < 0)[0], device=dev)
    assert (Y[pad].float() == 0).all()


def test_grouped_gemm_bad_offsets_reported(dev):
    """Offsets that do not cover the rows are rejected on the device: the
    affected tiles stay unwritten and the status reads FGFP8_ERR_DEVICE."""
    E, N, K, M = 2, 128, 256, 256
    Xq = torch.zeros((M, K), dtype=torch.uint8, device=dev)
    Xs = torch.ones((K // 128, M), dtype=torch.uint8, device=dev) * 127
    Wq = torch.zeros((E, N, K), dtype=torch.uint8, device=dev)
    Ws = torch.full((E, 1, K // 128), 127, dtype=torch.uint8, device=dev)
    offs = torch.tensor([0, 128, 128], dtype=torch.int32, device=dev)     # row block 1 uncovered
    Y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device=dev)
    fg.grouped_gemm(Xq, Xs, Wq, Ws, offs, UE8M0, Y=Y)
    with pytest.raises(fg.FGFP8Error) as ei:
        fg.check_device_status()
    assert ei.value.status == 7
    assert (Y[:128].float() == 0).all() and (Y[128:].float() == 7).all()
    fg.check_device_status()       # the status word was cleared


# ---------------------------------------------------------------- one-call linear layer
LINEAR_CASES = [(300, 640, 2048, F32), (513, 512, 4096, UE8M0), (1, 1280, 7168, UE8M0), (64, 256, 1024, F32),
                (33, 384, 512, F32), (4096, 4096, 4096, F32)]


@pytest.mark.parametrize("M,N,K,fmt", LINEAR_CASES)
def test_linear_equals_quant_then_gemm(dev, M, N, K, fmt):
    """fgfp8_linear (quantizer + GEMM launched as its programmatic dependent,
    weight tiles requested early) gives bit-for-bit the codes, scales and
    output of the two separate calls."""
    cfg = workloads.scaled_linear(workloads.TINY, M=M, N=N, K=K, seed=11 * M + N)
    X, W = workloads.linear_inputs(cfg, device=dev)
    Wq, Ws = fg.quant_weight(W, fmt)
    Xq1, Xs1 = fg.quant_act(X, fmt)
    Y1 = fg.gemm(Xq1, Xs1, Wq, Ws, fmt)
    Xq2 = torch.empty_like(Xq1)
    Xs2 = torch.empty_like(Xs1)
    Y2 = fg.linear(X, Wq, Ws, fmt, Xq=Xq2, Xs=Xs2)
    fg.check_device_status()
    assert torch.equal(Xq1, Xq2)
    assert torch.equal(Xs1[:, :M].contiguous().view(torch.uint8), Xs2[:, :M].contiguous().view(torch.uint8))
    assert torch.equal(Y1, Y2)


@pytest.mark.parametrize("M,N,K,fmt", [(129, 384, 1024, F32), (7, 256, 384, UE8M0)])
def test_linear_oracle_parity(dev, M, N, K, fmt):
    cfg = workloads.scaled_linear(workloads.TINY, M=M, N=N, K=K, seed=5 * M + K)
    X, W = workloads.linear_inputs(cfg)
    Wq, Ws = fg.quant_weight(W.to(dev), fmt)
    Y = fg.linear(X.to(dev), Wq, Ws, fmt)
    fg.check_device_status()
    Y_ref, S = oracle_linear(bits16(X), bits16(W), fmt)
    assert_gemm_close(y_to_f64(Y), Y_ref, S, f"linear {M}x{N}x{K}")


@pytest.mark.parametrize("M", [2, 300])
def test_linear_back_to_back_weight_updates(dev, M):
    """Weights re-quantized between layer calls on the same stream, with no
    host synchronisation: every call sees the weights written just before it
    (the early weight loads never overtake the preceding fgfp8_quant_weight)."""
    N, K = 512, 1024
    g = torch.Generator(device=dev).manual_seed(3)
    X = (torch.randn((M, K), generator=g, device=dev)).to(torch.bfloat16)
    Ws_list = [(torch.randn((N, K), generator=g, device=dev) * 0.02).to(torch.bfloat16) for _ in range(6)]
    Wq = torch.empty((N, K), dtype=torch.uint8, device=dev)
    Wsc = torch.empty((N // 128, K // 128), dtype=torch.float32, device=dev)
    outs = []
    for W in Ws_list:
        fg.quant_weight(W, F32, Wq=Wq, Ws=Wsc)
        outs.append(fg.linear(X, Wq, Wsc, F32))
    fg.check_device_status()
    for W, Y in zip(Ws_list, outs):
        Wq_i, Ws_i = fg.quant_weight(W, F32)
        Xq, Xs = fg.quant_act(X, F32)
        assert torch.equal(Y, fg.gemm(Xq, Xs, Wq_i, Ws_i, F32))


@pytest.mark.parametrize("fmt", [UE8M0, F32])
def test_grouped_linear_equals_two_calls(dev, fmt):
    cfg = workloads.scaled_moe(workloads.MOE, E=9, N=256, K=512, tokens=300, topk=3, fmt=fmt)
    r, X, Y1 = build_moe(cfg, dev)
    Wq = torch.empty((cfg.E, cfg.N, cfg.K), dtype=torch.uint8, device=dev)
    Ws = torch.empty((cfg.E, cfg.N // 128, cfg.K // 128), dtype=torch.float32 if fmt == F32 else torch.uint8,
                     device=dev)
    for e in range(cfg.E):
        fg.quant_weight(workloads.moe_expert_weight(cfg, e, device=dev), fmt, Wq=Wq[e], Ws=Ws[e])
    offs = torch.as_tensor(r.group_offs, device=dev)
    Y2 = fg.grouped_linear(X, Wq, Ws, offs, fmt)
    fg.check_device_status()
    assert torch.equal(Y1, Y2)


@pytest.mark.parametrize("fmt", [F32, UE8M0])
@pytest.mark.parametrize("M", [7, 200])
def test_gemm_output_beyond_bf16_range(dev, fmt, M):
    """Outputs whose exact value lies beyond the bf16 range round to +-inf,
    as the oracle's bf16 rounding of its fp64 result does; rows scaled down
    to stay in range keep the GEMM tolerance.  Operands are same-signed per
    row (|x| ~ 2^100, w ~ 2^20 up to 2^21), so no partial sum cancels: the
    K = 512 sum reaches ~2^130 on the large rows and ~2^120 on the scaled
    rows.  Covers the few-token kernel (M = 7) and the persistent one."""
    N, K = 256, 512
    g = torch.Generator().manual_seed(M + fmt)
    mag = (1.0 + torch.rand((M, K), generator=g)) * 2.0 ** 100
    sign = torch.where(torch.arange(M) % 2 == 0, 1.0, -1.0)[:, None]
    rowscale = torch.where(torch.arange(M) % 3 == 2, 2.0 ** -10, 1.0)[:, None]
    X = (mag * sign * rowscale).to(torch.bfloat16)
    W = ((1.0 + torch.rand((N, K), generator=g)) * 2.0 ** 20).to(torch.bfloat16)
    Y = gpu_linear(X.to(dev), W.to(dev), fmt)
    Y_ref, S = oracle_linear(bits16(X), bits16(W), fmt)
    Y_gpu = y_to_f64(Y)
    ref_bits = oracle.bf16_rne(Y_ref)
    over = np.abs(Y_ref) > 2.0 * float(np.finfo(np.float32).max)      # clearly beyond bf16 and fp32
    finite = np.abs(Y_ref) < 0.25 * 3.3895e38                          # clearly inside
    assert over.any() and finite.any()
    ref_over = torch.from_numpy(ref_bits[over].astype(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(Y_gpu[over], ref_over), "overflowing outputs differ from the oracle's bf16 rounding"
    assert np.isinf(Y_gpu[over]).all()
    assert_gemm_close(Y_gpu[finite], Y_ref[finite], S[finite], f"in-range rows fmt {fmt} M {M}")
