"""GPU parity of the masked (batched) expert GEMM: expert e's tokens occupy
rows [e * cap, e * cap + counts[e]) of a fixed [E * cap, K] buffer, the rest
is padding.  Token rows against the oracle (per expert, its own weights);
padding rows of Y never written; with every expert full the result equals the
contiguous grouped GEMM; an out-of-range count is reported without a fault."""
import numpy as np
import pytest
import torch

import fine_grained_fp8_token_b200 as fg
import oracle
import workloads
from parity import F32, UE8M0, assert_gemm_close, bits16, require_gpu, to_np, y_to_f64

pytestmark = pytest.mark.gpu
SENTINEL = 7.0


@pytest.fixture(scope="module")
def dev():
    d = require_gpu()
    fg.load()
    return d


def build(dev, E, cap, N, K, fmt, seed, nan_padding=True, counts=None):
    X = workloads.activations((E * cap, K), "normal_outliers", seed=seed)
    if nan_padding and counts is not None:
        for e, c in enumerate(counts):
            if c < cap:
                X[e * cap + c:(e + 1) * cap, ::7] = float("nan")     # padding may hold anything
    Wq = torch.empty((E, N, K), dtype=torch.uint8, device=dev)
    Ws = torch.empty((E, N // 128, K // 128), dtype=torch.float32 if fmt == F32 else torch.uint8, device=dev)
    W_list = []
    for e in range(E):
        W = workloads.weights((N, K), seed=seed + 1 + e)
        W_list.append(W)
        fg.quant_weight(W.to(dev), fmt, Wq=Wq[e], Ws=Ws[e])
    Xq, Xs = fg.quant_act(X.to(dev), fmt)
    return X, W_list, Xq, Xs, Wq, Ws


def check_rows(X, W_list, Y, counts, cap, fmt, what):
    for e, c in enumerate(counts):
        if c == 0:
            continue
        rows = slice(e * cap, e * cap + c)
        Xq_r, Xs_r = oracle.quant_act(bits16(X[rows]), fmt)
        Wq_r, Ws_r = oracle.quant_weight(bits16(W_list[e]), fmt)
        Y_ref, S = oracle.gemm(Xq_r, Xs_r, Wq_r, Ws_r, fmt)
        assert_gemm_close(y_to_f64(Y[rows]), Y_ref, S, f"{what} expert {e}")


@pytest.mark.parametrize("fmt", [F32, UE8M0])
@pytest.mark.parametrize("cap,counts,N", [(128, [0, 3, 128, 77, 1], 256), (256, [256, 130, 0, 200], 384)])
def test_masked_gemm(dev, fmt, cap, counts, N):
    E, K = len(counts), 512
    X, W_list, Xq, Xs, Wq, Ws = build(dev, E, cap, N, K, fmt, seed=cap + N + fmt, counts=counts)
    cnt = torch.tensor(counts, dtype=torch.int32, device=dev)
    Y = torch.full((E * cap, N), SENTINEL, dtype=torch.bfloat16, device=dev)
    fg.masked_gemm(Xq, Xs, Wq, Ws, cnt, fmt, Y=Y)
    fg.check_device_status()
    check_rows(X, W_list, Y, counts, cap, fmt, f"masked cap {cap}")
    for e, c in enumerate(counts):
        assert (Y[e * cap + c:(e + 1) * cap].float() == SENTINEL).all(), f"padding rows of expert {e} written"


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_masked_full_equals_grouped(dev, fmt):
    E, cap, N, K = 3, 256, 256, 1024
    X, W_list, Xq, Xs, Wq, Ws = build(dev, E, cap, N, K, fmt, seed=41, nan_padding=False)
    cnt = torch.full((E,), cap, dtype=torch.int32, device=dev)
    Y_m = fg.masked_gemm(Xq, Xs, Wq, Ws, cnt, fmt)
    offs = torch.arange(0, (E + 1) * cap, cap, dtype=torch.int32, device=dev)
    Y_g = fg.grouped_gemm(Xq, Xs, Wq, Ws, offs, fmt)
    fg.check_device_status()
    assert torch.equal(Y_m, Y_g)


def test_masked_bad_count_reported(dev):
    E, cap, N, K = 3, 128, 256, 256
    counts = [5, cap + 1, 128]
    X, W_list, Xq, Xs, Wq, Ws = build(dev, E, cap, N, K, F32, seed=7, counts=[5, cap, 128])
    cnt = torch.tensor(counts, dtype=torch.int32, device=dev)
    Y = torch.full((E * cap, N), SENTINEL, dtype=torch.bfloat16, device=dev)
    fg.masked_gemm(Xq, Xs, Wq, Ws, cnt, F32, Y=Y)
    with pytest.raises(fg.FGFP8Error) as ei:
        fg.check_device_status()
    assert ei.value.status == 7
    assert (Y[cap:2 * cap].float() == SENTINEL).all()          # the bad expert's rows untouched
    check_rows(X, W_list, Y, [5, 0, 128], cap, F32, "bad-count neighbours")
    fg.check_device_status()                                    # cleared


def test_masked_full_decode_step_every_expert(dev):
    """The 256-expert decode step the benchmark times (128 tokens top-8,
    Zipf-routed, cap = 128, UE8M0): the first and last token row of every
    active expert and every token row of the busiest experts, a middle one
    and the last active one against the oracle; every padding row of every
    expert untouched."""
    cfg, cap = workloads.MOE_DECODE, 128
    r = workloads.moe_routing(cfg)
    X = workloads.moe_masked_rows(workloads.moe_tokens(cfg, device=dev), r, cfg.E, cap)
    Wq = torch.empty((cfg.E, cfg.N, cfg.K), dtype=torch.uint8, device=dev)
    Ws = torch.empty((cfg.E, cfg.N // 128, cfg.K // 128), dtype=torch.uint8, device=dev)
    for e in range(cfg.E):
        fg.quant_weight(workloads.moe_expert_weight(cfg, e, device=dev), UE8M0, Wq=Wq[e], Ws=Ws[e])
    Xq, Xs = fg.quant_act(X, UE8M0)
    cnt = torch.as_tensor(r.counts.astype(np.int32), device=dev)
    Y = torch.full((cfg.E * cap, cfg.N), SENTINEL, dtype=torch.bfloat16, device=dev)
    fg.masked_gemm(Xq, Xs, Wq, Ws, cnt, UE8M0, Y=Y)
    fg.check_device_status()
    active = np.where(r.counts > 0)[0]
    full = set(np.unique(np.r_[np.argsort(-r.counts)[:3], active[len(active) // 2], active[-1]]).tolist())
    for e in active:
        c = int(r.counts[e])
        local = np.arange(c) if e in full else np.unique(np.r_[0, c - 1])
        rows = int(e) * cap + local
        Xq_r, Xs_r = oracle.quant_act(bits16(X[torch.as_tensor(rows, device=dev)]), UE8M0)
        Wq_r, Ws_r = oracle.quant_weight(bits16(workloads.moe_expert_weight(cfg, int(e), device=dev)), UE8M0)
        Y_ref, S = oracle.gemm(Xq_r, Xs_r, Wq_r, Ws_r, UE8M0)
        assert_gemm_close(y_to_f64(Y[torch.as_tensor(rows, device=dev)]), Y_ref, S, f"masked decode expert {e}")
    pad = torch.ones(cfg.E * cap, dtype=torch.bool, device=dev)
    for e in active:
        pad[int(e) * cap:int(e) * cap + int(r.counts[e])] = False
    assert (Y[pad].float() == SENTINEL).all(), "padding rows written"


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_quant_act_masked_token_rows_only(dev, fmt):
    """The masked quantizer writes exactly the token rows, bit-exact with the
    1x128 quantizer (and the oracle); padding rows (here NaN) are not read
    and their codes and scales stay as they were.  A count above cap
    quantizes the whole block, a negative one no row, and either is reported
    through the device status word."""
    E, cap, K = 4, 128, 896
    counts = [5, 0, 128, 77]
    X = workloads.activations((E * cap, K), "normal_outliers", seed=31)
    for e, c in enumerate(counts):
        X[e * cap + c:(e + 1) * cap, ::5] = float("nan")
    Xd = X.to(dev)
    Xq_all, Xs_all = fg.quant_act(Xd, fmt)
    sdt = torch.float32 if fmt == F32 else torch.uint8
    Xq = torch.full((E * cap, K), 0xAB, dtype=torch.uint8, device=dev)
    Xs = torch.full(Xs_all.shape, 3, dtype=sdt, device=dev)
    fg.quant_act_masked(Xd, torch.tensor(counts, dtype=torch.int32, device=dev), E, fmt, Xq=Xq, Xs=Xs)
    fg.check_device_status()
    tok = np.concatenate([np.arange(e * cap, e * cap + c) for e, c in enumerate(counts)])
    pad = np.setdiff1d(np.arange(E * cap), tok)
    assert torch.equal(Xq[tok], Xq_all[tok])
    assert torch.equal(Xs[:, tok].contiguous().view(torch.uint8), Xs_all[:, tok].contiguous().view(torch.uint8))
    Xq_r, Xs_r = oracle.quant_act(bits16(X[tok]), fmt)
    assert np.array_equal(to_np(Xq[tok]), Xq_r)
    assert (Xq[pad] == 0xAB).all() and (Xs[:, pad].float() == 3).all()
    # a count above cap: the whole block is quantized
    Xq2 = torch.zeros_like(Xq_all)
    Xs2 = torch.zeros_like(Xs_all)
    fg.quant_act_masked(Xd, torch.tensor([0, cap + 9, 0, 0], dtype=torch.int32, device=dev), E, fmt, Xq=Xq2, Xs=Xs2)
    with pytest.raises(fg.FGFP8Error) as ei:
        fg.check_device_status()
    assert ei.value.status == 7                                 # FGFP8_ERR_DEVICE
    blk = slice(cap, 2 * cap)
    assert torch.equal(Xq2[blk], Xq_all[blk])
    # a negative count: no row of that expert, the others as usual, reported
    Xq3 = torch.full((E * cap, K), 0xAB, dtype=torch.uint8, device=dev)
    fg.quant_act_masked(Xd, torch.tensor([-3, 0, 0, 4], dtype=torch.int32, device=dev), E, fmt, Xq=Xq3, Xs=Xs2)
    with pytest.raises(fg.FGFP8Error) as ei:
        fg.check_device_status()
    assert ei.value.status == 7
    assert (Xq3[:cap] == 0xAB).all()
    assert torch.equal(Xq3[3 * cap:3 * cap + 4], Xq_all[3 * cap:3 * cap + 4])
    fg.check_device_status()                                    # cleared


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_masked_linear_equals_two_calls(dev, fmt):
    """fgfp8_masked_linear (token-row quantizer + masked GEMM as its
    programmatic dependent) gives bit-for-bit the masked quantizer's codes
    and the masked GEMM's output; token rows also against the oracle."""
    E, cap, N, K = 5, 128, 256, 512
    counts = [3, 0, 128, 64, 1]
    X, W_list, _, _, Wq, Ws = build(dev, E, cap, N, K, fmt, seed=57, counts=counts)
    Xd = X.to(dev)
    cnt = torch.tensor(counts, dtype=torch.int32, device=dev)
    Xq1, Xs1 = fg.quant_act_masked(Xd, cnt, E, fmt)
    Y1 = torch.full((E * cap, N), SENTINEL, dtype=torch.bfloat16, device=dev)
    fg.masked_gemm(Xq1, Xs1, Wq, Ws, cnt, fmt, Y=Y1)
    Y2 = torch.full((E * cap, N), SENTINEL, dtype=torch.bfloat16, device=dev)
    fg.masked_linear(Xd, Wq, Ws, cnt, fmt, Y=Y2)
    fg.check_device_status()
    assert torch.equal(Y1, Y2)
    check_rows(X, W_list, Y2, counts, cap, fmt, "masked linear")
    for e, c in enumerate(counts):
        assert (Y2[e * cap + c:(e + 1) * cap].float() == SENTINEL).all()

