"""Sanitizer stand-in on the GPU (no memory checker runs on this hardware's
pool): the library built with its kernels' index checks compiled in
(libfgfp8_debug.so, -DFGFP8_DEBUG_CHECKS: tile origins, rows, columns and
experts checked against the problem bounds where they are formed and before
the stores they address) runs every kernel family on ragged and tail shapes
with no check failing, and writes the same bits as the release library,
inside canary bytes."""
import ctypes

import numpy as np
import pytest
import torch

import fine_grained_fp8_token_b200 as fg
import workloads
from fine_grained_fp8_token_b200 import build as fgbuild
from parity import F32, UE8M0, Guarded, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    require_gpu()
    release = fg.load()
    debug = ctypes.CDLL(fgbuild.build(debug=True))
    for name, (res, args) in fg.SIGNATURES.items():
        fn = getattr(debug, name)
        fn.restype, fn.argtypes = res, args
    return release, debug


def run_with(lib, monkeypatch, fn):
    """fn() with the binding routed to `lib`; the device status is checked
    (and cleared) through the same library."""
    with monkeypatch.context() as mp:
        mp.setattr(fg, "load", lambda build_if_missing=True: lib)
        out = fn()
        fg.check_device_status()
    return out


def dense_case(M, N, K, fmt, seed):
    def run():
        dev = torch.device("cuda:0")
        cfg = workloads.scaled_linear(workloads.TINY, M=M, N=N, K=K, seed=seed)
        X, W = workloads.linear_inputs(cfg, device=dev)
        Xq, Xs = fg.quant_act(X, fmt)
        Wq, Ws = fg.quant_weight(W, fmt)
        gY = Guarded((M, N), torch.bfloat16, dev)
        fg.gemm(Xq, Xs, Wq, Ws, fmt, Y=gY.t)
        torch.cuda.synchronize()
        gY.check("Y")
        return [Xq, Xs[:, :M], Wq, Ws, gY.t]          # scale entries m >= M are not written
    return run


CASES = [(1, 256, 512), (7, 128, 384), (64, 1280, 7168), (129, 384, 1024), (300, 640, 2048),
         (1200, 4096, 256), (2560, 2304, 384)]


@pytest.mark.parametrize("fmt", [F32, UE8M0])
@pytest.mark.parametrize("M,N,K", CASES)
def test_dense_and_decode_index_checks(libs, monkeypatch, M, N, K, fmt):
    rel, dbg = libs
    a = run_with(rel, monkeypatch, dense_case(M, N, K, fmt, seed=M + N + K + fmt))
    b = run_with(dbg, monkeypatch, dense_case(M, N, K, fmt, seed=M + N + K + fmt))
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


@pytest.mark.parametrize("fmt", [F32, UE8M0])
def test_grouped_and_masked_index_checks(libs, monkeypatch, fmt):
    rel, dbg = libs
    cfg = workloads.scaled_moe(workloads.MOE, E=24, N=256, K=512, tokens=600, topk=4, fmt=fmt)
    dev = torch.device("cuda:0")
    r = workloads.moe_routing(cfg)
    X = workloads.moe_grouped_rows(workloads.moe_tokens(cfg, device=dev), r)
    Wq = torch.empty((cfg.E, cfg.N, cfg.K), dtype=torch.uint8, device=dev)
    Ws = torch.empty((cfg.E, cfg.N // 128, cfg.K // 128), dtype=torch.float32 if fmt == F32 else torch.uint8,
                     device=dev)
    for e in range(cfg.E):
        run_with(rel, monkeypatch, lambda e=e: fg.quant_weight(workloads.moe_expert_weight(cfg, e, device=dev), fmt,
                                                               Wq=Wq[e], Ws=Ws[e]))
    offs = torch.as_tensor(r.group_offs, device=dev)
    cap = 128
    Xm = workloads.moe_masked_rows(workloads.moe_tokens(cfg, device=dev), r, cfg.E, cap)
    counts = torch.as_tensor(np.minimum(r.counts, cap).astype(np.int32), device=dev)

    def run():
        Xq, Xs = fg.quant_act(X, fmt)
        gY = Guarded((r.M_total, cfg.N), torch.bfloat16, dev, fill=0)
        fg.grouped_gemm(Xq, Xs, Wq, Ws, offs, fmt, Y=gY.t)
        gM = Guarded((cfg.E * cap, cfg.N), torch.bfloat16, dev, fill=0)
        Xqm = torch.zeros((cfg.E * cap, cfg.K), dtype=torch.uint8, device=dev)
        Xsm = torch.zeros((cfg.K // 128, fg.scale_rows(cfg.E * cap, fmt)), dtype=Xs.dtype, device=dev)
        fg.masked_linear(Xm, Wq, Ws, counts, fmt, Y=gM.t, Xq=Xqm, Xs=Xsm)
        torch.cuda.synchronize()
        gY.check("grouped Y")
        gM.check("masked Y")
        return [Xq, Xs[:, :r.M_total], gY.t, Xqm, Xsm, gM.t]

    a = run_with(rel, monkeypatch, run)
    b = run_with(dbg, monkeypatch, run)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_rowcol_and_fused_index_checks(libs, monkeypatch):
    rel, dbg = libs
    dev = torch.device("cuda:0")
    M, N, K, I = 300, 640, 1024, 384

    def run():
        X = workloads.activations((M, K), "normal_outliers", seed=3, device=dev)
        W = workloads.weights((N, K), seed=4, device=dev)
        Xq, sx = fg.quant_rows(X)
        Wq, sw = fg.quant_rows(W)
        gY = Guarded((M, N), torch.bfloat16, dev)
        fg.gemm_rowcol(Xq, sx, Wq, sw, Y=gY.t)
        Wg = workloads.weights((I, K), seed=5, device=dev)
        Wu = workloads.weights((I, K), seed=6, device=dev)
        Wq_gu, Ws_gu = fg.quant_weight(fg.interleave_gate_up(Wg, Wu), F32)
        Xq2, Xs2 = fg.quant_act(X, F32)
        ld = fg.scale_rows(M, F32)
        gH = Guarded((M, I), torch.uint8, dev)
        Hs = torch.zeros((I // 128, ld), dtype=torch.float32, device=dev)
        fg.gemm_swiglu_quant(Xq2, Xs2, Wq_gu, Ws_gu, Hq=gH.t, Hs=Hs, ld_h=ld)
        torch.cuda.synchronize()
        gY.check("rowcol Y")
        gH.check("Hq")
        return [Xq, sx, gY.t, gH.t, Hs[:, :M]]

    a = run_with(rel, monkeypatch, run)
    b = run_with(dbg, monkeypatch, run)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
