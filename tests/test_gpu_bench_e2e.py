"""The benchmark's end-to-end path streams a dense layer's token rows through
host copies in chunks on three streams (copy in, fgfp8_linear of the chunk,
copy out).  The chunked result read back to the host must equal the one-call
layer bit for bit (each output row depends on its own input row only), for
one layer and for the two-layer prefill step."""
import pytest
import torch

import bench
import workloads
from parity import require_gpu

pytestmark = pytest.mark.gpu


def run_streamed(parts, dev):
    X_hosts = [torch.empty(d.X.shape, dtype=d.X.dtype, pin_memory=True).copy_(d.X) for d in parts]
    Y_hosts = [torch.empty(d.Y.shape, dtype=d.Y.dtype, pin_memory=True) for d in parts]
    X_stages = [torch.empty_like(d.X) for d in parts]
    stream = torch.cuda.current_stream(dev)
    start = torch.cuda.Event()
    start.record(stream)
    bench.e2e_streamed(parts, X_hosts, X_stages, Y_hosts, stream, dev, start)
    torch.cuda.synchronize(dev)
    return Y_hosts


@pytest.mark.parametrize("fmt", [0, 1])
def test_streamed_dense_layer_equals_one_call(fmt):
    dev = require_gpu()
    cfg = workloads.replace(workloads.scaled_linear(workloads.TINY, M=2056, N=768, K=1024, seed=17), fmt=fmt)
    d = bench.DenseLayer(cfg, dev)
    d.linear()
    Y_ref = d.Y.clone().cpu()
    d.Y.zero_()
    (Y,) = run_streamed([d], dev)
    d.fg.check_device_status()
    assert torch.equal(Y, Y_ref)


def test_streamed_prefill_step_equals_one_call():
    dev = require_gpu()
    layer = bench.PrefillMLP(dev, tokens=1024)
    layer.linear()
    refs = [layer.gu.Y.clone().cpu(), layer.down.Y.clone().cpu()]
    layer.gu.Y.zero_()
    layer.down.Y.zero_()
    outs = run_streamed(bench.streamed_parts(layer), dev)
    layer.fg.check_device_status()
    for y, r in zip(outs, refs):
        assert torch.equal(y, r)
