"""The layer API: QuantizedLinear (graph replay per M bucket, eager beyond 32
tokens) and DecodeStep (a whole step of layers captured with its host copies)
must give the same bits as the eager calls."""
import pytest
import torch

import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth
from quantized_gemm_decode_b200.linear import DecodeStep, QuantizedLinear

pytestmark = pytest.mark.gpu


def _eager(layer, x):
    xq, sx = layer.quantize(x.cuda())
    return layer.gemm(xq, sx)


@pytest.mark.parametrize("fmt", ["fp8_dynamic", "w8a8_int8", "block_fp8"])
def test_bucket_graphs_match_eager(fmt):
    w = synth.weights(1024, 2048, seed=41).cuda()
    layer = QuantizedLinear(w, fmt)
    layer.capture()
    for M in (1, 3, 8, 13, 32, 40):
        x = synth.activations(M, 2048, seed=M, outliers=True)
        y = layer(x.cuda()).clone()
        ref = _eager(layer, x)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), f"M={M}"


@pytest.mark.parametrize("join_every,out_every", [(1, 1), (2, 1), (4, 1), (2, 2), (1, 3)])
def test_decode_step_with_host_io_matches_eager(join_every, out_every):
    layers = [QuantizedLinear(synth.weights(1536, 1024, seed=51).cuda(), "fp8_dynamic"),
              QuantizedLinear(synth.weights(1024, 2048, seed=52).cuda(), "w8a8_int8"),
              QuantizedLinear(synth.weights(512, 1024, seed=53).cuda(), "block_fp8")]
    ms = (4, 16, 1)
    xh = [synth.activations(m, l.K, seed=60 + i, outliers=True).pin_memory() for i, (l, m) in enumerate(zip(layers, ms))]
    yh = [torch.empty((m, l.N), dtype=torch.bfloat16).pin_memory() for l, m in zip(layers, ms)]
    step = DecodeStep(list(zip(layers, ms)), xh, yh, join_every=join_every, out_every=out_every)
    for rnd in range(2):
        if rnd == 1:  # new inputs in the same pinned buffers
            for i, (l, m) in enumerate(zip(layers, ms)):
                xh[i].copy_(synth.activations(m, l.K, seed=70 + i, outliers=True))
        step.replay()
        torch.cuda.synchronize()
        for i, (l, m) in enumerate(zip(layers, ms)):
            ref = _eager(l, xh[i]).cpu()
            assert torch.equal(yh[i].view(torch.int16), ref.view(torch.int16)), f"round {rnd} layer {i}"
    assert qgd.qgd_device_error() == 0
