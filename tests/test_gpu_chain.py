"""Parity of the dependent decode-layer chain (qkv -> o -> gate_up -> down).

Each layer call quantizes a column slice of an earlier layer's bf16 output,
read in place through its row stride, and runs its GEMM (fused into one
kernel where the layer plan says so); the whole chain is one CUDA graph.
Per layer, against the oracle applied to the very bf16 input the GPU layer
saw (its predecessor's output): the output within the FP8 tolerance.  That
is the parity bar; it holds layer by layer whatever rounding came before.
The chain runs once with the shipped plans and once with every layer's
quantizer forced into its GEMM.

End to end, the chain is also compared with a chain run entirely by the
oracle (which rounds each intermediate to bf16 itself).  The two inputs of
a layer then differ by the earlier layers' rounding, and a one-code change
in a requantized activation is not bounded by the per-layer tolerance, so
that comparison is a loose sanity check on the norm of the error only.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth
from quantized_gemm_decode_b200.linear import LAYER_8B, DecodeChain, QuantizedLinear
from paritylib import as_u8, bf16_to_f64, check_fp8_tolerance

pytestmark = pytest.mark.gpu

# a small layer with the same wiring as LAYER_8B (input 512 wide; qkv 768,
# o reads its first 512 columns, gate_up 3072, down reads its first 1536)
SMALL = ((768, 512), (512, 512), (3072, 512), (512, 1536))
SMALL_WIRING = (("qkv", -1, 512), ("o", 0, 512), ("gate_up", 1, 512), ("down", 2, 1536))
FULL = ((6144, 4096), (4096, 4096), (24576, 4096), (4096, 12288))


@pytest.fixture(autouse=True)
def _shipped_plans():
    qgd.lib()
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC)
    qgd.qgd_set_fused_override(qgd.FMT_FP8_DYNAMIC)
    yield
    qgd.qgd_set_fused_override(qgd.FMT_FP8_DYNAMIC)


def _chain(shapes, wiring, seed):
    ws = [synth.weights(n, k, seed + 10 * i) for i, (n, k) in enumerate(shapes)]
    layers = [QuantizedLinear(w.cuda(), "fp8_dynamic") for w in ws]
    return DecodeChain(layers, wiring), ws


def _check_layer(chain, ws, M, i, rows=None):
    """Layer i against the oracle on the GPU layer's own bf16 input (the
    oracle quantizes it itself; the layer call's codes are held to the
    oracle's bit for bit in the quantizer and fused-layer tests)."""
    x_in = chain.inputs(M)[i].float().cpu().to(torch.bfloat16).contiguous()
    oxq, osx = oracle.quant_rows(x_in, oracle.E4M3)
    w = ws[i] if rows is None else ws[i][torch.from_numpy(rows)]
    owq, osw = oracle.quant_rows(w, oracle.E4M3)
    yref, bound = oracle.gemm_rowscaled(oxq, osx, owq, osw, oracle.E4M3)
    y = bf16_to_f64(chain.outputs(M)[i])
    if rows is not None:
        y = y[:, rows]
    check_fp8_tolerance(y, yref, bound, x_in.shape[1], f"layer {i} ({chain.wiring[i][0]}) M={M}")


def _bf16_round(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("fused", [-1, 1])
@pytest.mark.parametrize("M", [1, 5, 32])
def test_small_chain_layer_by_layer_and_end_to_end(M, fused):
    qgd.qgd_set_fused_override(qgd.FMT_FP8_DYNAMIC, fused)
    chain, ws = _chain(SMALL, SMALL_WIRING, seed=71)
    x = synth.activations(M, SMALL[0][1], 71, outliers=True)
    y_last = chain.run(M, x.cuda())
    torch.cuda.synchronize()
    for i in range(4):
        _check_layer(chain, ws, M, i)
    # replaying again gives the same bits (deterministic reductions)
    first = [y.clone() for y in chain.outputs(M)]
    chain.run(M)
    torch.cuda.synchronize()
    for a, b in zip(first, chain.outputs(M)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # the whole chain by the oracle alone
    outs = []
    cur = x
    for i, (name, src, cols) in enumerate(SMALL_WIRING):
        inp = cur if src < 0 else outs[src][:, :cols].contiguous()
        xq, sx = oracle.quant_rows(inp, oracle.E4M3)
        wq, sw = oracle.quant_rows(ws[i], oracle.E4M3)
        y, _ = oracle.gemm_rowscaled(xq, sx, wq, sw, oracle.E4M3)
        outs.append(_bf16_round(y))
    ref = outs[-1].double().numpy()
    got = bf16_to_f64(y_last)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 0.1, f"chain end to end: relative error {rel:.3e}"


@pytest.mark.parametrize("M", [1, 32])
def test_full_size_8b_chain_sampled(M):
    chain, ws = _chain(FULL, LAYER_8B, seed=81)
    x = synth.activations(M, 4096, 81, outliers=True)
    chain.run(M, x.cuda())
    torch.cuda.synchronize()
    for i, (n, _) in enumerate(FULL):
        bands = [0, n // 256, n // 128 - 1]
        rows = np.concatenate([np.arange(b * 128, (b + 1) * 128) for b in bands])
        _check_layer(chain, ws, M, i, rows=rows)
    assert qgd.qgd_device_error() == 0


def test_chain_rejects_bad_wiring():
    layers = [QuantizedLinear(synth.weights(n, k, 3).cuda(), "fp8_dynamic") for n, k in SMALL]
    with pytest.raises(ValueError):
        DecodeChain(layers, (("qkv", -1, 512), ("o", 0, 1024), ("gate_up", 1, 512), ("down", 2, 1536)))
    with pytest.raises(ValueError):
        DecodeChain(layers, (("qkv", -1, 512), ("o", 1, 512), ("gate_up", 1, 512), ("down", 2, 1536)))


def test_strided_quantizer_matches_dense_copy():
    # a column slice read in place quantizes like a dense copy of it
    big = synth.activations(7, 6144, 5, outliers=True).cuda()
    view = big[:, :4096]
    xq_v, sx_v = qgd.quant_act_per_token(view, qgd.QTYPE_E4M3)
    xq_d, sx_d = qgd.quant_act_per_token(view.contiguous(), qgd.QTYPE_E4M3)
    assert torch.equal(xq_v.view(torch.uint8), xq_d.view(torch.uint8)) and torch.equal(sx_v, sx_d)
    gq_v, gs_v = qgd.quant_act_group128(view)
    gq_d, gs_d = qgd.quant_act_group128(view.contiguous())
    assert torch.equal(gq_v.view(torch.uint8), gq_d.view(torch.uint8)) and torch.equal(gs_v, gs_d)
    oxq, osx = oracle.quant_rows(view.cpu().contiguous(), oracle.E4M3)
    np.testing.assert_array_equal(as_u8(xq_v), oxq)
    np.testing.assert_array_equal(sx_v.cpu().numpy(), osx)
