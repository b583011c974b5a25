"""GPU parity of the dynamic quantizers against the oracle: codes and scales
must match bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth
from paritylib import as_u8

pytestmark = pytest.mark.gpu


def _per_token_both(x: torch.Tensor, qtype: int):
    xq, sx = qgd.quant_act_per_token(x.cuda(), qtype)
    torch.cuda.synchronize()
    oq, osx = oracle.quant_rows(x, oracle.E4M3 if qtype == qgd.QTYPE_E4M3 else oracle.INT8)
    return as_u8(xq), sx.cpu().numpy(), oq.view(np.uint8), osx


@pytest.mark.parametrize("qtype", [qgd.QTYPE_E4M3, qgd.QTYPE_INT8])
@pytest.mark.parametrize("M,K", [(1, 1024), (4, 1024), (3, 4096), (32, 4096), (7, 5120), (32, 12288),
                                 (5, 17408), (2, 25600), (3, 40), (1, 65536)])
def test_per_token_bit_exact(M, K, qtype):
    x = synth.activations(M, K, seed=M + K, outliers=True)
    q, s, oq, os_ = _per_token_both(x, qtype)
    np.testing.assert_array_equal(s.view(np.uint32), os_.view(np.uint32))
    np.testing.assert_array_equal(q, oq)


@pytest.mark.parametrize("qtype", [qgd.QTYPE_E4M3, qgd.QTYPE_INT8])
def test_per_token_edge_rows(qtype):
    K = 256
    rows = torch.zeros(6, K, dtype=torch.bfloat16)
    rows[1] = -0.0                                   # all negative zeros
    rows[2, 17] = 3.0                                # single nonzero
    ties = torch.tensor([448.0, 1.0625, 1.1875, 3 * 2.0 ** -10, 2.0 ** -10, -1.0625, 8.5, 9.5, 15.5])
    rows[3, :9] = ties                               # scale exactly 1: e4m3 midpoints
    rows[4, :6] = torch.tensor([127.0, 2.5, -2.5, 3.5, 0.5, -126.5])  # int8 half-way cases at scale 1
    rows[5] = synth.uniform_bf16((K,), -1e-3, 1e-3, seed=3)          # tiny magnitudes
    q, s, oq, os_ = _per_token_both(rows, qtype)
    np.testing.assert_array_equal(s.view(np.uint32), os_.view(np.uint32))
    np.testing.assert_array_equal(q, oq)


def test_per_channel_weights_bit_exact():
    w = synth.weights(1024, 4096, seed=11)
    for qtype in (qgd.QTYPE_E4M3, qgd.QTYPE_INT8):
        wq, sw = qgd.quant_weight_per_channel(w.cuda(), qtype)
        torch.cuda.synchronize()
        oq, osw = oracle.quant_rows(w, oracle.E4M3 if qtype == qgd.QTYPE_E4M3 else oracle.INT8)
        np.testing.assert_array_equal(sw.cpu().numpy().view(np.uint32), osw.view(np.uint32))
        np.testing.assert_array_equal(as_u8(wq), oq.view(np.uint8))


@pytest.mark.parametrize("M,K", [(1, 128), (4, 1024), (32, 5120), (13, 8192), (32, 25600), (300, 1024)])
def test_group128_bit_exact(M, K):
    x = synth.activations(M, K, seed=7 * M + K, outliers=True)
    x[0, :128] = 0.0  # an all-zero group
    xq, sx = qgd.quant_act_group128(x.cuda())
    torch.cuda.synchronize()
    oq, osx = oracle.quant_groups(x, 128)
    np.testing.assert_array_equal(sx.cpu().numpy().view(np.uint32), osx.view(np.uint32))
    np.testing.assert_array_equal(as_u8(xq), oq)


@pytest.mark.parametrize("N,K", [(128, 128), (512, 1024), (1280, 5120)])
def test_block128_bit_exact(N, K):
    w = synth.weights(N, K, seed=N + K)
    w[:128, :128] = 0.0  # an all-zero block
    wq, sw = qgd.quant_weight_block128(w.cuda())
    torch.cuda.synchronize()
    oq, osw = oracle.quant_blocks(w, 128)
    np.testing.assert_array_equal(sw.cpu().numpy().view(np.uint32), osw.view(np.uint32))
    np.testing.assert_array_equal(as_u8(wq), oq)


def test_block128_full_size_sampled_bands():
    # the largest Block_FP8 weight (51200 x 5120): every band quantized on the
    # GPU, a few bands checked against the oracle
    N, K = 51200, 5120
    w = synth.weights(N, K, seed=1003)
    wq, sw = qgd.quant_weight_block128(w.cuda())
    torch.cuda.synchronize()
    for band in (0, 17, 399):
        rows = slice(band * 128, (band + 1) * 128)
        oq, osw = oracle.quant_blocks(w[rows], 128)
        np.testing.assert_array_equal(sw[band].cpu().numpy().view(np.uint32), osw[0].view(np.uint32))
        np.testing.assert_array_equal(as_u8(wq[rows]), oq)


def test_empty_and_rejected_inputs():
    x = torch.zeros(0, 1024, dtype=torch.bfloat16, device="cuda")
    xq, sx = qgd.quant_act_per_token(x)
    assert xq.shape == (0, 1024)
    with pytest.raises(qgd.QGDError):
        qgd.quant_act_group128(torch.zeros(2, 100, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(qgd.QGDError):
        qgd.quant_weight_block128(torch.zeros(100, 128, dtype=torch.bfloat16, device="cuda"))
