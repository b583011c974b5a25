"""Pins for the oracle's quantized GEMMs (CPU only).

The oracle accumulates exact integers.  Here it is held against:
  * brute force: a numpy fp64 matmul of values dequantized through torch's
    own float8/int8 -> float64 conversion, with scales broadcast by numpy;
  * identity and one-hot weights, whose products have closed forms;
  * the transpose identity the Swap-AB variant relies on (the GEMM with the
    operands' roles exchanged is the transpose, bit for bit);
  * split-K invariance: any contiguous chunking of K sums to the same exact
    integer, which also equals a Python-integer brute-force sum.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_gemm_decode_b200 import synth


def deq_e4m3(q: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def deq_int8(q: np.ndarray) -> np.ndarray:
    return q.astype(np.float64)


@pytest.mark.parametrize("M,N,K", [(1, 8, 32), (3, 17, 96), (4, 40, 256), (5, 33, 160)])
@pytest.mark.parametrize("qtype", [oracle.E4M3, oracle.INT8])
def test_rowscaled_matches_brute_force(M, N, K, qtype):
    x = synth.activations(M, K, seed=M + N, outliers=True)
    w = synth.weights(N, K, seed=K)
    xq, sx = oracle.quant_rows(x, qtype)
    wq, sw = oracle.quant_rows(w, qtype)
    deq = deq_e4m3 if qtype == oracle.E4M3 else deq_int8
    xd = deq(xq) * sx.astype(np.float64)[:, None]
    wd = deq(wq) * sw.astype(np.float64)[:, None]
    ref = xd @ wd.T
    y, bound = oracle.gemm_rowscaled(xq, sx, wq, sw, qtype)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    np.testing.assert_allclose(bound, np.abs(xd) @ np.abs(wd).T, rtol=1e-12)


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (3, 256, 384), (2, 384, 256)])
def test_blockscaled_matches_brute_force(M, N, K):
    x = synth.activations(M, K, seed=100 + M, outliers=True)
    w = synth.weights(N, K, seed=200 + N)
    xq, sx = oracle.quant_groups(x, 128)
    wq, sw = oracle.quant_blocks(w, 128)
    # broadcast the scales to full [M,K] / [N,K] grids
    sxf = np.repeat(sx.astype(np.float64), 128, axis=1)
    swf = np.repeat(np.repeat(sw.astype(np.float64), 128, axis=0), 128, axis=1)
    xd = deq_e4m3(xq) * sxf
    wd = deq_e4m3(wq) * swf
    ref = xd @ wd.T
    y, bound = oracle.gemm_blockscaled(xq, sx, wq, sw, 128)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    np.testing.assert_allclose(bound, np.abs(xd) @ np.abs(wd).T, rtol=1e-12)


def test_identity_weight_returns_dequantized_activations():
    M, K = 4, 256
    x = synth.activations(M, K, seed=1, outliers=True)
    w = torch.eye(K, dtype=torch.bfloat16)
    xq, sx = oracle.quant_rows(x, oracle.E4M3)
    wq, sw = oracle.quant_rows(w, oracle.E4M3)
    assert np.all(np.diag(wq) == 0x7E)
    assert np.all(sw == np.float32(1.0) / np.float32(448.0))
    y, _ = oracle.gemm_rowscaled(xq, sx, wq, sw, oracle.E4M3)
    xd = deq_e4m3(xq) * sx.astype(np.float64)[:, None]
    np.testing.assert_allclose(y, xd, rtol=2.0 ** -22, atol=0)


def test_one_hot_rows_select_columns():
    M, K, N = 3, 128, 16
    x = synth.activations(M, K, seed=2, outliers=False)
    cols = np.random.default_rng(0).choice(K, size=N, replace=False)
    w = torch.zeros(N, K, dtype=torch.bfloat16)
    w[torch.arange(N), torch.from_numpy(cols)] = torch.tensor(
        np.linspace(-2.0, 3.0, N, dtype=np.float32)).to(torch.bfloat16)
    xq, sx = oracle.quant_rows(x, oracle.INT8)
    wq, sw = oracle.quant_rows(w, oracle.INT8)
    y, _, acc = oracle.gemm_rowscaled(xq, sx, wq, sw, oracle.INT8, want_acc=True)
    for n in range(N):
        np.testing.assert_array_equal(acc[:, n], xq[:, cols[n]].astype(np.int64) * int(wq[n, cols[n]]))


@pytest.mark.parametrize("qtype", [oracle.E4M3, oracle.INT8])
def test_transpose_identity(qtype):
    x = synth.activations(6, 256, seed=4, outliers=True)
    w = synth.weights(20, 256, seed=4)
    xq, sx = oracle.quant_rows(x, qtype)
    wq, sw = oracle.quant_rows(w, qtype)
    y, _, acc = oracle.gemm_rowscaled(xq, sx, wq, sw, qtype, want_acc=True)
    yt, _, acct = oracle.gemm_rowscaled(wq, sw, xq, sx, qtype, want_acc=True)
    np.testing.assert_array_equal(acc, acct.T)
    np.testing.assert_array_equal(y, yt.T)


@pytest.mark.parametrize("qtype", [oracle.E4M3, oracle.INT8])
def test_split_k_invariance(qtype):
    K = 1024
    x = synth.activations(2, K, seed=5, outliers=True)
    w = synth.weights(3, K, seed=5)
    xq, _ = oracle.quant_rows(x, qtype)
    wq, _ = oracle.quant_rows(w, qtype)
    if qtype == oracle.E4M3:
        xi = (deq_e4m3(xq) * 512).astype(np.int64)
        wi = (deq_e4m3(wq) * 512).astype(np.int64)
    else:
        xi, wi = xq.astype(np.int64), wq.astype(np.int64)
    for m in range(2):
        for n in range(3):
            exact = sum(int(a) * int(b) for a, b in zip(xi[m], wi[n]))
            for s in (1, 2, 3, 4, 8, 16, 32, 64, 128, 256):
                assert oracle.dot_split(xq, m, wq, n, qtype, s) == exact


def test_zero_activation_row_gives_zero_output():
    x = synth.activations(3, 256, seed=6, outliers=False)
    x[1] = 0.0
    w = synth.weights(8, 256, seed=6)
    for qtype in (oracle.E4M3, oracle.INT8):
        xq, sx = oracle.quant_rows(x, qtype)
        wq, sw = oracle.quant_rows(w, qtype)
        y, _ = oracle.gemm_rowscaled(xq, sx, wq, sw, qtype)
        assert np.all(y[1] == 0.0)
