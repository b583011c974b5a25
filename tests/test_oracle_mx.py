"""Pins of the oracle's MXFP8 functions (OCP Microscaling Formats v1.0: blocks
of 32 values along K sharing an E8M0 power-of-two scale, E4M3 elements),
each checked against something other than the oracle's own code: the
closed form of the block exponent, torch's own e4m3 cast of the scaled
values, and a numpy fp64 product of values dequantized through torch.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _e4m3_values(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def test_block_exponent_closed_form():
    # amax in [2^j, 2^(j+1)) -> scale 2^(j - 8), since 448 = 1.75 * 2^8
    rng = np.random.default_rng(1)
    rows = []
    want = []
    for j in (-20, -3, 0, 1, 5, 9, 14):
        for frac in (1.0, 1.25, 1.9921875):  # exact bf16 mantissas
            blk = rng.uniform(-1, 1, 32) * (2.0 ** j)
            blk[7] = -frac * 2.0 ** j  # the block's largest magnitude
            blk = np.clip(blk, -frac * 2.0 ** j, frac * 2.0 ** j)
            rows.append(blk)
            want.append(j - 8 + 127)
    x = _bf16(np.array(rows))
    _, se = oracle.quant_mx(x)
    assert se[:, 0].tolist() == want


def test_zero_block_and_exponent_clamp():
    x = np.zeros((2, 64), dtype=np.float32)
    x[1, 32:] = 2.0 ** -130  # below the smallest scale's reach: exponent clamps at -127
    q, se = oracle.quant_mx(_bf16(x))
    assert se[0].tolist() == [0, 0]      # all-zero block: the smallest scale
    assert not q[0].any()                # every code +0
    assert se[1, 1] == 0                 # -138 - 8 clamps to -127
    assert (q[1, 32:] != 0).all()        # 2^-130 / 2^-127 = 2^-3 is representable


def test_codes_match_torch_cast_of_scaled_values():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((16, 256)).astype(np.float32) * np.exp(rng.uniform(-8, 8, (16, 1))).astype(np.float32)
    xb = _bf16(x)
    q, se = oracle.quant_mx(xb)
    v = xb.float().numpy().astype(np.float64).reshape(16, 8, 32)
    scale = np.ldexp(1.0, se.astype(np.int64) - 127)[:, :, None]
    scaled = v / scale  # exact: division by a power of two
    assert np.abs(scaled).max() < 512
    sat = np.clip(scaled, -448, 448)  # saturation, then round to nearest even
    ref = torch.from_numpy(sat.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(q.reshape(16, 8, 32), ref)
    # the block maximum lands on the top binade of e4m3 (256 .. 448)
    top = np.abs(_e4m3_values(q).reshape(16, 8, 32)).max(axis=2)
    assert (top >= 256).all() and (top <= 448).all()


def test_dequantized_error_within_half_an_e4m3_step():
    # within half a step of e4m3 (3 mantissa bits) below 448 x scale; above
    # it the block maximum saturates, as the conversion rule says
    rng = np.random.default_rng(3)
    x = _bf16(rng.standard_normal((4, 128)))
    q, se = oracle.quant_mx(x)
    scale = np.repeat(np.ldexp(1.0, se.astype(np.int64) - 127), 32, axis=1)
    deq = _e4m3_values(q) * scale
    v = x.float().numpy().astype(np.float64)
    over = np.maximum(np.abs(v) - 448 * scale, 0.0)
    assert np.all(np.abs(deq - v) <= np.abs(v) * 2.0 ** -4 + 2.0 ** -10 * scale + over)
    assert np.all(np.abs(deq[over > 0]) == 448 * scale[over > 0])


@pytest.mark.parametrize("M,N,K", [(3, 17, 96), (1, 40, 256), (5, 8, 64)])
def test_mx_gemm_matches_brute_force(M, N, K):
    rng = np.random.default_rng(M * N + K)
    xq = rng.integers(0, 256, (M, K)).astype(np.uint8)
    wq = rng.integers(0, 256, (N, K)).astype(np.uint8)
    for a in (xq, wq):  # no NaN codes
        a[(a & 0x7F) == 0x7F] = 0x10
    sx = rng.integers(110, 140, (M, K // 32)).astype(np.uint8)
    sw = rng.integers(110, 140, (N, K // 32)).astype(np.uint8)
    y, bound = oracle.gemm_mx(xq, sx, wq, sw)
    xd = _e4m3_values(xq) * np.repeat(np.ldexp(1.0, sx.astype(np.int64) - 127), 32, axis=1)
    wd = _e4m3_values(wq) * np.repeat(np.ldexp(1.0, sw.astype(np.int64) - 127), 32, axis=1)
    ref = xd @ wd.T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(bound, np.abs(xd) @ np.abs(wd).T, rtol=1e-12, atol=1e-300)


def test_mx_gemm_scales_belong_to_their_own_block():
    # one-hot weights pick single activation values with their own block's scale
    K = 96
    x = _bf16(np.linspace(-3, 3, 2 * K).reshape(2, K) * np.array([[1.0], [64.0]]))
    xq, sx = oracle.quant_mx(x)
    w = np.zeros((3, K), dtype=np.float32)
    w[0, 5] = 1.0
    w[1, 40] = 1.0
    w[2, 95] = 1.0
    wq, sw = oracle.quant_mx(_bf16(w))
    y, _ = oracle.gemm_mx(xq, sx, wq, sw)
    xd = _e4m3_values(xq) * np.repeat(np.ldexp(1.0, sx.astype(np.int64) - 127), 32, axis=1)
    for n, k in enumerate((5, 40, 95)):
        np.testing.assert_allclose(y[:, n], xd[:, k], rtol=1e-15)
