"""Pins of the oracle's NVFP4 functions (E2M1 elements, an E4M3 scale per 16
values along K, an fp32 scale per row), each checked against something other
than the oracle's own code: the FP4 (E2M1) value table of the OCP
Microscaling Formats v1.0 specification, torch's own e4m3 cast of the block
scales, numpy's IEEE fp32 arithmetic for the row scales, the error bound the
rounding rule implies, and a numpy fp64 product of values dequantized through
the specification's table.
"""
import numpy as np
import pytest
import torch

import oracle

# OCP MX v1.0, FP4 (E2M1): the eight magnitudes, codes 0..7 (bit 3 is the sign)
SPEC_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _unpack(q: np.ndarray) -> np.ndarray:
    """Packed bytes [R, K/2] -> codes [R, K]: element 2i in the low nibble."""
    out = np.empty((q.shape[0], q.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = q & 0xF
    out[:, 1::2] = q >> 4
    return out


def _e2m1_values(codes: np.ndarray) -> np.ndarray:
    mag = np.asarray(SPEC_E2M1, dtype=np.float64)[codes & 0x7]
    return np.where(codes & 0x8, -mag, mag)


def _e4m3_values(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def test_e2m1_decode_matches_spec_table():
    got = [oracle.e2m1_decode(c) for c in range(16)]
    assert got[:8] == SPEC_E2M1
    assert got[8:] == [-v for v in SPEC_E2M1]
    assert np.signbit(got[8])  # code 0x8 is -0


def test_e2m1_round_trip_midpoints_and_saturation():
    for c in range(16):
        assert oracle.e2m1_encode(oracle.e2m1_decode(c)) == c
    for i in range(7):
        lo, hi = SPEC_E2M1[i], SPEC_E2M1[i + 1]
        mid = (lo + hi) / 2
        even = i if i % 2 == 0 else i + 1  # the code whose mantissa bit is clear
        assert oracle.e2m1_encode(mid) == even, (lo, hi)
        assert oracle.e2m1_encode(-mid) == 0x8 | even
        assert oracle.e2m1_encode(np.nextafter(mid, lo)) == i
        assert oracle.e2m1_encode(np.nextafter(mid, hi)) == i + 1
    for v in (6.0, 6.5, 7.0, 1e30):
        assert oracle.e2m1_encode(v) == 0x7 and oracle.e2m1_encode(-v) == 0xF
    assert oracle.e2m1_encode(0.2) == 0x0 and oracle.e2m1_encode(-0.2) == 0x8


def _rows(seed, R=6, K=256):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((R, K)).astype(np.float32) * np.exp(rng.uniform(-6, 6, (R, 1))).astype(np.float32)
    x[:, rng.choice(K, 5, replace=False)] *= 20.0  # outlier channels
    return _bf16(x)


@pytest.mark.parametrize("seed", [1, 2])
def test_row_and_block_scales_follow_ieee_fp32_and_torch_cast(seed):
    xb = _rows(seed)
    q, s, g = oracle.quant_nv(xb)
    v = xb.float().numpy()
    amax = np.abs(v).max(axis=1).astype(np.float32)
    np.testing.assert_array_equal(g, amax / np.float32(2688.0))  # numpy: correctly rounded fp32
    bmax = np.abs(v.reshape(v.shape[0], -1, 16)).max(axis=2).astype(np.float32)
    six_g = (np.float32(6.0) * g).astype(np.float32)
    ratio = (bmax / six_g[:, None]).astype(np.float32)
    assert ratio.max() <= 448.0 * (1 + 2 ** -20)
    ref = torch.from_numpy(np.minimum(ratio, 448.0)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(s, ref)


@pytest.mark.parametrize("seed", [3, 4])
def test_row_maximum_lands_on_six_with_scale_448(seed):
    xb = _rows(seed)
    q, s, g = oracle.quant_nv(xb)
    v = xb.float().numpy()
    codes = _unpack(q)
    for r in range(v.shape[0]):
        k = int(np.argmax(np.abs(v[r])))
        assert codes[r, k] & 0x7 == 0x7  # magnitude 6
        assert (codes[r, k] >> 3) == (1 if v[r, k] < 0 else 0)
        assert s[r, k // 16] == 0x7E  # 448


@pytest.mark.parametrize("seed", [5, 6])
def test_dequantized_error_within_half_an_e2m1_step(seed):
    # nearest rounding of the fp32 quotient t = x / d: |x - c d| is at most
    # half the spacing of E2M1 around t (0.25 below 2, 0.5 in [2, 4], 1 in
    # [4, 6]) plus the quotient's own fp32 rounding; past 6 (a block scale
    # rounded down to E4M3) the code saturates at 6.  d = dec(s) g in fp32.
    xb = _rows(seed)
    q, s, g = oracle.quant_nv(xb)
    v = xb.float().numpy().astype(np.float64)
    d = (np.repeat(_e4m3_values(s), 16, axis=1).astype(np.float32) * g[:, None]).astype(np.float32).astype(np.float64)
    c = _e2m1_values(_unpack(q))
    t = np.abs(v) / d
    half_step = np.where(t <= 2, 0.25, np.where(t <= 4, 0.5, 1.0))
    over = np.maximum(t - 6.0, 0.0)
    assert t.max() < 6 * 1.07  # the E4M3 block scale is within one step of exact
    assert np.all(np.abs(v - c * d) <= (half_step + over + t * 2 ** -23) * d * (1 + 2 ** -20))
    assert np.all(np.abs(c[t > 6]) == 6.0)


def test_zero_row_zero_block_and_signed_zero():
    x = np.zeros((2, 64), dtype=np.float32)
    x[1, 16:32] = 1.0
    x[1, 0] = -0.0
    q, s, g = oracle.quant_nv(_bf16(x))
    assert g[0] == np.float32(1e-12) / np.float32(2688.0)  # the amax floor
    assert not q[0].any() and not s[0].any()
    assert s[1, 0] == 0 and s[1, 1] == 0x7E  # an all-zero block gets scale 0, its codes stay +-0
    codes = _unpack(q)
    assert codes[1, 0] == 0x8  # -0 keeps its sign
    assert (codes[1, 16:32] == 0x7).all()


@pytest.mark.parametrize("M,N,K", [(3, 17, 64), (1, 40, 256), (5, 8, 512)])
def test_nv_gemm_matches_brute_force(M, N, K):
    rng = np.random.default_rng(M * 100 + N)
    xb = _bf16(rng.standard_normal((M, K)))
    wb = _bf16(rng.standard_normal((N, K)) * 0.02)
    xq, sx, gx = oracle.quant_nv(xb)
    wq, sw, gw = oracle.quant_nv(wb)
    y, bound = oracle.gemm_nv(xq, sx, gx, wq, sw, gw)
    xd = _e2m1_values(_unpack(xq)) * np.repeat(_e4m3_values(sx), 16, axis=1) * gx.astype(np.float64)[:, None]
    wd = _e2m1_values(_unpack(wq)) * np.repeat(_e4m3_values(sw), 16, axis=1) * gw.astype(np.float64)[:, None]
    ref = xd @ wd.T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    np.testing.assert_allclose(bound, np.abs(xd) @ np.abs(wd).T, rtol=1e-12)
    # and the product approximates the bf16 inputs' product to NVFP4 accuracy
    exact = xb.double().numpy() @ wb.double().numpy().T
    assert np.abs(y - exact).max() <= 0.25 * np.abs(exact).max() + 0.1 * bound.max()


def test_nv_gemm_block_scales_belong_to_their_own_block():
    # one non-zero block per operand row; a scale read from the wrong block
    # (or a product over the wrong K block) changes the result
    K = 64
    x = np.zeros((1, K), dtype=np.float32)
    w = np.zeros((2, K), dtype=np.float32)
    x[0, 16:32] = np.linspace(0.5, 3.0, 16)
    x[0, 48:64] = 100.0
    w[0, 16:32] = 1.0
    w[1, 48:64] = -0.25
    xq, sx, gx = oracle.quant_nv(_bf16(x))
    wq, sw, gw = oracle.quant_nv(_bf16(w))
    y, _ = oracle.gemm_nv(xq, sx, gx, wq, sw, gw)
    xd = _e2m1_values(_unpack(xq)) * np.repeat(_e4m3_values(sx), 16, axis=1) * float(gx[0])
    wd = _e2m1_values(_unpack(wq)) * np.repeat(_e4m3_values(sw), 16, axis=1) * gw.astype(np.float64)[:, None]
    assert np.all(wd[0, 16:32] == wd[0, 16]) and np.all(wd[1, 48:64] == wd[1, 48])
    assert abs(y[0, 0] - xd[0, 16:32].sum() * wd[0, 16]) <= 1e-12 * abs(y[0, 0])
    assert abs(y[0, 1] - xd[0, 48:64].sum() * wd[1, 48]) <= 1e-12 * abs(y[0, 1])
    assert abs(wd[0, 16] - 1.0) < 1e-6 and abs(wd[1, 48] + 0.25) < 1e-6
