"""Pins for the oracle's e4m3 and int8 codecs (CPU only).

The oracle's codecs are written from the format definition.  Here they are
held against things other than themselves: the OCP FP8 specification's named
values (tests/golden/e4m3_codes.txt), torch's independent CPU float8 cast,
numpy's round-half-even, and properties every correct nearest-even encoder
has (round trip, midpoints, saturation, signed zero).
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_codes.txt")


def torch_decode(code: int) -> float:
    return float(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64))


def test_decode_matches_spec_points():
    with open(GOLDEN) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(rows) >= 10
    for code, value in rows:
        got = oracle.e4m3_decode(int(code, 16))
        assert got == float(value), (code, got, value)
        assert np.signbit(got) == np.signbit(float(value)), code


def test_decode_all_codes_match_torch():
    for c in range(256):
        ours = oracle.e4m3_decode(c)
        ref = torch_decode(c)
        if c in (0x7F, 0xFF):
            assert np.isnan(ours) and np.isnan(ref)
        else:
            assert ours == ref, (hex(c), ours, ref)
            assert np.signbit(ours) == np.signbit(ref), hex(c)


def test_round_trip_all_finite_codes():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c, hex(c)


def test_midpoints_round_to_even_code():
    for sign in (0x00, 0x80):
        for c in range(0, 0x7E):
            lo = oracle.e4m3_decode(sign | c)
            hi = oracle.e4m3_decode(sign | (c + 1))
            mid = (lo + hi) / 2.0
            want = c if c % 2 == 0 else c + 1
            got = oracle.e4m3_encode(mid)
            assert got == (sign | want), (hex(c), mid, hex(got))
            # just off the midpoint goes to the nearer neighbour
            eps = (hi - lo) * 1e-6
            assert oracle.e4m3_encode(mid - np.copysign(eps, mid)) == (sign | c)
            assert oracle.e4m3_encode(mid + np.copysign(eps, mid)) == (sign | (c + 1))


def test_saturation_nan_and_signed_zero():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(448.0 * (1 + 2 ** -10)) == 0x7E
    assert oracle.e4m3_encode(464.0) == 0x7E
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(-500.0) == 0xFE
    assert oracle.e4m3_encode(float("nan")) == 0x7F
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(1e-30) == 0x00
    assert oracle.e4m3_encode(-1e-30) == 0x80
    # half the smallest subnormal ties to zero (even); just above it rounds up
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00
    assert oracle.e4m3_encode(2.0 ** -10 * 1.0001) == 0x01


def test_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(7)
    # log-uniform magnitudes across the whole e4m3 range, both signs
    mags = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), size=20000))
    vals = (mags * rng.choice([-1.0, 1.0], size=mags.shape)).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_encode(float(v)) for v in vals], dtype=np.uint8)
    np.testing.assert_array_equal(ours, ref)


def test_int8_encode_matches_rint_and_clamps():
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.uniform(-127.4, 127.4, size=5000),
        np.arange(-127, 127) + 0.5,  # every tie
        np.array([-0.5, 0.5, -1.5, 1.5, -126.5, 126.5]),
    ]).astype(np.float32)
    ours = np.array([oracle.int8_encode(float(v)) for v in vals], dtype=np.int8)
    np.testing.assert_array_equal(ours, np.rint(vals).astype(np.int8))
    assert oracle.int8_encode(127.6) == 127
    assert oracle.int8_encode(300.0) == 127
    assert oracle.int8_encode(-300.0) == -127
    assert oracle.int8_encode(-127.5) == -127


@pytest.mark.parametrize("K", [1024, 4096, 5120, 8192, 12288, 17408, 25600])
def test_int8_accumulator_fits_int32(K):
    # |sum_k q_x q_w| <= 127^2 K must stay below 2^31 for every K the
    # workloads use, so a signed 32-bit accumulator is exact.
    assert 127 * 127 * K < 2 ** 31
