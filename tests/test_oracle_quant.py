"""Pins for the oracle's dynamic quantizers (CPU only).

Checked against torch's CPU float8 cast / round applied to a separately
computed scale, against the invariant that the largest-magnitude element
lands exactly on the largest code, and against reshaping identities that
tie the group and block layouts to the per-row one.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_gemm_decode_b200 import synth


def torch_rows(x: torch.Tensor, qmax: float, as_int8: bool):
    """Library route: fp32 amax, fp32 divide, torch cast (RNE)."""
    xf = x.float()
    amax = xf.abs().amax(dim=-1, keepdim=True).clamp_min(torch.tensor(1e-12, dtype=torch.float32))
    s = amax / torch.tensor(qmax, dtype=torch.float32)
    v = xf / s
    if as_int8:
        q = torch.round(v).clamp(-127, 127).to(torch.int8).numpy()
    else:
        q = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return q, s.squeeze(-1).numpy()


@pytest.mark.parametrize("M,K", [(1, 128), (4, 1024), (7, 4096), (3, 5120)])
@pytest.mark.parametrize("qtype", [oracle.E4M3, oracle.INT8])
def test_rows_match_library_route(M, K, qtype):
    x = synth.activations(M, K, seed=M * 31 + K, outliers=True)
    q, s = oracle.quant_rows(x, qtype)
    rq, rs = torch_rows(x, 448.0 if qtype == oracle.E4M3 else 127.0, qtype == oracle.INT8)
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(q.view(np.uint8), rq.view(np.uint8))


@pytest.mark.parametrize("qtype,top", [(oracle.E4M3, 0x7E), (oracle.INT8, 127)])
def test_row_max_hits_top_code(qtype, top):
    x = synth.activations(16, 2048, seed=5, outliers=False)
    q, _ = oracle.quant_rows(x, qtype)
    xf = x.float().numpy()
    idx = np.abs(xf).argmax(axis=1)
    for m in range(16):
        code = int(q[m, idx[m]].view(np.uint8)) if qtype == oracle.E4M3 else int(q[m, idx[m]])
        if qtype == oracle.E4M3:
            assert code & 0x7F == top and (code >> 7) == (xf[m, idx[m]] < 0)
        else:
            assert abs(code) == top and (code < 0) == (xf[m, idx[m]] < 0)


def test_zero_row_and_signed_zero():
    x = torch.zeros(3, 256, dtype=torch.bfloat16)
    x[1, 5] = -0.0
    x[2] = -0.0
    q, s = oracle.quant_rows(x, oracle.E4M3)
    expect_s = np.float32(np.float32(1e-12) / np.float32(448.0))
    assert np.all(s == expect_s)
    assert np.all(q[0] == 0)
    assert q[1, 5] == 0x80 and np.all(np.delete(q[1], 5) == 0)
    assert np.all(q[2] == 0x80)
    qi, si = oracle.quant_rows(x, oracle.INT8)
    assert np.all(qi == 0)


def test_scale_one_row_exposes_codec_ties():
    # amax = 448 makes the scale exactly 1, so each code is E(x) itself:
    # midpoints must round to the even code.
    vals = [448.0, 1.0625, 1.1875, 3 * 2.0 ** -10, 2.0 ** -10, -1.0625, 8.5, 9.5, 15.5]
    x = torch.tensor([vals], dtype=torch.bfloat16)
    q, s = oracle.quant_rows(x, oracle.E4M3)
    assert s[0] == 1.0
    assert list(q[0]) == [0x7E, 0x38, 0x3A, 0x02, 0x00, 0xB8, 0x50, 0x52, 0x58]


def test_groups_equal_rows_of_reshaped_input():
    M, K = 5, 1024
    x = synth.activations(M, K, seed=3, outliers=True)
    q, s = oracle.quant_groups(x, 128)
    xr = x.reshape(M * K // 128, 128)
    rq, rs = torch_rows(xr, 448.0, False)
    np.testing.assert_array_equal(s.reshape(-1), rs)
    np.testing.assert_array_equal(q.reshape(-1, 128), rq)


def test_blocks_equal_rows_of_permuted_input():
    N, K, B = 256, 384, 128
    w = synth.weights(N, K, seed=9)
    q, s = oracle.quant_blocks(w, B)
    # gather each B x B block into one row of B*B values
    blocks = w.reshape(N // B, B, K // B, B).permute(0, 2, 1, 3).reshape(-1, B * B)
    rq, rs = torch_rows(blocks, 448.0, False)
    np.testing.assert_array_equal(s.reshape(-1), rs)
    qb = q.reshape(N // B, B, K // B, B).transpose(0, 2, 1, 3).reshape(-1, B * B)
    np.testing.assert_array_equal(qb, rq)
