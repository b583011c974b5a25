"""The pins hold the oracle to the pages and to mathematics: show it.

Each case below plants one plausible mistake in a copy of oracle/oracle.c (a
wrong exponent bias, ties to odd, a lost sign of zero, a dropped term, a
wrong scale index, ...), compiles the copy on the CPU, swaps it in for the
real oracle and runs the pin tests.  At least one pin must fail for every
mutant; the unmodified source must pass them all.  Every mutant keeps its
memory accesses inside the same buffers, so a mutant can only compute the
wrong numbers, never crash the test process.
"""
import os

import pytest

import oracle
import test_oracle_codec as codec
import test_oracle_gemm as gemm
import test_oracle_mx as mx
import test_oracle_nv as nv
import test_oracle_quant as quant

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "exponent bias 8": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "subnormal exponent": ("v = ldexp((double)m / 8.0, 1 - 7);", "v = ldexp((double)m / 8.0, 0 - 7);"),
    "ties to odd": ("best = (lo & 1) ? hi : lo;", "best = (lo & 1) ? lo : hi;"),
    "ties away from zero": ("best = (lo & 1) ? hi : lo;", "best = hi;"),
    "saturation loses sign": ("return (uint8_t)(sign | 0x7E);", "return (uint8_t)0x7E;"),
    "sign of zero lost": ("sign = signbit(v) ? 0x80 : 0x00;", "sign = (v < 0) ? 0x80 : 0x00;"),
    "int8 half away from zero": ("if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0))",
                                 "if (frac >= 0.5)"),
    "int8 clamps to -128": ("if (r < -ORC_INT8_MAX)\n        r = -ORC_INT8_MAX;",
                            "if (r < -ORC_INT8_MAX - 1.0)\n        r = -ORC_INT8_MAX - 1.0;"),
    "no amax floor": ("if (amax < ORC_AMAX_FLOOR)\n        amax = ORC_AMAX_FLOOR;", ""),
    "reciprocal multiply": ("float v = div_rn_f32(bf16_to_float(x[r * pitch + k]), s);",
                            "float v = bf16_to_float(x[r * pitch + k]) * (1.0f / s);"),
    "int8 scale uses 448": ("double qmax = (qtype == ORC_E4M3) ? ORC_E4M3_MAX : ORC_INT8_MAX;",
                            "double qmax = ORC_E4M3_MAX;"),
    "dropped first term": ("for (k = k0; k < k1; k++) {", "for (k = k0 + 1; k < k1; k++) {"),
    "sign of first product": ("acc += p;", "acc += (k == k0) ? -p : p;"),
    "weight scale indexed by token": ("double scale = (double)sx[m] * (double)sw[n];",
                                      "double scale = (double)sx[m] * (double)sw[m];"),
    "e4m3 integer unit": ("return (int64_t)ldexp(orc_e4m3_decode(code), 9);",
                          "return (int64_t)ldexp(orc_e4m3_decode(code), 10);"),
    "block scale ignores K block": ("(double)sx[m * kbs + kb] * (double)sw[(n / G) * kbs + kb];",
                                    "(double)sx[m * kbs + kb] * (double)sw[(n / G) * kbs];"),
    "group offset": ("s[m * ng + g] = quant_group(x + m * K + g * G, 1, G, K, ORC_E4M3,",
                     "s[m * ng + g] = quant_group(x + m * K + g * (G / 2), 1, G, K, ORC_E4M3,"),
    "block row pitch": ("quant_group(w + nb * B * K + kb * B, B, B, K, ORC_E4M3,",
                        "quant_group(w + nb * B * K + kb * B, B, B, B, ORC_E4M3,"),
    "split chunk drops tail": ("if (k1 > K)\n            k1 = K;", "if (k1 >= K)\n            k1 = K - 1;"),
    "mx exponent off by one": ("ex = ex - 1 - 8;", "ex = ex - 8;"),
    "mx emax of 7": ("ex = ex - 1 - 8;", "ex = ex - 1 - 7;"),
    "mx zero block scale": ("        return -127;\n    frexp", "        return 0;\n    frexp"),
    "mx weight scale of the next block": ("(int)sw[n * nb + b] - 127);", "(int)sw[n * nb + (b + 1) % nb] - 127);"),
    "mx scales added to exponent bias once": ("double scale = ldexp(1.0, (int)sx[m * nb + b] - 127 +",
                                              "double scale = ldexp(1.0, (int)sx[m * nb + b] +"),
    "e2m1 exponent bias 2": ("v = ldexp(1.0 + (double)m / 2.0, e - 1);", "v = ldexp(1.0 + (double)m / 2.0, e - 2);"),
    "e2m1 ties to odd": ("best = (lo % 2 == 0) ? lo : hi;", "best = (lo % 2 == 0) ? hi : lo;"),
    "e2m1 saturation loses sign": ("return (uint8_t)(sign | 0x7);", "return (uint8_t)0x7;"),
    "nv row scale over 448": ("gr = div_rn_f32(amax, 2688.0f);", "gr = div_rn_f32(amax, 448.0f);"),
    "nv block maximum over half the block": (
        "for (k = 0; k < 16; k++) {\n                float a = fabsf(bf16_to_float(x[r * K + b * 16 + k]));",
        "for (k = 0; k < 8; k++) {\n                float a = fabsf(bf16_to_float(x[r * K + b * 16 + k]));"),
    # (the nibble order of the product alone is no mistake: swapping both
    # operands' pairs inside a block leaves every block sum unchanged)
    "nv nibble order of the codes": ("q[r * (K / 2) + i / 2] |= (uint8_t)((i & 1) ? (c << 4) : c);",
                                     "q[r * (K / 2) + i / 2] |= (uint8_t)((i & 1) ? c : (c << 4));"),
    "nv weight row scale dropped": ("double unit = ldexp((double)gx[m] * (double)gw[n], -20);",
                                    "double unit = ldexp((double)gx[m], -20);"),
    "nv weight block scale of the token": ("sc = e4m3_units(sx[m * nb + b]) * e4m3_units(sw[n * nb + b]);",
                                           "sc = e4m3_units(sx[m * nb + b]) * e4m3_units(sw[m * nb + b]);"),
}


def pin_suite():
    """The pins, run as plain calls; raises on the first that fails."""
    codec.test_decode_matches_spec_points()
    codec.test_decode_all_codes_match_torch()
    codec.test_round_trip_all_finite_codes()
    codec.test_midpoints_round_to_even_code()
    codec.test_saturation_nan_and_signed_zero()
    codec.test_encode_matches_torch_cast_in_range()
    codec.test_int8_encode_matches_rint_and_clamps()
    for qt in (oracle.E4M3, oracle.INT8):
        quant.test_rows_match_library_route(4, 1024, qt)
        gemm.test_rowscaled_matches_brute_force(3, 17, 96, qt)
        gemm.test_transpose_identity(qt)
        gemm.test_split_k_invariance(qt)
    quant.test_row_max_hits_top_code(oracle.E4M3, 0x7E)
    quant.test_row_max_hits_top_code(oracle.INT8, 127)
    quant.test_zero_row_and_signed_zero()
    quant.test_scale_one_row_exposes_codec_ties()
    quant.test_groups_equal_rows_of_reshaped_input()
    quant.test_blocks_equal_rows_of_permuted_input()
    gemm.test_blockscaled_matches_brute_force(3, 256, 384)
    gemm.test_identity_weight_returns_dequantized_activations()
    gemm.test_one_hot_rows_select_columns()
    gemm.test_zero_activation_row_gives_zero_output()
    mx.test_block_exponent_closed_form()
    mx.test_zero_block_and_exponent_clamp()
    mx.test_codes_match_torch_cast_of_scaled_values()
    mx.test_dequantized_error_within_half_an_e4m3_step()
    for shape in ((3, 17, 96), (1, 40, 256), (5, 8, 64)):
        mx.test_mx_gemm_matches_brute_force(*shape)
    mx.test_mx_gemm_scales_belong_to_their_own_block()
    nv.test_e2m1_decode_matches_spec_table()
    nv.test_e2m1_round_trip_midpoints_and_saturation()
    for seed in (1, 2):
        nv.test_row_and_block_scales_follow_ieee_fp32_and_torch_cast(seed)
        nv.test_row_maximum_lands_on_six_with_scale_448(seed + 2)
        nv.test_dequantized_error_within_half_an_e2m1_step(seed + 4)
    nv.test_zero_row_zero_block_and_signed_zero()
    for shape in ((3, 17, 64), (1, 40, 256), (5, 8, 512)):
        nv.test_nv_gemm_matches_brute_force(*shape)
    nv.test_nv_gemm_block_scales_belong_to_their_own_block()


@pytest.fixture
def swap_oracle():
    saved = oracle.lib()

    def use(path):
        oracle._lib = oracle.load_library(path)

    yield use
    oracle._lib = saved


def test_unmodified_oracle_passes_the_pin_suite():
    pin_suite()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_planted_mistake_is_caught(name, tmp_path, swap_oracle):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not found exactly once"
    mpath = tmp_path / "oracle_mutant.c"
    mpath.write_text(src.replace(old, new))
    so = oracle.compile_source(str(mpath), str(tmp_path / "liboracle_mutant.so"))
    swap_oracle(so)
    with pytest.raises(AssertionError):
        pin_suite()
