"""Plant plausible mistakes in copies of the oracle's C source (on the CPU) and
require every one to be caught by at least one pin.  This shows the pins would
notice a dropped term, a wrong sign or index, a transposed operand, a reversed
tie rule or order, a broken inverse permutation or a wrong gate slot."""
import os
import shutil

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "silu_sign": ("a / (1.0 + exp(-a))", "a / (1.0 + exp(a))"),
    "gate_up_swapped": ("a[i] = silu(sg) * su;", "a[i] = silu(su) * sg;"),
    "tie_to_higher_index": ("l[e] > l[best]", "l[e] >= l[best]"),
    "router_transposed": ("wr[(size_t)h * E + e]", "wr[(size_t)e * H + h]"),
    "bias_dropped": ("acc = acc + bias[e];", "acc = acc;"),
    "softmax_short_sum": ("for (int j = 0; j < k; ++j) s += exp",
                          "for (int j = 0; j < k - 1; ++j) s += exp"),
    "down_transposed": ("d[(size_t)o * I + i]", "d[(size_t)i * H + o]"),
    "inverse_perm_wrong": ("flat_to_sorted[f] = pos;", "flat_to_sorted[f] = f;"),
    "ffn_dropped_term": ("        for (int h = 0; h < H; ++h) {\n            sg +=",
                         "        for (int h = 1; h < H; ++h) {\n            sg +="),
    "combine_wrong_gate_slot": ("double g = j->gate[(size_t)t * j->k + q];",
                                "double g = j->gate[(size_t)t * j->k];"),
    "router_order_reversed": ("        for (int h = 0; h < H; ++h) {\n            float a",
                              "        for (int h = H - 1; h >= 0; --h) {\n            float a"),
    "tile_rows_not_clipped": ("(c - r) < bm ? (c - r) : bm", "bm"),
    "permute_offsets_shifted": ("offsets[e] = pos;", "offsets[e] = pos + (e > 0);"),
    "e4m3_tie_away": ("(d == bd && (c & 1) == 0 && (best & 1) == 1)", "(d == bd && c > best)"),
    "fp8_scale_transposed": ("sb[(size_t)(n / 128) * KB + kb]", "sb[(size_t)kb * (N / 128) + n / 128]"),
    "fp8_act_scale_dropped": ("acc += (double)sa[kb] * (double)sb", "acc += (double)sb"),
    "fp8_amax_448_off": ("float s = amax / 448.0f;", "float s = amax / 440.0f;"),
    "fp8_h_not_requantised": ("fp8_row_gemm(H, I, qh, sh,", "fp8_row_gemm(H, I, qh, sx,"),
    "shared_gate_up_swapped": ("expert_ffn(j->H, j->I, 0, xt, j->wg, j->wu, j->wd,",
                               "expert_ffn(j->H, j->I, 0, xt, j->wu, j->wg, j->wd,"),
    "mx_tie_away": ("(d == bd && !(c & 1) && (best & 1))", "(d == bd && c > best)"),
    "mx_scale_exponent_off": ("int X = ex - 1 - emax;", "int X = ex - emax;"),
    "mx_act_scale_dropped": ("acc += ldexp(1.0, (int)xa[kb] - 127) * ldexp", "acc += ldexp"),
    "mx_h_wrong_format": ("oracle_mx_quantize_rows(1, I, h, MX_E4M3, qh, sh);",
                          "oracle_mx_quantize_rows(1, I, h, MX_E2M1, qh, sh);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = open(oracle.SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique/present"
    msrc = tmp_path / "moe_oracle_mutant.c"
    msrc.write_text(src.replace(old, new))
    lib = oracle.build(str(msrc), str(tmp_path / "libmutant.so"), force=True)
    orc = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
