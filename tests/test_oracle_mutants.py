"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch each one.  The committed oracle is never modified: each mutant is a
text substitution compiled to a temporary library on the CPU, swapped in for
the duration of one test.
"""
import ctypes
import os
import subprocess
import tempfile

import pytest

import oracle
from tests import test_oracle_attention as att
from tests import test_oracle_layout as lay
from tests import test_oracle_numbers as num
from tests import test_oracle_quantizer as qz
from tests import test_oracle_rotation as rot
from tests import test_oracle_groups as grp

SRC = os.path.join(os.path.dirname(oracle.__file__), "kvq_oracle.c")

MUTANTS = {
    "truncate_instead_of_round": ("float r = nearbyintf(t);", "float r = floorf(t);"),
    "zero_from_max": ("mn = mn + 0.0f;", "mn = mx + 0.0f;"),
    "levels_off_by_one": ("float levels = (float)((1 << bits) - 1);",
                          "float levels = (float)(1 << bits);"),
    "no_negative_zero_fix": ("mn = mn + 0.0f; /* a -0 minimum becomes +0 */", ""),
    "no_negative_zero_fix_max": ("mx = mx + 0.0f; /* and so does a -0 maximum */", ""),
    "k_slice_index": ("int slice = (d % 8) / 2;", "int slice = d % 4;"),
    "v_half_swapped": ("int bit = 16 * (k % 2) + b * ((d / 8) % E);\n  int n",
                       "int bit = 16 * (1 - k % 2) + b * ((d / 8) % E);\n  int n"),
    "v_lane_transposed": ("int lane = 4 * (d % 8) + (k % 8) / 2;",
                          "int lane = (d % 8) + 8 * ((k % 8) / 2);"),
    "dequant_sign": ("out[d] = prod + zero;", "out[d] = prod - zero;"),
    "no_softmax_scale": ("s[t] = acc * sm_scale;", "s[t] = acc;"),
    # first occurrence: the packed-cache attention
    "gqa_modulo": ("int hq = h * gq + j;", "int hq = j * Hkv + h;"),
    "f16_ties_away": ("double n = nearbyint(a / spacing);", "double n = round(a / spacing);"),
    # key-only rotation
    "fwht_butterfly_swapped": ("        x[i] = a + b;\n        x[i + h] = a - b;",
                               "        x[i] = a - b;\n        x[i + h] = a + b;"),
    "rotated_query_not_divided": ("for (int d = 0; d < D; ++d) qd[d] /= (double)D;", ""),
    "keys_not_rotated": ("if (which == 0 && rotate_keys) ora_fwht(x, D);", ""),
    "values_rotated_too": ("if (which == 0 && rotate_keys) ora_fwht(x, D);",
                           "if (rotate_keys) ora_fwht(x, D);"),
    # separate key and value groups
    # (keys quantized with the values' coarser groups; writes stay inside the
    # key-parameter array, which is sized for the finer groups)
    "key_groups_from_values": ("int G = which == 0 ? Gk : Gv;", "int G = Gv;"),
}

PINS = [
    lambda o: num.test_f32_to_f16_edges(o, 2.0 ** -25),
    lambda o: num.test_f32_to_f16_edges(o, 2.5 * 2.0 ** -24),
    lambda o: num.test_f32_to_f16_random_patterns(o),
    lambda o: qz.test_exact_grid(o, 2),
    lambda o: qz.test_ties_round_half_even(o),
    lambda o: qz.test_negative_zero_minimum_is_canonical(o),
    lambda o: qz.test_signed_zero_extremes_give_positive_zero_params(o),
    lambda o: qz.test_codes_are_nearest_levels_exact_rationals(o, 4),
    lambda o: qz.test_cache_dequant_within_error_bound(o, 0, 4),
    lambda o: lay.test_k_row_fields_tile_the_row(o, 128, 4),
    lambda o: lay.test_k_rows_feed_score_fragments(o, 128, 4),
    lambda o: lay.test_v_tiles_feed_output_fragments(o, 128, 2),
    lambda o: att.test_single_token_returns_its_value(o),
    lambda o: att.test_brute_force_tiny(o, 3),
    lambda o: att.test_library_softmax_gqa(o, 4, 2, 64),
    lambda o: rot.test_fwht_is_the_sylvester_hadamard_product(o, 64),
    lambda o: rot.test_rotated_keys_dequantise_near_the_rotated_row(o),
    lambda o: rot.test_rotated_decode_matches_dense_attention_at_8_bits(o),
    lambda o: grp.test_each_array_uses_its_own_groups(o, 32, 128),
]


@pytest.fixture()
def mutant_lib(ora, request):
    old, new = MUTANTS[request.param]
    src = open(SRC).read()
    assert src.count(old) >= 1, request.param
    tmp = tempfile.mkdtemp()
    c_path = os.path.join(tmp, "m.c")
    so_path = os.path.join(tmp, "m.so")
    open(c_path, "w").write(src.replace(old, new, 1))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           c_path, "-o", so_path, "-lm"])
    saved = ora._lib
    ora._lib = ora._load(so_path)
    yield ora
    ora._lib = saved


@pytest.mark.parametrize("mutant_lib", sorted(MUTANTS), indirect=True)
def test_some_pin_catches_the_mutant(mutant_lib):
    caught = 0
    for pin in PINS:
        try:
            pin(mutant_lib)
        except AssertionError:
            caught += 1
    assert caught > 0
