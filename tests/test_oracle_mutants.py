"""Planted-mistake controls for the oracle's pins (CPU only).

Each case copies ``oracle/oracle.c``, plants one plausible mistake (a dropped
term, a wrong sign, index or operand, a broken tie rule), builds it, and runs
the pins against that build.  At least one pin must fail for every mutant;
otherwise the pins would not be able to tell that mistake from the method.
"""
import os

import pytest

import oracle
import test_oracle_codec as codec
import test_oracle_ffn as ffn
import test_oracle_mx as mx
import test_oracle_route as route

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "decode_subnormal_exponent": ("m * ldexp(1.0, -9)", "m * ldexp(1.0, -10)"),
    "decode_nan_policy": ("mag = 0.0;                         /* NaN", "mag = NAN;                         /* NaN"),
    "decode_bias": ("ldexp(1.0, e - 7)", "ldexp(1.0, e - 8)"),
    "encode_ties_to_odd": ("(c & 1) == 0 && (best & 1) == 1", "(c & 1) == 1 && (best & 1) == 0"),
    "encode_no_saturation": ("if (a >= 448.0) return (uint8_t)(0x7E | (neg << 7));", ""),
    "quant_wrong_max": ("amax / 448.0f", "amax / 447.0f"),
    "quant_zero_scale_rule": ("if (sv == 0.0f) sv = 1.0f;", "if (sv == 0.0f) sv = 2.0f;"),
    "route_tie_to_higher_id": ("l[e] > l[best]", "l[e] >= l[best]"),
    "route_weights_not_normalised": ("/ den;", "/ (den + 1.0);"),
    "route_nan_selectable": ("return !isnan(v) && !(isinf(v) && v < 0);", "return !(isinf(v) && v < 0);"),
    "permute_unstable": ("sorted_pairs[next[e]++] = (int32_t)p;",
                         "sorted_pairs[offsets[e + 1] - 1 - (next[e]++ - offsets[e])] = (int32_t)p;"),
    "ffn_gate_scale_dropped": ("dec[Wg[n * H + kk]] * (double)Sg[(n / 128) * GH + kk / 128]", "dec[Wg[n * H + kk]]"),
    "ffn_act_scale_dropped": ("* (double)act_scales[t * GH + kk / 128]", "* 1.0"),
    "ffn_silu_sign": ("double h64 = g / (1.0 + exp(-g)) * u;", "double h64 = g / (1.0 + exp(g)) * u;"),
    "ffn_clamped_silu": ("double h64 = g / (1.0 + exp(-g)) * u;",
                         "double h64 = g / (1.0 + exp(-g)) * (u > 10 ? 10 : u < -10 ? -10 : u);"),
    "ffn_up_gate_swapped": ("* u;\n", "* g;\n"),
    "ffn_no_requant": ("for (int64_t i = 0; i < I; ++i) hd[i] = dec[hq_use[i]] * (double)sh_use[i / 128];",
                       "for (int64_t i = 0; i < I; ++i) hd[i] = h_override_codes ? dec[hq_use[i]] * (double)sh_use[i / 128] : (double)h32[i];"),
    "ffn_down_transposed": ("acc += hd[i] * (dec[Wd[n * I + i]] * (double)", "acc += hd[i] * (dec[Wd[i * H + n]] * (double)"),
    "ffn_down_scale_index": ("Sd[(n / 128) * GI + i / 128]", "Sd[(n / 128) * GI]"),
    "ffn_routing_weight_dropped": ("orow[n] += wj * o[n];", "orow[n] += o[n];"),
    "ffn_routed_scaling_dropped": ("orow[n] *= routed_scaling;\n        }\n        free(xd);\n        free(o);",
                                   "orow[n] *= 1.0;\n        }\n        free(xd);\n        free(o);"),
    "ffn_last_group_full_width": ("int64_t nc = (I - c0 < 128) ? (I - c0) : 128;", "int64_t nc = 128;"),
    # the MXFP8 variant
    "mx_ue8m0_bias": ("return ldexp(1.0, (int)x - 127);", "return ldexp(1.0, (int)x - 128);"),
    "mx_shared_exponent_off_by_one": ("se = (ex - 1) - 8;", "se = (ex - 1) - 7;"),
    "mx_weight_scale_dropped": ("g += xd[kk] * (dec[Wg[n * H + kk]] * sdec[Sg[n * BH + kk / 32]]);",
                                "g += xd[kk] * (dec[Wg[n * H + kk]]);"),
    "mx_block_of_64": ("sdec[act_scales[t * BH + kk / 32]]", "sdec[act_scales[t * BH + kk / 64]]"),
    "mx_no_requant": ("hd[i] = dec[hq[i]] * sdec[sh[i / 32]];", "hd[i] = (double)h32[i];"),
    "mx_zero_block_scale": ("if (amax == 0.0) {\n        se = -127;", "if (amax == 0.0) {\n        se = 0;"),
}

PINS = [
    (codec.test_decode_page_rules_golden, ()),
    (codec.test_decode_exhaustive_vs_torch_float8, ()),
    (codec.test_encode_midpoints_ties_to_even, ()),
    (codec.test_encode_special_values, ()),
    (codec.test_quant_group_zero_and_nonfinite, ()),
    (codec.test_quant_group_partial_and_tiny, ()),
    (codec.test_quant_act_vs_torch_ops, ()),
    (route.test_route_vs_full_sort, ("tiny",)),
    (route.test_route_special_logits, ()),
    (route.test_permute_vs_stable_argsort, (300, 8, 64)),
    (ffn.test_ffn_vs_dense_bruteforce, ("i192",)),
    (ffn.test_ffn_vs_dense_bruteforce, ("i320",)),
    (ffn.test_ffn_exact_integer_gate_up, ()),
    (ffn.test_ffn_invariants, ()),
    (ffn.test_ffn_nan_stays_in_its_row, ()),
    (mx.test_ue8m0_decode_exhaustive, ()),
    (mx.test_block_power_of_two_max, (3,)),
    (mx.test_block_zero_and_nonfinite, ()),
    (mx.test_block_vs_torch_restatement, ()),
    (mx.test_mx_layer_vs_dense_bruteforce, ("tiny",)),
]


def test_unmutated_source_passes_all_pins(tmp_path):
    lib = oracle.open_library(oracle.build(force=True, src=SRC, out=str(tmp_path / "same.so")))
    with oracle.using(lib):
        for fn, args in PINS:
            fn(*args)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique in oracle.c"
    mpath = tmp_path / f"{name}.c"
    mpath.write_text(src.replace(old, new))
    lib = oracle.open_library(oracle.build(force=True, src=str(mpath), out=str(tmp_path / f"{name}.so")))
    caught = []
    with oracle.using(lib):
        for fn, args in PINS:
            try:
                fn(*args)
            except AssertionError:
                caught.append(fn.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
