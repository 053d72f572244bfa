"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check
that the pins catch every one of them.

Each mutant is the oracle's C source with one textual change, built into a
temporary directory; the committed oracle is never modified."""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "k3moe_oracle.c")

MUTANTS = {
    "nibble_order": ("unsigned code = (c & 1) ? (byte >> 4) : (byte & 0xFu);",
                     "unsigned code = (c & 1) ? (byte & 0xFu) : (byte >> 4);"),
    "e2m1_table": ("{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}",
                   "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0}"),
    "e2m1_sign": ("return (nib & 8u) ? -v : v;", "return v;"),
    "e8m0_bias": ("(int)(e & 0xFFu) - 127", "(int)(e & 0xFFu) - 128"),
    "scale_block": ("scale[r * (cols / 32) + c / 32]", "scale[r * (cols / 32) + c / 64]"),
    "silu_on_up": ("g[i] = silu(g[i]) * u[i];\n    oracle_mxfp4_matvec(p[4]",
                   "g[i] = g[i] * silu(u[i]);\n    oracle_mxfp4_matvec(p[4]"),
    "gate_up_swapped": ("oracle_mxfp4_matvec(p[0], p[1], ff, d, xv, g);\n"
                        "    oracle_mxfp4_matvec(p[2], p[3], ff, d, xv, u);",
                        "oracle_mxfp4_matvec(p[2], p[3], ff, d, xv, g);\n"
                        "    oracle_mxfp4_matvec(p[0], p[1], ff, d, xv, u);"),
    "softmax_unnormalised": ("p[e] = exp(l[e] - m) / z;", "p[e] = exp(l[e] - m);"),
    "topk_ties_high": ("return (i > j) - (i < j);", "return (i < j) - (i > j);"),
    "topk_ascending": ("if (li > lj) return -1;\n    if (li < lj) return 1;",
                       "if (li < lj) return -1;\n    if (li > lj) return 1;"),
    "combine_wrong_slot_weight": ("double w = weight[t * k + s];", "double w = weight[t * k];"),
    "bias_ignored": ("if (bias) s += (double)bias[e];", ""),
    "shared_dropped": ("if (wg && wu && wd && ffs > 0)", "if (0)"),
    "router_token0_only": ("s += oracle_bf16_value(x[t * d + j]) * (double)w[e * d + j];",
                           "s += oracle_bf16_value(x[j]) * (double)w[e * d + j];"),
    "down_scale_rows": ("oracle_mxfp4_matvec(p[4], p[5], d, ff, g, out);",
                        "oracle_mxfp4_matvec(p[4], p[3], d, ff, g, out);"),
    # routing variants, RMSNorm, residual add
    "renorm_unscaled": ("weight[t * k + j] = renorm ? pj / z : pj;", "weight[t * k + j] = pj;"),
    "select_bias_in_softmax": ("oracle_router_logits(x, T, w, bias_select_only ? NULL : bias, d, E, l);",
                               "oracle_router_logits(x, T, w, bias, d, E, l);"),
    "select_bias_ignored": ("sel[e] = lt[e] + ((bias_select_only && bias) ? (double)bias[e] : 0.0);",
                            "sel[e] = lt[e];"),
    "rmsnorm_sum_not_mean": ("const double r = 1.0 / sqrt(ss / (double)d + eps);",
                             "const double r = 1.0 / sqrt(ss + eps);"),
    "rmsnorm_eps_outside": ("const double r = 1.0 / sqrt(ss / (double)d + eps);",
                            "const double r = 1.0 / sqrt(ss / (double)d) + eps;"),
    "rmsnorm_no_weight": ("oracle_bf16_rne(oracle_bf16_value(h[t * d + j]) * r * oracle_bf16_value(g[j]));",
                          "oracle_bf16_rne(oracle_bf16_value(h[t * d + j]) * r);"),
    "residual_dropped": ("out[i] = oracle_bf16_value(h[i]) + y[i];", "out[i] = y[i];"),
}

BATTERY = [
    pins.test_e2m1_all_codes, pins.test_e8m0_scales, pins.test_mxfp4_element_layout,
    pins.test_mxfp4_matvec_exact_bruteforce, pins.test_router_logits_exact_bruteforce,
    pins.test_softmax_closed_forms, pins.test_topk_bruteforce_random_and_ties,
    pins.test_routing_worked_example, pins.test_expert_ffn_worked_example,
    pins.test_scale_plus_one_doubles, pins.test_layer_k1_no_shared_is_single_expert,
    pins.test_layer_k_equals_E_is_full_mixture, pins.test_layer_shared_only_adds,
    pins.test_bias_shifts_routing,
    lambda o: pins.test_torch_fp64_second_opinion(o, "tiny"),
    lambda o: pins.test_torch_fp64_second_opinion(o, "small_bias"),
    pins.test_route_variants_closed_forms, pins.test_route_variants_selection_ties_go_to_lower_index,
    pins.test_route_variants_invariants, pins.test_rmsnorm_worked_example,
    pins.test_rmsnorm_constant_token_gives_the_weights, pins.test_rmsnorm_scale_invariance_and_eps,
    pins.test_residual_add,
]


def _build_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/absent"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                           "-std=c11", "-o", str(lib), str(path), "-lm"])
    return oracle.Oracle(oracle.load(str(lib)))


def test_unmutated_passes_battery():
    o = oracle.oracle()
    for check in BATTERY:
        check(o)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    mut = _build_mutant(tmp_path, name)
    failures = 0
    for check in BATTERY:
        try:
            check(mut)
        except AssertionError:
            failures += 1
    assert failures > 0, f"mutant {name} survived every pin"
