"""Planted mistakes in copies of the oracle must each fail at least one pin.

Every mutant is a plausible slip (a swapped operand, a dropped term, a wrong sign,
an unstable order, a missing pad) that stays inside its buffers. The copies are
compiled to a temporary directory; the real oracle is never touched.
"""
import os

import pytest

import oracle
import oracle_pins as P

SRC = open(oracle.SRC).read()

MUTANTS = {
    "gate_up_swapped": (
        "g[n] += xh * bf16_to_double(w[n]);\n      u[n] += xh * bf16_to_double(w[I + n]);",
        "g[n] += xh * bf16_to_double(w[I + n]);\n      u[n] += xh * bf16_to_double(w[n]);"),
    "silu_sign": ("return v / (1.0 + exp(-v));", "return v / (1.0 + exp(v));"),
    "sigmoid_not_silu": ("return v / (1.0 + exp(-v));", "return 1.0 / (1.0 + exp(-v));"),
    "routing_weight_dropped": ("yt[m] += w * z[m];", "yt[m] += z[m];"),
    "preactivation_into_w2": ("z[m] += a[n] * bf16_to_double(w[m]);",
                              "z[m] += g[n] * bf16_to_double(w[m]);"),
    "up_not_multiplied": ("a[n] = silu(g[n]) * u[n];", "a[n] = silu(g[n]);"),
    "plan_unstable_order": (
        "  for (int64_t f = 0; f < pairs; ++f) {\n    int32_t e = topk_idx[f];\n    if (e < 0) {",
        "  for (int64_t f = pairs - 1; f >= 0; --f) {\n    int32_t e = topk_idx[f];\n    if (e < 0) {"),
    "plan_no_padding": ("offsets[e + 1] = offsets[e] + (int32_t)round_up(counts[e], tile);",
                        "offsets[e + 1] = offsets[e] + counts[e];"),
    "pool_padding_not_zero": ("(f >= 0) ? x[(int64_t)(f / k) * H + h] : (uint16_t)0;",
                              "(f >= 0) ? x[(int64_t)(f / k) * H + h] : x[h];"),
    "pool_wrong_token": ("x[(int64_t)(f / k) * H + h]", "x[(int64_t)(f % (k > 1 ? k : 1)) * H + h]"),
    "combine_skips_first": (
        "for (int32_t j = 0; j < k; ++j) {\n        int32_t p = pool_row[t * k + j];",
        "for (int32_t j = 1; j < k; ++j) {\n        int32_t p = pool_row[t * k + j];"),
    "identity_counts_dropped": ("if (topk_idx[t * k + j] >= 0)\n          acc +=", "acc +="),
    "bad_index_accepted": ("if (e < -1 || e >= E) return ORACLE_ERR_BAD_INDEX;\n  }\n  for (int32_t e = 0; e < E; ++e) counts[e] = 0;",
                           "if (e < -1 || e >= E) e = 0;\n  }\n  for (int32_t e = 0; e < E; ++e) counts[e] = 0;"),
    "route_tie_to_higher_index": ("if (!taken[e] && (best < 0 || v[e] > v[best])) best = e;",
                                  "if (!taken[e] && (best < 0 || v[e] >= v[best])) best = e;"),
    "route_no_renorm": ("for (int32_t j = 0; j < k; ++j) w[t * k + j] /= sum;",
                        "for (int32_t j = 0; j < k; ++j) w[t * k + j] /= sum + 1.0;"),
    "route_smallest_first": ("if (!taken[e] && (best < 0 || v[e] > v[best])) best = e;",
                             "if (!taken[e] && (best < 0 || v[e] < v[best])) best = e;"),
    "route_bias_ignored": ("v[e] = bias ? logits[t * E + e] + bias[e] : logits[t * E + e];",
                           "v[e] = logits[t * E + e];"),
    "bwd_silu_grad_is_sigmoid": ("return s * (1.0 + v * (1.0 - s));", "return s;"),
    "bwd_dg_du_swapped": (
        "acc += bf16_to_double(w1[q]) * dg[q] + bf16_to_double(w1[I + q]) * du[q];",
        "acc += bf16_to_double(w1[q]) * du[q] + bf16_to_double(w1[I + q]) * dg[q];"),
    "bwd_routing_weight_not_applied": ("dz[m] = w * dym;", "dz[m] = dym;"),
    "bwd_dw_weighted": ("s += dym * z[m];", "s += w * dym * z[m];"),
    "bwd_w2_transposed": ("          for (int32_t m = 0; m < H; ++m) da += bf16_to_double(w2[m]) * dz[m];",
                          "          for (int32_t m = 0; m < H; ++m) da += bf16_to_double(W2[e][(int64_t)m * I + q]) * dz[m];"),
    "bwd_du_uses_gate_only": ("          du[q] = da * silu(g[q]);", "          du[q] = da * g[q];"),
    "wgrad_w2_transposed": ("\n      for (int32_t m = 0; m < H; ++m) da += bf16_to_double(w2[m]) * dz[m];",
                            "\n      for (int32_t m = 0; m < H; ++m) da += bf16_to_double(W2e[(int64_t)m * I + q]) * dz[m];"),
    "wgrad_du_uses_gate_only": ("\n      du[q] = da * silu(g[q]);", "\n      du[q] = da * g[q];"),
    "wgrad_gate_up_swapped": ("row[q] += xh * dg[q];\n        row[I + q] += xh * du[q];",
                              "row[q] += xh * du[q];\n        row[I + q] += xh * dg[q];"),
    "wgrad_w2_no_routing_weight": (
        "for (int32_t m = 0; m < H; ++m) dz[m] = w * bf16_to_double(dy[t * H + m]);",
        "for (int32_t m = 0; m < H; ++m) dz[m] = bf16_to_double(dy[t * H + m]);"),
    "wgrad_w2_uses_preactivation": ("for (int32_t m = 0; m < H; ++m) row[m] += a[q] * dz[m];",
                                    "for (int32_t m = 0; m < H; ++m) row[m] += g[q] * dz[m];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(name, tmp_path):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation site for {name} not unique"
    src = tmp_path / f"{name}.c"
    src.write_text(SRC.replace(old, new))
    lib = oracle.build(str(src), str(tmp_path / f"lib{name}.so"))
    mut = oracle.Oracle(lib)
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin(mut)
        except (AssertionError, oracle.OracleError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
