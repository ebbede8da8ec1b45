"""Plant plausible mistakes in copies of the oracle and check that a pin catches each.

Every mutant is a textual edit of moe_oracle.c (at every occurrence of its
site) compiled into a temporary
library on the CPU; the real oracle is never modified.  A mutant that passes
every pin would mean the pins cannot tell that mistake from the definition.
"""

import os
import subprocess
import tempfile

import pytest

import oracle
from tests import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

MUTANTS = {
    "gate_and_up_swapped": ("h[r] = g / (1.0 + exp(-g)) * u;", "h[r] = u / (1.0 + exp(-u)) * g;"),
    "silu_sign": ("h[r] = g / (1.0 + exp(-g)) * u;", "h[r] = g / (1.0 + exp(g)) * u;"),
    "silu_dropped": ("h[r] = g / (1.0 + exp(-g)) * u;", "h[r] = g * u;"),
    "down_proj_transposed": ("z += bf16_value(W2[c * f + r]) * h[r];", "z += bf16_value(W2[r * d + c]) * h[r];"),
    "gate_weight_dropped": ("y[c] += gate * z;", "y[c] += z;"),
    "bias_dropped": ("s += (double)bias[e];", "s += 0.0;"),
    "widening_shift": ("uint32_t u = (uint32_t)bits << 16;", "uint32_t u = (uint32_t)bits << 15;"),
    "tie_to_higher_index": ("return ia < ib;", "return ia > ib;"),
    "nan_ranks_first": ("return bn;          /* the non-NaN one ranks first */", "return an;"),
    "gates_unnormalised": ("w[t * k + j] = exp((double)row[idx[t * k + j]] - top) / z;",
                           "w[t * k + j] = exp((double)row[idx[t * k + j]] - top);"),
    "permutation_unstable": ("for (int64_t q = 0; q < P; q++) {      /* ascending q keeps each segment stable */",
                             "for (int64_t q = P - 1; q >= 0; q--) {"),
    "shared_expert_dropped": ("if (J->fs > 0)\n            expert_ffn_add", "if (0)\n            expert_ffn_add"),
    "up_uses_gate_weights": ("u += bf16_value(W3[r * d + c]) * xc;", "u += bf16_value(W1[r * d + c]) * xc;"),
    "gate_proj_transposed": ("g += bf16_value(W1[r * d + c]) * xc;", "g += bf16_value(W1[c * f + r]) * xc;"),
    "shared_expert_gated": ("expert_ffn_add(J->Ws1, J->Ws3, J->Ws2, xt, J->d, J->fs, 1.0, h, y);",
                            "expert_ffn_add(J->Ws1, J->Ws3, J->Ws2, xt, J->d, J->fs, J->w[t * J->k], h, y);"),
    "gate_of_first_pair_for_all": ("J->f, J->w[t * J->k + j], h, y);", "J->f, J->w[t * J->k], h, y);"),
    "router_weights_transposed": ("s += bf16_value(x[t * d + c]) * bf16_value(Wg[e * d + c]);",
                                  "s += bf16_value(x[t * d + c]) * bf16_value(Wg[c * E + e]);"),
    "bias_subtracted": ("s += (double)bias[e];", "s -= (double)bias[e];"),
    "perm_holds_token_not_pair": ("perm[pos] = (int32_t)q;", "perm[pos] = (int32_t)(q / k * k);"),
    "inv_perm_is_perm": ("inv_perm[q] = pos;", "inv_perm[q] = (int32_t)q;"),
    "x_row_stride": ("const uint16_t *xt = J->x + t * J->d;", "const uint16_t *xt = J->x + t;"),
    "fp8_h_requant_dropped": ("h[r] = e4m3_value(hq[r]) * sh[r / 128];", "h[r] = h[r];"),
    "fp8_h_scale_not_stored": ("sh[b] = sc;", "sh[b] = 1.0;"),
    "fp8_h_codes_unscaled": ("hq[b * 128 + r] = oracle_e4m3_encode_fast(h[b * 128 + r] / sc);",
                             "hq[b * 128 + r] = oracle_e4m3_encode_fast(h[b * 128 + r]);"),
    "fp8_weight_scale_transposed": ("g += e4m3_value(W1q[r * d + c]) * s1[(r / 128) * db + c / 128] * xc;",
                                    "g += e4m3_value(W1q[r * d + c]) * s1[(c / 128) * db + r / 128] * xc;"),
    "fp8_ties_away_from_zero": ("double m = nearbyint((2.0 * frac - 1.0) * 8.0);",
                                "double m = round((2.0 * frac - 1.0) * 8.0);"),
    "fp8_scale_not_smallest": ("while (amax <= ldexp(448.0, e - 1) && e > -127)",
                               "while (amax <= ldexp(448.0, e - 2) && e > -127)"),
    "fp8_scale_below_ue8m0": ("while (amax <= ldexp(448.0, e - 1) && e > -127)",
                              "while (amax <= ldexp(448.0, e - 1) && e > -160)"),
    "fp8_exponent_bias": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "fp8_activation_scale_dropped": ("double xc = e4m3_value(xq[c]) * sx[c / 128];", "double xc = e4m3_value(xq[c]);"),
    "fp8_activation_first_block_scale": ("double xc = e4m3_value(xq[c]) * sx[c / 128];",
                                         "double xc = e4m3_value(xq[c]) * sx[0];"),
    "fp8_h_requant_block0_amax": ("amax = fmax(amax, fabs(h[b * 128 + r]));", "amax = fmax(amax, fabs(h[r]));"),
    "fp4_exponent_bias": ("double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);",
                          "double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 2);"),
    "fp4_subnormal_value": ("double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);",
                            "double v = e == 0 ? 0.25 * m : ldexp(1.0 + 0.5 * m, e - 1);"),
    "fp4_ties_to_odd": ("if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {\n            best = (uint8_t)c;\n            best_err = err;\n        }\n    }\n    return sign | best;\n}\n\n/* Smallest power of two s with amax / s <= 6",
                        "if (err < best_err || (err == best_err && (c & 1) == 1 && (best & 1) == 0)) {\n            best = (uint8_t)c;\n            best_err = err;\n        }\n    }\n    return sign | best;\n}\n\n/* Smallest power of two s with amax / s <= 6"),
    "fp4_scale_not_smallest": ("while (amax <= ldexp(6.0, e - 1) && e > -127)",
                               "while (amax <= ldexp(3.0, e - 1) && e > -127)"),
    "fp4_block_of_64": ("g += oracle_e2m1_decode(W1q[r * d + c]) * s1[r * (d / 32) + c / 32] * xc;",
                        "g += oracle_e2m1_decode(W1q[r * d + c]) * s1[r * (d / 32) + c / 64] * xc;"),
    "fp4_up_scale_of_gate": ("u += oracle_e2m1_decode(W3q[r * d + c]) * s3[r * (d / 32) + c / 32] * xc;",
                             "u += oracle_e2m1_decode(W3q[r * d + c]) * s1[r * (d / 32) + c / 32] * xc;"),
    "fp4_down_scale_transposed": ("z += oracle_e2m1_decode(W2q[c * f + r]) * s2[c * (f / 32) + r / 32] * h[r];",
                                  "z += oracle_e2m1_decode(W2q[c * f + r]) * s2[r * (d / 32) + c / 32] * h[r];"),
    "fp8_down_scale_transposed": ("z += e4m3_value(W2q[c * f + r]) * s2[(c / 128) * fb + r / 128] * h[r];",
                                  "z += e4m3_value(W2q[c * f + r]) * s2[(r / 128) * fb + c / 128] * h[r];"),
}


@pytest.fixture(scope="module")
def tmpdir_mod():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmpdir_mod):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    # a site shared by the bf16 and the FP8 expert FFN is mutated in both
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    path_c = os.path.join(tmpdir_mod, f"{name}.c")
    path_so = os.path.join(tmpdir_mod, f"lib_{name}.so")
    open(path_c, "w").write(src.replace(old, new))
    subprocess.run(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared", "-o", path_so, path_c,
                    "-lm", "-lpthread"], check=True)
    prev = oracle.use(oracle.load(path_so))
    caught = []
    try:
        for pin in P.ALL_PINS:
            try:
                pin()
            except (AssertionError, oracle.OracleError) as e:
                caught.append(pin.__name__)
                break
    finally:
        oracle.use(prev)
    assert caught, f"no pin caught the planted mistake {name}"
