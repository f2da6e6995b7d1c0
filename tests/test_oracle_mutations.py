"""The oracle's pins must catch plausible mistakes (CPU only).

Each case copies the oracle source, plants one mistake by text substitution,
compiles the copy into a temporary library and reruns the pin suite against
it; at least one pin must fail. Nothing here touches a GPU.
"""
import ctypes
import os
import subprocess
import tempfile

import pytest

from oracle import oracle as oracle_module

import test_oracle_bruteforce as bf
import test_oracle_closed_form as cf
import test_oracle_epilogue as ep
import test_oracle_formats as ff
import test_oracle_w4a4 as w4

MUTATIONS = {
    "nibble_order": ("(c % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4)", "(c % 2 == 0) ? (byte >> 4) : (byte & 0x0Fu)"),
    "scale_block_32": ("scales[c / 16]", "scales[c / 32]"),
    "silu_on_up": ("silu((double)G) * (double)U", "silu((double)U) * (double)G"),
    "tie_to_higher_index": ("logits[e] > logits[best]", "logits[e] >= logits[best]"),
    "bias_dropped": ("if (L->router_bias) l = l + L->router_bias[e];", ""),
    "no_normalisation": ("g[s] = exp((double)logits[ids[s]] - lmax) / den;", "g[s] = exp((double)logits[ids[s]] - lmax);"),
    "down_uses_up_global": ("L->down_global[e], I, dd", "L->up_global[e], I, dd"),
    "e4m3_bias_8": ("ldexp(1.0, (int)e - 7)", "ldexp(1.0, (int)e - 8)"),
    "e2m1_subnormal_one": ("0.5 * (double)m :", "1.0 * (double)m :"),
    "router_drops_last_term": ("for (int h = 0; h < H; ++h)\n            acc +=", "for (int h = 0; h < H - 1; ++h)\n            acc +="),
    "token_row_offset": ("const double *xr = xd + (size_t)t * H;", "const double *xr = xd;"),
    "combine_slot0_weight": ("acc += g[p] * y[p * H + h];", "acc += g[(size_t)t * k] * y[p * H + h];"),
    "gate_up_swapped_codes": ("dequant_row(L->gate_codes + row * (H / 2), L->gate_scales", "dequant_row(L->up_codes + row * (H / 2), L->gate_scales"),
    "bf16_ties_away": ("rint(ldexp(a, -q_exp))", "round(ldexp(a, -q_exp))"),
    "bf16_truncate": ("rint(ldexp(a, -q_exp))", "floor(ldexp(a, -q_exp))"),
    "gate_not_rounded_fp32": ("a[(size_t)p * I + j] = oracle_round_bf16(silu((double)G) * (double)U);",
                              "a[(size_t)p * I + j] = oracle_round_bf16(silu(sg) * su);"),
    "shared_down_uses_up_global": ("L->sh_down_global, Is, dd", "L->sh_up_global, Is, dd"),
    "shared_output_dropped": ("acc += y_sh[o];", ";"),
    "shared_gate_up_swapped": ("oracle_round_bf16(silu((double)G) * (double)U);\n            }\n        }\n        free(dg);\n        free(du);\n    }\n#pragma omp parallel num_threads(nthreads)\n    {\n        double *dd = (double *)malloc(sizeof(double) * Is);",
                               "oracle_round_bf16(silu((double)U) * (double)G);\n            }\n        }\n        free(dg);\n        free(du);\n    }\n#pragma omp parallel num_threads(nthreads)\n    {\n        double *dd = (double *)malloc(sizeof(double) * Is);"),
    "shared_down_row_stride": ("L->sh_down_codes + (size_t)h * (Is / 2)", "L->sh_down_codes + (size_t)h * (H / 2)"),
    "residual_dropped": ("if (res) acc += oracle_bf16_to_double(res[o]);", ""),
    "norm_sum_not_mean": ("sqrt(ss / (double)H + eps)", "sqrt(ss + eps)"),
    "norm_eps_outside_root": ("1.0 / sqrt(ss / (double)H + eps)", "1.0 / (sqrt(ss / (double)H) + eps)"),
    "norm_gamma_column_0": ("oracle_bf16_to_double(gamma[h])", "oracle_bf16_to_double(gamma[0])"),
    "norm_mean_off_by_one": ("sqrt(ss / (double)H + eps)", "sqrt(ss / (double)(H - 1) + eps)"),
    "act_e2m1_tie_away_from_zero": ("if (a <= 0.25) c = 0;", "if (a < 0.25) c = 0;"),
    "act_global_over_448": ("amax / 2688.0f", "amax / 448.0f"),
    "act_block_scale_from_row_amax": ("float ratio = amax_b / six_g;", "float ratio = amax / six_g;"),
    "act_e4m3_truncates": ("rint(ldexp(v, -q_exp))", "floor(ldexp(v, -q_exp))"),
    "w4a4_down_reads_unquantised_a": ("const double *aq = ad ? ad + (size_t)p * I : NULL;", "const double *aq = NULL;"),
}


def _all_pins(mod):
    """Run every pin function with the given oracle module; return the number that failed."""
    failures = 0
    cases = []
    for name in dir(ff):
        if name.startswith("test_") and name != "test_round_bf16_hand_cases":
            cases.append(lambda n=name: getattr(ff, n)(mod))
    for value, bits in [(1.0 + 2.0 ** -8, 0x3F80), (1.0 + 3 * 2.0 ** -8, 0x3F82),
                        (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81), (3 * 2.0 ** -134, 0x0002)]:
        cases.append(lambda v=value, b=bits: ff.test_round_bf16_hand_cases(mod, v, b))
    for name in dir(cf):
        if name.startswith("test_"):
            cases.append(lambda n=name: getattr(cf, n)(mod))
    cases.append(lambda: bf.test_oracle_matches_brute_force_tiny(mod, 64, 32, 4, 2, 4, 12))
    cases.append(lambda: bf.test_oracle_matches_brute_force_with_bias(mod))
    cases.append(lambda: bf.test_oracle_matches_brute_force_tiny_layer_shape(mod))
    for name in dir(ep):
        if name.startswith("test_") and name not in ("test_shared_expert_residual_and_norm_match_dense",
                                                     "test_norm_of_constant_row_is_sign_when_eps_is_zero"):
            cases.append(lambda n=name: getattr(ep, n)(mod))
    cases.append(lambda: ep.test_shared_expert_residual_and_norm_match_dense(mod, 64, 32, 4, 2, 32, 3, 21))
    cases.append(lambda: ep.test_norm_of_constant_row_is_sign_when_eps_is_zero(mod, 0.75))
    for name in dir(w4):
        if name.startswith("test_") and name != "test_w4a4_forward_matches_dense":
            cases.append(lambda n=name: getattr(w4, n)(mod))
    cases.append(lambda: w4.test_w4a4_forward_matches_dense(mod, 64, 32, 4, 2, 3, 61))
    for c in cases:
        try:
            c()
        except Exception:
            failures += 1
    return failures


class _Variant:
    """An oracle module bound to a different compiled library."""

    def __init__(self, path):
        self._cdll = ctypes.CDLL(path)
        saved = oracle_module._lib
        oracle_module._lib = None
        real_build = oracle_module.build
        oracle_module.build = lambda force=False: path
        try:
            self._bound = oracle_module.lib()
        finally:
            oracle_module._lib = saved
            oracle_module.build = real_build

    def __getattr__(self, name):
        fn = getattr(oracle_module, name)
        if not callable(fn) or name in ("lib",):
            return fn

        def call(*a, **kw):
            saved = oracle_module._lib
            oracle_module._lib = self._bound
            try:
                return fn(*a, **kw)
            finally:
                oracle_module._lib = saved
        return call


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(mutation):
    src = open(oracle_module.SRC).read()
    old, new = MUTATIONS[mutation]
    assert src.count(old) >= 1, f"mutation anchor not found: {mutation}"
    mutated = src.replace(old, new)
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "m.c")
        so = os.path.join(d, f"libm_{mutation}.so")
        open(c, "w").write(mutated)
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC",
                               "-std=c11", c, "-o", so, "-lm"])
        failures = _all_pins(_Variant(so))
    assert failures > 0, f"no pin caught the planted mistake '{mutation}'"


def test_unmutated_oracle_passes_all_pins():
    assert _all_pins(oracle_module) == 0
