"""The oracle pins must catch plausible mistakes in the oracle.

Each case compiles a copy of ``oracle/flare_oracle.c`` (or of the gradient
file ``oracle/flare_oracle_bwd.c``) with one planted mistake (a dropped term,
a wrong index, a transposed operand, an off-by-one mask), swaps it in, and
checks that at least one pin of ``test_oracle_pins`` (``test_oracle_bwd_pins``)
fails.  Everything runs on the CPU.
"""
import contextlib
import ctypes
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_bwd_pins as bwd_pins
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "flare_oracle.c")
SRC_BWD = os.path.join(os.path.dirname(oracle.__file__), "flare_oracle_bwd.c")

MUTATIONS = {
    "decode_exp_drops_scale": ("double p = exp(scale * dot(k, Qg + m * D, D) - nu);",
                               "double p = exp(dot(k, Qg + m * D, D) - nu);"),
    "encode_wrong_normaliser": ("den += w;", "den += 1.0;"),
    "encode_uses_keys_as_values": ("z[d] += w * Vh[n * D + d];", "z[d] += w * Kh[n * D + d];"),
    "project_transposed_weight": ("x[c] * W[c * C + h * D + d]", "x[c] * W[(h * D + d) * C + c]"),
    "decode_mask_off_by_one": ("if (n >= L) continue;", "if (n > L) continue;"),
    "encode_mask_ignored": ("long L = valid_len(lengths, b, N);\n        for (long d = 0; d < D; ++d) z[d] = 0.0;",
                            "long L = N;\n        for (long d = 0; d < D; ++d) z[d] = 0.0;"),
    "encode_query_group_ignores_batch": ("long g = q_per_batch ? b * H + h : h;\n        const double *q",
                                         "long g = h;\n        const double *q"),
    "decode_max_not_subtracted_sign": ("double p = exp(scale * dot(k, Qg + m * D, D) - nu);",
                                       "double p = exp(scale * dot(k, Qg + m * D, D) + nu);"),
}

PIN_FUNCS = [
    lambda m: pins.test_flarepp_matches_torch_sdpa_chain(m, True),
    lambda m: pins.test_flare_matches_torch_sdpa_chain(m),
    lambda m: pins.test_project_matches_matmul(m),
    lambda m: pins.test_materialised_mixing_matrix(m, "flarepp"),
    lambda m: pins.test_two_tokens_one_latent_closed_form(m),
    lambda m: pins.test_identical_keys_give_token_mean(m),
    lambda m: pins.test_zero_queries_give_uniform_routing(m),
    lambda m: pins.test_zero_seeds_give_mean_synthesis_values(m),
    lambda m: pins.test_mask_equals_truncation(m),
    lambda m: pins.test_hard_max_limit(m),
]


BWD_MUTATIONS = {
    "encode_bwd_drops_gamma": ("(dot_bwd(dz, Vh + n * D, D) - gamma)", "dot_bwd(dz, Vh + n * D, D)"),
    "decode_bwd_drops_delta": ("(dot_bwd(dy, Zh + m * D, D) - delta)", "dot_bwd(dy, Zh + m * D, D)"),
    "encode_bwd_dv_uses_query": ("dVh[n * D + d] += A[n] * dz[d];", "dVh[n * D + d] += A[n] * q[d];"),
    "decode_bwd_dk_drops_scale": ("dk[d] += scale * dS * Qg[m * D + d];", "dk[d] += dS * Qg[m * D + d];"),
    "encode_bwd_dq_wrong_sign": ("dq[d] += scale * dS * Kh[n * D + d];", "dq[d] -= scale * dS * Kh[n * D + d];"),
    "fold_ignores_batch": ("const long g = q_per_batch ? b * H + h : h;", "const long g = h;"),
    "project_bwd_dw_transposed": ("dW[i * C + h * D + d] += s;", "dW[(h * D + d) * C + i] += s;"),
    "decode_bwd_mask_ignored": ("long L = valid_len_bwd(lengths, b, N);\n        const double *Qg",
                                "long L = N;\n        const double *Qg"),
    "decode_bwd_dz_uses_keys": ("dZh[m * D + d] += P[m] * dy[d];", "dZh[m * D + d] += P[m] * k[d];"),
}

BWD_PIN_FUNCS = [
    lambda m: bwd_pins.test_flarepp_grads_match_torch_autograd(m, True),
    lambda m: bwd_pins.test_flare_grads_match_torch_autograd(m),
    lambda m: bwd_pins.test_flarepp_directional_derivatives(m),
    lambda m: bwd_pins.test_flare_directional_derivatives_masked(m),
    lambda m: bwd_pins.test_encoder_key_gradients_sum_to_zero(m),
    lambda m: bwd_pins.test_decoder_query_gradients_sum_to_zero(m),
    lambda m: bwd_pins.test_row_stochastic_sum_rules(m),
    lambda m: bwd_pins.test_single_latent(m),
    lambda m: bwd_pins.test_masked_tokens_get_no_gradient_and_match_truncation(m),
]


@contextlib.contextmanager
def mutated_oracle(tmp_path, name, bwd=False):
    old, new = (BWD_MUTATIONS if bwd else MUTATIONS)[name]
    target = SRC_BWD if bwd else SRC
    text = open(target).read()
    assert text.count(old) == 1, name
    src = tmp_path / f"{name}.c"
    src.write_text(text.replace(old, new))
    other = SRC if bwd else SRC_BWD
    so = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC",
                    "-shared", "-o", str(so), str(src), other, "-lm"], check=True)
    good = oracle._load()
    bad = ctypes.CDLL(str(so))
    for fn in ("flare_oracle_project", "flare_oracle_encode", "flare_oracle_decode",
               "flare_oracle_encode_bwd", "flare_oracle_decode_bwd", "flare_oracle_project_bwd"):
        getattr(bad, fn).argtypes = getattr(good, fn).argtypes
        getattr(bad, fn).restype = None
    oracle._lib = bad
    try:
        yield
    finally:
        oracle._lib = good


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    failures = 0
    with mutated_oracle(tmp_path, name):
        for f in PIN_FUNCS:
            try:
                f(oracle)
            except AssertionError:
                failures += 1
    assert failures >= 1, f"no pin caught the planted mistake {name}"


@pytest.mark.parametrize("name", sorted(BWD_MUTATIONS))
def test_gradient_pins_catch_planted_mistake(tmp_path, name):
    failures = 0
    with mutated_oracle(tmp_path, name, bwd=True):
        for f in BWD_PIN_FUNCS:
            try:
                f(oracle)
            except AssertionError:
                failures += 1
    assert failures >= 1, f"no gradient pin caught the planted mistake {name}"
