"""CPU tests: the fp64 oracle against its pins, the chunked algebra against the oracle,
and deliberately broken copies of the oracle against the pins (each must be caught)."""
from __future__ import annotations

import os
import tempfile

import numpy as np
import pytest

import oracle
import oracle_pins
from chunked_ref import chunk_fwd
from oracle_pins import ALL_PINS, random_inputs


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


@pytest.mark.parametrize("T,chunk,strong", [(1, 64, False), (16, 16, False), (37, 16, True),
                                            (130, 64, False), (150, 64, True)])
def test_chunked_algebra_matches_oracle(T, chunk, strong, oracle_lib):
    """The WY/UT chunked form with 16-token sub-blocks equals the token loop (fp64)."""
    q, k, v, g, beta, S0 = random_inputs(100 + T, T, 2, 16, 8, strong=strong)
    if strong:
        g = g * 2.0   # cumulative decay over a chunk far beyond exp's fp32 range
    o_ref, S_ref = oracle.kda_fwd(q, k, v, g, beta, 0.9, S0, lib=oracle_lib)
    o, S = chunk_fwd(q, k, v, g, beta, 0.9, S0, chunk=chunk)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-11 * max(1, np.abs(o_ref).max()))
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-11 * max(1, np.abs(S_ref).max()))


def test_chunked_algebra_varlen(oracle_lib):
    lens = [70, 5, 64, 129]
    cu = np.cumsum([0] + lens)
    q, k, v, g, beta, _ = random_inputs(200, cu[-1], 2, 8, 8)
    h0 = np.random.default_rng(201).normal(0, 0.02, (4, 2, 8, 8))
    o_ref, S_ref = oracle.kda_fwd(q, k, v, g, beta, 1.0, h0, cu, lib=oracle_lib)
    o, S = chunk_fwd(q, k, v, g, beta, 1.0, h0, cu)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, atol=1e-12)


# Plausible mistakes, each a one-line change of the oracle's C source.
MUTANTS = {
    "residual_sign": ("u[j] = vt[j] - r;", "u[j] = vt[j] + r;"),
    "beta_dropped": ("const double bk = bt * kt[i];", "const double bk = kt[i];"),
    "scalar_gate": ("const double a = exp(gt[i]);", "const double a = exp(gt[0]);"),
    "gate_on_columns": ("S[(size_t)i * dv + j] *= a;", "S[(size_t)i * dv + j] *= exp(gt[j]);"),
    "gate_sign": ("const double a = exp(gt[i]);", "const double a = exp(-gt[i]);"),
    "readout_with_q": ("r += S[(size_t)i * dv + j] * kt[i];", "r += S[(size_t)i * dv + j] * qt[i];"),
    "output_with_k": ("r += S[(size_t)i * dv + j] * qt[i];\n            ot[j]",
                      "r += S[(size_t)i * dv + j] * kt[i];\n            ot[j]"),
    "scale_dropped": ("* qt[i];\n            ot[j] = c->scale * r;", "* qt[i];\n            ot[j] = r;"),
    "h0_ignored": ("* (size_t)dv);\n    const size_t sbase = ((size_t)n * H + h) * (size_t)dk * dv;\n"
                   "    if (c->h0) memcpy(S, c->h0 + sbase, sizeof(double) * (size_t)dk * dv);\n"
                   "    else memset(S, 0, sizeof(double) * (size_t)dk * dv);\n\n    for (int64_t t = bos",
                   "* (size_t)dv);\n    const size_t sbase = ((size_t)n * H + h) * (size_t)dk * dv;\n"
                   "    memset(S, 0, sizeof(double) * (size_t)dk * dv);\n\n    for (int64_t t = bos"),
    "conv_taps_reversed": ("z += w[(size_t)c * K + j] * ext[t + j];",
                           "z += w[(size_t)c * K + (K - 1 - j)] * ext[t + j];"),
    "conv_no_silu": ("y[(size_t)(bos + t) * C + c] = z / (1.0 + exp(-z));",
                     "y[(size_t)(bos + t) * C + c] = z;"),
    "cache_not_advanced": ("cache_out[((size_t)n * C + c) * P + p] = ext[L + p];",
                           "cache_out[((size_t)n * C + c) * P + p] = ext[p];"),
    "l2_eps_outside": ("const double inv = 1.0 / sqrt(ss + eps);",
                       "const double inv = 1.0 / (sqrt(ss) + eps);"),
    "gdn_gate_missing": ("at * (S[(size_t)i * dv + j] - bt * kt[i] * kS[j])",
                         "(S[(size_t)i * dv + j] - bt * kt[i] * kS[j])"),
    "gate_positive": ("g[i] = -a * sp;", "g[i] = a * sp;"),
    "gate_dt_bias_dropped": ("const double z = x[i] + dt_bias[(size_t)h * dk + c];",
                             "const double z = x[i];"),
    "gate_dt_bias_per_head": ("const double z = x[i] + dt_bias[(size_t)h * dk + c];",
                              "const double z = x[i] + dt_bias[h];"),
    "gate_softplus_as_exp": ("log1p(exp(-z)) : log1p(exp(z));", "log1p(exp(-z)) : exp(z);"),
    "gate_without_exp": ("const double a = exp(A_log[h]);", "const double a = A_log[h];"),
    "sigmoid_sign": ("beta[i] = 1.0 / (1.0 + exp(-b_raw[i]));", "beta[i] = 1.0 / (1.0 + exp(b_raw[i]));"),
    "rmsnorm_sum_not_mean": ("const double inv = 1.0 / sqrt(ss / dv + eps);",
                             "const double inv = 1.0 / sqrt(ss + eps);"),
    "rmsnorm_weight_dropped": ("y[i] = o[i] * inv * w[j] * (1.0", "y[i] = o[i] * inv * (1.0"),
    "transition_decay_on_columns": ("M[(size_t)r * dk + col] *= decay;",
                                    "M[(size_t)r * dk + col] *= exp(gt[col]);"),
    "transition_readout_transposed": ("acc += kt[r] * M[(size_t)r * dk + col];",
                                      "acc += kt[r] * M[(size_t)col * dk + r];"),
    "transition_beta_dropped": ("M[(size_t)r * dk + col] -= bt * kt[r] * w[col];",
                                "M[(size_t)r * dk + col] -= kt[r] * w[col];"),
    "transition_update_sign": ("M[(size_t)r * dk + col] -= bt * kt[r] * w[col];",
                               "M[(size_t)r * dk + col] += bt * kt[r] * w[col];"),
    "rmsnorm_gate_silu": ("y[i] = o[i] * inv * w[j] * (1.0 / (1.0 + exp(-z[i])));",
                          "y[i] = o[i] * inv * w[j] * (z[i] / (1.0 + exp(-z[i])));"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    src = open(oracle._SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    with tempfile.TemporaryDirectory() as tmp:
        path = os.path.join(tmp, "mut.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle.load(oracle.compile_oracle(path, os.path.join(tmp, "mut.so")))
        caught = []
        for pin in ALL_PINS:
            try:
                pin(lib)
            except AssertionError:
                caught.append(pin.__name__)
        assert caught, f"no pin catches the mutant {name}"


def test_pin_module_lists_every_pin():
    names = {n for n in dir(oracle_pins) if n.startswith("pin_")}
    assert names == {p.__name__ for p in ALL_PINS}
