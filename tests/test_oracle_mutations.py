"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the C oracle (on the CPU, in a
temporary directory), builds it, and runs a fast subset of the pins from
test_oracle_pins.py against it: at least one pin must fail for every mutant,
and all of them must pass for the unmodified source."""
import ctypes
import os
import subprocess
import tempfile

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "mesa_oracle.c")

MUTANTS = {
    "beta dropped from the H update": ("Hm[(size_t)i * dk + j] = g * Hm[(size_t)i * dk + j] + bta * kt[i] * kt[j];",
                                       "Hm[(size_t)i * dk + j] = g * Hm[(size_t)i * dk + j] + kt[i] * kt[j];"),
    "decay dropped from the H update": ("Hm[(size_t)i * dk + j] = g * Hm[(size_t)i * dk + j] + bta * kt[i] * kt[j];",
                                        "Hm[(size_t)i * dk + j] = Hm[(size_t)i * dk + j] + bta * kt[i] * kt[j];"),
    "G built as k v^T": ("Gm[(size_t)i * dk + j] = g * Gm[(size_t)i * dk + j] + bta * vt[i] * kt[j];",
                         "Gm[(size_t)i * dk + j] = g * Gm[(size_t)i * dk + j] + bta * vt[j] * kt[i];"),
    "CG residual sign": ("r[i] -= alpha * y[i];", "r[i] += alpha * y[i];"),
    "CG rho inverted": ("const double rho = rr_new / rr;", "const double rho = rr / rr_new;"),
    "CG direction not conjugated": ("p[i] = r[i] + rho * p[i];", "p[i] = r[i];"),
    "chunk diagonal term dropped": ("for (int j = 0; j <= t; ++j) {\n        const double m = c->betac[j]",
                                    "for (int j = 0; j < t; ++j) {\n        const double m = c->betac[j]"),
    "chunk decay sign": ("const double m = c->betac[j] * exp(c->bcum[t] - c->bcum[j]);",
                         "const double m = c->betac[j] * exp(c->bcum[j] - c->bcum[t]);"),
    "Cholesky back-substitution transposed": ("for (int m = i + 1; m < n; ++m) s -= A[(size_t)m * n + i] * x[m];",
                                              "for (int m = i + 1; m < n; ++m) s -= A[(size_t)i * n + m] * x[m];"),
    "Lambda applied twice": ("A[(size_t)i * dk + i] += lambda[(size_t)h * dk + i];",
                             "A[(size_t)i * dk + i] += 2.0 * lambda[(size_t)h * dk + i];"),
    "preprocessing convolution looks ahead": (
        "for (int w = 0; w < W && w <= t; ++w)\n                    u += conv[((size_t)h * W + w) * d + i] * xs[(size_t)(t - w) * d + i];",
        "for (int w = 0; w < W && t + w < T; ++w)\n                    u += conv[((size_t)h * W + w) * d + i] * xs[(size_t)(t + w) * d + i];"),
    "preprocessing weights read with the lag reversed": (
        "u += conv[((size_t)h * W + w) * d + i] * xs[(size_t)(t - w) * d + i];",
        "u += conv[((size_t)h * W + (W - 1 - w)) * d + i] * xs[(size_t)(t - w) * d + i];"),
    "warm start residual sign": ("for (int i = 0; i < n; ++i) { r[i] = b[i] - y[i]; p[i] = r[i]; }",
                                 "for (int i = 0; i < n; ++i) { r[i] = b[i] + y[i]; p[i] = r[i]; }"),
    "warm start drops x0 from x": ("for (int i = 0; i < n; ++i) x[i] = x0[i];\n        mv(ctx, x, y);",
                                   "for (int i = 0; i < n; ++i) x[i] = x0[i];\n        mv(ctx, x, y);\n        for (int i = 0; i < n; ++i) x[i] = 0.0;"),
    "warm stopping test relative to the first residual": ("const double bnorm = sqrt(dot(n, b, b));",
                                                          "const double bnorm = sqrt(rr);"),
    "preprocessing norm left out": ("const double inv = 1.0 / (nrm > 1e-6 ? nrm : 1e-6);", "const double inv = 1.0;"),
    "backward dk without the transposed H total": (
        "s += (Hbar[(size_t)i * dk + j] + Hbar[(size_t)j * dk + i]) * kt[j];",
        "s += 2.0 * Hbar[(size_t)i * dk + j] * kt[j];"),
    "backward dgamma against the state after the token": ("const double* Hprev = Hs + (size_t)t * SH;",
                                                          "const double* Hprev = Hs + (size_t)(t + 1) * SH;"),
    "backward totals not decayed": ("const double gnext = (t + 1 < T) ? gamma[bt + 1] : 0.0;",
                                    "const double gnext = (t + 1 < T) ? 1.0 : 0.0;"),
    "backward dlambda sign": ("part[(size_t)bh * dk + i] -= ut[i] * xt[i];",
                              "part[(size_t)bh * dk + i] += ut[i] * xt[i];"),
    "adjoint right-hand side G do instead of G^T do": ("for (int i = 0; i < dv; ++i) s += Gm[(size_t)i * dk + j] * dot_[i];",
                                                       "for (int i = 0; i < dv; ++i) s += Gm[(size_t)j * dk + i] * dot_[i];"),
    "backward dbeta without the value statistics": (
        "for (int j = 0; j < dk; ++j) db += vt[i] * Gbar[(size_t)i * dk + j] * kt[j];",
        "for (int j = 0; j < dk; ++j) db += 0.0 * vt[i] * Gbar[(size_t)i * dk + j] * kt[j];"),
    "warm forward starts every token from the sequence's first guess": (
        "x0 ? x0 + bt * dk : NULL", "x0 ? x0 + (size_t)bh * T * dk : NULL"),
    "warm forward returns the guesses as the solutions": (
        "if (x_out) memcpy(x_out + bt * dk, x, sizeof(double) * (size_t)dk);",
        "if (x_out) memcpy(x_out + bt * dk, x0 ? x0 + bt * dk : x, sizeof(double) * (size_t)dk);"),
    "backward dlambda from one batch row only": ("for (int b = 0; b < B; ++b) s += part[((size_t)b * H + h) * dk + i];",
                                                 "for (int b = 0; b < 1; ++b) s += part[((size_t)b * H + h) * dk + i];"),
}


class _Mutant:
    """The oracle module's Python API bound to another build of the C source."""

    def __init__(self, lib):
        self.lib = lib

    def __getattr__(self, name):
        fn = getattr(oracle, name)

        def call(*a, **kw):
            saved = oracle._lib
            oracle._lib = self.lib
            try:
                return fn(*a, **kw)
            finally:
                oracle._lib = saved
        return call


def build_variant(src_text, tmp):
    c = os.path.join(tmp, "m.c")
    h = os.path.join(tmp, "mesa_oracle.h")
    with open(c, "w") as f:
        f.write(src_text)
    with open(os.path.join(os.path.dirname(SRC), "mesa_oracle.h")) as f, open(h, "w") as g:
        g.write(f.read())
    so = os.path.join(tmp, "libm.so")
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-I", tmp,
                    "-o", so, c, "-lm"], check=True)
    return _Mutant(oracle._configure(ctypes.CDLL(so)))


PIN_SUBSET = [
    lambda o: pins.test_cg_iterates_equal_krylov_galerkin(o, 9),
    lambda o: pins.test_cg_one_step_closed_form(o),
    lambda o: pins.test_cholesky_minimises_the_mesa_objective(o, 3, 2, 6),
    lambda o: pins.test_gamma_beta_one_gives_plain_sums(o),
    lambda o: pins.test_first_token_and_gamma_zero_match_sherman_morrison(o),
    lambda o: pins.test_unconverged_cg_equals_galerkin_on_explicit_statistics(o),
    lambda o: pins.test_chunked_equals_per_token(o, 8, 0.0),
    lambda o: pins.test_large_lambda_gives_linear_attention(o),
    lambda o: pins.test_preprocess_matches_numpy_convolution(o),
    lambda o: pins.test_preprocess_causal_and_scale_invariant(o),
    lambda o: pins.test_warm_cg_equals_shifted_cold_cg(o),
    lambda o: pins.test_warm_cg_from_the_solution_stops_at_once(o),
    lambda o: pins.test_warm_forward_is_the_shifted_cold_solve_per_token(o),
    lambda o: pins.test_warm_forward_from_the_exact_solutions(o),
    lambda o: pins.test_backward_matches_finite_differences_of_the_exact_layer(o),
    lambda o: pins.test_backward_one_step_closed_form(o),
    lambda o: pins.test_backward_respects_the_beta_lambda_scale_invariance(o),
]


def failing_pins(mod):
    failed = 0
    for pin in PIN_SUBSET:
        try:
            pin(mod)
        except (AssertionError, RuntimeError, FloatingPointError, ValueError, IndexError):
            failed += 1
    return failed


def test_unmodified_source_passes_the_subset():
    with open(SRC) as f:
        text = f.read()
    with tempfile.TemporaryDirectory() as tmp:
        assert failing_pins(build_variant(text, tmp)) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        text = f.read()
    assert text.count(old) >= 1, f"mutation anchor missing: {name}"
    with tempfile.TemporaryDirectory() as tmp:      # the first occurrence is mutated
        assert failing_pins(build_variant(text.replace(old, new, 1), tmp)) >= 1, name
