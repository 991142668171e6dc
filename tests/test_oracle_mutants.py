"""Mutation check of the oracle's pins: each test plants one plausible mistake in a copy of the
oracle source (on the CPU), builds it, and requires that at least one pin rejects it.

The planted mistakes are the kinds the pins are meant to catch: a dropped term, a wrong sign,
a wrong index or mask bound, a transposed operand, a missing normalisation.
"""
import os
import subprocess

import pytest

import test_oracle_pins as pins
from oracle import oracle

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "rsa_oracle.c")

MUTANTS = {
    "score scale dropped": ("s[j] = acc * scale;", "s[j] = acc;"),
    "causal bound off by one": ("score_row(qi, Kh, L, d, causal ? i + 1 : L, scale, p);",
                                "score_row(qi, Kh, L, d, causal ? i + 2 : L, scale, p);"),
    "softmax not normalised": ("for (long j = 0; j < L; ++j) s[j] /= l;", ""),
    "lse without log": ("return m + log(l);", "return m + l;"),
    "dS sign flipped": ("double ds = p[j] * (dp[j] - D);", "double ds = p[j] * (D - dp[j]);"),
    "D term dropped": ("            D += p[j] * acc;\n        }\n        for (long k = 0; k < d; ++k) dQh",
                       "        }\n        for (long k = 0; k < d; ++k) dQh"),
    "dK transposed operand": ("dKh[j * d + k] += scale * ds * qi[k];",
                              "dKh[j * d + k] += scale * ds * Kh[i * d + k];"),
    "dV uses dP": ("dVh[j * d + k] += p[j] * doi[k];", "dVh[j * d + k] += dp[j] * doi[k];"),
    "dQ scale dropped": ("dQh[i * d + k] += scale * ds * Kh[j * d + k];",
                         "dQh[i * d + k] += ds * Kh[j * d + k];"),
    "ring skips its own block": ("if (causal && (m > n || j > i)) {", "if (causal && (m >= n || j > i)) {"),
    "ring wrong key block": ("acc += S[ii * L + m * c + jj] * Vh[(m * c + jj) * d + k];",
                             "acc += S[ii * L + m * c + jj] * Vh[(n * c + jj) * d + k];"),
    "ring dV wrong row": ("dVh[j * d + k] += p * dOh[i * d + k];", "dVh[j * d + k] += p * dOh[j * d + k];"),
    "linear bias dropped": ("            if (b) acc += b[n];\n", ""),
    "GELU half dropped": ("if (gelu) acc = 0.5 * acc * (1.0 + erf(acc / sqrt(2.0)));",
                          "if (gelu) acc = acc * (1.0 + erf(acc / sqrt(2.0)));"),
    "residual inside the GELU": (
        "            if (gelu) acc = 0.5 * acc * (1.0 + erf(acc / sqrt(2.0)));\n            if (R) acc += R[m * N + n];",
        "            if (R) acc += R[m * N + n];\n            if (gelu) acc = 0.5 * acc * (1.0 + erf(acc / sqrt(2.0)));"),
    "linear weight row/column swapped": ("acc += X[m * K + k] * W[n * K + k];",
                                         "acc += X[m * K + k] * W[(k % N) * K + (n % K)];"),
}


def _battery(orc):
    """A quick subset of the pins; returns the names of those that reject the library."""
    checks = [
        ("brute force", lambda: pins.test_forward_matches_decimal_brute_force(orc, 5, 4, 2.0, False)),
        ("brute force causal", lambda: pins.test_forward_matches_decimal_brute_force(orc, 5, 4, 2.0, True)),
        ("zero queries causal", lambda: pins.test_zero_queries_give_running_mean(orc, True)),
        ("ring fwd", lambda: pins.test_ring_forward_equals_unchunked(orc, 16, False)),
        ("ring fwd causal", lambda: pins.test_ring_forward_equals_unchunked(orc, 16, True)),
        ("ring bwd", lambda: pins.test_ring_backward_equals_unchunked(orc, 8, False)),
        ("ring bwd causal", lambda: pins.test_ring_backward_equals_unchunked(orc, 8, True)),
        ("finite differences", lambda: pins.test_backward_matches_finite_differences(orc, 5, 3, False)),
        ("finite differences causal", lambda: pins.test_backward_matches_finite_differences(orc, 5, 3, True)),
        ("invariants", lambda: pins.test_backward_invariants(orc, False)),
        ("linear", lambda: pins.test_linear_matches_plain_python(orc, False, True, False)),
        ("linear gelu residual", lambda: pins.test_linear_matches_plain_python(orc, True, True, True)),
        ("gelu values", lambda: pins.test_gelu_values_and_symmetry(orc)),
    ]
    failed = []
    for name, fn in checks:
        try:
            fn()
        except Exception:  # an assertion, or an error code from the library
            failed.append(name)
    return failed


def test_unmutated_oracle_passes_battery():
    assert _battery(oracle) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {old!r}"
    mutated = src.replace(old, new)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "libmutant.so"
    c_path.write_text(mutated)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", str(so_path),
                    str(c_path), "-lm"], check=True)
    lib = oracle.open_library(str(so_path))
    with oracle.using_library(lib):
        failed = _battery(oracle)
    assert failed, f"no pin rejects the mutant '{name}'"
