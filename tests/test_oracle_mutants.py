"""Plant plausible mistakes in copies of the oracle and check that the pins catch each.

Every mutant is a one-line textual edit of ``oracle/ttt_oracle.c`` compiled into a
temporary library; the original source is never touched.  A mutant "survives"
when every pin still passes, which would mean the pins cannot tell that mistake
from the method.  No GPU is involved.
"""
import os

import pytest

import oracle
from oracle_pins import all_pins

MUTANTS = {
    "no factor 2 in the linear gradient": ("dy[j] = 2.0 * r; /* d l / d y */", "dy[j] = r;"),
    "gamma dropped from d l / d xhat": ("dout[j] = 2.0 * r * m->gamma[j];", "dout[j] = 2.0 * r;"),
    "update with the wrong sign": ("W[p] -= eta[t] * grad[p];", "W[p] += eta[t] * grad[p];"),
    "gradient base is the current state (online GD)": (
        "if (t % b == 0) memcpy(Wbase, W, sizeof(double) * P);", "memcpy(Wbase, W, sizeof(double) * P);"),
    "output before the token's own update (exclusive diagonal)": (
        "    model_loss_grad(m, Wbase, k, v, grad, &sc); /* G_t at the mini-batch base */\n"
        "    for (long p = 0; p < P; ++p) W[p] -= eta[t] * grad[p];\n"
        "    model_apply(m, W, q, Z + (long)t * d, &sc); /* output at the updated W_t */\n",
        "    model_apply(m, W, q, Z + (long)t * d, &sc);\n"
        "    model_loss_grad(m, Wbase, k, v, grad, &sc);\n"
        "    for (long p = 0; p < P; ++p) W[p] -= eta[t] * grad[p];\n"),
    "step size of the mini-batch's first token": ("W[p] -= eta[t] * grad[p];", "W[p] -= eta[t - t % b] * grad[p];"),
    "unbiased variance in LN": ("var /= d;", "var /= (d - 1);"),
    "epsilon outside the square root": ("1.0 / sqrt(var + eps);", "1.0 / (sqrt(var) + eps);"),
    "transposed W in the output": (
        "for (int i = 0; i < d; ++i) acc += x[i] * W[(long)i * d + j];",
        "for (int i = 0; i < d; ++i) acc += x[i] * W[(long)j * d + i];"),
    "LN Jacobian without the xhat xhat term": ("- 1.0 / d - xhat[i] * xhat[j] / d", "- 1.0 / d"),
    "LN Jacobian without the mean term": ("- 1.0 / d - xhat[i] * xhat[j] / d", "- xhat[i] * xhat[j] / d"),
    "GELU derivative without x phi(x)": ("return Phi + x * phi;", "return Phi;"),
    "tanh GELU instead of the exact one": (
        "static double gelu(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }",
        "static double gelu(double x) { return 0.5 * x * (1.0 + tanh(0.7978845608 * (x + 0.044715 * x * x * x))); }"),
    "residual dropped from the output": (
        "out[j] = x[j] + (m->gamma[j] * sc->xhat[j] + m->beta[j]);",
        "out[j] = (m->gamma[j] * sc->xhat[j] + m->beta[j]);"),
    "beta dropped from the loss": (
        "k[j] + (m->gamma[j] * xhat[j] + m->beta[j]) - v[j];", "k[j] + (m->gamma[j] * xhat[j]) - v[j];"),
    "W2 gradient from the pre-activation": ("gW2[(long)i * d + j] = s[i] * dy[j];",
                                           "gW2[(long)i * d + j] = a[i] * dy[j];"),
    "W1 gradient without GELU'": ("a[i] = ds * gelu_deriv(a[i]);", "a[i] = ds;"),
}


@pytest.fixture(scope="module")
def source():
    with open(oracle.SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", list(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) >= 1, f"anchor for '{name}' not found in the oracle source"
    src = tmp_path / "mutant.c"
    src.write_text(source.replace(old, new, 1))
    lib = oracle.load(oracle.build(str(src), str(tmp_path / "libmutant.so"), force=True))
    orc = oracle.Oracle(lib)
    caught = []
    for pin_name, pin in all_pins():
        try:
            pin(orc)
        except (AssertionError, ValueError):
            caught.append(pin_name)
    assert caught, f"mutant '{name}' passes every pin"


def test_unmutated_copy_passes(source, tmp_path):
    """The copy-and-compile route itself does not change results."""
    src = tmp_path / "same.c"
    src.write_text(source)
    orc = oracle.Oracle(oracle.load(oracle.build(str(src), str(tmp_path / "libsame.so"), force=True)))
    from test_oracle_momentum import momentum_pins
    for _, pin in all_pins() + momentum_pins():
        pin(orc)


MOMENTUM_MUTANTS = {
    "momentum without alpha": ("S[p] = alpha[t] * S[p] - eta[t] * grad[p];", "S[p] = S[p] - eta[t] * grad[p];"),
    "decay applied to the momentum": ("W[p] = (1.0 - lam[t]) * W[p] + S[p];",
                                      "W[p] = W[p] + (1.0 - lam[t]) * S[p];"),
    "momentum gradient at the current state": (
        "    if (t % b == 0) memcpy(Wbase, W, sizeof(double) * P);\n"
        "    const double *k = K + (long)t * d, *v = V + (long)t * d, *q = Q + (long)t * d;\n"
        "    model_loss_grad(m, Wbase, k, v, grad, &sc);\n"
        "    for (long p = 0; p < P; ++p) {\n      S[p]",
        "    memcpy(Wbase, W, sizeof(double) * P);\n"
        "    const double *k = K + (long)t * d, *v = V + (long)t * d, *q = Q + (long)t * d;\n"
        "    model_loss_grad(m, Wbase, k, v, grad, &sc);\n"
        "    for (long p = 0; p < P; ++p) {\n      S[p]"),
    "decay of the previous token": ("W[p] = (1.0 - lam[t]) * W[p] + S[p];",
                                    "W[p] = (1.0 - lam[t > 0 ? t - 1 : 0]) * W[p] + S[p];"),
    "state updated with the previous momentum": (
        "      S[p] = alpha[t] * S[p] - eta[t] * grad[p];\n      W[p] = (1.0 - lam[t]) * W[p] + S[p];",
        "      W[p] = (1.0 - lam[t]) * W[p] + S[p];\n      S[p] = alpha[t] * S[p] - eta[t] * grad[p];"),
}


@pytest.mark.parametrize("name", list(MOMENTUM_MUTANTS))
def test_momentum_mutant_is_caught(name, source, tmp_path):
    """The same for the momentum and decay variant, against its own pins."""
    from test_oracle_momentum import momentum_pins
    old, new = MOMENTUM_MUTANTS[name]
    assert source.count(old) == 1, f"anchor for '{name}' not unique in the oracle source"
    src = tmp_path / "mutant.c"
    src.write_text(source.replace(old, new, 1))
    orc = oracle.Oracle(oracle.load(oracle.build(str(src), str(tmp_path / "libmutant.so"), force=True)))
    caught = []
    for pin_name, pin in momentum_pins():
        try:
            pin(orc)
        except (AssertionError, ValueError):
            caught.append(pin_name)
    assert caught, f"mutant '{name}' passes every momentum pin"
