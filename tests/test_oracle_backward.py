"""Pins of the backward oracle (oracle/backward.py, fp64 autograd through the
primal rule), each against something other than autograd itself: central
finite differences of the separately written C forward oracle, and closed forms
of special cases.  No GPU."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as OB

EPS_LN = 1e-5


def _inputs(seed, B=1, H=2, T=8, d=4):
    rng = np.random.default_rng(seed)
    Q, K, V, dZ = (rng.standard_normal((B, H, T, d)) for _ in range(4))
    eta = 0.1 + 0.1 * rng.random((B, H, T))
    W0 = 0.3 * rng.standard_normal((H, d, d))
    gamma = 1 + 0.1 * rng.standard_normal((H, d))
    beta = 0.1 * rng.standard_normal((H, d))
    dWT = rng.standard_normal((B, H, d, d))
    return rng, dict(Q=Q, K=K, V=V, eta=eta, W0=W0, gamma=gamma, beta=beta), dZ, dWT


def _objective(x, b, ln, dZ, dWT):
    """L = <dZ, Z> + <dW_T, W_T> from the C forward oracle."""
    if ln:
        Z, W = oracle.ttt_linear_ln(x["Q"], x["K"], x["V"], x["eta"], x["W0"], b, x["gamma"], x["beta"],
                                    EPS_LN)
    else:
        Z, W = oracle.ttt_linear(x["Q"], x["K"], x["V"], x["eta"], x["W0"], b)
    return float((Z * dZ).sum() + (W * dWT).sum())


@pytest.mark.parametrize("ln", [False, True])
@pytest.mark.parametrize("b", [1, 4, 8])
def test_directional_derivatives_match_finite_differences(ln, b):
    rng, x, dZ, dWT = _inputs(seed=10 * b + ln)
    g = OB.ttt_linear_backward(x["Q"], x["K"], x["V"], x["eta"], x["W0"], b, dZ, dWT, ln, x["gamma"],
                               x["beta"], EPS_LN)
    names = ["Q", "K", "V", "eta", "W0"] + (["gamma", "beta"] if ln else [])
    for name in names:
        direction = rng.standard_normal(x[name].shape)
        h = 1e-6
        xp, xm = dict(x), dict(x)
        xp[name] = x[name] + h * direction
        xm[name] = x[name] - h * direction
        fd = (_objective(xp, b, ln, dZ, dWT) - _objective(xm, b, ln, dZ, dWT)) / (2 * h)
        grad = g["d" + name]
        if name in ("W0", "gamma", "beta"):   # per-unit gradients of a per-head parameter
            grad = grad.sum(axis=0)
        an = float((grad * direction).sum())
        # Central differences with h = 1e-6 carry O(h^2) truncation and about
        # 1e-16 |L| / h rounding: 1e-6 relative, far below what a dropped term
        # or a wrong sign gives.
        assert abs(an - fd) <= 1e-6 * max(1.0, abs(fd)), (name, an, fd)


def test_one_mini_batch_dV_closed_form():
    """b = T, f linear: Z = Q W0 - tril(Q K^T) diag(eta) 2 (K W0 - V), so
    dL/dV = 2 diag(eta) tril(Q K^T)^T dZ."""
    _, x, dZ, _ = _inputs(seed=3)
    T = x["Q"].shape[2]
    g = OB.ttt_linear_backward(x["Q"], x["K"], x["V"], x["eta"], x["W0"], T, dZ)
    for hi in range(2):
        q, k, e = x["Q"][0, hi], x["K"][0, hi], x["eta"][0, hi]
        A = np.tril(q @ k.T)
        np.testing.assert_allclose(g["dV"][0, hi], 2 * e[:, None] * (A.T @ dZ[0, hi]), rtol=1e-12,
                                   atol=1e-12)


@pytest.mark.parametrize("ln", [False, True])
def test_zero_learning_rate(ln):
    """eta = 0: Z = f(Q; W0) and W_T = W0, so K and V get no gradient, and dQ, dW0
    are those of f alone (torch's own layer_norm for the LN case)."""
    _, x, dZ, dWT = _inputs(seed=4)
    x["eta"] = np.zeros_like(x["eta"])
    g = OB.ttt_linear_backward(x["Q"], x["K"], x["V"], x["eta"], x["W0"], 4, dZ, dWT, ln, x["gamma"],
                               x["beta"], EPS_LN)
    assert np.all(g["dK"] == 0) and np.all(g["dV"] == 0)
    for hi in range(2):
        q = torch.tensor(x["Q"][0, hi], requires_grad=True)
        w = torch.tensor(x["W0"][hi], requires_grad=True)
        y = q @ w
        if ln:
            y = q + torch.nn.functional.layer_norm(y, (y.shape[-1],), torch.tensor(x["gamma"][hi]),
                                                   torch.tensor(x["beta"][hi]), EPS_LN)
        dq, dw = torch.autograd.grad((y * torch.tensor(dZ[0, hi])).sum(), (q, w))
        np.testing.assert_allclose(g["dQ"][0, hi], dq.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g["dW0"][0, hi], dw.numpy() + dWT[0, hi], rtol=1e-12, atol=1e-12)


_MUTANTS = {
    "update sign": ("Ws = [W - eta[t] * g for", "Ws = [W + eta[t] * g for"),
    "gradient at the current state": ("        if t % b == 0:\n            base = Ws\n", "        base = Ws\n"),
    "output before the update": (
        "        Ws = [W - eta[t] * g for W, g in zip(Ws, grads)]\n        Z.append(f(q[t], Ws))",
        "        Z.append(f(q[t], Ws))\n        Ws = [W - eta[t] * g for W, g in zip(Ws, grads)]"),
    "residual dropped": ("return x + _ln(y, gamma, beta, eps) if ln else y",
                         "return _ln(y, gamma, beta, eps) if ln else y"),
    "tanh GELU in the MLP": ("torch.nn.functional.gelu(x @ Ws[0])",
                             "torch.nn.functional.gelu(x @ Ws[0], approximate='tanh')"),
    "MLP without residual": ("return x + _ln(torch.nn.functional.gelu", "return _ln(torch.nn.functional.gelu"),
}


@pytest.mark.parametrize("mutant", sorted(_MUTANTS))
def test_planted_mistakes_are_caught(mutant, monkeypatch):
    """A copy of the backward oracle with one plausible mistake fails the pins."""
    import types
    src = open(OB.__file__).read()
    old, new = _MUTANTS[mutant]
    assert src.count(old) == 1
    mod = types.ModuleType("backward_mutant")
    exec(compile(src.replace(old, new), "backward_mutant", "exec"), mod.__dict__)
    monkeypatch.setattr(__import__(__name__), "OB", mod)
    failed = 0
    pins = [lambda: test_directional_derivatives_match_finite_differences(False, 1),
            lambda: test_directional_derivatives_match_finite_differences(True, 4),
            lambda: test_mlp_directional_derivatives_match_finite_differences(4)]
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed, f"mutant '{mutant}' passed every pin"


def _mlp_inputs(seed, B=1, H=2, T=8, d=4, h=8):
    rng = np.random.default_rng(seed)
    Q, K, V, dZ = (rng.standard_normal((B, H, T, d)) for _ in range(4))
    x = dict(Q=Q, K=K, V=V, eta=0.1 + 0.1 * rng.random((B, H, T)),
             W1=0.4 * rng.standard_normal((H, d, h)), W2=0.4 * rng.standard_normal((H, h, d)),
             gamma=1 + 0.1 * rng.standard_normal((H, d)), beta=0.1 * rng.standard_normal((H, d)))
    dW1T, dW2T = rng.standard_normal((B, H, d, h)), rng.standard_normal((B, H, h, d))
    return rng, x, dZ, dW1T, dW2T


@pytest.mark.parametrize("b", [1, 4])
def test_mlp_directional_derivatives_match_finite_differences(b):
    rng, x, dZ, dW1T, dW2T = _mlp_inputs(seed=20 + b)
    g = OB.ttt_mlp_backward(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], b, dZ, x["gamma"],
                            x["beta"], EPS_LN, dW1T, dW2T)

    def objective(y):
        Z, W1, W2 = oracle.ttt_mlp(y["Q"], y["K"], y["V"], y["eta"], y["W1"], y["W2"], b, y["gamma"],
                                   y["beta"], EPS_LN)
        return float((Z * dZ).sum() + (W1 * dW1T).sum() + (W2 * dW2T).sum())

    for name in ("Q", "K", "V", "eta", "W1", "W2", "gamma", "beta"):
        direction = rng.standard_normal(x[name].shape)
        h = 1e-6
        xp, xm = dict(x), dict(x)
        xp[name] = x[name] + h * direction
        xm[name] = x[name] - h * direction
        fd = (objective(xp) - objective(xm)) / (2 * h)
        grad = g["d" + name]
        if name in ("W1", "W2", "gamma", "beta"):
            grad = grad.sum(axis=0)
        an = float((grad * direction).sum())
        assert abs(an - fd) <= 1e-6 * max(1.0, abs(fd)), (name, an, fd)


def test_mlp_zero_learning_rate():
    """eta = 0: Z = Q + LN(GELU(Q W1) W2) with torch's own layer_norm and gelu."""
    _, x, dZ, _, _ = _mlp_inputs(seed=5)
    x["eta"] = np.zeros_like(x["eta"])
    g = OB.ttt_mlp_backward(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], 4, dZ, x["gamma"],
                            x["beta"], EPS_LN)
    assert np.all(g["dK"] == 0) and np.all(g["dV"] == 0)
    for hi in range(2):
        q = torch.tensor(x["Q"][0, hi], requires_grad=True)
        w1 = torch.tensor(x["W1"][hi], requires_grad=True)
        w2 = torch.tensor(x["W2"][hi], requires_grad=True)
        y = torch.nn.functional.gelu(q @ w1) @ w2
        z = q + torch.nn.functional.layer_norm(y, (y.shape[-1],), torch.tensor(x["gamma"][hi]),
                                               torch.tensor(x["beta"][hi]), EPS_LN)
        dq, dw1, dw2 = torch.autograd.grad((z * torch.tensor(dZ[0, hi])).sum(), (q, w1, w2))
        np.testing.assert_allclose(g["dQ"][0, hi], dq.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g["dW1"][0, hi], dw1.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g["dW2"][0, hi], dw2.numpy(), rtol=1e-12, atol=1e-12)
