"""The per-mini-batch dual form of the momentum and decay update on the TTT-MLP
memory that the CUDA-core momentum kernel computes, restated in fp64 numpy and
checked against the oracle's token-by-token recursion (the Titans article,
§二.1(2)-(3), with the TTT write-up's mini-batch rule, §03.6, and its MLP inner
model, §03.9).  Within a mini-batch with base state (W1, W2, S1, S2) and all
gradients taken there, the recursion S_t = alpha_t S_{t-1} - eta_t g_t,
W_t = (1 - lambda_t) W_{t-1} + S_t gives, per layer,

  Zq1 = diag(Lam) Q W1 + diag(C) Q S1 - (c o tril(Q K^T)) diag(eta) G2
  Zq3 = diag(Lam) Zq2 W2 + diag(C) Zq2 S2 - (c o tril(Zq2 X2^T)) diag(eta) G3

with the coefficients of the linear case (Lam, A, C, a, c over the b tokens), and
the mini-batch's last rows of c and a give the next base state.  The derivation
is this build's; a planted mistake must fail."""
import numpy as np
import pytest
from scipy.special import ndtr

import oracle

D, HID, MB = 64, 256, 16


def gelu(x):
    return x * ndtr(x)


def gelu_grad(x):
    return ndtr(x) + x * np.exp(-0.5 * x * x) / np.sqrt(2.0 * np.pi)


def ln_grad(y, k, v, gamma, beta, eps):
    """dl/dy of l = ||k + LN_{gamma,beta}(y) - v||^2 per row."""
    mu = y.mean(axis=1, keepdims=True)
    sig = np.sqrt(((y - mu) ** 2).mean(axis=1, keepdims=True) + eps)
    xh = (y - mu) / sig
    dxh = 2.0 * (k + gamma * xh + beta - v) * gamma
    return (dxh - dxh.mean(axis=1, keepdims=True) - xh * (dxh * xh).mean(axis=1, keepdims=True)) / sig


def layer_norm(y, gamma, beta, eps):
    mu = y.mean(axis=1, keepdims=True)
    return gamma * (y - mu) / np.sqrt(((y - mu) ** 2).mean(axis=1, keepdims=True) + eps) + beta


def coefficients(alpha, lam, mistake=None):
    n = len(alpha)
    om = 1.0 - lam
    Lam, A, C = np.cumprod(om), np.cumprod(alpha), np.zeros(n)
    for t in range(n):
        C[t] = (om[t] * C[t - 1] if t else 0.0) + A[t]
    a, c = np.zeros((n, n)), np.zeros((n, n))
    for s in range(n):
        a[s, s] = c[s, s] = 1.0
        for t in range(s + 1, n):
            a[t, s] = alpha[t] * a[t - 1, s]
            c[t, s] = om[t] * c[t - 1, s] + a[t, s]
    if mistake == "no_momentum_in_outputs":
        C = np.zeros(n)
    return Lam, A, C, a, c


def dual_form(Q, K, V, eta, alpha, lam, W1, W2, gamma, beta, eps=1e-6, mistake=None):
    T = Q.shape[0]
    S1, S2 = np.zeros_like(W1), np.zeros_like(W2)
    Z = np.zeros_like(Q)
    for t0 in range(0, T, MB):
        r = slice(t0, t0 + MB)
        q, k, v, e = Q[r], K[r], V[r], eta[r]
        Lam, A, C, a, c = coefficients(alpha[r], lam[r], mistake)
        # Gradients of every token of the mini-batch at its base state.
        X1 = k @ W1
        X2 = gelu(X1)
        G3 = ln_grad(X2 @ W2, k, v, gamma, beta, eps)
        G2 = (G3 @ W2.T) * gelu_grad(X1)
        ce = np.tril(c) * e[None, :]  # c_{t,s} eta_s for s <= t
        Zq1 = Lam[:, None] * (q @ W1) + C[:, None] * (q @ S1) - (ce * (q @ k.T)) @ G2
        Zq2 = gelu(Zq1)
        Zq3 = Lam[:, None] * (Zq2 @ W2) + C[:, None] * (Zq2 @ S2) - (ce * (Zq2 @ X2.T)) @ G3
        Z[r] = q + layer_norm(Zq3, gamma, beta, eps)
        L = MB - 1
        cL, aL = c[L] * e, a[L] * e
        W1, S1 = Lam[L] * W1 + C[L] * S1 - (k * cL[:, None]).T @ G2, A[L] * S1 - (k * aL[:, None]).T @ G2
        W2, S2 = Lam[L] * W2 + C[L] * S2 - (X2 * cL[:, None]).T @ G3, A[L] * S2 - (X2 * aL[:, None]).T @ G3
    return Z, W1, W2, S1, S2


def case(T, seed, rates="mixed"):
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.standard_normal((T, D)) / np.sqrt(D) for _ in range(3))
    eta = 0.2 / (1.0 + np.exp(-rng.standard_normal(T)))
    if rates == "mixed":
        alpha, lam = rng.uniform(0.0, 0.9, T), rng.uniform(0.0, 0.05, T)
    else:  # extremes: no carried momentum, full forgetting
        alpha, lam = rng.choice([0.0, 1.0], T), rng.choice([0.0, 1.0], T)
    W1, W2 = 0.02 * rng.standard_normal((D, HID)), 0.02 * rng.standard_normal((HID, D))
    gamma, beta = 1.0 + 0.01 * rng.standard_normal(D), 0.01 * rng.standard_normal(D)
    return Q, K, V, eta, alpha, lam, W1, W2, gamma, beta


def recursion(Q, K, V, eta, alpha, lam, W1, W2, gamma, beta, eps=1e-6):
    params = np.concatenate([W1.ravel(), W2.ravel()])[None]
    Zr, Wr, Sr = oracle.default().momentum_forward(
        oracle.MLP_LN, Q[None, None], K[None, None], V[None, None], eta[None, None], alpha[None, None],
        lam[None, None], params, MB, gamma[None], beta[None], eps, hidden=HID)
    n1 = D * HID
    return (Zr[0, 0], Wr[0, 0, :n1].reshape(D, HID), Wr[0, 0, n1:].reshape(HID, D),
            Sr[0, 0, :n1].reshape(D, HID), Sr[0, 0, n1:].reshape(HID, D))


def rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("rates", ["mixed", "extremes"])
@pytest.mark.parametrize("T", [16, 48])
def test_mini_batch_dual_form_equals_the_recursion(T, rates):
    args = case(T, seed=T, rates=rates)
    got = dual_form(*args)
    ref = recursion(*args)
    for g, r in zip(got, ref):
        if np.linalg.norm(r) > 0:
            assert rel(g, r) < 1e-10


def test_planted_mistake_fails():
    args = case(48, seed=5)
    Z, *_ = dual_form(*args, mistake="no_momentum_in_outputs")
    Zr, *_ = recursion(*args)
    assert rel(Z, Zr) > 1e-2
