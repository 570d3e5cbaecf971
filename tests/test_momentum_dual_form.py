"""The chunked dual form of the momentum and decay update that the tensor-core
momentum kernel computes, restated in fp64 numpy and checked against the oracle's
token-by-token recursion (the Titans article, §二.1(2), kept to the mini-batch
rule of the TTT write-up, §03.6).  The kernel's formulas are derived, not printed
on the pages, so this pins the derivation apart from the GPU: with W_c, S_c the
state at the start of a 64-token chunk,

  W_t = Lam_t W_c + C_t S_c - sum_{s<=t} c_{t,s} eta_s g_s
  S_t = A_t S_c - sum_{s<=t} a_{t,s} eta_s g_s

with Lam_t = prod (1 - lambda), A_t = prod alpha, C_t = (1 - lambda_t) C_{t-1} + A_t,
a_{t,s} = alpha_t a_{t-1,s} and c_{t,s} = (1 - lambda_t) c_{t-1,s} + a_{t,s}
(a_{s,s} = c_{s,s} = 1), walked up each column s as the kernel's table is.  Planted
mistakes in the coefficients must fail."""
import numpy as np
import pytest

import oracle

D, MB, CHUNK = 64, 16, 64


def grad_wrt_y(y, k, v, ln, gamma, beta, eps):
    """dl/dy of l = ||f - v||^2 per row, f = y (plain) or k + LN_{gamma,beta}(y)."""
    if not ln:
        return 2.0 * (y - v)
    mu = y.mean(axis=1, keepdims=True)
    sig = np.sqrt(((y - mu) ** 2).mean(axis=1, keepdims=True) + eps)
    xh = (y - mu) / sig
    dxh = 2.0 * (k + gamma * xh + beta - v) * gamma
    return (dxh - dxh.mean(axis=1, keepdims=True) - xh * (dxh * xh).mean(axis=1, keepdims=True)) / sig


def output(zpre, q, ln, gamma, beta, eps):
    if not ln:
        return zpre
    mu = zpre.mean(axis=1, keepdims=True)
    sig = np.sqrt(((zpre - mu) ** 2).mean(axis=1, keepdims=True) + eps)
    return q + gamma * (zpre - mu) / sig + beta


def coefficients(alpha, lam, mistake=None):
    """Lam, A, C per token and the tables a, c [t][s] of one chunk (fp64)."""
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
    if mistake == "c_is_a":
        c = a.copy()
    elif mistake == "strict_diagonal":
        c = c - np.eye(n)
    elif mistake == "decay_on_s":
        C = A.copy()
    return Lam, A, C, a, c


def dual_form(Q, K, V, eta, alpha, lam, W0, ln, gamma=None, beta=None, eps=1e-6, mistake=None):
    """One unit: Q, K, V [T, d], eta, alpha, lam [T], W0 [d, d]; returns Z, W, S."""
    T = Q.shape[0]
    W, S = W0.copy(), np.zeros_like(W0)
    Z = np.zeros_like(Q)
    for c0 in range(0, T, CHUNK):
        n = min(CHUNK, T - c0)
        q, k, v, e = Q[c0:c0 + n], K[c0:c0 + n], V[c0:c0 + n], eta[c0:c0 + n]
        Lam, A, C, a, c = coefficients(alpha[c0:c0 + n], lam[c0:c0 + n], mistake)
        X, Y = np.vstack([k, q]) @ W, np.vstack([k, q]) @ S  # [K;Q] W_c, [K;Q] S_c
        G = np.zeros((n, D))
        for m in range(n // MB):
            rows = slice(MB * m, MB * m + MB)
            base = MB * m - 1  # the state the mini-batch's gradients are taken at
            rho, kap = (Lam[base], C[base]) if base >= 0 else (1.0, 0.0)
            y = rho * X[rows] + kap * Y[rows]
            if base >= 0:
                coef = c[base, :base + 1] * e[:base + 1]
                y = y - (k[rows] @ k[:base + 1].T * coef) @ G[:base + 1]
            G[rows] = grad_wrt_y(y, k[rows], v[rows], ln, gamma, beta, eps)
        for t in range(n):
            coef = c[t, :t + 1] * e[:t + 1]
            zpre = Lam[t] * X[n + t] + C[t] * Y[n + t] - (k[:t + 1] @ q[t] * coef) @ G[:t + 1]
            Z[c0 + t] = output(zpre[None], q[t][None], ln, gamma, beta, eps)[0]
        L = n - 1
        W, S = (Lam[L] * W + C[L] * S - (k * (c[L] * e)[:, None]).T @ G,
                A[L] * S - (k * (a[L] * e)[:, None]).T @ G)
    return Z, W, S


def case(T, seed, ln, rates="mixed"):
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.standard_normal((T, D)) / np.sqrt(D) for _ in range(3))
    eta = 0.5 * (1.0 / D) / (1.0 + np.exp(-rng.standard_normal(T)))
    if rates == "mixed":
        alpha, lam = rng.uniform(0.5, 1.0, T), rng.uniform(0.0, 0.1, T)
    elif rates == "zero":
        alpha, lam = np.zeros(T), np.zeros(T)
    else:  # extremes: no carried momentum, full forgetting
        alpha, lam = rng.choice([0.0, 1.0], T), rng.choice([0.0, 1.0], T)
    W0 = 0.02 * rng.standard_normal((D, D))
    gamma = 1.0 + 0.01 * rng.standard_normal(D) if ln else None
    beta = 0.01 * rng.standard_normal(D) if ln else None
    return Q, K, V, eta, alpha, lam, W0, gamma, beta


def recursion(Q, K, V, eta, alpha, lam, W0, ln, gamma, beta, eps=1e-6):
    kind = oracle.LINEAR_LN if ln else oracle.LINEAR
    Zr, Wr, Sr = oracle.default().momentum_forward(
        kind, Q[None, None], K[None, None], V[None, None], eta[None, None], alpha[None, None],
        lam[None, None], W0.reshape(1, -1), MB, gamma[None] if ln else None, beta[None] if ln else None, eps)
    return Zr[0, 0], Wr[0, 0].reshape(D, D), Sr[0, 0].reshape(D, D)


def rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("rates", ["mixed", "zero", "extremes"])
@pytest.mark.parametrize("T", [16, 48, 64, 128, 208])
@pytest.mark.parametrize("ln", [False, True])
def test_chunked_dual_form_equals_the_recursion(ln, T, rates):
    args = case(T, seed=T + 7 * ln, ln=ln, rates=rates)
    Z, W, S = dual_form(*args[:7], ln, args[7], args[8])
    Zr, Wr, Sr = recursion(*args[:7], ln, args[7], args[8])
    assert rel(Z, Zr) < 1e-11 and rel(W, Wr) < 1e-11
    if np.linalg.norm(Sr) > 0:
        assert rel(S, Sr) < 1e-11


@pytest.mark.parametrize("mistake", ["c_is_a", "strict_diagonal", "decay_on_s"])
def test_planted_coefficient_mistakes_fail(mistake):
    args = case(128, seed=3, ln=True)
    Zr, Wr, Sr = recursion(*args[:7], True, args[7], args[8])
    Z, W, S = dual_form(*args[:7], True, args[7], args[8], mistake=mistake)
    assert max(rel(Z, Zr), rel(W, Wr)) > 1e-3, mistake
