"""Pins of the oracle's momentum and decay variant (the Titans-style memory update:
S_t = alpha_t S_{t-1} - eta_t grad l(W_t'), W_t = (1 - lambda_t) W_{t-1} + S_t),
each against something other than the recursion itself: the TTT rule it reduces
to, and closed forms built from the separately pinned gradient and apply routines."""
import numpy as np
import pytest

import oracle

KINDS = [(oracle.LINEAR, 0), (oracle.LINEAR_LN, 0), (oracle.MLP_LN, 16)]


def _setup(kind, hidden, B=2, H=2, T=12, d=6, seed=0):
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.standard_normal((B, H, T, d)) for _ in range(3))
    eta = 0.05 + 0.1 * rng.random((B, H, T))
    P = 2 * d * hidden if kind == oracle.MLP_LN else d * d
    params = 0.2 * rng.standard_normal((H, P))
    gamma = 1.0 + 0.1 * rng.standard_normal((H, d))
    beta = 0.1 * rng.standard_normal((H, d))
    return rng, Q, K, V, eta, params, gamma, beta


@pytest.mark.parametrize("kind,hidden", KINDS)
def test_no_momentum_no_decay_is_ttt(kind, hidden, o=None):
    """alpha = lambda = 0: the variant is the TTT mini-batch rule."""
    _, Q, K, V, eta, params, gamma, beta = _setup(kind, hidden)
    zero = np.zeros_like(eta)
    o = o or oracle.default()
    Z, W, S = o.momentum_forward(kind, Q, K, V, eta, zero, zero, params, 4, gamma, beta, 1e-5, hidden)
    Zt, Wt = o.forward(kind, Q, K, V, eta, params, 4, gamma, beta, 1e-5, hidden)
    assert np.array_equal(Z, Zt) and np.array_equal(W, Wt)


@pytest.mark.parametrize("kind,hidden", KINDS)
def test_decay_alone_with_zero_gradients(kind, hidden, o=None):
    """K = 0 zeroes every gradient (each is k^T times something, or passes through
    GELU(0 W1) = 0), so S stays 0 and W_t = prod_{s<=t} (1 - lambda_s) W0."""
    rng, Q, K, V, eta, params, gamma, beta = _setup(kind, hidden, seed=1)
    K = np.zeros_like(K)
    alpha = rng.random(eta.shape)
    lam = 0.3 * rng.random(eta.shape)
    o = o or oracle.default()
    Z, W, S = o.momentum_forward(kind, Q, K, V, eta, alpha, lam, params, 3, gamma, beta, 1e-5, hidden)
    assert np.all(S == 0.0)
    B, H, T, d = Q.shape
    for bi in range(B):
        for hi in range(H):
            decay = np.cumprod(1.0 - lam[bi, hi])
            for t in range(T):
                Wt = decay[t] * params[hi]
                zt = o.apply(kind, Wt, Q[bi, hi, t], gamma[hi], beta[hi], 1e-5, hidden)
                np.testing.assert_allclose(Z[bi, hi, t], zt, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(W[bi, hi], decay[-1] * params[hi], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("kind,hidden", KINDS)
def test_momentum_in_one_mini_batch(kind, hidden, o=None):
    """b = T, lambda = 0: every gradient g_s is taken at W0, so
    S_t = -sum_{s<=t} (prod_{s<r<=t} alpha_r) eta_s g_s and W_t = W0 + sum_{u<=t} S_u."""
    rng, Q, K, V, eta, params, gamma, beta = _setup(kind, hidden, seed=2)
    alpha = rng.random(eta.shape)
    lam = np.zeros_like(eta)
    B, H, T, d = Q.shape
    o = o or oracle.default()
    Z, W, S = o.momentum_forward(kind, Q, K, V, eta, alpha, lam, params, T, gamma, beta, 1e-5, hidden)
    for bi in range(B):
        for hi in range(H):
            g = np.stack([o.loss_grad(kind, params[hi], K[bi, hi, s], V[bi, hi, s], gamma[hi],
                                      beta[hi], 1e-5, hidden)[1] for s in range(T)])
            Wt = params[hi].copy()
            for t in range(T):
                St = np.zeros_like(Wt)
                for s in range(t + 1):
                    St -= np.prod(alpha[bi, hi, s + 1:t + 1]) * eta[bi, hi, s] * g[s]
                Wt = Wt + St
                zt = o.apply(kind, Wt, Q[bi, hi, t], gamma[hi], beta[hi], 1e-5, hidden)
                np.testing.assert_allclose(Z[bi, hi, t], zt, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(W[bi, hi], Wt, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(S[bi, hi], St, rtol=1e-10, atol=1e-12)


def test_hand_example_scalar(o=None):
    """d = 1, T = b = 2 (both gradients at W0 = 0.5), worked by hand:
    token 1: k=1, v=0, q=1, eta=0.5, alpha=0.5, lambda=0.5
      g1 = 2 k (k w0 - v) = 1,  S1 = -0.5,  W1 = 0.5 * 0.5 - 0.5 = -0.25,  z1 = -0.25
    token 2: k=2, v=1, q=3, eta=0.25, alpha=0.5, lambda=0.5
      g2 = 2 * 2 * (2 * 0.5 - 1) = 0,  S2 = 0.5 * -0.5 = -0.25,
      W2 = 0.5 * -0.25 - 0.25 = -0.375,  z2 = 3 * -0.375 = -1.125."""
    sh = (1, 1, 2, 1)
    Q = np.array([1.0, 3.0]).reshape(sh)
    K = np.array([1.0, 2.0]).reshape(sh)
    V = np.array([0.0, 1.0]).reshape(sh)
    eta = np.array([0.5, 0.25]).reshape(1, 1, 2)
    alpha = np.full((1, 1, 2), 0.5)
    lam = np.full((1, 1, 2), 0.5)
    Z, W, S = (o or oracle.default()).momentum_forward(oracle.LINEAR, Q, K, V, eta, alpha, lam,
                                                       np.array([[0.5]]), 2)
    assert Z.ravel().tolist() == [-0.25, -1.125]
    assert W.ravel().tolist() == [-0.375] and S.ravel().tolist() == [-0.25]


def momentum_pins():
    """(name, callable(orc)) for every momentum pin, for the planted-mistake test."""
    pins = [("hand_example_scalar", lambda orc: test_hand_example_scalar(orc))]
    for kind, hidden in KINDS:
        for fn in (test_no_momentum_no_decay_is_ttt, test_decay_alone_with_zero_gradients,
                   test_momentum_in_one_mini_batch):
            pins.append((f"{fn.__name__[5:]}[{kind}]",
                         (lambda f, k, h: (lambda orc: f(k, h, orc)))(fn, kind, hidden)))
    return pins
