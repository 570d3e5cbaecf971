"""The reverse dual-form step that the backward kernel implements, restated in
fp64 numpy exactly as the kernel's header writes it (per mini-batch: recompute
G, E, A and the output LN from the checkpointed base, then P, M, dQ, dE, deta,
dG, the VJP of the gradient's LN, dK, dV, dW), must equal the autograd oracle to
rounding.  This pins the derivation itself, independently of the GPU.  No GPU."""
import numpy as np
import pytest

from oracle import backward as OB


def _norm(y, eps):
    mu = y.mean(-1, keepdims=True)
    var = ((y - mu) ** 2).mean(-1, keepdims=True)
    return (y - mu) / np.sqrt(var + eps), 1.0 / np.sqrt(var + eps)


def _grad(Y, K, V, ln, g, bt, eps):
    if not ln:
        return 2 * (Y - V), None
    xh, rs = _norm(Y, eps)
    r = K + g * xh + bt - V
    gx = 2 * g * r
    m1, m2 = gx.mean(-1, keepdims=True), (gx * xh).mean(-1, keepdims=True)
    return rs * (gx - m1 - xh * m2), (xh, rs, r, gx, m2)


def reverse_dual_form(q, k, v, eta, W0, b, dZ, dWT, ln, g, bt, eps):
    T, d = q.shape
    N = T // b
    ck, W = [], W0.copy()
    for n in range(N):
        s = slice(n * b, (n + 1) * b)
        ck.append(W.copy())
        G, _ = _grad(k[s] @ W, k[s], v[s], ln, g, bt, eps)
        W = W - k[s].T @ (eta[s, None] * G)
    tril = np.tril(np.ones((b, b)))
    dW = dWT.copy()
    out = {n: np.zeros((T, d)) for n in ("dQ", "dK", "dV")}
    out.update(deta=np.zeros(T), dgamma=np.zeros(d), dbeta=np.zeros(d))
    for n in reversed(range(N)):
        s = slice(n * b, (n + 1) * b)
        Q, K, V, e, W = q[s], k[s], v[s], eta[s, None], ck[n]
        G, ctx = _grad(K @ W, K, V, ln, g, bt, eps)
        E, A = e * G, tril * (Q @ K.T)
        if ln:
            zh, rz = _norm(Q @ W - A @ E, eps)
            gz = dZ[s] * g
            P = rz * (gz - gz.mean(-1, keepdims=True) - zh * (gz * zh).mean(-1, keepdims=True))
            out["dgamma"] += (dZ[s] * zh).sum(0)
            out["dbeta"] += dZ[s].sum(0)
        else:
            P = dZ[s]
        M = tril * (P @ E.T)
        out["dQ"][s] = P @ W.T - M @ K + (dZ[s] if ln else 0)
        dE = -A.T @ P - K @ dW
        out["deta"][s] = (dE * G).sum(-1)
        dG = e * dE
        if ln:
            xh, rs, r, gx, m2 = ctx
            u = rs * dG
            mu, mux = u.mean(-1, keepdims=True), (u * xh).mean(-1, keepdims=True)
            dsig = -(u * G).sum(-1, keepdims=True)
            dgx = u - mu - xh * mux
            dr = 2 * g * dgx
            out["dgamma"] += (2 * r * dgx + xh * dr).sum(0)
            out["dbeta"] += dr.sum(0)
            dx = -m2 * u - gx * mux + g * dr
            dY = rs * (dx - dx.mean(-1, keepdims=True) - xh * (dx * xh).mean(-1, keepdims=True)) \
                + xh * dsig / d
            out["dV"][s] = -dr
        else:
            dY = 2 * dG
            dr = 0
            out["dV"][s] = -dY
        out["dK"][s] = -M.T @ Q - E @ dW.T + dY @ W.T + dr
        dW = dW + Q.T @ P + K.T @ dY
    out["dW0"] = dW
    return out


@pytest.mark.parametrize("ln", [False, True])
@pytest.mark.parametrize("b", [1, 3, 8])
def test_reverse_dual_form_equals_autograd(ln, b):
    rng = np.random.default_rng(100 + b + 10 * ln)
    T, d = 24, 6
    q, k, v, dZ = (rng.standard_normal((T, d)) for _ in range(4))
    eta = 0.05 + 0.2 * rng.random(T)
    W0 = 0.3 * rng.standard_normal((d, d))
    g, bt = 1 + 0.2 * rng.standard_normal(d), 0.2 * rng.standard_normal(d)
    dWT = rng.standard_normal((d, d))
    got = reverse_dual_form(q, k, v, eta, W0, b, dZ, dWT, ln, g, bt, 1e-5)
    ref = OB.ttt_linear_backward(q[None, None], k[None, None], v[None, None], eta[None, None],
                                 W0[None], b, dZ[None, None], dWT[None, None], ln, g[None], bt[None],
                                 1e-5)
    keys = ["dQ", "dK", "dV", "deta", "dW0"] + (["dgamma", "dbeta"] if ln else [])
    for key in keys:
        r = ref[key][0, 0]
        assert np.abs(got[key] - r).max() <= 1e-12 * max(1.0, np.abs(r).max()), key
