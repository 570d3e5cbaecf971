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


def _gelu(x):
    from scipy.special import erf
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def _gelu_d(x):
    from scipy.special import erf
    phi = np.exp(-0.5 * x * x) / np.sqrt(2.0 * np.pi)
    return 0.5 * (1.0 + erf(x / np.sqrt(2.0))) + x * phi


def _gelu_dd(x):
    phi = np.exp(-0.5 * x * x) / np.sqrt(2.0 * np.pi)
    return phi * (2.0 - x * x)


def _ln_loss_grad(X3, K, V, g, bt, eps):
    """G3 = dl/dX3 of l = ||k + LN(X3) - v||^2 with the context of its VJP."""
    xh, rs = _norm(X3, eps)
    r = K + g * xh + bt - V
    gx = 2 * g * r
    m2 = (gx * xh).mean(-1, keepdims=True)
    return rs * (gx - gx.mean(-1, keepdims=True) - xh * m2), (xh, rs, r, gx, m2)


def _ln_loss_grad_vjp(dG, G, ctx, g):
    """(dX3, dr, dgamma, dbeta) of the map X3 -> G3 at cotangent dG."""
    xh, rs, r, gx, m2 = ctx
    d = xh.shape[-1]
    u = rs * dG
    mu, mux = u.mean(-1, keepdims=True), (u * xh).mean(-1, keepdims=True)
    dsig = -(u * G).sum(-1, keepdims=True)
    dgx = u - mu - xh * mux
    dr = 2 * g * dgx
    dx = -m2 * u - gx * mux + g * dr
    dX3 = rs * (dx - dx.mean(-1, keepdims=True) - xh * (dx * xh).mean(-1, keepdims=True)) + xh * dsig / d
    return dX3, dr, (2 * r * dgx + xh * dr).sum(0), dr.sum(0)


def mlp_reverse_dual_form(q, k, v, eta, W1_0, W2_0, b, dZ, dW1T, dW2T, g, bt, eps):
    """The TTT-MLP reverse step per mini-batch (the derivation a CUDA kernel would
    follow).  Forward, at the base (W1, W2) with E = diag(eta):
      X1 = K W1, X2 = GELU(X1), G3 = dl/dX3 at X3 = X2 W2, H = G3 W2^T,
      G2 = H * GELU'(X1), E2 = E G2, E3 = E G3,
      Z1 = Q W1 - A1 E2 (A1 = tril(Q K^T)), Z2 = GELU(Z1),
      Z3 = Z2 W2 - A2 E3 (A2 = tril(Z2 X2^T)), Z = Q + LN(Z3),
      W1' = W1 - K^T E2, W2' = W2 - X2^T E3.
    Reverse, given dZ, dW1', dW2': P3 = LN backward of dZ;
      M2 = tril(P3 E3^T): dZ2 = P3 W2^T - M2 X2, dX2 = -M2^T Z2 - E3 dW2'^T,
      dE3 = -A2^T P3 - X2 dW2',  dW2 = dW2' + Z2^T P3;
      dZ1 = dZ2 * GELU'(Z1), M1 = tril(dZ1 E2^T): dQ += dZ1 W1^T - M1 K,
      dK = -M1^T Q - E2 dW1'^T, dE2 = -A1^T dZ1 - K dW1', dW1 = dW1' + Q^T dZ1;
      deta = rowsum(dE2 G2 + dE3 G3), dG2 = E dE2, dG3 = E dE3;
      dH = dG2 * GELU'(X1), dX1 = dG2 * H * GELU''(X1),
      dG3 += dH W2, dW2 += dH^T G3;
      (dX3, dr) = VJP of the LN loss gradient at dG3: dK += dr, dV = -dr;
      dX2 += dX3 W2^T, dW2 += X2^T dX3;  dX1 += dX2 * GELU'(X1);
      dK += dX1 W1^T, dW1 += K^T dX1."""
    T, d = q.shape
    N = T // b
    ck, W1, W2 = [], W1_0.copy(), W2_0.copy()
    for n in range(N):
        s = slice(n * b, (n + 1) * b)
        ck.append((W1.copy(), W2.copy()))
        X1 = k[s] @ W1
        X2 = _gelu(X1)
        G3, _ = _ln_loss_grad(X2 @ W2, k[s], v[s], g, bt, eps)
        G2 = (G3 @ W2.T) * _gelu_d(X1)
        e = eta[s, None]
        W1, W2 = W1 - k[s].T @ (e * G2), W2 - X2.T @ (e * G3)
    tril = np.tril(np.ones((b, b)))
    dW1, dW2 = dW1T.copy(), dW2T.copy()
    out = {n: np.zeros((T, d)) for n in ("dQ", "dK", "dV")}
    out.update(deta=np.zeros(T), dgamma=np.zeros(d), dbeta=np.zeros(d))
    for n in reversed(range(N)):
        s = slice(n * b, (n + 1) * b)
        Q, K, V, e = q[s], k[s], v[s], eta[s, None]
        W1, W2 = ck[n]
        X1 = K @ W1
        X2 = _gelu(X1)
        G3, ctx = _ln_loss_grad(X2 @ W2, K, V, g, bt, eps)
        H = G3 @ W2.T
        G2 = H * _gelu_d(X1)
        E2, E3 = e * G2, e * G3
        A1 = tril * (Q @ K.T)
        Z1 = Q @ W1 - A1 @ E2
        Z2 = _gelu(Z1)
        A2 = tril * (Z2 @ X2.T)
        zh, rz = _norm(Z2 @ W2 - A2 @ E3, eps)
        gz = dZ[s] * g
        P3 = rz * (gz - gz.mean(-1, keepdims=True) - zh * (gz * zh).mean(-1, keepdims=True))
        out["dgamma"] += (dZ[s] * zh).sum(0)
        out["dbeta"] += dZ[s].sum(0)
        M2 = tril * (P3 @ E3.T)
        dZ2 = P3 @ W2.T - M2 @ X2
        dX2 = -M2.T @ Z2 - E3 @ dW2.T
        dE3 = -A2.T @ P3 - X2 @ dW2
        dW2n = dW2 + Z2.T @ P3
        dZ1 = dZ2 * _gelu_d(Z1)
        M1 = tril * (dZ1 @ E2.T)
        dQ = dZ[s] + dZ1 @ W1.T - M1 @ K
        dK = -M1.T @ Q - E2 @ dW1.T
        dE2 = -A1.T @ dZ1 - K @ dW1
        dW1n = dW1 + Q.T @ dZ1
        out["deta"][s] = (dE2 * G2).sum(-1) + (dE3 * G3).sum(-1)
        dG2, dG3 = e * dE2, e * dE3
        dH = dG2 * _gelu_d(X1)
        dX1 = dG2 * H * _gelu_dd(X1)
        dG3 = dG3 + dH @ W2
        dW2n = dW2n + dH.T @ G3
        dX3, dr, dgam, dbet = _ln_loss_grad_vjp(dG3, G3, ctx, g)
        out["dgamma"] += dgam
        out["dbeta"] += dbet
        dK = dK + dr
        out["dV"][s] = -dr
        dX2 = dX2 + dX3 @ W2.T
        dW2n = dW2n + X2.T @ dX3
        dX1 = dX1 + dX2 * _gelu_d(X1)
        dK = dK + dX1 @ W1.T
        dW1n = dW1n + K.T @ dX1
        out["dQ"][s], out["dK"][s] = dQ, dK
        dW1, dW2 = dW1n, dW2n
    out["dW1"], out["dW2"] = dW1, dW2
    return out


@pytest.mark.parametrize("b", [1, 3, 8])
def test_mlp_reverse_dual_form_equals_autograd(b):
    rng = np.random.default_rng(200 + b)
    T, d, h = 24, 4, 16
    q, k, v, dZ = (rng.standard_normal((T, d)) for _ in range(4))
    eta = 0.05 + 0.2 * rng.random(T)
    W1, W2 = 0.4 * rng.standard_normal((d, h)), 0.4 * rng.standard_normal((h, d))
    g, bt = 1 + 0.2 * rng.standard_normal(d), 0.2 * rng.standard_normal(d)
    dW1T, dW2T = rng.standard_normal((d, h)), rng.standard_normal((h, d))
    got = mlp_reverse_dual_form(q, k, v, eta, W1, W2, b, dZ, dW1T, dW2T, g, bt, 1e-5)
    ref = OB.ttt_mlp_backward(q[None, None], k[None, None], v[None, None], eta[None, None], W1[None],
                              W2[None], b, dZ[None, None], g[None], bt[None], 1e-5, dW1T[None, None],
                              dW2T[None, None])
    for key in ("dQ", "dK", "dV", "deta", "dW1", "dW2", "dgamma", "dbeta"):
        r = ref[key][0, 0]
        assert np.abs(got[key] - r).max() <= 1e-11 * max(1.0, np.abs(r).max()), key
