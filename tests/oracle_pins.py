"""Pins of the fp64 oracle to things other than itself.

Each pin takes an ``oracle.Oracle`` handle and raises AssertionError when the
oracle disagrees with an independent statement of the method:

* hand-derived worked examples (``golden/hand_linear.json``);
* the dual form (TTT write-up §03.7): whole mini-batches as masked matrix
  products, with the gradient with respect to the pre-activations taken by
  torch.autograd instead of any hand-written backward;
* online GD (b = 1, §03.6) and batch GD (one mini-batch, §03.8) stated through
  autograd of the loss, not through the oracle's gradient code;
* eta = 0: the output is f(Q; W0), checked against torch's own layer_norm and
  exact GELU, and the state is returned unchanged;
* W0 = 0 with one mini-batch: TTT-Linear reduces to (unnormalised, causal)
  linear attention scaled by 2 eta (§03.8 "theoretical equivalence");
* central finite differences of the oracle's own loss against its gradient;
* descent: a small step lowers that token's loss (§03.1, Fig. 5);
* segmentation: the fixed-size state carries across calls.

The pins run at small sizes (d = 8, h = 4d, b = 4) where every check finishes in
well under a second, and with parameters scaled so that each term is visible:
a widely spread LN gamma, a non-zero beta, non-symmetric W and an epsilon large
enough for its placement to matter.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch
import torch.nn.functional as F

from oracle import LINEAR, LINEAR_LN, MLP_LN

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
KIND_NAMES = {LINEAR: "linear", LINEAR_LN: "linear_ln", MLP_LN: "mlp"}
TOL = 1e-10  # fp64 reorderings differ by ~1e-15; any real mistake is >> 1e-6


def rel_err(a, b) -> float:
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def rand_case(kind, seed, B=2, H=2, T=12, d=8, b=4, eta_scale=0.05, eps=1e-2):
    rng = np.random.default_rng(seed)
    h = 4 * d
    c = {"kind": kind, "b": b, "d": d, "h": h, "eps": eps}
    c["Q"] = rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    c["K"] = rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    c["V"] = rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    c["eta"] = eta_scale * (0.5 + rng.random((B, H, T)))
    if kind == MLP_LN:
        c["params"] = np.concatenate([0.4 * rng.standard_normal((H, d * h)),
                                      0.2 * rng.standard_normal((H, h * d))], axis=1)
    else:
        c["params"] = 0.3 * rng.standard_normal((H, d * d))
    c["gamma"] = 1.0 + 0.3 * rng.standard_normal((H, d))
    c["beta"] = 0.3 * rng.standard_normal((H, d))
    return c


def run_oracle(orc, c, nthreads=0):
    ln = c["kind"] != LINEAR
    return orc.forward(c["kind"], c["Q"], c["K"], c["V"], c["eta"], c["params"], c["b"],
                       c["gamma"] if ln else None, c["beta"] if ln else None, c["eps"],
                       hidden=c["h"] if c["kind"] == MLP_LN else 0, nthreads=nthreads)


# --- torch statement of f (library layer_norm and exact GELU) --------------

def t_split(kind, P, d, h):
    if kind == MLP_LN:
        return P[: d * h].reshape(d, h), P[d * h:].reshape(h, d)
    return (P.reshape(d, d),)


def t_f(kind, P, x, gamma, beta, eps, d, h):
    """f(x; W) for rows x [n, d]."""
    if kind == MLP_LN:
        W1, W2 = t_split(kind, P, d, h)
        y = F.gelu(x @ W1, approximate="none") @ W2
    else:
        y = x @ t_split(kind, P, d, h)[0]
    if kind == LINEAR:
        return y
    return x + F.layer_norm(y, (d,), gamma, beta, eps)


def _unit(c, bi, hi):
    T = lambda a: torch.tensor(a, dtype=torch.float64)  # noqa: E731
    return (T(c["Q"][bi, hi]), T(c["K"][bi, hi]), T(c["V"][bi, hi]), T(c["eta"][bi, hi]),
            T(c["params"][hi]), T(c["gamma"][hi]), T(c["beta"][hi]))


# --- pins --------------------------------------------------------------------

def pin_hand_examples(orc):
    """Hand-derived TTT-Linear examples (mini-batch and online) match exactly."""
    with open(os.path.join(GOLDEN, "hand_linear.json")) as f:
        data = json.load(f)
    for case in data["cases"]:
        d = case["d"]
        Q, K, V = (np.array(case[k], np.float64)[None, None] for k in ("Q", "K", "V"))
        eta = np.array(case["eta"], np.float64)[None, None]
        W0 = np.array(case["W0"], np.float64).reshape(1, d * d)
        for res in case["results"]:
            Z, W = orc.forward(LINEAR, Q, K, V, eta, W0, res["b"])
            assert np.allclose(Z[0, 0], np.array(res["Z"]), rtol=0, atol=1e-14), (case["name"], res["b"], Z)
            assert np.allclose(W[0, 0], np.array(res["W"]).ravel(), rtol=0, atol=1e-14), (case["name"], res["b"], W)


def dual_form_unit(c, bi, hi):
    """Dual form over whole mini-batches (§03.7), gradients w.r.t. pre-activations by
    autograd.  Returns (Z [T,d], params [P])."""
    kind, b, d, h, eps = c["kind"], c["b"], c["d"], c["h"], c["eps"]
    Q, K, V, eta, P, gamma, beta = _unit(c, bi, hi)
    T = Q.shape[0]
    LN = lambda y: F.layer_norm(y, (d,), gamma, beta, eps)  # noqa: E731
    Zs = []
    if kind == MLP_LN:
        W1, W2 = t_split(kind, P, d, h)
    else:
        (W,) = t_split(kind, P, d, h)
    for n in range(T // b):
        s = slice(n * b, (n + 1) * b)
        Qn, Kn, Vn, en = Q[s], K[s], V[s], eta[s]
        A = torch.tril(Qn @ Kn.T) * en[None, :]  # (q_t . k_s) eta_s for s <= t
        if kind == MLP_LN:
            X1 = (Kn @ W1).detach().requires_grad_(True)
            X2 = F.gelu(X1, approximate="none")
            X3 = X2 @ W2
            loss = ((Kn + LN(X3) - Vn) ** 2).sum()
            G2, G3 = torch.autograd.grad(loss, [X1, X3])
            X2 = X2.detach()
            Zq1 = Qn @ W1 - A @ G2
            Zq2 = F.gelu(Zq1, approximate="none")
            A2 = torch.tril(Zq2 @ X2.T) * en[None, :]
            Zq3 = Zq2 @ W2 - A2 @ G3
            Zs.append(Qn + LN(Zq3))
            W1 = W1 - Kn.T @ (en[:, None] * G2)
            W2 = W2 - X2.T @ (en[:, None] * G3)
        else:
            Y = (Kn @ W).detach().requires_grad_(True)
            out = Y if kind == LINEAR else Kn + LN(Y)
            (G,) = torch.autograd.grad(((out - Vn) ** 2).sum(), [Y])
            Zpre = Qn @ W - A @ G
            Zs.append(Zpre if kind == LINEAR else Qn + LN(Zpre))
            W = W - Kn.T @ (en[:, None] * G)
    Pn = torch.cat([W1.reshape(-1), W2.reshape(-1)]) if kind == MLP_LN else W.reshape(-1)
    return torch.cat(Zs).numpy(), Pn.detach().numpy()


def pin_dual_form(orc, kind, seed=0, **kw):
    """Primal oracle == dual form on every unit, to fp64 reordering error."""
    c = rand_case(kind, seed, **kw)
    Z, W = run_oracle(orc, c)
    B, H = c["Q"].shape[:2]
    for bi in range(B):
        for hi in range(H):
            Zd, Wd = dual_form_unit(c, bi, hi)
            assert rel_err(Z[bi, hi], Zd) < TOL, (KIND_NAMES[kind], "Z", rel_err(Z[bi, hi], Zd))
            assert rel_err(W[bi, hi], Wd) < TOL, (KIND_NAMES[kind], "W", rel_err(W[bi, hi], Wd))


def pin_online_gd(orc, kind, seed=1):
    """b = 1 is online GD: W_t = W_{t-1} - eta_t grad l(W_{t-1}; k_t, v_t), z_t = f(q_t; W_t),
    with the gradient taken by autograd."""
    c = rand_case(kind, seed, B=1, H=2, T=6, b=1)
    Z, W = run_oracle(orc, c)
    d, h, eps = c["d"], c["h"], c["eps"]
    for hi in range(2):
        Q, K, V, eta, P, gamma, beta = _unit(c, 0, hi)
        Zr = []
        for t in range(Q.shape[0]):
            Pl = P.clone().requires_grad_(True)
            loss = ((t_f(kind, Pl, K[t:t + 1], gamma, beta, eps, d, h) - V[t:t + 1]) ** 2).sum()
            (g,) = torch.autograd.grad(loss, [Pl])
            P = P - eta[t] * g
            Zr.append(t_f(kind, P, Q[t:t + 1], gamma, beta, eps, d, h))
        Zr = torch.cat(Zr).detach().numpy()
        assert rel_err(Z[0, hi], Zr) < TOL, (KIND_NAMES[kind], rel_err(Z[0, hi], Zr))
        assert rel_err(W[0, hi], P.detach().numpy()) < TOL, KIND_NAMES[kind]


def pin_batch_gd(orc, kind, seed=2):
    """One mini-batch (T = b) is batch GD from W0.  The state after token t is
    W0 - grad_W sum_{s<=t} eta_s l(W0; k_s, v_s): the gradient of an eta-weighted
    prefix loss, taken by autograd in one call per prefix."""
    c = rand_case(kind, seed, B=1, H=1, T=5, b=5)
    Z, W = run_oracle(orc, c)
    d, h, eps = c["d"], c["h"], c["eps"]
    Q, K, V, eta, P0, gamma, beta = _unit(c, 0, 0)
    Zr = []
    for t in range(5):
        Pl = P0.clone().requires_grad_(True)
        per_tok = ((t_f(kind, Pl, K[: t + 1], gamma, beta, eps, d, h) - V[: t + 1]) ** 2).sum(1)
        (g,) = torch.autograd.grad((eta[: t + 1] * per_tok).sum(), [Pl])
        Pt = P0 - g
        Zr.append(t_f(kind, Pt, Q[t:t + 1], gamma, beta, eps, d, h))
    Zr = torch.cat(Zr).detach().numpy()
    assert rel_err(Z[0, 0], Zr) < TOL, (KIND_NAMES[kind], rel_err(Z[0, 0], Zr))
    assert rel_err(W[0, 0], Pt.detach().numpy()) < TOL, KIND_NAMES[kind]


def pin_eta_zero(orc, kind, seed=3):
    """eta = 0: Z = f(Q; W0) (torch layer_norm, exact GELU) and the state is unchanged."""
    c = rand_case(kind, seed)
    c["eta"] = np.zeros_like(c["eta"])
    Z, W = run_oracle(orc, c)
    B, H = c["Q"].shape[:2]
    for bi in range(B):
        for hi in range(H):
            Q, K, V, eta, P, gamma, beta = _unit(c, bi, hi)
            Zr = t_f(kind, P, Q, gamma, beta, c["eps"], c["d"], c["h"]).numpy()
            assert rel_err(Z[bi, hi], Zr) < TOL, (KIND_NAMES[kind], rel_err(Z[bi, hi], Zr))
            assert np.array_equal(W[bi, hi], c["params"][hi]), KIND_NAMES[kind]


def pin_linear_attention(orc, seed=4):
    """TTT-Linear, W0 = 0, one mini-batch: z_t = sum_{s<=t} 2 eta_s (q_t . k_s) v_s and
    W = sum_s 2 eta_s k_s^T v_s (causal linear attention scaled by 2 eta)."""
    c = rand_case(LINEAR, seed, B=1, H=1, T=6, b=6)
    c["params"] = np.zeros_like(c["params"])
    Z, W = run_oracle(orc, c)
    q, k, v, eta = c["Q"][0, 0], c["K"][0, 0], c["V"][0, 0], c["eta"][0, 0]
    d = c["d"]
    Zr = np.zeros((6, d))
    Wr = np.zeros((d, d))
    for t in range(6):
        for s in range(t + 1):
            Zr[t] += 2.0 * eta[s] * float(np.dot(q[t], k[s])) * v[s]
    for s in range(6):
        Wr += 2.0 * eta[s] * np.outer(k[s], v[s])
    assert rel_err(Z[0, 0], Zr) < TOL, rel_err(Z[0, 0], Zr)
    assert rel_err(W[0, 0], Wr.ravel()) < TOL, rel_err(W[0, 0], Wr.ravel())


def pin_gradient(orc, kind, seed=5):
    """The oracle's per-token loss equals ||f(k;W) - v||^2 from torch, its gradient equals
    autograd's, and central finite differences of its own loss agree with its gradient."""
    c = rand_case(kind, seed, B=1, H=1, T=1, b=1)
    d, h, eps = c["d"], c["h"], c["eps"]
    P, k, v = c["params"][0], c["K"][0, 0, 0], c["V"][0, 0, 0]
    gamma, beta = c["gamma"][0], c["beta"][0]
    hid = h if kind == MLP_LN else 0
    loss, grad = orc.loss_grad(kind, P, k, v, gamma, beta, eps, hidden=hid)
    Pt = torch.tensor(P, requires_grad=True)
    tk, tv = torch.tensor(k)[None], torch.tensor(v)[None]
    lt = ((t_f(kind, Pt, tk, torch.tensor(gamma), torch.tensor(beta), eps, d, h) - tv) ** 2).sum()
    (gt,) = torch.autograd.grad(lt, [Pt])
    assert abs(loss - lt.item()) <= TOL * max(1.0, abs(loss)), (KIND_NAMES[kind], loss, lt.item())
    assert rel_err(grad, gt.numpy()) < TOL, (KIND_NAMES[kind], rel_err(grad, gt.numpy()))
    rng = np.random.default_rng(seed)
    hstep = 1e-5
    for _ in range(4):
        u = rng.standard_normal(P.shape)
        u /= np.linalg.norm(u)
        lp, _ = orc.loss_grad(kind, P + hstep * u, k, v, gamma, beta, eps, hidden=hid)
        lm, _ = orc.loss_grad(kind, P - hstep * u, k, v, gamma, beta, eps, hidden=hid)
        fd = (lp - lm) / (2 * hstep)
        an = float(np.dot(grad, u))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (KIND_NAMES[kind], fd, an)


def pin_descent(orc, kind, seed=6):
    """With a small step, the token's own loss falls after its update (b = 1)."""
    c = rand_case(kind, seed, B=1, H=1, T=8, b=1, eta_scale=1e-3)
    d, h, eps = c["d"], c["h"], c["eps"]
    hid = h if kind == MLP_LN else 0
    gamma, beta = c["gamma"][0], c["beta"][0]
    P = c["params"]
    for t in range(8):
        sl = lambda a: a[:, :, t:t + 1]  # noqa: E731
        _, Wn = orc.forward(kind, sl(c["Q"]), sl(c["K"]), sl(c["V"]), sl(c["eta"]), P, 1,
                            gamma[None] if kind != LINEAR else None,
                            beta[None] if kind != LINEAR else None, eps, hidden=hid)
        k, v = c["K"][0, 0, t], c["V"][0, 0, t]
        before, _ = orc.loss_grad(kind, P[0], k, v, gamma, beta, eps, hidden=hid)
        after, _ = orc.loss_grad(kind, Wn[0, 0], k, v, gamma, beta, eps, hidden=hid)
        assert after < before, (KIND_NAMES[kind], t, before, after)
        P = Wn[0]


def pin_segmentation(orc, kind, seed=7):
    """Running [0, T) equals running [0, T1) then [T1, T) from the carried state."""
    c = rand_case(kind, seed, B=1, H=2, T=12, b=4)
    Z, W = run_oracle(orc, c)
    first = dict(c, Q=c["Q"][:, :, :8], K=c["K"][:, :, :8], V=c["V"][:, :, :8], eta=c["eta"][:, :, :8])
    Z1, W1 = run_oracle(orc, first)
    second = dict(c, Q=c["Q"][:, :, 8:], K=c["K"][:, :, 8:], V=c["V"][:, :, 8:], eta=c["eta"][:, :, 8:],
                  params=W1[0])
    Z2, W2 = run_oracle(orc, second)
    assert rel_err(np.concatenate([Z1, Z2], axis=2), Z) < TOL, KIND_NAMES[kind]
    assert rel_err(W2, W) < TOL, KIND_NAMES[kind]


ALL_KINDS = (LINEAR, LINEAR_LN, MLP_LN)


def all_pins():
    """(name, callable(orc)) for every pin."""
    pins = [("hand_examples", pin_hand_examples), ("linear_attention", pin_linear_attention)]
    for kind in ALL_KINDS:
        n = KIND_NAMES[kind]
        for fn in (pin_dual_form, pin_online_gd, pin_batch_gd, pin_eta_zero, pin_gradient,
                   pin_descent, pin_segmentation):
            pins.append((f"{fn.__name__[4:]}[{n}]", (lambda f, k: (lambda orc: f(orc, k)))(fn, kind)))
    return pins
