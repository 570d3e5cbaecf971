"""fp64 CPU oracle of the TTT-Linear backward pass (gradients of the forward).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import it.

The TTT write-up trains its layer end to end: the forward has a matching
backward pass through the mini-batch chain (§04 "Implementation details", and
the dual form's use for the backward in §04.3).  What it computes is fixed by
the forward alone: for a scalar objective L = <dZ, Z> + <dW_T, W_T> (dZ, dW_T
the incoming cotangents), the gradients of L with respect to Q, K, V, eta, W0,
gamma and beta.  This oracle is that definition written out: the forward is the
primal token-by-token mini-batch rule (each gradient taken at the state its
mini-batch started from, §03.6; z_t = f(q_t; W_t) at the updated state, §03.1),
the inner gradient grad_W l(W; k, v) of l = ||f(k; W) - v||^2 (§03.5) is taken
by torch.autograd with create_graph, and the outer gradients by autograd again,
all in float64 on the CPU.  No blocking, no dual form, no hand-written adjoint.

f is  x W            (TTT-Linear), or
      x + LN(x W)    (TTT-Linear with LayerNorm and residual, §03.9; population
                      variance, eps inside the square root, affine gamma, beta),
      x + LN(GELU(x W1) W2)   (TTT-MLP, §03.9: hidden width 4d, exact GELU).
"""
from __future__ import annotations

import numpy as np
import torch

_f64 = torch.float64


def _ln(y, gamma, beta, eps):
    mu = y.mean(-1, keepdim=True)
    var = ((y - mu) ** 2).mean(-1, keepdim=True)
    return gamma * (y - mu) / torch.sqrt(var + eps) + beta


def _f(x, W, ln, gamma, beta, eps):
    y = x @ W
    return x + _ln(y, gamma, beta, eps) if ln else y


def _f_mlp(x, Ws, gamma, beta, eps):
    return x + _ln(torch.nn.functional.gelu(x @ Ws[0]) @ Ws[1], gamma, beta, eps)


def _unit_forward_states(q, k, v, eta, W0s, b, f):
    """Primal rule for one (batch, head) unit with the state a list of matrices
    and f(x, states); returns Z [T, d] and the final states.  Every W0 must
    require grad (every state is then a node of the graph)."""
    Ws = list(W0s)
    base = Ws
    Z = []
    for t in range(q.shape[0]):
        if t % b == 0:
            base = Ws
        # grad_W l(W_base; k_t, v_t), kept differentiable in W_base, k, v, gamma, beta.
        loss = ((f(k[t], base) - v[t]) ** 2).sum()
        grads = torch.autograd.grad(loss, base, create_graph=True)
        Ws = [W - eta[t] * g for W, g in zip(Ws, grads)]
        Z.append(f(q[t], Ws))
    return torch.stack(Z), Ws


def _unit_forward(q, k, v, eta, W0, b, ln, gamma, beta, eps):
    """TTT-Linear (or with LN) for one unit; returns Z [T, d] and the final W."""
    Z, Ws = _unit_forward_states(q, k, v, eta, [W0], b,
                                 lambda x, Ws: _f(x, Ws[0], ln, gamma, beta, eps))
    return Z, Ws[0]


def ttt_linear_backward(Q, K, V, eta, W0, b, dZ, dW_T=None, ln=False, gamma=None, beta=None,
                        eps=1e-6):
    """Gradients of L = <dZ, Z> + <dW_T, W_T> through the TTT-Linear forward.

    Q, K, V, dZ [B,H,T,d]; eta [B,H,T]; W0 [H,d,d] (per head); gamma, beta [H,d]
    (LN only); dW_T [B,H,d,d] or None (zero).  Returns a dict of float64 arrays:
    dQ, dK, dV [B,H,T,d], deta [B,H,T], dW0 [B,H,d,d] (per unit: a W0 shared by
    the batch has the sum over the batch as its gradient), and for LN dgamma,
    dbeta [B,H,d] (per unit likewise).
    """
    Q, K, V, eta, dZ = (np.asarray(x, np.float64) for x in (Q, K, V, eta, dZ))
    W0 = np.asarray(W0, np.float64)
    B, H, T, d = Q.shape
    out = {k: np.zeros((B, H, T, d)) for k in ("dQ", "dK", "dV")}
    out["deta"] = np.zeros((B, H, T))
    out["dW0"] = np.zeros((B, H, d, d))
    if ln:
        out["dgamma"] = np.zeros((B, H, d))
        out["dbeta"] = np.zeros((B, H, d))
    for bi in range(B):
        for hi in range(H):
            leaves = [torch.tensor(x[bi, hi], dtype=_f64, requires_grad=True) for x in (Q, K, V, eta)]
            w0 = torch.tensor(W0[hi], dtype=_f64, requires_grad=True)
            g = bt = None
            if ln:
                g = torch.tensor(np.asarray(gamma, np.float64)[hi], requires_grad=True)
                bt = torch.tensor(np.asarray(beta, np.float64)[hi], requires_grad=True)
            Z, W = _unit_forward(*leaves, w0, b, ln, g, bt, eps)
            L = (Z * torch.tensor(dZ[bi, hi])).sum()
            if dW_T is not None:
                L = L + (W * torch.tensor(np.asarray(dW_T, np.float64)[bi, hi])).sum()
            wrt = leaves + [w0] + ([g, bt] if ln else [])
            grads = torch.autograd.grad(L, wrt, allow_unused=True)
            grads = [np.zeros(x.shape) if gr is None else gr.detach().numpy() for gr, x in zip(grads, wrt)]
            out["dQ"][bi, hi], out["dK"][bi, hi], out["dV"][bi, hi] = grads[0], grads[1], grads[2]
            out["deta"][bi, hi] = grads[3]
            out["dW0"][bi, hi] = grads[4]
            if ln:
                out["dgamma"][bi, hi], out["dbeta"][bi, hi] = grads[5], grads[6]
    return out


def ttt_mlp_backward(Q, K, V, eta, W1, W2, b, dZ, gamma, beta, eps=1e-6, dW1_T=None, dW2_T=None):
    """Gradients of L = <dZ, Z> + <dW1_T, W1_T> + <dW2_T, W2_T> through the TTT-MLP
    forward.  Q, K, V, dZ [B,H,T,d]; eta [B,H,T]; W1 [H,d,h], W2 [H,h,d], gamma,
    beta [H,d] (per head); dW1_T [B,H,d,h], dW2_T [B,H,h,d] or None.  Returns a
    dict of float64 arrays: dQ, dK, dV, deta, and per (batch, head) unit dW1,
    dW2 (of the initial states), dgamma, dbeta."""
    Q, K, V, eta, dZ = (np.asarray(x, np.float64) for x in (Q, K, V, eta, dZ))
    W1, W2 = np.asarray(W1, np.float64), np.asarray(W2, np.float64)
    B, H, T, d = Q.shape
    h = W1.shape[-1]
    out = {k: np.zeros((B, H, T, d)) for k in ("dQ", "dK", "dV")}
    out["deta"] = np.zeros((B, H, T))
    out["dW1"] = np.zeros((B, H, d, h))
    out["dW2"] = np.zeros((B, H, h, d))
    out["dgamma"] = np.zeros((B, H, d))
    out["dbeta"] = np.zeros((B, H, d))
    for bi in range(B):
        for hi in range(H):
            leaves = [torch.tensor(x[bi, hi], dtype=_f64, requires_grad=True) for x in (Q, K, V, eta)]
            w1 = torch.tensor(W1[hi], requires_grad=True)
            w2 = torch.tensor(W2[hi], requires_grad=True)
            g = torch.tensor(np.asarray(gamma, np.float64)[hi], requires_grad=True)
            bt = torch.tensor(np.asarray(beta, np.float64)[hi], requires_grad=True)
            Z, (W1T, W2T) = _unit_forward_states(*leaves, [w1, w2], b,
                                                 lambda x, Ws: _f_mlp(x, Ws, g, bt, eps))
            L = (Z * torch.tensor(dZ[bi, hi])).sum()
            if dW1_T is not None:
                L = L + (W1T * torch.tensor(np.asarray(dW1_T, np.float64)[bi, hi])).sum()
            if dW2_T is not None:
                L = L + (W2T * torch.tensor(np.asarray(dW2_T, np.float64)[bi, hi])).sum()
            wrt = leaves + [w1, w2, g, bt]
            grads = torch.autograd.grad(L, wrt, allow_unused=True)
            grads = [np.zeros(x.shape) if gr is None else gr.detach().numpy() for gr, x in zip(grads, wrt)]
            for key, gr in zip(("dQ", "dK", "dV", "deta", "dW1", "dW2", "dgamma", "dbeta"), grads):
                out[key][bi, hi] = gr
    return out
