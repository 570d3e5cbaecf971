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
                      variance, eps inside the square root, affine gamma, beta).
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


def _unit_forward(q, k, v, eta, W0, b, ln, gamma, beta, eps):
    """Primal rule for one (batch, head) unit; returns Z [T, d] and the final W.
    W0 must require grad (every state is then a node of the graph)."""
    T = q.shape[0]
    W = W0
    Wbase = W0
    Z = []
    for t in range(T):
        if t % b == 0:
            Wbase = W
        # grad_W l(W_base; k_t, v_t), kept differentiable in W_base, k, v, gamma, beta.
        loss = ((_f(k[t], Wbase, ln, gamma, beta, eps) - v[t]) ** 2).sum()
        g, = torch.autograd.grad(loss, Wbase, create_graph=True)
        W = W - eta[t] * g
        Z.append(_f(q[t], W, ln, gamma, beta, eps))
    return torch.stack(Z), W


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
