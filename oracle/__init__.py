"""fp64 CPU oracle of the TTT layer forward (primal, token-by-token mini-batch rule).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library and its Python binding never import it.

The arithmetic lives in ``ttt_oracle.c`` (plain C, float64); this module only
marshals numpy arrays into it.  Method, sources and readings are stated in the
header of ``ttt_oracle.c``: output rule z_t = f(q_t; W_t) at the updated
weight and update W_t = W_{t-1} - eta_t * grad l(W_{t'}; k_t, v_t) with
t' = t - mod(t, b) (TTT write-up, §03.1 "TTT hidden state" and §03.6
"mini-batch TTT"), loss ||f(k; W) - v||^2 (§03.5), f linear, linear + LN +
residual, or a GELU MLP + LN + residual (§03.9 "two variants").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ttt_oracle.c")
LIB = os.path.join(HERE, "libttt_oracle.so")

LINEAR, LINEAR_LN, MLP_LN = 0, 1, 2
KINDS = {"linear": LINEAR, "linear_ln": LINEAR_LN, "mlp": MLP_LN}

_dp = ctypes.POINTER(ctypes.c_double)
_lib_handle = None


def build(src: str = SRC, out: str = LIB, extra_flags=(), force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
           *extra_flags, "-o", out + ".tmp", src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def load(path: str | None = None):
    """Load (building first if needed) the oracle library; returns a ctypes handle."""
    global _lib_handle
    if path is None and _lib_handle is not None:
        return _lib_handle
    lib = ctypes.CDLL(path or build())
    lib.oracle_ttt_forward_f64.restype = ctypes.c_int
    lib.oracle_ttt_forward_f64.argtypes = [
        ctypes.c_int, _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp, ctypes.c_double, _dp, _dp,
        ctypes.c_int]
    lib.oracle_loss_grad_f64.restype = ctypes.c_double
    lib.oracle_loss_grad_f64.argtypes = [ctypes.c_int, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                         _dp, _dp, ctypes.c_double, _dp]
    lib.oracle_apply_f64.restype = ctypes.c_int
    lib.oracle_apply_f64.argtypes = [ctypes.c_int, _dp, _dp, ctypes.c_int, ctypes.c_int, _dp, _dp,
                                     ctypes.c_double, _dp]
    lib.oracle_default_threads.restype = ctypes.c_int
    lib.oracle_ttt_momentum_forward_f64.restype = ctypes.c_int
    lib.oracle_ttt_momentum_forward_f64.argtypes = [
        ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp, ctypes.c_double, _dp, _dp, _dp]
    if path is None:
        _lib_handle = lib
    return lib


def _f64(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


class Oracle:
    """Bound oracle library (the default build, or another build of the same source)."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    def default_threads(self) -> int:
        return int(self.lib.oracle_default_threads())

    def forward(self, kind, Q, K, V, eta, params, b, gamma=None, beta=None, eps=1e-6,
                hidden=0, nthreads=0):
        """Run the primal rule.  params: [H, P] flat per-head parameters.
        Returns (Z [B,H,T,d], W_out [B,H,P])."""
        Q, K, V, eta, params = map(_f64, (Q, K, V, eta, params))
        gamma, beta = _f64(gamma), _f64(beta)
        B, H, T, d = Q.shape
        P = params.shape[-1]
        Z = np.zeros((B, H, T, d))
        W_out = np.zeros((B, H, P))
        rc = self.lib.oracle_ttt_forward_f64(
            int(kind), _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(params), B, H, T, d,
            int(hidden), int(b), _ptr(gamma), _ptr(beta), float(eps), _ptr(Z), _ptr(W_out),
            int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle_ttt_forward_f64 failed with status {rc}")
        return Z, W_out

    def ttt_linear(self, Q, K, V, eta, W0, b, nthreads=0):
        """TTT-Linear, f(x) = x W.  W0 [H,d,d] -> (Z [B,H,T,d], W [B,H,d,d])."""
        W0 = _f64(W0)
        H, d, _ = W0.shape
        Z, W = self.forward(LINEAR, Q, K, V, eta, W0.reshape(H, d * d), b, nthreads=nthreads)
        return Z, W.reshape(W.shape[0], H, d, d)

    def ttt_linear_ln(self, Q, K, V, eta, W0, b, gamma, beta, eps=1e-6, nthreads=0):
        """TTT-Linear with LN + residual, f(x) = x + LN(x W)."""
        W0 = _f64(W0)
        H, d, _ = W0.shape
        Z, W = self.forward(LINEAR_LN, Q, K, V, eta, W0.reshape(H, d * d), b, gamma, beta, eps,
                            nthreads=nthreads)
        return Z, W.reshape(W.shape[0], H, d, d)

    def ttt_mlp(self, Q, K, V, eta, W1, W2, b, gamma, beta, eps=1e-6, nthreads=0):
        """TTT-MLP, f(x) = x + LN(GELU(x W1) W2).  W1 [H,d,h], W2 [H,h,d]."""
        W1, W2 = _f64(W1), _f64(W2)
        H, d, h = W1.shape
        params = np.concatenate([W1.reshape(H, d * h), W2.reshape(H, h * d)], axis=1)
        Z, W = self.forward(MLP_LN, Q, K, V, eta, params, b, gamma, beta, eps, hidden=h,
                            nthreads=nthreads)
        Bn = W.shape[0]
        return Z, W[:, :, : d * h].reshape(Bn, H, d, h), W[:, :, d * h:].reshape(Bn, H, h, d)

    def momentum_forward(self, kind, Q, K, V, eta, alpha, lam, params, b, gamma=None, beta=None,
                         eps=1e-6, hidden=0):
        """The momentum and decay variant (Titans-style): S_t = alpha_t S_{t-1} - eta_t grad,
        W_t = (1 - lambda_t) W_{t-1} + S_t, gradients at the mini-batch base.
        Returns (Z [B,H,T,d], W_out [B,H,P], S_out [B,H,P])."""
        Q, K, V, eta, alpha, lam, params = map(_f64, (Q, K, V, eta, alpha, lam, params))
        gamma, beta = _f64(gamma), _f64(beta)
        B, H, T, d = Q.shape
        P = params.shape[-1]
        Z = np.zeros((B, H, T, d))
        W_out = np.zeros((B, H, P))
        S_out = np.zeros((B, H, P))
        rc = self.lib.oracle_ttt_momentum_forward_f64(
            int(kind), _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(alpha), _ptr(lam), _ptr(params),
            B, H, T, d, int(hidden), int(b), _ptr(gamma), _ptr(beta), float(eps), _ptr(Z),
            _ptr(W_out), _ptr(S_out))
        if rc != 0:
            raise ValueError(f"oracle_ttt_momentum_forward_f64 failed with status {rc}")
        return Z, W_out, S_out

    def loss_grad(self, kind, params, k, v, gamma=None, beta=None, eps=1e-6, hidden=0):
        """Loss ||f(k; W) - v||^2 of one head and its gradient (flat, like params)."""
        params, k, v = _f64(params).ravel(), _f64(k), _f64(v)
        gamma, beta = _f64(gamma), _f64(beta)
        grad = np.zeros_like(params)
        loss = self.lib.oracle_loss_grad_f64(int(kind), _ptr(params), _ptr(k), _ptr(v), k.shape[0],
                                             int(hidden), _ptr(gamma), _ptr(beta), float(eps),
                                             _ptr(grad))
        return float(loss), grad

    def apply(self, kind, params, x, gamma=None, beta=None, eps=1e-6, hidden=0):
        """f(x; W) of one head for one row x[d]."""
        params, x = _f64(params).ravel(), _f64(x)
        gamma, beta = _f64(gamma), _f64(beta)
        out = np.zeros_like(x)
        rc = self.lib.oracle_apply_f64(int(kind), _ptr(params), _ptr(x), x.shape[0], int(hidden),
                                       _ptr(gamma), _ptr(beta), float(eps), _ptr(out))
        if rc != 0:
            raise ValueError(f"oracle_apply_f64 failed with status {rc}")
        return out


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def ttt_linear(*a, **k):
    return default().ttt_linear(*a, **k)


def ttt_linear_ln(*a, **k):
    return default().ttt_linear_ln(*a, **k)


def ttt_mlp(*a, **k):
    return default().ttt_mlp(*a, **k)
