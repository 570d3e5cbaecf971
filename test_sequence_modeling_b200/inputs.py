"""Seeded synthetic inputs for the TTT layer forward.

This module holds none of the method's arithmetic: only random draws, their
scaling to the stated distributions, and the rounding of Q, K, V to the input
dtype.  Both the CUDA path and the fp64 oracle are fed from it.

Every (batch, head) unit draws from its own counter-seeded stream
``default_rng([seed, 1, batch, head])`` and every head's parameters from
``default_rng([seed, 2, head])``, so any unit of a full-size workload can be
regenerated alone (this is how full-size runs are sampled for parity).

Distributions (the five workloads of the TTT layer forward):
  Q, K, V  ~ N(0, 1/d), drawn in float32, then rounded to bf16 (round to nearest
             even) for the bf16 workloads;
  eta_t    = constant, or scale * sigmoid(N(0, 1)) per (batch, head, token);
  W0 (W1, W2) ~ N(0, 0.02^2) in float32, one per head, shared by the batch;
  gamma    ~ 1 + N(0, 0.01^2), beta ~ N(0, 0.01^2), one per head.
Draw order within a unit stream: Q, K, V, eta noise.  Within a head stream:
W0 (or W1 then W2), gamma, beta.

Two more streams serve the widened paths: ``default_rng([seed, 3, s])`` draws the
momentum factors alpha ~ U[0, 0.9) and weight decays lambda ~ U[0, 0.05) of the
momentum and decay update, ``default_rng([seed, 4, s])`` the incoming gradients
dZ ~ N(0, 1/d), dW_T ~ N(0, 1/d^2) of the TTT-Linear backward pass, and
``default_rng([seed, 5, s])`` those of the TTT-MLP backward (dZ ~ N(0, 1/d),
dW1_T, dW2_T ~ N(0, 1/(d h))).
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np

VARIANTS = ("linear", "linear_ln", "mlp")


@dataclass(frozen=True)
class TTTConfig:
    name: str
    variant: str  # "linear" | "linear_ln" | "mlp"
    dtype: str  # dtype of Q, K, V: "f32" | "bf16"
    B: int
    H: int
    T: int
    d: int = 64
    b: int = 16
    hidden: int = 256  # MLP hidden width (4 d)
    eta: str = "sigmoid"  # "const" | "sigmoid"
    eta_scale: float = 0.1
    seed: int = 0
    ln_eps: float = 1e-6

    def replace(self, **kw) -> "TTTConfig":
        return replace(self, **kw)

    @property
    def units(self) -> int:
        return self.B * self.H

    @property
    def head_tokens(self) -> int:
        return self.B * self.H * self.T


CONFIGS = {
    # TTT-Linear, fp32 throughout, constant eta = 0.1, seed 0.
    "linear_f32_B1H1T256": TTTConfig("linear_f32_B1H1T256", "linear", "f32", 1, 1, 256,
                                     eta="const", eta_scale=0.1, seed=0),
    # TTT-Linear, bf16 Q/K/V, eta = 0.1 sigmoid(N(0,1)).
    "linear_bf16_B16H12T2048": TTTConfig("linear_bf16_B16H12T2048", "linear", "bf16", 16, 12,
                                         2048, eta_scale=0.1, seed=1),
    # TTT-Linear with LN + residual, 1.3B-layer shape (32 heads x 64), 8k context.
    "linear_ln_B16H32T8192": TTTConfig("linear_ln_B16H32T8192", "linear_ln", "bf16", 16, 32, 8192,
                                       eta_scale=1.0 / 64, seed=2),
    # Long-context TTT-Linear with LN + residual.
    "linear_ln_B1H32T32768": TTTConfig("linear_ln_B1H32T32768", "linear_ln", "bf16", 1, 32, 32768,
                                       eta_scale=1.0 / 64, seed=3),
    # TTT-MLP (hidden 4d, GELU) with LN + residual.
    "mlp_B8H32T8192": TTTConfig("mlp_B8H32T8192", "mlp", "bf16", 8, 32, 8192,
                                eta_scale=1.0 / 64, seed=4),
}
CONFIG_ORDER = list(CONFIGS)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of bf16-exact float32 values (the bf16 encoding)."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> np.uint32(16)).astype(
        np.uint16)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 encodings to float32 (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def unit_inputs(cfg: TTTConfig, bi: int, hi: int, T: int | None = None):
    """Q, K, V [T, d] and eta [T] of unit (bi, hi), as float32 (bf16-exact for bf16)."""
    T = cfg.T if T is None else T
    rng = np.random.default_rng([cfg.seed, 1, bi, hi])
    scale = np.float32(1.0 / math.sqrt(cfg.d))
    out = []
    for _ in range(3):
        x = rng.standard_normal((T, cfg.d), dtype=np.float32) * scale
        out.append(round_to_bf16(x) if cfg.dtype == "bf16" else x)
    if cfg.eta == "const":
        eta = np.full(T, cfg.eta_scale, dtype=np.float32)
    else:
        eta = (cfg.eta_scale * _sigmoid(rng.standard_normal(T))).astype(np.float32)
    return out[0], out[1], out[2], eta


def head_params(cfg: TTTConfig, hi: int) -> dict:
    """Per-head parameters: W0 [d,d] (or W1 [d,h], W2 [h,d]), gamma [d], beta [d]."""
    rng = np.random.default_rng([cfg.seed, 2, hi])
    d, h = cfg.d, cfg.hidden
    p = {}
    if cfg.variant == "mlp":
        p["W1"] = (0.02 * rng.standard_normal((d, h))).astype(np.float32)
        p["W2"] = (0.02 * rng.standard_normal((h, d))).astype(np.float32)
    else:
        p["W0"] = (0.02 * rng.standard_normal((d, d))).astype(np.float32)
    p["gamma"] = (1.0 + 0.01 * rng.standard_normal(d)).astype(np.float32)
    p["beta"] = (0.01 * rng.standard_normal(d)).astype(np.float32)
    return p


def params(cfg: TTTConfig) -> dict:
    """All heads' parameters stacked on a leading H axis."""
    per = [head_params(cfg, hi) for hi in range(cfg.H)]
    return {k: np.stack([p[k] for p in per]) for k in per[0]}


def make_inputs(cfg: TTTConfig, threads: int = 8, bf16_as_bits: bool = True,
                batch_offset: int = 0) -> dict:
    """Full workload.  Q, K, V [B,H,T,d]: float32, or (bf16 with bf16_as_bits) uint16
    bf16 encodings; eta [B,H,T] float32; plus the per-head parameters.  Batch row i
    holds the units of global batch index batch_offset + i (how a data-parallel
    rank draws its own shard)."""
    B, H, T, d = cfg.B, cfg.H, cfg.T, cfg.d
    as_bits = cfg.dtype == "bf16" and bf16_as_bits
    qkv_dt = np.uint16 if as_bits else np.float32
    Q = np.empty((B, H, T, d), qkv_dt)
    K = np.empty((B, H, T, d), qkv_dt)
    V = np.empty((B, H, T, d), qkv_dt)
    eta = np.empty((B, H, T), np.float32)

    def fill(u):
        bi, hi = divmod(u, H)
        q, k, v, e = unit_inputs(cfg, batch_offset + bi, hi)
        if as_bits:
            q, k, v = bf16_bits(q), bf16_bits(k), bf16_bits(v)
        Q[bi, hi], K[bi, hi], V[bi, hi], eta[bi, hi] = q, k, v, e

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(fill, range(B * H)))
    out = {"Q": Q, "K": K, "V": V, "eta": eta, "qkv_bits": as_bits}
    out.update(params(cfg))
    return out


def momentum_rates(cfg: TTTConfig, seed: int = 0):
    """Per-token momentum factors alpha in [0, 0.9) and weight decays lambda in
    [0, 0.05), [B, H, T] float32 each, for the momentum and decay update."""
    rng = np.random.default_rng([cfg.seed, 3, seed])
    alpha = (0.9 * rng.random((cfg.B, cfg.H, cfg.T))).astype(np.float32)
    lam = (0.05 * rng.random((cfg.B, cfg.H, cfg.T))).astype(np.float32)
    return alpha, lam


def cotangents(cfg: TTTConfig, seed: int = 0):
    """Incoming gradients for the backward pass: dZ [B, H, T, d] ~ N(0, 1/d) and
    dW_T [B, H, d, d] ~ N(0, 1/d^2), float32."""
    rng = np.random.default_rng([cfg.seed, 4, seed])
    dZ = (rng.standard_normal((cfg.B, cfg.H, cfg.T, cfg.d), dtype=np.float32) / np.float32(math.sqrt(cfg.d)))
    dWT = (rng.standard_normal((cfg.B, cfg.H, cfg.d, cfg.d), dtype=np.float32) / np.float32(cfg.d))
    return dZ, dWT


def mlp_cotangents(cfg: TTTConfig, seed: int = 0):
    """Incoming gradients for the TTT-MLP backward: dZ [B, H, T, d] ~ N(0, 1/d) and
    dW1_T [B, H, d, h], dW2_T [B, H, h, d] ~ N(0, 1/(d h)), float32, from the stream
    default_rng([seed, 5, s])."""
    rng = np.random.default_rng([cfg.seed, 5, seed])
    dZ = (rng.standard_normal((cfg.B, cfg.H, cfg.T, cfg.d), dtype=np.float32) / np.float32(math.sqrt(cfg.d)))
    sc = np.float32(1.0 / math.sqrt(cfg.d * cfg.hidden))
    dW1 = rng.standard_normal((cfg.B, cfg.H, cfg.d, cfg.hidden), dtype=np.float32) * sc
    dW2 = rng.standard_normal((cfg.B, cfg.H, cfg.hidden, cfg.d), dtype=np.float32) * sc
    return dZ, dW1, dW2


def unit_as_f64(cfg: TTTConfig, bi: int, hi: int, T: int | None = None) -> dict:
    """One unit's inputs and its head's parameters in float64, shaped [1,1,T,d] and
    [1,...] for feeding a per-unit reference computation."""
    q, k, v, e = unit_inputs(cfg, bi, hi, T)
    p = head_params(cfg, hi)
    out = {"Q": q[None, None].astype(np.float64), "K": k[None, None].astype(np.float64),
           "V": v[None, None].astype(np.float64), "eta": e[None, None].astype(np.float64)}
    out.update({kk: vv[None].astype(np.float64) for kk, vv in p.items()})
    return out
