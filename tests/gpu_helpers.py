"""Shared helpers of the GPU parity tests: seeded inputs to device tensors, one call
of the CUDA path through the binding, and per-unit comparison with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import test_sequence_modeling_b200 as ttt
from test_sequence_modeling_b200 import inputs as I

# Max relative Frobenius error per (batch, head) unit and output: 1e-5 for fp32
# inputs, 2e-3 for bf16 inputs with fp32 state and accumulation.
TOL = {"f32": 1e-5, "bf16": 2e-3}


def to_device(cfg, data, device="cuda"):
    if data["qkv_bits"]:
        qkv = [torch.from_numpy(data[k].view(np.int16)).to(device).view(torch.bfloat16)
               for k in ("Q", "K", "V")]
    else:
        qkv = [torch.from_numpy(np.ascontiguousarray(data[k])).to(device) for k in ("Q", "K", "V")]
    dev = {"Q": qkv[0], "K": qkv[1], "V": qkv[2]}
    for k in ("eta", "W0", "W1", "W2", "gamma", "beta"):
        if k in data:
            dev[k] = torch.from_numpy(np.ascontiguousarray(data[k])).to(device)
    return dev


def run_gpu(cfg, dev, **kw):
    """One forward through the binding; returns a dict of host numpy outputs."""
    if cfg.variant == "linear":
        Z, W = ttt.ttt_linear_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], cfg.b, **kw)
        out = {"Z": Z, "W": W}
    elif cfg.variant == "linear_ln":
        Z, W = ttt.ttt_linear_ln_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"],
                                     dev["gamma"], dev["beta"], cfg.b, cfg.ln_eps, **kw)
        out = {"Z": Z, "W": W}
    else:
        Z, W1, W2 = ttt.ttt_mlp_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W1"], dev["W2"],
                                    dev["gamma"], dev["beta"], cfg.b, cfg.ln_eps, **kw)
        out = {"Z": Z, "W1": W1, "W2": W2}
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


def oracle_unit(cfg, bi, hi):
    """The oracle's outputs for one unit, in float64: {"Z": [T,d], "W"/"W1"/"W2": ...}."""
    u = I.unit_as_f64(cfg, bi, hi)
    if cfg.variant == "linear":
        Z, W = oracle.ttt_linear(u["Q"], u["K"], u["V"], u["eta"], u["W0"], cfg.b, nthreads=1)
        return {"Z": Z[0, 0], "W": W[0, 0]}
    if cfg.variant == "linear_ln":
        Z, W = oracle.ttt_linear_ln(u["Q"], u["K"], u["V"], u["eta"], u["W0"], cfg.b, u["gamma"],
                                    u["beta"], cfg.ln_eps, nthreads=1)
        return {"Z": Z[0, 0], "W": W[0, 0]}
    Z, W1, W2 = oracle.ttt_mlp(u["Q"], u["K"], u["V"], u["eta"], u["W1"], u["W2"], cfg.b,
                               u["gamma"], u["beta"], cfg.ln_eps, nthreads=1)
    return {"Z": Z[0, 0], "W1": W1[0, 0], "W2": W2[0, 0]}


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def compare(cfg, gpu, units):
    """Max relative Frobenius error over the given units and every output."""
    worst = {}
    for bi, hi in units:
        ref = oracle_unit(cfg, bi, hi)
        for k, r in ref.items():
            e = rel_fro(gpu[k][bi, hi], r)
            assert np.all(np.isfinite(gpu[k][bi, hi])), (k, bi, hi)
            worst[k] = max(worst.get(k, 0.0), e)
    return worst


def all_units(cfg):
    return [(bi, hi) for bi in range(cfg.B) for hi in range(cfg.H)]


def sample_units(cfg, n, seed=0):
    """First, last and n-2 random units."""
    rng = np.random.default_rng(seed)
    idx = {0, cfg.units - 1} | set(rng.choice(cfg.units, size=min(n, cfg.units), replace=False).tolist())
    return [divmod(int(u), cfg.H) for u in sorted(idx)][: max(n, 2)]
