"""GPU parity of the momentum and decay decode step (the Titans-style memory
update): run token by token over a sequence, the calls must reproduce the fp64
oracle's outputs, final state and final momentum, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import test_sequence_modeling_b200 as ttt
from test_sequence_modeling_b200 import inputs as I
from gpu_helpers import rel_fro, to_device
from test_momentum_tolerance import MLP_MOMENTUM_TOL

pytestmark = pytest.mark.gpu

# fp32 arithmetic from exactly the oracle's inputs, as for the plain decode step.
DECODE_TOL = 1e-5


def run_sequence(cfg, dev, alpha, lam):
    B, H, T, d = cfg.B, cfg.H, cfg.T, cfg.d
    W = dev["W0"].unsqueeze(0).expand(B, H, d, d).contiguous()
    W_base = W.clone()
    S = torch.zeros_like(W)
    Z = torch.empty(B, H, T, d, dtype=torch.float32, device="cuda")
    for t in range(T):
        q, k, v = (dev[n][:, :, t].contiguous() for n in ("Q", "K", "V"))
        eta, al, lm = (x[:, :, t].contiguous() for x in (dev["eta"], alpha, lam))
        if cfg.variant == "linear":
            Z[:, :, t] = ttt.ttt_linear_momentum_decode(q, k, v, eta, al, lm, W, W_base, S, cfg.b,
                                                        t % cfg.b)
        else:
            Z[:, :, t] = ttt.ttt_linear_ln_momentum_decode(q, k, v, eta, al, lm, W, W_base, S,
                                                           dev["gamma"], dev["beta"], cfg.b,
                                                           t % cfg.b, cfg.ln_eps)
    torch.cuda.synchronize()
    assert ttt.last_device_status() == 0
    return Z.cpu().numpy(), W.cpu().numpy(), S.cpu().numpy(), W_base


@pytest.mark.parametrize("b", [1, 16])
@pytest.mark.parametrize("name", ["linear_f32_B1H1T256", "linear_bf16_B16H12T2048",
                                  "linear_ln_B16H32T8192"])
def test_momentum_decode_matches_oracle(name, b):
    cfg = I.CONFIGS[name].replace(B=2, H=3, T=48, b=b)
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = I.momentum_rates(cfg)
    Z, W, S, W_base = run_sequence(cfg, dev, torch.from_numpy(alpha).cuda(),
                                   torch.from_numpy(lam).cuda())
    kind = oracle.LINEAR if cfg.variant == "linear" else oracle.LINEAR_LN
    worst = {"Z": 0.0, "W": 0.0, "S": 0.0}
    for bi in range(cfg.B):
        for hi in range(cfg.H):
            u = I.unit_as_f64(cfg, bi, hi)
            Zr, Wr, Sr = oracle.default().momentum_forward(
                kind, u["Q"], u["K"], u["V"], u["eta"], alpha[bi, hi][None, None].astype(np.float64),
                lam[bi, hi][None, None].astype(np.float64), u["W0"].reshape(1, -1), cfg.b,
                u["gamma"], u["beta"], cfg.ln_eps)
            for key, g, r in (("Z", Z[bi, hi], Zr[0, 0]), ("W", W[bi, hi].ravel(), Wr[0, 0]),
                              ("S", S[bi, hi].ravel(), Sr[0, 0])):
                assert np.all(np.isfinite(g))
                worst[key] = max(worst[key], rel_fro(g, r))
    assert max(worst.values()) <= DECODE_TOL, worst
    # T is a whole number of mini-batches: the base state is the final state.
    assert torch.equal(W_base.cpu(), torch.from_numpy(W))


def test_zero_momentum_and_decay_is_the_plain_step():
    """alpha = lambda = 0 gives the plain decode step up to rounding (the plain step
    fuses the multiply and add of W - k^T (eta G), the momentum step rounds S first)."""
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=2, H=2, T=32)
    dev = to_device(cfg, I.make_inputs(cfg))
    zero = torch.zeros(cfg.B, cfg.H, cfg.T, device="cuda")
    Zm, Wm, _, _ = run_sequence(cfg, dev, zero, zero)
    W = dev["W0"].unsqueeze(0).expand(cfg.B, cfg.H, 64, 64).contiguous()
    Wb = W.clone()
    Z = torch.empty(cfg.B, cfg.H, cfg.T, 64, device="cuda")
    for t in range(cfg.T):
        q, k, v = (dev[n][:, :, t].contiguous() for n in ("Q", "K", "V"))
        Z[:, :, t] = ttt.ttt_linear_ln_decode(q, k, v, dev["eta"][:, :, t].contiguous(), W, Wb,
                                              dev["gamma"], dev["beta"], cfg.b, t % cfg.b, cfg.ln_eps)
    torch.cuda.synchronize()
    np.testing.assert_allclose(Zm, Z.cpu().numpy(), rtol=0, atol=1e-6)
    np.testing.assert_allclose(Wm, W.cpu().numpy(), rtol=0, atol=1e-7)


@pytest.mark.parametrize("b", [1, 16])
def test_mlp_momentum_decode_matches_oracle(b):
    cfg = I.CONFIGS["mlp_B8H32T8192"].replace(B=2, H=3, T=32, b=b)
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = I.momentum_rates(cfg)
    al_d, lm_d = torch.from_numpy(alpha).cuda(), torch.from_numpy(lam).cuda()
    B, H, T, d, h = cfg.B, cfg.H, cfg.T, cfg.d, cfg.hidden
    W1 = dev["W1"].unsqueeze(0).expand(B, H, d, h).contiguous()
    W2 = dev["W2"].unsqueeze(0).expand(B, H, h, d).contiguous()
    W1b, W2b = W1.clone(), W2.clone()
    S1, S2 = torch.zeros_like(W1), torch.zeros_like(W2)
    Z = torch.empty(B, H, T, d, dtype=torch.float32, device="cuda")
    for t in range(T):
        q, k, v = (dev[n][:, :, t].contiguous() for n in ("Q", "K", "V"))
        eta, al, lm = (x[:, :, t].contiguous() for x in (dev["eta"], al_d, lm_d))
        Z[:, :, t] = ttt.ttt_mlp_momentum_decode(q, k, v, eta, al, lm, W1, W2, W1b, W2b, S1, S2,
                                                 dev["gamma"], dev["beta"], cfg.b, t % cfg.b, cfg.ln_eps)
    torch.cuda.synchronize()
    assert ttt.last_device_status() == 0
    Z, W1, W2, S1, S2 = (x.cpu().numpy() for x in (Z, W1, W2, S1, S2))
    worst = {}
    for bi in range(B):
        for hi in range(H):
            u = I.unit_as_f64(cfg, bi, hi)
            params = np.concatenate([u["W1"].reshape(1, -1), u["W2"].reshape(1, -1)], axis=1)
            Zr, Wr, Sr = oracle.default().momentum_forward(
                oracle.MLP_LN, u["Q"], u["K"], u["V"], u["eta"],
                alpha[bi, hi][None, None].astype(np.float64), lam[bi, hi][None, None].astype(np.float64),
                params, cfg.b, u["gamma"], u["beta"], cfg.ln_eps, hidden=h)
            n1 = d * h
            for key, g, r in (("Z", Z[bi, hi], Zr[0, 0]), ("W1", W1[bi, hi].ravel(), Wr[0, 0, :n1]),
                              ("W2", W2[bi, hi].ravel(), Wr[0, 0, n1:]),
                              ("S1", S1[bi, hi].ravel(), Sr[0, 0, :n1]),
                              ("S2", S2[bi, hi].ravel(), Sr[0, 0, n1:])):
                assert np.all(np.isfinite(g))
                worst[key] = max(worst.get(key, 0.0), rel_fro(g, r))
    # fp32 rounding grows along the sequence under momentum with b = 1: the tolerance
    # is derived from an independent fp32 evaluation in test_momentum_tolerance.py.
    assert max(worst.values()) <= MLP_MOMENTUM_TOL, worst
    assert torch.equal(W1b.cpu(), torch.from_numpy(W1))
    assert torch.equal(W2b.cpu(), torch.from_numpy(W2))
