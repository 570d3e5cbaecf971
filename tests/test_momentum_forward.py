"""GPU parity of the whole-sequence forward with the momentum and decay update
(ttt_linear_momentum_fwd / ttt_linear_ln_momentum_fwd) against the fp64
oracle's momentum variant, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import test_sequence_modeling_b200 as ttt
from test_sequence_modeling_b200 import inputs as I
from gpu_helpers import rel_fro, to_device

pytestmark = pytest.mark.gpu

# fp32 arithmetic from exactly the oracle's inputs, as for the decode step.
TOL = 1e-5
NAMES = ["linear_f32_B1H1T256", "linear_bf16_B16H12T2048", "linear_ln_B16H32T8192"]


def run_gpu(cfg, dev, alpha, lam):
    ln = cfg.variant == "linear_ln"
    kw = dict(gamma=dev["gamma"], beta=dev["beta"], eps=cfg.ln_eps) if ln else {}
    Z, W, S = ttt.ttt_linear_momentum_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], alpha, lam, dev["W0"],
                                          cfg.b, **kw)
    torch.cuda.synchronize()
    assert ttt.last_device_status() == 0
    return Z, W, S


@pytest.mark.parametrize("b", [1, 4, 16])
@pytest.mark.parametrize("name", NAMES)
def test_momentum_forward_matches_oracle(name, b):
    cfg = I.CONFIGS[name].replace(B=2, H=3, T=48, b=b)
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = I.momentum_rates(cfg)
    Z, W, S = (x.cpu().numpy() for x in run_gpu(cfg, dev, torch.from_numpy(alpha).cuda(),
                                                 torch.from_numpy(lam).cuda()))
    kind = oracle.LINEAR if cfg.variant == "linear" else oracle.LINEAR_LN
    worst = {"Z": 0.0, "W": 0.0, "S": 0.0}
    for bi in range(cfg.B):
        for hi in range(cfg.H):
            u = I.unit_as_f64(cfg, bi, hi)
            Zr, Wr, Sr = oracle.default().momentum_forward(
                kind, u["Q"], u["K"], u["V"], u["eta"], alpha[bi, hi][None, None].astype(np.float64),
                lam[bi, hi][None, None].astype(np.float64), u["W0"].reshape(1, -1), b, u["gamma"],
                u["beta"], cfg.ln_eps)
            for key, g, r in (("Z", Z[bi, hi], Zr[0, 0]), ("W", W[bi, hi].ravel(), Wr[0, 0]),
                              ("S", S[bi, hi].ravel(), Sr[0, 0])):
                assert np.all(np.isfinite(g))
                worst[key] = max(worst[key], rel_fro(g, r))
    assert max(worst.values()) <= TOL, worst


def test_momentum_forward_agrees_with_the_decode_steps():
    """The kernel and a sequence of momentum decode calls run the same per-element
    arithmetic (one mini-batch's gradients at its base, then the token updates)."""
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=2, H=2, T=64, b=16)
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = (torch.from_numpy(x).cuda() for x in I.momentum_rates(cfg))
    Z, W, S = run_gpu(cfg, dev, alpha, lam)
    Wd = dev["W0"].unsqueeze(0).expand(cfg.B, cfg.H, 64, 64).contiguous()
    Wb, Sd = Wd.clone(), torch.zeros_like(Wd)
    Zd = torch.empty_like(Z)
    for t in range(cfg.T):
        q, k, v = (dev[n][:, :, t].contiguous() for n in ("Q", "K", "V"))
        e, a, l_ = (x[:, :, t].contiguous() for x in (dev["eta"], alpha, lam))
        Zd[:, :, t] = ttt.ttt_linear_ln_momentum_decode(q, k, v, e, a, l_, Wd, Wb, Sd, dev["gamma"],
                                                        dev["beta"], cfg.b, t % cfg.b, cfg.ln_eps)
    torch.cuda.synchronize()
    torch.testing.assert_close(Z, Zd, rtol=1e-6, atol=1e-6)
    torch.testing.assert_close(W, Wd, rtol=1e-6, atol=1e-7)
    torch.testing.assert_close(S, Sd, rtol=1e-6, atol=1e-7)


def test_momentum_forward_empty_sequence():
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=2, H=2, T=0)
    dev = to_device(cfg, I.make_inputs(cfg))
    e = torch.empty(2, 2, 0, device="cuda")
    Z, W, S = run_gpu(cfg, dev, e, e)
    assert Z.numel() == 0
    assert torch.equal(W, dev["W0"].unsqueeze(0).expand(2, 2, 64, 64))
    assert torch.all(S == 0)


def test_momentum_forward_full_size_sampled_units():
    """The full linear + LN workload (B16 H32 T8192, b = 16), first and last units."""
    cfg = I.CONFIGS["linear_ln_B16H32T8192"]
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = I.momentum_rates(cfg)
    Z, W, S = run_gpu(cfg, dev, torch.from_numpy(alpha).cuda(), torch.from_numpy(lam).cuda())
    assert bool(torch.isfinite(Z).all()) and bool(torch.isfinite(W).all())
    worst = {}
    for bi, hi in ((0, 0), (cfg.B - 1, cfg.H - 1)):
        u = I.unit_as_f64(cfg, bi, hi)
        Zr, Wr, Sr = oracle.default().momentum_forward(
            oracle.LINEAR_LN, u["Q"], u["K"], u["V"], u["eta"], alpha[bi, hi][None, None].astype(np.float64),
            lam[bi, hi][None, None].astype(np.float64), u["W0"].reshape(1, -1), cfg.b, u["gamma"],
            u["beta"], cfg.ln_eps)
        for key, g, r in (("Z", Z[bi, hi].cpu().numpy(), Zr[0, 0]), ("W", W[bi, hi].cpu().numpy().ravel(), Wr[0, 0]),
                          ("S", S[bi, hi].cpu().numpy().ravel(), Sr[0, 0])):
            worst[key] = max(worst.get(key, 0.0), rel_fro(g, r))
    assert max(worst.values()) <= TOL, worst
