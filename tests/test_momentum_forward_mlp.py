"""GPU parity of the TTT-MLP forward with the momentum and decay update
(ttt_mlp_momentum_fwd) against the fp64 oracle's momentum variant, through the C
ABI: every unit at reduced sizes, alpha = lambda = 0 against the plain TTT-MLP
forward, and sampled units of a launch with the full workload's B8 H32 shape."""
import numpy as np
import pytest
import torch

import oracle
import test_sequence_modeling_b200 as ttt
from test_sequence_modeling_b200 import inputs as I
from gpu_helpers import rel_fro, to_device
from test_momentum_tolerance import MLP_MOMENTUM_TOL

pytestmark = pytest.mark.gpu

# fp32 arithmetic from exactly the oracle's inputs, at the momentum tolerance:
# an independent fp32 evaluation of this recursion already spreads above 1e-5
# from the oracle for b = 1, for fp32 inputs and for longer sequences
# (test_momentum_tolerance.py), and the kernel lands where it does.
BASE = I.CONFIGS["mlp_B8H32T8192"]


def tol(b):
    return MLP_MOMENTUM_TOL


def run_gpu(cfg, dev, alpha, lam):
    out = ttt.ttt_mlp_momentum_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], alpha, lam, dev["W1"], dev["W2"],
                                   dev["gamma"], dev["beta"], cfg.b, cfg.ln_eps)
    torch.cuda.synchronize()
    assert ttt.last_device_status() == 0
    return [x.cpu().numpy() for x in out]


def compare(cfg, got, units, alpha, lam):
    Z, W1, W2, S1, S2 = got
    n1 = cfg.d * cfg.hidden
    worst = {}
    for bi, hi in units:
        u = I.unit_as_f64(cfg, bi, hi)
        params = np.concatenate([u["W1"].reshape(1, -1), u["W2"].reshape(1, -1)], axis=1)
        Zr, Wr, Sr = oracle.default().momentum_forward(
            oracle.MLP_LN, u["Q"], u["K"], u["V"], u["eta"], alpha[bi, hi][None, None].astype(np.float64),
            lam[bi, hi][None, None].astype(np.float64), params, cfg.b, u["gamma"], u["beta"], cfg.ln_eps,
            hidden=cfg.hidden)
        for key, g, r in (("Z", Z[bi, hi], Zr[0, 0]), ("W1", W1[bi, hi].ravel(), Wr[0, 0, :n1]),
                          ("W2", W2[bi, hi].ravel(), Wr[0, 0, n1:]), ("S1", S1[bi, hi].ravel(), Sr[0, 0, :n1]),
                          ("S2", S2[bi, hi].ravel(), Sr[0, 0, n1:])):
            assert np.all(np.isfinite(g)), (key, bi, hi)
            worst[key] = max(worst.get(key, 0.0), rel_fro(g, r))
    return worst


@pytest.mark.parametrize("b", [1, 4, 16])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mlp_momentum_forward_matches_oracle(dtype, b):
    cfg = BASE.replace(B=2, H=3, T=48, b=b, dtype=dtype)
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = I.momentum_rates(cfg)
    got = run_gpu(cfg, dev, torch.from_numpy(alpha).cuda(), torch.from_numpy(lam).cuda())
    worst = compare(cfg, got, [(bi, hi) for bi in range(cfg.B) for hi in range(cfg.H)], alpha, lam)
    print(f"b={b} {dtype}: {worst}")
    assert max(worst.values()) <= tol(b), worst


def test_mlp_momentum_forward_without_momentum_or_decay_is_ttt():
    """alpha = lambda = 0: the exact-fp32 TTT-MLP forward's outputs, and zero momenta."""
    cfg = BASE.replace(B=2, H=3, T=64, b=16)
    dev = to_device(cfg, I.make_inputs(cfg))
    zeros = torch.zeros(cfg.B, cfg.H, cfg.T, device="cuda")
    Z, W1, W2, S1, S2 = run_gpu(cfg, dev, zeros, zeros)
    prev = ttt.set_path(ttt.TTT_PATH_SIMT)
    try:
        Zr, W1r, W2r = ttt.ttt_mlp_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W1"], dev["W2"],
                                       dev["gamma"], dev["beta"], cfg.b, cfg.ln_eps)
    finally:
        ttt.set_path(prev)
    for g, r in ((Z, Zr), (W1, W1r), (W2, W2r)):  # two fp32 evaluations of one quantity
        assert rel_fro(g, r.cpu().numpy()) <= 1e-5
    # S_T = -eta_T grad at the last token (alpha = 0): nonzero, and W_T - W_{T-1} = S_T.
    assert np.abs(S1).max() > 0 and np.abs(S2).max() > 0


def test_mlp_momentum_forward_full_shape_sampled_units():
    """The full workload's B8 H32 shape (256 units) at T = 256, checked on its first
    and last units against the oracle, and everywhere finite."""
    cfg = BASE.replace(T=256)
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = I.momentum_rates(cfg)
    got = run_gpu(cfg, dev, torch.from_numpy(alpha).cuda(), torch.from_numpy(lam).cuda())
    for x in got:
        assert np.all(np.isfinite(x))
    worst = compare(cfg, got, [(0, 0), (cfg.B - 1, cfg.H - 1)], alpha, lam)
    print(f"full shape T=256: {worst}")
    assert max(worst.values()) <= MLP_MOMENTUM_TOL, worst
