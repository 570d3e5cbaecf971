"""GPU parity of the TTT-MLP backward pass (ttt_mlp_bwd) against the fp64 autograd
oracle, through the C ABI: every unit at reduced sizes for several mini-batch
sizes and both input dtypes, the checkpoints against the oracle's forward, the
absent final-state cotangent, T = 0, and sampled units of a launch with the full
workload's B8 H32 shape."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as OB
import test_sequence_modeling_b200 as ttt
from test_sequence_modeling_b200 import inputs as I
from gpu_helpers import rel_fro, to_device

pytestmark = pytest.mark.gpu

# fp32 arithmetic from exactly the oracle's inputs (bf16 inputs are upcast
# exactly): the forward's fp32 tolerance for b = 16, and 1e-4 for smaller
# mini-batches, where an fp32 evaluation of the same recursion in another
# operation order already lands 3-5e-5 from the oracle
# (test_backward_mlp_tolerance.py).
BWD_TOL = 1e-5
SMALL_B_TOL = 1e-4


def tol(b):
    return BWD_TOL if b >= 16 else SMALL_B_TOL


KEYS = ("dQ", "dK", "dV", "deta", "dW1", "dW2", "dgamma", "dbeta")
BASE = I.CONFIGS["mlp_B8H32T8192"]


def run_gpu(cfg, dev, dZ, dW1T, dW2T):
    out = ttt.ttt_mlp_bwd(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W1"], dev["W2"], dev["gamma"],
                          dev["beta"], dZ, cfg.b, cfg.ln_eps, dW1_T=dW1T, dW2_T=dW2T)
    torch.cuda.synchronize()
    assert ttt.last_device_status() == 0
    return out


def oracle_unit(cfg, bi, hi, dZ, dW1T, dW2T):
    u = I.unit_as_f64(cfg, bi, hi)
    sl = lambda a: None if a is None else a[bi:bi + 1, hi:hi + 1].astype(np.float64)
    return OB.ttt_mlp_backward(u["Q"], u["K"], u["V"], u["eta"], u["W1"], u["W2"], cfg.b, sl(dZ),
                               u["gamma"], u["beta"], cfg.ln_eps, sl(dW1T), sl(dW2T))


def compare(cfg, gpu, units, dZ, dW1T, dW2T):
    worst = {}
    host = {k: gpu[k].cpu().numpy() for k in KEYS}
    for bi, hi in units:
        ref = oracle_unit(cfg, bi, hi, dZ, dW1T, dW2T)
        for k in KEYS:
            g = host[k][bi, hi]
            assert np.all(np.isfinite(g)), (k, bi, hi)
            worst[k] = max(worst.get(k, 0.0), rel_fro(g, ref[k][0, 0]))
    return worst


def cuda(*xs):
    return [None if x is None else torch.from_numpy(x).cuda() for x in xs]


@pytest.mark.parametrize("b", [1, 4, 16])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mlp_backward_matches_oracle(dtype, b):
    cfg = BASE.replace(B=2, H=3, T=48, b=b, dtype=dtype)
    dev = to_device(cfg, I.make_inputs(cfg))
    dZ, dW1T, dW2T = I.mlp_cotangents(cfg)
    out = run_gpu(cfg, dev, *cuda(dZ, dW1T, dW2T))
    units = [(bi, hi) for bi in range(cfg.B) for hi in range(cfg.H)]
    worst = compare(cfg, out, units, dZ, dW1T, dW2T)
    print(f"b={b} {dtype}: {worst}")
    assert max(worst.values()) <= tol(b), worst
    # The checkpoints: the initial state first, the forward's state at the last base.
    ck1, ck2 = out["W1_ckpt"].cpu().numpy(), out["W2_ckpt"].cpu().numpy()
    N = cfg.T // b
    assert np.array_equal(ck1[:, :, 0], np.broadcast_to(dev["W1"].cpu().numpy(), ck1[:, :, 0].shape))
    assert np.array_equal(ck2[:, :, 0], np.broadcast_to(dev["W2"].cpu().numpy(), ck2[:, :, 0].shape))
    for bi, hi in units[:2]:
        u = I.unit_as_f64(cfg, bi, hi)
        Tn = (N - 1) * b
        sl = {k: u[k][:, :, :Tn] for k in ("Q", "K", "V")}
        _, W1, W2 = oracle.ttt_mlp(sl["Q"], sl["K"], sl["V"], u["eta"][:, :, :Tn], u["W1"], u["W2"], b,
                                   u["gamma"], u["beta"], cfg.ln_eps, nthreads=1)
        assert rel_fro(ck1[bi, hi, N - 1], W1[0, 0]) <= tol(b)
        assert rel_fro(ck2[bi, hi, N - 1], W2[0, 0]) <= tol(b)


def test_mlp_backward_without_final_state_cotangents():
    """dW1_T = dW2_T = None are zero cotangents: bit-identical to passing zeros."""
    cfg = BASE.replace(B=1, H=3, T=32, b=16)
    dev = to_device(cfg, I.make_inputs(cfg))
    dZ, _, _ = I.mlp_cotangents(cfg)
    dZd = cuda(dZ)[0]
    a = run_gpu(cfg, dev, dZd, None, None)
    z = run_gpu(cfg, dev, dZd, torch.zeros(1, 3, 64, 256, device="cuda"), torch.zeros(1, 3, 256, 64, device="cuda"))
    for k in a:
        assert torch.equal(a[k], z[k]), k
    worst = compare(cfg, a, [(0, h) for h in range(cfg.H)], dZ, None, None)
    assert max(worst.values()) <= BWD_TOL, worst


def test_mlp_backward_empty_sequence():
    """T = 0: the state cotangents pass through and the LN parameters get nothing."""
    cfg = BASE.replace(B=2, H=2, T=0)
    dev = to_device(cfg, I.make_inputs(cfg))
    dW1T, dW2T = torch.randn(2, 2, 64, 256, device="cuda"), torch.randn(2, 2, 256, 64, device="cuda")
    out = run_gpu(cfg, dev, torch.empty(2, 2, 0, 64, device="cuda"), dW1T, dW2T)
    assert torch.equal(out["dW1"], dW1T) and torch.equal(out["dW2"], dW2T)
    assert torch.all(out["dgamma"] == 0) and torch.all(out["dbeta"] == 0)


def test_mlp_backward_full_shape_sampled_units():
    """The full workload's B8 H32 shape (256 units, two waves) at T = 256, checked on
    its first and last units against the oracle, and everywhere finite."""
    cfg = BASE.replace(T=256)
    dev = to_device(cfg, I.make_inputs(cfg))
    dZ, dW1T, dW2T = I.mlp_cotangents(cfg)
    out = run_gpu(cfg, dev, *cuda(dZ, dW1T, dW2T))
    for k in KEYS:
        assert bool(torch.isfinite(out[k]).all()), k
    worst = compare(cfg, out, [(0, 0), (cfg.B - 1, cfg.H - 1)], dZ, dW1T, dW2T)
    assert max(worst.values()) <= BWD_TOL, worst
