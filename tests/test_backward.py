"""GPU parity of the backward pass (ttt_linear_bwd / ttt_linear_ln_bwd) against the
fp64 autograd oracle, through the C ABI, on every unit at reduced sizes and on
sampled units of the full-size linear + LN workload."""
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
# exactly): the forward's fp32 tolerance.
BWD_TOL = 1e-5


def run_gpu(cfg, dev, dZ, dWT):
    ln = cfg.variant == "linear_ln"
    kw = dict(gamma=dev["gamma"], beta=dev["beta"], eps=cfg.ln_eps) if ln else {}
    out = ttt.ttt_linear_bwd(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], dZ, cfg.b, dW_T=dWT, **kw)
    torch.cuda.synchronize()
    assert ttt.last_device_status() == 0
    return out


def oracle_unit(cfg, bi, hi, dZ, dWT):
    u = I.unit_as_f64(cfg, bi, hi)
    ln = cfg.variant == "linear_ln"
    dwt = None if dWT is None else dWT[bi:bi + 1, hi:hi + 1].astype(np.float64)
    return OB.ttt_linear_backward(u["Q"], u["K"], u["V"], u["eta"], u["W0"], cfg.b,
                                  dZ[bi:bi + 1, hi:hi + 1].astype(np.float64), dwt, ln, u["gamma"],
                                  u["beta"], cfg.ln_eps)


def compare(cfg, gpu, units, dZ, dWT):
    worst = {}
    keys = ["dQ", "dK", "dV", "deta", "dW0"] + (["dgamma", "dbeta"] if cfg.variant == "linear_ln" else [])
    host = {k: gpu[k].cpu().numpy() for k in keys}
    for bi, hi in units:
        ref = oracle_unit(cfg, bi, hi, dZ, dWT)
        for k in keys:
            g = host[k][bi, hi]
            assert np.all(np.isfinite(g)), (k, bi, hi)
            worst[k] = max(worst.get(k, 0.0), rel_fro(g, ref[k][0, 0]))
    return worst


NAMES = ["linear_f32_B1H1T256", "linear_bf16_B16H12T2048", "linear_ln_B16H32T8192"]


@pytest.mark.parametrize("b", [1, 4, 16])
@pytest.mark.parametrize("name", NAMES)
def test_backward_matches_oracle(name, b):
    cfg = I.CONFIGS[name].replace(B=2, H=3, T=48, b=b)
    dev = to_device(cfg, I.make_inputs(cfg))
    dZ, dWT = I.cotangents(cfg)
    out = run_gpu(cfg, dev, torch.from_numpy(dZ).cuda(), torch.from_numpy(dWT).cuda())
    units = [(bi, hi) for bi in range(cfg.B) for hi in range(cfg.H)]
    worst = compare(cfg, out, units, dZ, dWT)
    assert max(worst.values()) <= BWD_TOL, worst
    # The checkpoints: W0 at the first base, the forward's state at the last one.
    ck = out["W_ckpt"].cpu().numpy()
    N = cfg.T // b
    assert np.array_equal(ck[:, :, 0], np.broadcast_to(dev["W0"].cpu().numpy(), ck[:, :, 0].shape))
    for bi, hi in units[:2]:
        u = I.unit_as_f64(cfg, bi, hi)
        Tn = (N - 1) * b
        sl = {k: u[k][:, :, :Tn] for k in ("Q", "K", "V")}
        if cfg.variant == "linear_ln":
            _, W = oracle.ttt_linear_ln(sl["Q"], sl["K"], sl["V"], u["eta"][:, :, :Tn], u["W0"], b,
                                        u["gamma"], u["beta"], cfg.ln_eps, nthreads=1)
        else:
            _, W = oracle.ttt_linear(sl["Q"], sl["K"], sl["V"], u["eta"][:, :, :Tn], u["W0"], b, nthreads=1)
        assert rel_fro(ck[bi, hi, N - 1], W[0, 0]) <= BWD_TOL


@pytest.mark.parametrize("name", ["linear_bf16_B16H12T2048", "linear_ln_B16H32T8192"])
def test_backward_without_final_state_cotangent(name):
    """dW_T = None is a zero cotangent: bit-identical to passing zeros, and parity."""
    cfg = I.CONFIGS[name].replace(B=1, H=3, T=32, b=16)
    dev = to_device(cfg, I.make_inputs(cfg))
    dZ, _ = I.cotangents(cfg)
    dZd = torch.from_numpy(dZ).cuda()
    a = run_gpu(cfg, dev, dZd, None)
    z = run_gpu(cfg, dev, dZd, torch.zeros(cfg.B, cfg.H, 64, 64, device="cuda"))
    for k in a:
        assert torch.equal(a[k], z[k]), k
    worst = compare(cfg, a, [(0, h) for h in range(cfg.H)], dZ, None)
    assert max(worst.values()) <= BWD_TOL, worst


def test_backward_empty_sequence():
    """T = 0: dW0 is dW_T itself and the LN parameters get no gradient."""
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=2, H=2, T=0)
    dev = to_device(cfg, I.make_inputs(cfg))
    dWT = torch.randn(2, 2, 64, 64, device="cuda")
    dZ = torch.empty(2, 2, 0, 64, device="cuda")
    out = run_gpu(cfg, dev, dZ, dWT)
    assert torch.equal(out["dW0"], dWT)
    assert torch.all(out["dgamma"] == 0) and torch.all(out["dbeta"] == 0)


def test_backward_full_size_sampled_units():
    """The full linear + LN workload (B16 H32 T8192, b = 16) in one launch, checked
    on its first and last units against the oracle, and everywhere finite."""
    cfg = I.CONFIGS["linear_ln_B16H32T8192"]
    dev = to_device(cfg, I.make_inputs(cfg))
    dZ, dWT = I.cotangents(cfg)
    out = run_gpu(cfg, dev, torch.from_numpy(dZ).cuda(), torch.from_numpy(dWT).cuda())
    for k in ("dQ", "dK", "dV", "deta", "dW0", "dgamma", "dbeta"):
        assert bool(torch.isfinite(out[k]).all()), k
    worst = compare(cfg, out, [(0, 0), (cfg.B - 1, cfg.H - 1)], dZ, dWT)
    assert max(worst.values()) <= BWD_TOL, worst
