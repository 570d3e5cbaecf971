"""GPU parity of the primal-form decode step: run token by token over a sequence,
the calls must reproduce the fp64 oracle's outputs and final state (the oracle
is the primal mini-batch rule, token by token), through the C ABI."""
import numpy as np
import pytest
import torch

import test_sequence_modeling_b200 as ttt
from test_sequence_modeling_b200 import inputs as I
from gpu_helpers import all_units, compare, to_device

pytestmark = pytest.mark.gpu

# The decode step computes in fp32 from exactly the oracle's inputs.
DECODE_TOL = 1e-5


def decode_sequence(cfg, dev):
    B, H, T, d = cfg.B, cfg.H, cfg.T, cfg.d
    W = dev["W0"].unsqueeze(0).expand(B, H, d, d).contiguous()
    W_base = W.clone()
    Z = torch.empty(B, H, T, d, dtype=torch.float32, device="cuda")
    for t in range(T):
        q, k, v = (dev[n][:, :, t].contiguous() for n in ("Q", "K", "V"))
        eta = dev["eta"][:, :, t].contiguous()
        if cfg.variant == "linear":
            Z[:, :, t] = ttt.ttt_linear_decode(q, k, v, eta, W, W_base, cfg.b, t % cfg.b)
        else:
            Z[:, :, t] = ttt.ttt_linear_ln_decode(q, k, v, eta, W, W_base, dev["gamma"], dev["beta"],
                                                  cfg.b, t % cfg.b, cfg.ln_eps)
    torch.cuda.synchronize()
    return {"Z": Z.cpu().numpy(), "W": W.cpu().numpy()}, W_base


@pytest.mark.parametrize("b", [1, 4, 16])
@pytest.mark.parametrize("name", ["linear_f32_B1H1T256", "linear_bf16_B16H12T2048",
                                  "linear_ln_B16H32T8192"])
def test_decode_matches_oracle(name, b):
    cfg = I.CONFIGS[name].replace(B=2, H=3, T=48, b=b)
    dev = to_device(cfg, I.make_inputs(cfg))
    out, W_base = decode_sequence(cfg, dev)
    worst = compare(cfg, out, all_units(cfg))
    assert max(worst.values()) <= DECODE_TOL, worst
    # T is a whole number of mini-batches: the base state is the final state.
    assert torch.equal(W_base.cpu(), torch.from_numpy(out["W"]))


def test_decode_mid_mini_batch_keeps_base():
    """Within a mini-batch the base state stays put; only the last position moves it."""
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=1, H=2, T=16)
    dev = to_device(cfg, I.make_inputs(cfg))
    W = dev["W0"].unsqueeze(0).expand(1, 2, 64, 64).contiguous()
    W_base = W.clone()
    W0 = W.clone()
    for t in range(3):
        q, k, v = (dev[n][:, :, t].contiguous() for n in ("Q", "K", "V"))
        ttt.ttt_linear_ln_decode(q, k, v, dev["eta"][:, :, t].contiguous(), W, W_base, dev["gamma"],
                                 dev["beta"], 16, t)
    torch.cuda.synchronize()
    assert torch.equal(W_base, W0)
    assert not torch.equal(W, W0)
    assert ttt.last_device_status() == 0


def decode_sequence_mlp(cfg, dev):
    B, H, T, d, h = cfg.B, cfg.H, cfg.T, cfg.d, cfg.hidden
    W1 = dev["W1"].unsqueeze(0).expand(B, H, d, h).contiguous()
    W2 = dev["W2"].unsqueeze(0).expand(B, H, h, d).contiguous()
    W1b, W2b = W1.clone(), W2.clone()
    Z = torch.empty(B, H, T, d, dtype=torch.float32, device="cuda")
    for t in range(T):
        q, k, v = (dev[n][:, :, t].contiguous() for n in ("Q", "K", "V"))
        Z[:, :, t] = ttt.ttt_mlp_decode(q, k, v, dev["eta"][:, :, t].contiguous(), W1, W2, W1b, W2b,
                                        dev["gamma"], dev["beta"], cfg.b, t % cfg.b, cfg.ln_eps)
    torch.cuda.synchronize()
    return {"Z": Z.cpu().numpy(), "W1": W1.cpu().numpy(), "W2": W2.cpu().numpy()}, (W1b, W2b)


@pytest.mark.parametrize("b", [1, 16])
def test_mlp_decode_matches_oracle(b):
    cfg = I.CONFIGS["mlp_B8H32T8192"].replace(B=2, H=3, T=32, b=b)
    dev = to_device(cfg, I.make_inputs(cfg))
    out, (W1b, W2b) = decode_sequence_mlp(cfg, dev)
    worst = compare(cfg, out, all_units(cfg))
    assert max(worst.values()) <= DECODE_TOL, worst
    assert torch.equal(W1b.cpu(), torch.from_numpy(out["W1"]))
    assert torch.equal(W2b.cpu(), torch.from_numpy(out["W2"]))
