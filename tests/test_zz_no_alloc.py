"""The backward entry point that allocates nothing (ttt_linear_ln_bwd_noalloc).

Some callers cannot call cudaMalloc: an operator hosted by a framework that owns
the device allocator, or a serving process that reserves all device memory at
start-up.  ttt_linear_ln_bwd asks such a caller for a workspace (the states its
reverse pass reads back); ttt_linear_ln_bwd_noalloc keeps them in a fixed array
inside the library instead.  These tests call it through the C ABI and check
that its outputs match ttt_linear_ln_bwd's on the same inputs, on two calls in a
row: the array keeps the first call's contents, so a second call that read a
stale state would differ.

This file sorts last so that a run stopping at the first failure has run every
other test before it; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from test_sequence_modeling_b200 import _lib as L
from test_sequence_modeling_b200 import inputs as I

pytestmark = pytest.mark.gpu

# The backward's tolerance (fp32 arithmetic from exactly the same inputs).
BWD_TOL = 1e-5
KEYS = ("dQ", "dK", "dV", "deta", "dW0", "dgamma", "dbeta")


def _device_inputs(cfg, seed_offset):
    cfg = cfg.replace(seed=cfg.seed + seed_offset)
    data = I.make_inputs(cfg)
    qkv = [torch.from_numpy(data[k].view(np.int16)).cuda().view(torch.bfloat16) for k in ("Q", "K", "V")]
    dev = {"Q": qkv[0], "K": qkv[1], "V": qkv[2]}
    for k in ("eta", "W0", "gamma", "beta"):
        dev[k] = torch.from_numpy(np.ascontiguousarray(data[k])).cuda()
    dZ, dWT = I.cotangents(cfg)
    dev["dZ"] = torch.from_numpy(dZ).cuda()
    dev["dW_T"] = torch.from_numpy(dWT).cuda()
    return cfg, dev


def _outputs(cfg):
    B, H, T, d = cfg.B, cfg.H, cfg.T, cfg.d
    shapes = {"dQ": (B, H, T, d), "dK": (B, H, T, d), "dV": (B, H, T, d), "deta": (B, H, T),
              "dW0": (B, H, d, d), "dgamma": (B, H, d), "dbeta": (B, H, d)}
    # NaN-filled, so that an element the call does not write cannot pass.
    return {k: torch.full(s, float("nan"), device="cuda") for k, s in shapes.items()}


def _call_existing(lib, cfg, dev, stream):
    out = _outputs(cfg)
    ckpt = torch.empty(cfg.B, cfg.H, cfg.T // cfg.b, cfg.d, cfg.d, device="cuda")
    st = lib.ttt_linear_ln_bwd(
        dev["Q"].data_ptr(), dev["K"].data_ptr(), dev["V"].data_ptr(), L.TTT_BF16, dev["eta"].data_ptr(),
        dev["W0"].data_ptr(), dev["gamma"].data_ptr(), dev["beta"].data_ptr(), cfg.ln_eps,
        dev["dZ"].data_ptr(), dev["dW_T"].data_ptr(), cfg.B, cfg.H, cfg.T, cfg.d, cfg.b,
        *[out[k].data_ptr() for k in KEYS], ckpt.data_ptr(), stream)
    assert st == L.TTT_OK, L.status_string(st)
    return out


def _call_noalloc(lib, cfg, dev, stream):
    out = _outputs(cfg)
    st = lib.ttt_linear_ln_bwd_noalloc(
        dev["Q"].data_ptr(), dev["K"].data_ptr(), dev["V"].data_ptr(), L.TTT_BF16, dev["eta"].data_ptr(),
        dev["W0"].data_ptr(), dev["gamma"].data_ptr(), dev["beta"].data_ptr(), cfg.ln_eps,
        dev["dZ"].data_ptr(), dev["dW_T"].data_ptr(), cfg.B, cfg.H, cfg.T, cfg.d, cfg.b,
        *[out[k].data_ptr() for k in KEYS], stream)
    assert st == L.TTT_OK, L.status_string(st)
    return out


def _rel_fro(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def test_noalloc_backward_matches_existing_entry_point_on_two_calls_in_a_row():
    lib = L.load()
    stream = torch.cuda.current_stream().cuda_stream
    base = I.CONFIGS["linear_ln_B16H32T8192"]
    # First a small call, then one that fills the whole array (4 x 32 units x 32
    # mini-batches = 4096 states) with other inputs: the second call overwrites
    # and re-reads every state the first one left behind.
    cases = [(base.replace(B=2, H=3, T=48), 10), (base.replace(B=4, H=32, T=512), 20)]
    assert cases[1][0].B * cases[1][0].H * cases[1][0].T // cases[1][0].b == L.TTT_NOALLOC_BWD_MAX_STATES
    for cfg, seed_offset in cases:
        cfg, dev = _device_inputs(cfg, seed_offset)
        got = _call_noalloc(lib, cfg, dev, stream)
        ref = _call_existing(lib, cfg, dev, stream)
        torch.cuda.synchronize()
        assert lib.ttt_last_device_status(stream) == L.TTT_OK
        for k in KEYS:
            assert bool(torch.isfinite(got[k]).all()), k
            err = _rel_fro(got[k], ref[k])
            assert err <= BWD_TOL, (cfg.B, cfg.H, cfg.T, k, err)


def test_noalloc_backward_rejects_more_states_than_its_array_holds():
    lib = L.load()
    cfg, dev = _device_inputs(I.CONFIGS["linear_ln_B16H32T8192"].replace(B=4, H=32, T=528), 30)
    assert cfg.B * cfg.H * cfg.T // cfg.b > L.TTT_NOALLOC_BWD_MAX_STATES
    out = _outputs(cfg)
    st = lib.ttt_linear_ln_bwd_noalloc(
        dev["Q"].data_ptr(), dev["K"].data_ptr(), dev["V"].data_ptr(), L.TTT_BF16, dev["eta"].data_ptr(),
        dev["W0"].data_ptr(), dev["gamma"].data_ptr(), dev["beta"].data_ptr(), cfg.ln_eps,
        dev["dZ"].data_ptr(), dev["dW_T"].data_ptr(), cfg.B, cfg.H, cfg.T, cfg.d, cfg.b,
        *[out[k].data_ptr() for k in KEYS], torch.cuda.current_stream().cuda_stream)
    assert st == L.TTT_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert all(bool(torch.isnan(out[k]).all()) for k in KEYS)  # nothing was launched
