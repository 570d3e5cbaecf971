"""Where the TTT-MLP backward's GPU tolerance comes from (CPU, no GPU).

The reverse dual-form step (``mlp_reverse_dual_form`` in
test_backward_derivation.py, pinned there against the fp64 autograd oracle to
1e-11) is evaluated again with every intermediate rounded to float32, an
operation order unrelated to the kernel's.  For small mini-batches the second
derivative of the LN of the loss gradient amplifies fp32 rounding: this
evaluation lands above 1e-5 from the oracle for b = 1 and b = 4 (so 1e-5 is below
what fp32 reaches there) and below 1e-5 for b = 16.  The GPU test therefore uses
1e-4 for b < 16 and keeps 1e-5 for b = 16.
"""
import numpy as np
import pytest

import test_backward_derivation as TD
from oracle import backward as OB
from test_sequence_modeling_b200 import inputs as I

KEYS = ("dQ", "dK", "dV", "deta", "dW1", "dW2", "dgamma", "dbeta")


@pytest.fixture
def fp32_helpers(monkeypatch):
    as32 = lambda x: np.asarray(x, np.float32)
    for name in ("_gelu", "_gelu_d", "_gelu_dd"):
        fn = getattr(TD, name)
        monkeypatch.setattr(TD, name, lambda x, fn=fn: as32(fn(x)))
    norm = TD._norm
    monkeypatch.setattr(TD, "_norm", lambda y, eps: tuple(as32(v) for v in norm(y, eps)))
    lg = TD._ln_loss_grad
    monkeypatch.setattr(TD, "_ln_loss_grad",
                        lambda *a: (lambda G, ctx: (as32(G), tuple(as32(v) for v in ctx)))(*lg(*a)))
    vjp = TD._ln_loss_grad_vjp
    monkeypatch.setattr(TD, "_ln_loss_grad_vjp", lambda *a: tuple(as32(v) for v in vjp(*a)))


def fp32_error(b):
    cfg = I.CONFIGS["mlp_B8H32T8192"].replace(B=2, H=3, T=48, b=b)
    dZ, dW1T, dW2T = I.mlp_cotangents(cfg)
    worst = 0.0
    for bi, hi in ((0, 0), (1, 2)):
        u = I.unit_as_f64(cfg, bi, hi)
        sl = lambda a: a[bi:bi + 1, hi:hi + 1].astype(np.float64)
        ref = OB.ttt_mlp_backward(u["Q"], u["K"], u["V"], u["eta"], u["W1"], u["W2"], b, sl(dZ),
                                  u["gamma"], u["beta"], cfg.ln_eps, sl(dW1T), sl(dW2T))
        f = lambda x: np.asarray(x, np.float32)
        got = TD.mlp_reverse_dual_form(f(u["Q"][0, 0]), f(u["K"][0, 0]), f(u["V"][0, 0]), f(u["eta"][0, 0]),
                                       f(u["W1"][0]), f(u["W2"][0]), b, f(dZ[bi, hi]), f(dW1T[bi, hi]),
                                       f(dW2T[bi, hi]), f(u["gamma"][0]), f(u["beta"][0]), np.float32(cfg.ln_eps))
        for k in KEYS:
            r = ref[k][0, 0]
            worst = max(worst, float(np.linalg.norm(np.asarray(got[k], np.float64) - r) / np.linalg.norm(r)))
    return worst


@pytest.mark.parametrize("b", [1, 4])
def test_fp32_lands_above_1e5_for_small_mini_batches(fp32_helpers, b):
    e = fp32_error(b)
    assert 1e-5 < e < 1e-4, e


def test_fp32_stays_below_1e5_for_b16(fp32_helpers):
    e = fp32_error(16)
    assert e < 1e-5, e
