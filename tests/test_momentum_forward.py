"""GPU parity of the whole-sequence forward with the momentum and decay update
(ttt_linear_momentum_fwd / ttt_linear_ln_momentum_fwd) against the fp64
oracle's momentum variant, through the C ABI: the exact-fp32 register-state
kernel (the CUDA-core path) to 1e-5, and the tensor-core dual form (TTT-Linear +
LN, bf16 inputs, b = 16, the default path there) to the bf16-input tolerance with
a regression bound."""
import numpy as np
import pytest
import torch

import oracle
import test_sequence_modeling_b200 as ttt
from test_sequence_modeling_b200 import _lib, inputs as I
from gpu_helpers import rel_fro, to_device

pytestmark = pytest.mark.gpu

# fp32 arithmetic from exactly the oracle's inputs, as for the decode step.
TOL = 1e-5
# The tensor-core path: bf16 inputs with fp32 accumulation (the method's 2e-3),
# and a regression bound a few times the 2.9-3.5e-4 it measures (fp16 operands
# of the coefficient-weighted Gram, eta G and the weighted K of the update).
TC_TOL, TC_REGRESSION = 2e-3, 1e-3
NAMES = ["linear_f32_B1H1T256", "linear_bf16_B16H12T2048", "linear_ln_B16H32T8192"]


def run_gpu(cfg, dev, alpha, lam, path=ttt.TTT_PATH_SIMT):
    ln = cfg.variant == "linear_ln"
    kw = dict(gamma=dev["gamma"], beta=dev["beta"], eps=cfg.ln_eps) if ln else {}
    prev = ttt.set_path(path)
    try:
        Z, W, S = ttt.ttt_linear_momentum_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], alpha, lam, dev["W0"],
                                              cfg.b, **kw)
        torch.cuda.synchronize()
    finally:
        ttt.set_path(prev)
    assert ttt.last_device_status() == 0
    return Z, W, S


def oracle_unit(cfg, alpha, lam, bi, hi):
    u = I.unit_as_f64(cfg, bi, hi)
    kind = oracle.LINEAR if cfg.variant == "linear" else oracle.LINEAR_LN
    return oracle.default().momentum_forward(
        kind, u["Q"], u["K"], u["V"], u["eta"], alpha[bi, hi][None, None].astype(np.float64),
        lam[bi, hi][None, None].astype(np.float64), u["W0"].reshape(1, -1), cfg.b, u["gamma"], u["beta"],
        cfg.ln_eps)


def worst_error(cfg, out, alpha, lam, units):
    Z, W, S = (x.cpu().numpy() for x in out)
    worst = {"Z": 0.0, "W": 0.0, "S": 0.0}
    for bi, hi in units:
        Zr, Wr, Sr = oracle_unit(cfg, alpha, lam, bi, hi)
        for key, g, r in (("Z", Z[bi, hi], Zr[0, 0]), ("W", W[bi, hi].ravel(), Wr[0, 0]),
                          ("S", S[bi, hi].ravel(), Sr[0, 0])):
            assert np.all(np.isfinite(g)), key
            worst[key] = max(worst[key], rel_fro(g, r))
    return worst


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


@pytest.mark.parametrize("path", [ttt.TTT_PATH_SIMT, ttt.TTT_PATH_AUTO])
def test_momentum_forward_empty_sequence(path):
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=2, H=2, T=0)
    dev = to_device(cfg, I.make_inputs(cfg))
    e = torch.empty(2, 2, 0, device="cuda")
    Z, W, S = run_gpu(cfg, dev, e, e, path)
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


# ---- the tensor-core dual form ------------------------------------------------------

TC_NAMES = ["linear_ln_B16H32T8192", "linear_bf16_B16H12T2048"]


def tc_case(T, B=2, H=3, name="linear_ln_B16H32T8192"):
    cfg = I.CONFIGS[name].replace(B=B, H=H, T=T, b=16)
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = I.momentum_rates(cfg)
    return cfg, dev, alpha, lam


@pytest.mark.parametrize("T", [16, 48, 64, 128, 208])
@pytest.mark.parametrize("name", TC_NAMES)
def test_tc_momentum_forward_matches_oracle(name, T):
    """Every unit, one to four chunks, ragged last chunks (T % 64 != 0); TTT-Linear
    with and without LN."""
    cfg, dev, alpha, lam = tc_case(T, name=name)
    out = run_gpu(cfg, dev, torch.from_numpy(alpha).cuda(), torch.from_numpy(lam).cuda(), ttt.TTT_PATH_TC)
    worst = worst_error(cfg, out, alpha, lam, [(b, h) for b in range(cfg.B) for h in range(cfg.H)])
    print(f"tensor-core momentum {cfg.variant} T={T}: {worst}")
    assert max(worst.values()) <= TC_REGRESSION, worst


@pytest.mark.parametrize("name", TC_NAMES)
def test_tc_momentum_forward_agrees_with_cuda_core_path(name):
    """The two CUDA paths on the same inputs, far below the oracle tolerance."""
    cfg, dev, alpha, lam = tc_case(512, B=2, H=4, name=name)
    a, l_ = torch.from_numpy(alpha).cuda(), torch.from_numpy(lam).cuda()
    tc = [x.cpu().numpy() for x in run_gpu(cfg, dev, a, l_, ttt.TTT_PATH_TC)]
    cc = [x.cpu().numpy() for x in run_gpu(cfg, dev, a, l_, ttt.TTT_PATH_SIMT)]
    for x, y in zip(tc, cc):
        assert rel_fro(x, y) < TC_REGRESSION


@pytest.mark.parametrize("name", TC_NAMES)
def test_tc_momentum_without_momentum_or_decay_is_ttt(name):
    """alpha = lambda = 0 makes the dual form's coefficients the causal mask: the
    TTT-Linear (+ LN) tensor-core forward's outputs, and S_T = -eta_T g_T."""
    cfg, dev, _, _ = tc_case(256, name=name)
    z = torch.zeros(cfg.B, cfg.H, cfg.T, device="cuda")
    Z, W, S = run_gpu(cfg, dev, z, z, ttt.TTT_PATH_TC)
    if cfg.variant == "linear_ln":
        Zt, Wt = ttt.ttt_linear_ln_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], dev["gamma"],
                                       dev["beta"], cfg.b, cfg.ln_eps)
    else:
        Zt, Wt = ttt.ttt_linear_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], cfg.b)
    torch.cuda.synchronize()
    assert rel_fro(Z.cpu().numpy(), Zt.cpu().numpy()) < 1e-4
    assert rel_fro(W.cpu().numpy(), Wt.cpu().numpy()) < 1e-4
    assert torch.isfinite(S).all() and S.abs().max() > 0


@pytest.mark.parametrize("name", TC_NAMES)
def test_tc_momentum_forward_full_size_sampled_units(name):
    """The full workload (linear + LN B16 H32 T8192, linear B16 H12 T2048), first and
    last units."""
    cfg = I.CONFIGS[name]
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = I.momentum_rates(cfg)
    out = run_gpu(cfg, dev, torch.from_numpy(alpha).cuda(), torch.from_numpy(lam).cuda(), ttt.TTT_PATH_AUTO)
    assert all(bool(torch.isfinite(x).all()) for x in out)
    worst = worst_error(cfg, out, alpha, lam, [(0, 0), (cfg.B - 1, cfg.H - 1)])
    print(f"tensor-core momentum full size {name}: {worst}")
    assert max(worst.values()) <= TC_REGRESSION, worst


def test_tc_momentum_bounded_wait_expiry_is_reported_and_recoverable():
    """The timeout path without a fault, as for the other tensor-core kernels."""
    cfg, dev, alpha, lam = tc_case(128)
    a, l_ = torch.from_numpy(alpha).cuda(), torch.from_numpy(lam).cuda()
    ttt.debug_inject_timeout(1)
    prev = ttt.set_path(ttt.TTT_PATH_TC)
    try:
        ttt.ttt_linear_momentum_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], a, l_, dev["W0"], cfg.b,
                                    gamma=dev["gamma"], beta=dev["beta"], eps=cfg.ln_eps)
        torch.cuda.synchronize()
    finally:
        ttt.debug_inject_timeout(0)
        ttt.set_path(prev)
    assert ttt.last_device_status() == ttt.TTT_ERR_TIMEOUT
    out = run_gpu(cfg, dev, a, l_, ttt.TTT_PATH_TC)
    worst = worst_error(cfg, out, alpha, lam, [(0, 0), (1, 2)])
    assert max(worst.values()) <= TC_REGRESSION, worst


def test_tc_path_rejects_cases_without_a_tensor_core_kernel():
    """Under TTT_PATH_TC a case the dual form does not take (fp32 inputs) is refused,
    as for the plain forwards; AUTO runs it on the CUDA cores."""
    cfg = I.CONFIGS["linear_f32_B1H1T256"].replace(B=1, H=2, T=32, b=16)
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = (torch.from_numpy(x).cuda() for x in I.momentum_rates(cfg))
    prev = ttt.set_path(ttt.TTT_PATH_TC)
    try:
        with pytest.raises(ttt.TTTError) as e:
            ttt.ttt_linear_momentum_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], alpha, lam, dev["W0"], cfg.b)
        assert e.value.status == _lib.TTT_ERR_UNSUPPORTED
    finally:
        ttt.set_path(prev)
    run_gpu(cfg, dev, alpha, lam, ttt.TTT_PATH_AUTO)


def test_tc_momentum_forward_is_deterministic_and_stays_in_bounds():
    """Two runs agree bit for bit, and outputs carved from one larger buffer leave the
    guard bytes around them untouched (ragged last chunk: T = 208)."""
    cfg, dev, alpha, lam = tc_case(208)
    a, l_ = torch.from_numpy(alpha).cuda(), torch.from_numpy(lam).cuda()
    nz = cfg.B * cfg.H * cfg.T * cfg.d
    nw = cfg.B * cfg.H * cfg.d * cfg.d
    outs = []
    for _ in range(2):
        buf = torch.full((nz + 2 * nw + 4 * 1024,), 7.0, device="cuda")
        Z = buf[1024:1024 + nz].view(cfg.B, cfg.H, cfg.T, cfg.d)
        W = buf[2048 + nz:2048 + nz + nw].view(cfg.B, cfg.H, cfg.d, cfg.d)
        S = buf[3072 + nz + nw:3072 + nz + 2 * nw].view(cfg.B, cfg.H, cfg.d, cfg.d)
        prev = ttt.set_path(ttt.TTT_PATH_TC)
        try:
            ttt.ttt_linear_momentum_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], a, l_, dev["W0"], cfg.b,
                                        gamma=dev["gamma"], beta=dev["beta"], eps=cfg.ln_eps, Z=Z, W_out=W,
                                        S_out=S)
            torch.cuda.synchronize()
        finally:
            ttt.set_path(prev)
        assert ttt.last_device_status() == 0
        h = buf.cpu().numpy()
        assert np.all(h[:1024] == 7.0) and np.all(h[1024 + nz:2048 + nz] == 7.0)
        assert np.all(h[2048 + nz + nw:3072 + nz + nw] == 7.0) and np.all(h[3072 + nz + 2 * nw:] == 7.0)
        outs.append(h)
    assert np.array_equal(outs[0], outs[1])


def test_tc_momentum_forward_long_sequence():
    """512 chunks (T = 32768): no drift of the dual form's error along the sequence."""
    cfg = I.CONFIGS["linear_ln_B1H32T32768"].replace(H=2)
    dev = to_device(cfg, I.make_inputs(cfg))
    alpha, lam = I.momentum_rates(cfg)
    out = run_gpu(cfg, dev, torch.from_numpy(alpha).cuda(), torch.from_numpy(lam).cuda(), ttt.TTT_PATH_TC)
    worst = worst_error(cfg, out, alpha, lam, [(0, 0), (0, 1)])
    print(f"tensor-core momentum T=32768: {worst}")
    assert max(worst.values()) <= TC_REGRESSION, worst
