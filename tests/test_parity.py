"""GPU parity: the CUDA path against the fp64 oracle, through the C ABI.

Reduced sizes compare every unit element by element; the full workloads (in the
same launch configuration the benchmark times) compare sampled units.
"""
import numpy as np
import pytest
import torch

import test_sequence_modeling_b200 as ttt
from test_sequence_modeling_b200 import inputs as I
from gpu_helpers import TOL, all_units, compare, run_gpu, sample_units, to_device

pytestmark = pytest.mark.gpu

PATHS = {"auto": ttt.TTT_PATH_AUTO, "simt": ttt.TTT_PATH_SIMT, "tc": ttt.TTT_PATH_TC}


def tc_capable(cfg):
    return cfg.dtype == "bf16" and cfg.b == 16


@pytest.fixture(autouse=True)
def _restore_path():
    yield
    ttt.set_path(ttt.TTT_PATH_AUTO)


def reduced(cfg):
    """Several mini-batches, several units and an odd unit count."""
    if cfg.name.startswith("linear_f32"):
        return cfg.replace(B=3, H=5, T=256)
    return cfg.replace(B=3, H=5, T=128 if cfg.variant == "mlp" else 256)


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", I.CONFIG_ORDER)
def test_reduced_config_every_unit(name, path):
    cfg = reduced(I.CONFIGS[name])
    if path == "tc" and not tc_capable(cfg):
        pytest.skip("no tensor-core kernel for this case")
    ttt.set_path(PATHS[path])
    dev = to_device(cfg, I.make_inputs(cfg))
    out = run_gpu(cfg, dev)
    worst = compare(cfg, out, all_units(cfg))
    tol = TOL[cfg.dtype]
    assert max(worst.values()) <= tol, (name, path, worst)


# Regression bounds of the default path at full size, a few times the error each
# path measures (printed by the test): the exact-fp32 path for fp32 inputs; for
# TTT-Linear, W as bf16 hi + lo and fp16 chain and update operands (measured
# 2.2e-4 plain, 7.4e-5 with LN); tf32 and fp16 operands for TTT-MLP.  A
# precision change shows here long before it reaches the oracle tolerance.
REGRESSION = {"linear_f32_B1H1T256": 1e-6, "linear_bf16_B16H12T2048": 1e-3,
              "linear_ln_B16H32T8192": 3e-4, "linear_ln_B1H32T32768": 3e-4,
              "mlp_B8H32T8192": 1.5e-3}


@pytest.mark.parametrize("name", I.CONFIG_ORDER)
def test_full_size_sampled_units(name):
    cfg = I.CONFIGS[name]
    dev = to_device(cfg, I.make_inputs(cfg))
    out = run_gpu(cfg, dev)
    n = 6 if cfg.variant != "mlp" else 3
    worst = compare(cfg, out, sample_units(cfg, n))
    print(f"{name}: max relative Frobenius error per output {worst}")
    assert max(worst.values()) <= TOL[cfg.dtype], (name, worst)
    assert max(worst.values()) <= REGRESSION[name], (name, worst)
    # Properties that hold at any size: finite everywhere, no unit left unwritten.
    for k, v in out.items():
        assert np.all(np.isfinite(v)), k
        assert np.all(np.abs(v).reshape(cfg.B * cfg.H, -1).max(axis=1) > 0), k


@pytest.mark.parametrize("variant", ["linear", "linear_ln", "mlp"])
@pytest.mark.parametrize("b", [1, 4, 16, 64])
def test_mini_batch_sizes(variant, b):
    if variant == "mlp" and b > 16:
        pytest.skip("TTT-MLP supports b <= 16")
    base = {"linear": "linear_bf16_B16H12T2048", "linear_ln": "linear_ln_B16H32T8192",
            "mlp": "mlp_B8H32T8192"}[variant]
    cfg = I.CONFIGS[base].replace(B=2, H=2, T=max(2 * b, 64), b=b)
    dev = to_device(cfg, I.make_inputs(cfg))
    worst = compare(cfg, run_gpu(cfg, dev), all_units(cfg))
    assert max(worst.values()) <= TOL[cfg.dtype], (variant, b, worst)


@pytest.mark.parametrize("name", ["linear_bf16_B16H12T2048", "linear_ln_B16H32T8192", "mlp_B8H32T8192"])
def test_empty_sequence_copies_initial_state(name):
    cfg = I.CONFIGS[name].replace(B=2, H=3, T=0)
    dev = to_device(cfg, I.make_inputs(cfg))
    out = run_gpu(cfg, dev)
    for k in ("W0", "W1", "W2"):
        if k in dev:
            key = "W" if k == "W0" else k
            ref = np.broadcast_to(dev[k].cpu().numpy()[None], out[key].shape)
            assert np.array_equal(out[key], ref)


def test_deterministic_and_stream_ordered():
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=2, H=4, T=512)
    dev = to_device(cfg, I.make_inputs(cfg))
    a = run_gpu(cfg, dev)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = run_gpu(cfg, dev, stream=s)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_outputs_stay_in_bounds():
    """Outputs carved from a larger buffer: the guard bytes around them stay untouched."""
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=2, H=3, T=64)
    dev = to_device(cfg, I.make_inputs(cfg))
    nz = cfg.B * cfg.H * cfg.T * cfg.d
    nw = cfg.B * cfg.H * cfg.d * cfg.d
    buf = torch.full((nz + nw + 3 * 1024,), 7.0, device="cuda")
    Z = buf[1024:1024 + nz].view(cfg.B, cfg.H, cfg.T, cfg.d)
    W = buf[2048 + nz:2048 + nz + nw].view(cfg.B, cfg.H, cfg.d, cfg.d)
    ttt.ttt_linear_ln_fwd(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], dev["gamma"],
                          dev["beta"], cfg.b, cfg.ln_eps, Z=Z, W_out=W)
    torch.cuda.synchronize()
    h = buf.cpu().numpy()
    assert np.all(h[:1024] == 7.0) and np.all(h[1024 + nz:2048 + nz] == 7.0)
    assert np.all(h[2048 + nz + nw:] == 7.0)


def test_device_status_clean_after_runs():
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=1, H=2, T=64)
    dev = to_device(cfg, I.make_inputs(cfg))
    run_gpu(cfg, dev)
    assert ttt.last_device_status() == 0


BASES = {"linear": "linear_bf16_B16H12T2048", "linear_ln": "linear_ln_B16H32T8192",
         "mlp": "mlp_B8H32T8192"}


@pytest.mark.parametrize("variant", ["linear", "linear_ln", "mlp"])
@pytest.mark.parametrize("T", [16, 48, 80, 208, 1040])
def test_tensor_core_ragged_chunks(variant, T):
    """Sequences whose length is not a multiple of the 64-token chunk."""
    base = BASES[variant]
    cfg = I.CONFIGS[base].replace(B=2, H=3, T=T)
    ttt.set_path(ttt.TTT_PATH_TC)
    dev = to_device(cfg, I.make_inputs(cfg))
    worst = compare(cfg, run_gpu(cfg, dev), all_units(cfg))
    assert max(worst.values()) <= TOL[cfg.dtype], (variant, T, worst)


def test_bounded_wait_expiry_on_the_four_cta_kernel():
    """A grid that the launch runs on the 4-CTA-per-SM register budget (more units
    than 2 per SM hold): expiry reported, context usable, next call exact."""
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=10, H=32, T=128)
    dev = to_device(cfg, I.make_inputs(cfg))
    ttt.set_path(ttt.TTT_PATH_TC)
    ttt.debug_inject_timeout(True)
    try:
        run_gpu(cfg, dev)
        assert ttt.last_device_status() == ttt.TTT_ERR_TIMEOUT
    finally:
        ttt.debug_inject_timeout(False)
    out = run_gpu(cfg, dev)
    assert ttt.last_device_status() == 0
    worst = compare(cfg, out, sample_units(cfg, 6))
    assert max(worst.values()) <= REGRESSION[cfg.name], worst


# Agreement of the tensor-core path with the exact-fp32 CUDA-core path: fp16
# chain and update operands (11-bit significand) for TTT-Linear, tf32 and fp16
# operands for TTT-MLP, both far below the oracle tolerance.
AGREE = {"linear_bf16_B16H12T2048": 1e-3, "linear_ln_B16H32T8192": 5e-4, "mlp_B8H32T8192": 1e-3}


@pytest.mark.parametrize("name", list(AGREE))
def test_tensor_core_matches_cuda_core_path(name):
    """The two CUDA paths agree far below the oracle tolerance."""
    cfg = I.CONFIGS[name].replace(B=2, H=4, T=1024 if not name.startswith("mlp") else 512)
    dev = to_device(cfg, I.make_inputs(cfg))
    ttt.set_path(ttt.TTT_PATH_TC)
    a = run_gpu(cfg, dev)
    ttt.set_path(ttt.TTT_PATH_SIMT)
    b = run_gpu(cfg, dev)
    for k in a:
        rel = np.linalg.norm(a[k] - b[k]) / np.linalg.norm(b[k])
        assert rel < AGREE[name], (k, rel)


@pytest.mark.parametrize("variant", ["linear", "linear_ln", "mlp"])
def test_bounded_wait_expiry_is_reported_and_recoverable(variant):
    """The timeout path without a fault: every CTA waits on a barrier that nothing
    arrives at, the bounded wait expires, the status word reports it, and the
    context stays usable (the next call is exact again)."""
    base = BASES[variant]
    cfg = I.CONFIGS[base].replace(B=2, H=3, T=320)
    dev = to_device(cfg, I.make_inputs(cfg))
    ttt.set_path(ttt.TTT_PATH_TC)
    assert ttt.last_device_status() == 0
    ttt.debug_inject_timeout(True)
    try:
        run_gpu(cfg, dev)
        assert ttt.last_device_status() == ttt.TTT_ERR_TIMEOUT
        assert ttt.last_device_status() == 0, "reading the status word clears it"
    finally:
        ttt.debug_inject_timeout(False)
    worst = compare(cfg, run_gpu(cfg, dev), all_units(cfg))
    assert ttt.last_device_status() == 0
    assert max(worst.values()) <= TOL[cfg.dtype], worst
