"""GPU: the host-memory forward (ttt_fwd_host through the C ABI: copies of batch
chunks overlapped with the forwards on three streams) gives exactly the
device-resident forward's outputs."""
import numpy as np
import pytest
import torch

from test_sequence_modeling_b200 import inputs as I
from test_sequence_modeling_b200.host import HostForward
from gpu_helpers import run_gpu, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["linear_bf16_B16H12T2048", "linear_ln_B16H32T8192", "mlp_B8H32T8192"])
@pytest.mark.parametrize("chunks", [1, 3])
def test_host_forward_equals_device_forward(name, chunks):
    cfg = I.CONFIGS[name].replace(B=5, H=3, T=128)
    data = I.make_inputs(cfg)
    dev = to_device(cfg, data)
    ref = run_gpu(cfg, dev)
    host = {k: v.cpu().pin_memory() for k, v in dev.items()}
    Z = torch.empty(cfg.B, cfg.H, cfg.T, cfg.d, pin_memory=True)
    if cfg.variant == "mlp":
        params = [host[k] for k in ("W1", "W2", "gamma", "beta")]
        w_shapes = [(cfg.H, cfg.d, cfg.hidden), (cfg.H, cfg.hidden, cfg.d)]
        outs, keys = [torch.empty((cfg.B,) + s[1:], pin_memory=True) for s in
                      [(0, cfg.H, cfg.d, cfg.hidden), (0, cfg.H, cfg.hidden, cfg.d)]], ["W1", "W2"]
    else:
        params = [host["W0"]] + ([host["gamma"], host["beta"]] if cfg.variant == "linear_ln" else [])
        w_shapes = [(cfg.H, cfg.d, cfg.d)]
        outs, keys = [torch.empty(cfg.B, cfg.H, cfg.d, cfg.d, pin_memory=True)], ["W"]
    fwd = HostForward(cfg.variant, host["Q"], w_shapes, [p.shape for p in params], chunks=chunks)
    done = fwd.run(host["Q"], host["K"], host["V"], host["eta"], params, cfg.b, cfg.ln_eps, Z, outs)
    done.synchronize()
    assert np.array_equal(Z.numpy(), ref["Z"])
    for k, o in zip(keys, outs):
        assert np.array_equal(o.numpy(), ref[k]), k


def test_back_to_back_calls_do_not_overlap():
    """Two calls in a row on different inputs (no event passed between them): each
    output equals the device forward of its own inputs."""
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=6, H=4, T=256)
    runs = []
    for seed in (11, 12):
        c = cfg.replace(seed=seed)
        dev = to_device(c, I.make_inputs(c))
        runs.append((dev, run_gpu(c, dev)))
    fwd = None
    outs = []
    for dev, _ in runs:
        host = {k: v.cpu().pin_memory() for k, v in dev.items()}
        params = [host["W0"], host["gamma"], host["beta"]]
        if fwd is None:
            fwd = HostForward("linear_ln", host["Q"], [(cfg.H, cfg.d, cfg.d)], [p.shape for p in params],
                              chunks=3)
        Z = torch.empty(cfg.B, cfg.H, cfg.T, cfg.d, pin_memory=True)
        W = torch.empty(cfg.B, cfg.H, cfg.d, cfg.d, pin_memory=True)
        fwd.run(host["Q"], host["K"], host["V"], host["eta"], params, cfg.b, cfg.ln_eps, Z, [W])
        outs.append((Z, W))
    fwd.done.synchronize()
    for (Z, W), (_, ref) in zip(outs, runs):
        assert np.array_equal(Z.numpy(), ref["Z"])
        assert np.array_equal(W.numpy(), ref["W"])


def test_host_forward_edges():
    """T = 0 (states pass through), more chunks than batch rows, pageable host
    memory, and a workspace one byte short (rejected before anything runs)."""
    from test_sequence_modeling_b200 import ttt
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=2, H=3, T=64)
    dev = to_device(cfg, I.make_inputs(cfg))
    ref = run_gpu(cfg, dev)
    host = {k: v.cpu() for k, v in dev.items()}          # pageable
    params = [host["W0"], host["gamma"], host["beta"]]
    n = ttt.fwd_host_workspace_bytes("linear_ln", tuple(host["Q"].shape), host["Q"].dtype)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    Z = torch.empty(cfg.B, cfg.H, cfg.T, cfg.d)
    W = torch.empty(cfg.B, cfg.H, cfg.d, cfg.d)
    ttt.ttt_fwd_host("linear_ln", host["Q"], host["K"], host["V"], host["eta"], params, cfg.b, cfg.ln_eps,
                     Z, [W], ws, chunks=7)
    torch.cuda.synchronize()
    assert np.array_equal(Z.numpy(), ref["Z"]) and np.array_equal(W.numpy(), ref["W"])
    with pytest.raises(ttt.TTTError):
        ttt.ttt_fwd_host("linear_ln", host["Q"], host["K"], host["V"], host["eta"], params, cfg.b,
                         cfg.ln_eps, Z, [W], ws[: n - 1], chunks=2)
    # T = 0: no tokens; the final state is the initial one for every unit.
    e = {k: torch.empty(cfg.B, cfg.H, 0, cfg.d, dtype=host[k].dtype) for k in ("Q", "K", "V")}
    eta0 = torch.empty(cfg.B, cfg.H, 0)
    Z0 = torch.empty(cfg.B, cfg.H, 0, cfg.d)
    W0 = torch.zeros(cfg.B, cfg.H, cfg.d, cfg.d)
    ws0 = torch.empty(ttt.fwd_host_workspace_bytes("linear_ln", (cfg.B, cfg.H, 0, cfg.d), host["Q"].dtype),
                      dtype=torch.uint8, device="cuda")
    ttt.ttt_fwd_host("linear_ln", e["Q"], e["K"], e["V"], eta0, params, cfg.b, cfg.ln_eps, Z0, [W0], ws0)
    torch.cuda.synchronize()
    assert np.array_equal(W0.numpy(), np.broadcast_to(host["W0"].numpy(), W0.shape))
