"""TTT layers (mini-batch TTT) on NVIDIA B200, sm_100a: the dual-form forward of
TTT-Linear, TTT-Linear + LN and TTT-MLP, its backward (TTT-Linear, + LN), the
primal-form decode step, and the momentum and decay (Titans-style) update.

The computation lives in ``libttt.so`` (C ABI in ``include/ttt.h``); the
functions below are its Python binding over torch CUDA tensors.  ``inputs``
holds the seeded synthetic workloads; ``host`` the forward over host buffers.
"""
from ._lib import (TTT_BF16, TTT_ERR_TIMEOUT, TTT_F32, TTT_OK, TTT_PATH_AUTO,  # noqa: F401
                   TTT_PATH_SIMT, TTT_PATH_TC, TTTError)


def __getattr__(name):
    # The torch-facing binding is imported on first use so that ``inputs`` and the
    # ABI constants stay importable without touching CUDA.
    if name in ("ttt_linear_fwd", "ttt_linear_ln_fwd", "ttt_mlp_fwd", "set_path",
                "last_device_status", "launch_count", "debug_inject_timeout",
                "ttt_linear_decode", "ttt_linear_ln_decode", "ttt_mlp_decode",
                "ttt_linear_momentum_decode", "ttt_linear_ln_momentum_decode",
                "ttt_mlp_momentum_decode", "ttt_linear_bwd", "ttt_linear_momentum_fwd",
                "ttt_linear_ln_bwd_noalloc", "ttt_mlp_bwd",
                "ttt_mlp_momentum_fwd", "ttt_fwd_host", "fwd_host_workspace_bytes"):
        from . import ttt
        return getattr(ttt, name)
    raise AttributeError(name)
