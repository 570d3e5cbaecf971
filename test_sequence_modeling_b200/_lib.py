"""ctypes view of the C ABI declared in ``include/ttt.h`` (libttt.so, built in-tree)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libttt.so")

TTT_OK, TTT_ERR_ARG, TTT_ERR_ALIGN, TTT_ERR_UNSUPPORTED, TTT_ERR_CUDA, TTT_ERR_TIMEOUT = (
    0, -1, -2, -3, -4, -5)
TTT_F32, TTT_BF16 = 0, 1
TTT_PATH_AUTO, TTT_PATH_SIMT, TTT_PATH_TC = 0, 1, 2
TTT_VARIANT_LINEAR, TTT_VARIANT_LINEAR_LN, TTT_VARIANT_MLP = 0, 1, 2
# Capacity of ttt_linear_ln_bwd_noalloc's built-in state array (d x d fp32 states).
TTT_NOALLOC_BWD_MAX_STATES = 4096

_vp, _fp, _i, _f = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float

SIGNATURES = {
    "ttt_linear_fwd": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _i, _i, _i, _i, _i, _fp, _fp, _vp]),
    "ttt_linear_ln_fwd": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _f, _i, _i, _i, _i, _i,
                               _fp, _fp, _vp]),
    "ttt_mlp_fwd": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _fp, _f, _i, _i, _i, _i, _i, _i,
                         _fp, _fp, _fp, _vp]),
    "ttt_status_string": (ctypes.c_char_p, [_i]),
    "ttt_last_device_status": (_i, [_vp]),
    "ttt_set_path": (_i, [_i]),
    "ttt_launch_count": (ctypes.c_longlong, []),
    "ttt_debug_inject_timeout": (_i, [_i]),
    "ttt_linear_momentum_fwd": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _i, _i, _i, _i, _i, _fp, _fp,
                                     _fp, _vp]),
    "ttt_linear_ln_momentum_fwd": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _fp, _fp, _f, _i, _i, _i,
                                        _i, _i, _fp, _fp, _fp, _vp]),
    "ttt_linear_bwd": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _i, _i, _i, _i, _i, _fp, _fp, _fp,
                            _fp, _fp, _fp, _vp]),
    "ttt_linear_ln_bwd": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _f, _fp, _fp, _i, _i, _i, _i, _i,
                               _fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _vp]),
    "ttt_mlp_momentum_fwd": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _f, _i, _i, _i, _i,
                                  _i, _i, _fp, _fp, _fp, _fp, _fp, _vp]),
    "ttt_mlp_bwd": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _fp, _f, _fp, _fp, _fp, _i, _i, _i, _i,
                         _i, _i, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _vp]),
    "ttt_linear_ln_bwd_noalloc": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _f, _fp, _fp, _i, _i, _i, _i,
                                       _i, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _vp]),
    "ttt_linear_decode": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _i, _i, _i, _i, _i, _fp, _vp]),
    "ttt_linear_ln_decode": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _fp, _f, _i, _i, _i, _i, _i,
                                  _fp, _vp]),
    "ttt_linear_momentum_decode": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _fp, _fp, _i, _i, _i,
                                        _i, _i, _fp, _vp]),
    "ttt_linear_ln_momentum_decode": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp,
                                           _f, _i, _i, _i, _i, _i, _fp, _vp]),
    "ttt_mlp_momentum_decode": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp,
                                     _fp, _fp, _f, _i, _i, _i, _i, _i, _i, _fp, _vp]),
    "ttt_mlp_decode": (_i, [_vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _f, _i, _i, _i, _i,
                            _i, _i, _fp, _vp]),
    "ttt_fwd_host_workspace_bytes": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i, _i]),
    "ttt_fwd_host": (_i, [_i, _vp, _vp, _vp, _i, _fp, _fp, _fp, _fp, _fp, _f, _i, _i, _i, _i, _i, _i,
                          _fp, _fp, _fp, _vp, ctypes.c_size_t, _i, _vp]),
}

_lib = None


class TTTError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {status_string(status)} (status {status})")


def load(path: str = LIB_PATH):
    """Load libttt.so.  Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is not built; run "
                           "`python -m test_sequence_modeling_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().ttt_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != TTT_OK:
        raise TTTError(status, where)
