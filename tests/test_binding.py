"""The Python binding's marshalling without a GPU: every entry point hands the C
ABI exactly the arguments its declared signature has, with the sizes in place,
and rejects tensors whose shapes do not match before any call (the C ABI reads
plain pointers, so a size mismatch could only show up as an out-of-bounds read).
The device check is lifted and the library replaced by a recorder."""
import contextlib

import pytest
import torch

from test_sequence_modeling_b200 import _lib as L
from test_sequence_modeling_b200 import ttt


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name not in L.SIGNATURES:
            raise AttributeError(name)

        def call(*args):
            assert len(args) == len(L.SIGNATURES[name][1]), (name, len(args))
            self.calls.append((name, args))
            return L.TTT_OK
        return call


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()

    def cuda_any_device(t, name, dtype=None):
        if not isinstance(t, torch.Tensor):
            raise TypeError(name)
        if dtype is not None and t.dtype != dtype:
            raise TypeError(name)
        return t

    monkeypatch.setattr(ttt, "_cuda", cuda_any_device)
    monkeypatch.setattr(L, "load", lambda *a, **k: r)
    monkeypatch.setattr(ttt, "_stream", lambda s, d: 0)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    return r


B, H, T, d, b, h = 2, 3, 32, 64, 16, 256


def _z(*shape):
    return torch.zeros(*shape)


def _qkv(dt=torch.bfloat16):
    return [torch.zeros(B, H, T, d, dtype=dt) for _ in range(3)]


def test_forward_entry_points(rec):
    Q, K, V = _qkv()
    ttt.ttt_linear_fwd(Q, K, V, _z(B, H, T), _z(H, d, d), b)
    ttt.ttt_linear_ln_fwd(Q, K, V, _z(B, H, T), _z(H, d, d), _z(H, d), _z(H, d), b)
    ttt.ttt_mlp_fwd(Q, K, V, _z(B, H, T), _z(H, d, h), _z(H, h, d), _z(H, d), _z(H, d), b)
    names = [c[0] for c in rec.calls]
    assert names == ["ttt_linear_fwd", "ttt_linear_ln_fwd", "ttt_mlp_fwd"]
    assert rec.calls[0][1][3] == L.TTT_BF16 and rec.calls[0][1][6:11] == (B, H, T, d, b)
    assert rec.calls[1][1][9:14] == (B, H, T, d, b)
    assert rec.calls[2][1][10:16] == (B, H, T, d, h, b)


def test_backward_and_momentum_entry_points(rec):
    Q, K, V = _qkv(torch.float32)
    g = ttt.ttt_linear_bwd(Q, K, V, _z(B, H, T), _z(H, d, d), _z(B, H, T, d), b)
    assert g["W_ckpt"].shape == (B, H, T // b, d, d)
    g = ttt.ttt_linear_bwd(Q, K, V, _z(B, H, T), _z(H, d, d), _z(B, H, T, d), b, dW_T=_z(B, H, d, d),
                           gamma=_z(H, d), beta=_z(H, d))
    assert g["dgamma"].shape == (B, H, d)
    ttt.ttt_linear_momentum_fwd(Q, K, V, _z(B, H, T), _z(B, H, T), _z(B, H, T), _z(H, d, d), b)
    ttt.ttt_linear_momentum_fwd(Q, K, V, _z(B, H, T), _z(B, H, T), _z(B, H, T), _z(H, d, d), b,
                                gamma=_z(H, d), beta=_z(H, d))
    names = [c[0] for c in rec.calls]
    assert names == ["ttt_linear_bwd", "ttt_linear_ln_bwd", "ttt_linear_momentum_fwd",
                     "ttt_linear_ln_momentum_fwd"]
    assert rec.calls[0][1][3] == L.TTT_F32 and rec.calls[0][1][8:13] == (B, H, T, d, b)
    assert rec.calls[0][1][7] is None  # no dW_T: a NULL pointer
    assert rec.calls[1][1][11:16] == (B, H, T, d, b)
    assert rec.calls[2][1][8:13] == (B, H, T, d, b)
    assert rec.calls[3][1][11:16] == (B, H, T, d, b)


def test_decode_entry_points(rec):
    q, k, v = (torch.zeros(B, H, d) for _ in range(3))
    W, Wb, S = _z(B, H, d, d), _z(B, H, d, d), _z(B, H, d, d)
    e = _z(B, H)
    ttt.ttt_linear_decode(q, k, v, e, W, Wb, b, 3)
    ttt.ttt_linear_ln_decode(q, k, v, e, W, Wb, _z(H, d), _z(H, d), b, 3)
    ttt.ttt_linear_momentum_decode(q, k, v, e, e, e, W, Wb, S, b, 3)
    ttt.ttt_linear_ln_momentum_decode(q, k, v, e, e, e, W, Wb, S, _z(H, d), _z(H, d), b, 3)
    W1, W2 = _z(B, H, d, h), _z(B, H, h, d)
    ttt.ttt_mlp_decode(q, k, v, e, W1, W2, W1.clone(), W2.clone(), _z(H, d), _z(H, d), b, 3)
    ttt.ttt_mlp_momentum_decode(q, k, v, e, e, e, W1, W2, W1.clone(), W2.clone(), W1.clone(), W2.clone(),
                                _z(H, d), _z(H, d), b, 3)
    assert [c[0] for c in rec.calls] == ["ttt_linear_decode", "ttt_linear_ln_decode",
                                         "ttt_linear_momentum_decode", "ttt_linear_ln_momentum_decode",
                                         "ttt_mlp_decode", "ttt_mlp_momentum_decode"]
    assert rec.calls[0][1][7:12] == (B, H, d, b, 3)
    assert rec.calls[4][1][12:18] == (B, H, d, h, b, 3)


@pytest.mark.parametrize("case", ["W0 heads", "eta length", "gamma width", "dZ", "alpha", "decode gamma",
                                  "mlp W2", "mlp decode eta"])
def test_shape_mismatches_are_rejected_before_any_call(rec, case):
    Q, K, V = _qkv()
    with pytest.raises(ValueError):
        if case == "W0 heads":
            ttt.ttt_linear_fwd(Q, K, V, _z(B, H, T), _z(1, d, d), b)
        elif case == "eta length":
            ttt.ttt_linear_fwd(Q, K, V, _z(B, H, T - 1), _z(H, d, d), b)
        elif case == "gamma width":
            ttt.ttt_linear_ln_fwd(Q, K, V, _z(B, H, T), _z(H, d, d), _z(H, d - 1), _z(H, d), b)
        elif case == "dZ":
            ttt.ttt_linear_bwd(Q, K, V, _z(B, H, T), _z(H, d, d), _z(B, H, T, d - 1), b)
        elif case == "alpha":
            ttt.ttt_linear_momentum_fwd(Q, K, V, _z(B, H, T), _z(B, H), _z(B, H, T), _z(H, d, d), b)
        elif case == "decode gamma":
            q = torch.zeros(B, H, d)
            ttt.ttt_linear_ln_decode(q, q, q, _z(B, H), _z(B, H, d, d), _z(B, H, d, d), _z(1, d), _z(H, d), b, 0)
        elif case == "mlp W2":
            ttt.ttt_mlp_fwd(Q, K, V, _z(B, H, T), _z(H, d, h), _z(H, h, d + 1), _z(H, d), _z(H, d), b)
        else:
            q = torch.zeros(B, H, d)
            W1, W2 = _z(B, H, d, h), _z(B, H, h, d)
            ttt.ttt_mlp_decode(q, q, q, _z(B), W1, W2, W1.clone(), W2.clone(), _z(H, d), _z(H, d), b, 0)
    assert rec.calls == []
