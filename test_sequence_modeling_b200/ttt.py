"""Python binding of the TTT layer library (forward, backward, decode, momentum and
decay variants): marshals torch CUDA tensors into the C ABI.

Every step of the computation runs in the CUDA kernels of libttt.so; this module
only checks shapes and dtypes, allocates outputs when the caller passes none,
and hands raw device pointers and the current CUDA stream to the library.  There
is no CPU path: tensors that are not on a CUDA device are rejected.
"""
from __future__ import annotations

import torch

from . import _lib
from ._lib import TTT_BF16, TTT_F32, TTTError, check  # noqa: F401

_QKV_DTYPES = {torch.float32: TTT_F32, torch.bfloat16: TTT_BF16}


def _cuda(t, name, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _shaped(t, name, shape):
    """A float32 CUDA tensor of exactly this shape: the C ABI reads plain pointers, so
    a size mismatch has to be caught here."""
    _cuda(t, name, torch.float32)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _qkv(Q, K, V):
    for n, t in (("Q", Q), ("K", K), ("V", V)):
        _cuda(t, n)
    if not (Q.dtype == K.dtype == V.dtype) or Q.dtype not in _QKV_DTYPES:
        raise TypeError("Q, K, V must share one dtype, float32 or bfloat16")
    if not (Q.shape == K.shape == V.shape) or Q.dim() != 4:
        raise ValueError("Q, K, V must have the same shape [B, H, T, d]")
    return _QKV_DTYPES[Q.dtype]


def _out(t, shape, device, name):
    if t is None:
        return torch.empty(shape, dtype=torch.float32, device=device)
    _cuda(t, name, torch.float32)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}")
    return t


def _stream(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes_stream(s)


def ctypes_stream(s) -> int:
    return int(s.cuda_stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def ttt_linear_fwd(Q, K, V, eta, W0, b, Z=None, W_out=None, stream=None):
    """TTT-Linear forward.  Q, K, V [B,H,T,d] (f32 or bf16), eta [B,H,T] f32, W0 [H,d,d] f32.
    Returns (Z [B,H,T,d] f32, W_out [B,H,d,d] f32)."""
    dt = _qkv(Q, K, V)
    B, H, T, d = Q.shape
    _shaped(eta, "eta", (B, H, T))
    _shaped(W0, "W0", (H, d, d))
    Z = _out(Z, (B, H, T, d), Q.device, "Z")
    W_out = _out(W_out, (B, H, d, d), Q.device, "W_out")
    with torch.cuda.device(Q.device):
        st = _lib.load().ttt_linear_fwd(_ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(W0), B, H, T,
                                        d, int(b), _ptr(Z), _ptr(W_out), _stream(stream, Q.device))
    check(st, "ttt_linear_fwd")
    return Z, W_out


VARIANTS = {"linear": _lib.TTT_VARIANT_LINEAR, "linear_ln": _lib.TTT_VARIANT_LINEAR_LN,
            "mlp": _lib.TTT_VARIANT_MLP}


def fwd_host_workspace_bytes(variant, shape, qkv_dtype, hidden=0) -> int:
    """Device workspace bytes ttt_fwd_host needs for inputs of `shape` [B,H,T,d]."""
    B, H, T, d = shape
    dt = TTT_BF16 if qkv_dtype == torch.bfloat16 else TTT_F32
    n = _lib.load().ttt_fwd_host_workspace_bytes(VARIANTS[variant], dt, B, H, T, d, int(hidden))
    if n == 0:
        raise TTTError(f"ttt_fwd_host_workspace_bytes: invalid arguments for {variant} {tuple(shape)}")
    return int(n)


def _host(t, name, dtype, shape):
    """A contiguous host tensor of this dtype and shape (the C ABI reads plain pointers)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cpu" or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def ttt_fwd_host(variant, Q, K, V, eta, params, b, eps, Z, W_outs, workspace, chunks=4, stream=None):
    """The forward with inputs and outputs in host memory (pinned for overlap).
    params: (W0,) | (W0, gamma, beta) | (W1, W2, gamma, beta) per variant; Z and
    W_outs ((W_out,) or (W1_out, W2_out)): host outputs written in place.  workspace:
    a uint8 CUDA tensor of at least fwd_host_workspace_bytes.  Enqueues on `stream`
    (default: the current stream of the workspace's device) and returns; the outputs
    are valid once that stream has reached this point."""
    if Q.dtype not in _QKV_DTYPES or Q.dim() != 4:
        raise TypeError("Q must be a [B, H, T, d] float32 or bfloat16 tensor")
    B, H, T, d = Q.shape
    dt = _QKV_DTYPES[Q.dtype]
    for n, t in (("Q", Q), ("K", K), ("V", V)):
        _host(t, n, Q.dtype, (B, H, T, d))
    _host(eta, "eta", torch.float32, (B, H, T))
    _host(Z, "Z", torch.float32, (B, H, T, d))
    if variant == "mlp":
        hidden = params[0].shape[-1]
        pshapes = [(H, d, hidden), (H, hidden, d), (H, d), (H, d)]
        wshapes = [(B, H, d, hidden), (B, H, hidden, d)]
    else:
        hidden = 0
        pshapes = [(H, d, d)] + ([(H, d), (H, d)] if variant == "linear_ln" else [])
        wshapes = [(B, H, d, d)]
    if len(params) != len(pshapes) or len(W_outs) != len(wshapes):
        raise ValueError(f"ttt_fwd_host: {variant} takes {len(pshapes)} parameters and {len(wshapes)} states")
    for i, (t, shp) in enumerate(zip(params, pshapes)):
        _host(t, f"params[{i}]", torch.float32, shp)
    for i, (t, shp) in enumerate(zip(W_outs, wshapes)):
        _host(t, f"W_outs[{i}]", torch.float32, shp)
    if not (isinstance(workspace, torch.Tensor) and workspace.is_cuda and workspace.dtype == torch.uint8):
        raise TypeError("ttt_fwd_host: workspace must be a uint8 CUDA tensor")
    W0 = params[0]
    W2_0 = params[1] if variant == "mlp" else None
    gamma, beta = (params[-2], params[-1]) if variant != "linear" else (None, None)
    W2_out = W_outs[1] if variant == "mlp" else None
    with torch.cuda.device(workspace.device):
        st = _lib.load().ttt_fwd_host(VARIANTS[variant], _ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(W0),
                                      _ptr(W2_0), _ptr(gamma), _ptr(beta), float(eps), B, H, T, d, int(hidden),
                                      int(b), _ptr(Z), _ptr(W_outs[0]), _ptr(W2_out), _ptr(workspace),
                                      workspace.numel(), int(chunks), _stream(stream, workspace.device))
    check(st, "ttt_fwd_host")


def ttt_linear_ln_fwd(Q, K, V, eta, W0, gamma, beta, b, eps=1e-6, Z=None, W_out=None, stream=None):
    """TTT-Linear with LN + residual.  gamma, beta [H,d] f32."""
    dt = _qkv(Q, K, V)
    B, H, T, d = Q.shape
    for n, t, shp in (("eta", eta, (B, H, T)), ("W0", W0, (H, d, d)), ("gamma", gamma, (H, d)),
                      ("beta", beta, (H, d))):
        _shaped(t, n, shp)
    Z = _out(Z, (B, H, T, d), Q.device, "Z")
    W_out = _out(W_out, (B, H, d, d), Q.device, "W_out")
    with torch.cuda.device(Q.device):
        st = _lib.load().ttt_linear_ln_fwd(_ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(W0),
                                           _ptr(gamma), _ptr(beta), float(eps), B, H, T, d, int(b),
                                           _ptr(Z), _ptr(W_out), _stream(stream, Q.device))
    check(st, "ttt_linear_ln_fwd")
    return Z, W_out


def ttt_mlp_fwd(Q, K, V, eta, W1, W2, gamma, beta, b, eps=1e-6, Z=None, W1_out=None, W2_out=None,
                stream=None):
    """TTT-MLP forward.  W1 [H,d,h], W2 [H,h,d] f32.  Returns (Z, W1_out, W2_out)."""
    dt = _qkv(Q, K, V)
    B, H, T, d = Q.shape
    _cuda(W1, "W1", torch.float32)
    hidden = W1.shape[-1]
    for n, t, shp in (("eta", eta, (B, H, T)), ("W1", W1, (H, d, hidden)), ("W2", W2, (H, hidden, d)),
                      ("gamma", gamma, (H, d)), ("beta", beta, (H, d))):
        _shaped(t, n, shp)
    Z = _out(Z, (B, H, T, d), Q.device, "Z")
    W1_out = _out(W1_out, (B, H, d, hidden), Q.device, "W1_out")
    W2_out = _out(W2_out, (B, H, hidden, d), Q.device, "W2_out")
    with torch.cuda.device(Q.device):
        st = _lib.load().ttt_mlp_fwd(_ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(W1), _ptr(W2),
                                     _ptr(gamma), _ptr(beta), float(eps), B, H, T, d, hidden,
                                     int(b), _ptr(Z), _ptr(W1_out), _ptr(W2_out),
                                     _stream(stream, Q.device))
    check(st, "ttt_mlp_fwd")
    return Z, W1_out, W2_out


def ttt_linear_momentum_fwd(Q, K, V, eta, alpha, lam, W0, b, gamma=None, beta=None, eps=1e-6, Z=None,
                            W_out=None, S_out=None, stream=None):
    """Forward of TTT-Linear (with gamma and beta: TTT-Linear + LN) with the momentum and
    decay update (see include/ttt.h).  alpha, lam [B,H,T] f32 like eta.  Returns
    (Z [B,H,T,d], W_out [B,H,d,d], S_out [B,H,d,d]), all f32."""
    dt = _qkv(Q, K, V)
    B, H, T, d = Q.shape
    ln = gamma is not None
    for n, t in (("eta", eta), ("alpha", alpha), ("lam", lam)):
        _cuda(t, n, torch.float32)
        if tuple(t.shape) != (B, H, T):
            raise ValueError(f"{n} must have shape {(B, H, T)}")
    _shaped(W0, "W0", (H, d, d))
    if ln:
        for n, t in (("gamma", gamma), ("beta", beta)):
            _shaped(t, n, (H, d))
    Z = _out(Z, (B, H, T, d), Q.device, "Z")
    W_out = _out(W_out, (B, H, d, d), Q.device, "W_out")
    S_out = _out(S_out, (B, H, d, d), Q.device, "S_out")
    with torch.cuda.device(Q.device):
        if ln:
            st = _lib.load().ttt_linear_ln_momentum_fwd(
                _ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(alpha), _ptr(lam), _ptr(W0), _ptr(gamma),
                _ptr(beta), float(eps), B, H, T, d, int(b), _ptr(Z), _ptr(W_out), _ptr(S_out),
                _stream(stream, Q.device))
        else:
            st = _lib.load().ttt_linear_momentum_fwd(
                _ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(alpha), _ptr(lam), _ptr(W0), B, H, T, d,
                int(b), _ptr(Z), _ptr(W_out), _ptr(S_out), _stream(stream, Q.device))
    check(st, "ttt_linear_ln_momentum_fwd" if ln else "ttt_linear_momentum_fwd")
    return Z, W_out, S_out


def ttt_linear_bwd(Q, K, V, eta, W0, dZ, b, dW_T=None, gamma=None, beta=None, eps=1e-6, stream=None):
    """Backward of ttt_linear_fwd (or, with gamma and beta, of ttt_linear_ln_fwd): the
    gradients of <dZ, Z> + <dW_T, W_T>.  dZ [B,H,T,d] f32, dW_T [B,H,d,d] f32 or None.
    Returns a dict: dQ, dK, dV, deta, dW0 (per unit [B,H,d,d]), W_ckpt [B,H,T/b,d,d]
    (the state at every mini-batch start) and, with LN, dgamma, dbeta [B,H,d]."""
    dt = _qkv(Q, K, V)
    B, H, T, d = Q.shape
    ln = gamma is not None
    _shaped(eta, "eta", (B, H, T))
    _shaped(W0, "W0", (H, d, d))
    _shaped(dZ, "dZ", (B, H, T, d))
    if dW_T is not None:
        _cuda(dW_T, "dW_T", torch.float32)
        if tuple(dW_T.shape) != (B, H, d, d):
            raise ValueError(f"dW_T must have shape {(B, H, d, d)}")
    if ln:
        for n, t in (("gamma", gamma), ("beta", beta)):
            _shaped(t, n, (H, d))
    if b <= 0 or T % b:
        raise ValueError("T must be a multiple of b")
    dev = Q.device
    out = {n: torch.empty(B, H, T, d, device=dev) for n in ("dQ", "dK", "dV")}
    out["deta"] = torch.empty(B, H, T, device=dev)
    out["dW0"] = torch.empty(B, H, d, d, device=dev)
    out["W_ckpt"] = torch.empty(B, H, T // b, d, d, device=dev)
    if ln:
        out["dgamma"] = torch.empty(B, H, d, device=dev)
        out["dbeta"] = torch.empty(B, H, d, device=dev)
    o = {k: _ptr(v) for k, v in out.items()}
    dwt = _ptr(dW_T)
    with torch.cuda.device(dev):
        if ln:
            st = _lib.load().ttt_linear_ln_bwd(
                _ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(W0), _ptr(gamma), _ptr(beta), float(eps),
                _ptr(dZ), dwt, B, H, T, d, int(b), o["dQ"], o["dK"], o["dV"], o["deta"], o["dW0"],
                o["dgamma"], o["dbeta"], o["W_ckpt"], _stream(stream, dev))
        else:
            st = _lib.load().ttt_linear_bwd(
                _ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(W0), _ptr(dZ), dwt, B, H, T, d, int(b),
                o["dQ"], o["dK"], o["dV"], o["deta"], o["dW0"], o["W_ckpt"], _stream(stream, dev))
    check(st, "ttt_linear_ln_bwd" if ln else "ttt_linear_bwd")
    return out


def ttt_mlp_momentum_fwd(Q, K, V, eta, alpha, lam, W1, W2, gamma, beta, b, eps=1e-6, stream=None):
    """TTT-MLP forward with the momentum and decay update.  Q, K, V [B,H,T,d]; eta,
    alpha, lam [B,H,T] f32; W1 [H,d,h], W2 [H,h,d]; gamma, beta [H,d].  Returns
    (Z [B,H,T,d], W1 [B,H,d,h], W2 [B,H,h,d], S1 [B,H,d,h], S2 [B,H,h,d])."""
    dt = _qkv(Q, K, V)
    B, H, T, d = Q.shape
    h = W1.shape[-1]
    for n, t in (("eta", eta), ("alpha", alpha), ("lambda", lam)):
        _shaped(t, n, (B, H, T))
    _shaped(W1, "W1", (H, d, h))
    _shaped(W2, "W2", (H, h, d))
    for n, t in (("gamma", gamma), ("beta", beta)):
        _shaped(t, n, (H, d))
    dev = Q.device
    Z = torch.empty(B, H, T, d, device=dev)
    W1o, S1o = (torch.empty(B, H, d, h, device=dev) for _ in range(2))
    W2o, S2o = (torch.empty(B, H, h, d, device=dev) for _ in range(2))
    with torch.cuda.device(dev):
        st = _lib.load().ttt_mlp_momentum_fwd(
            _ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(alpha), _ptr(lam), _ptr(W1), _ptr(W2),
            _ptr(gamma), _ptr(beta), float(eps), B, H, T, d, h, int(b), _ptr(Z), _ptr(W1o), _ptr(W2o),
            _ptr(S1o), _ptr(S2o), _stream(stream, dev))
    check(st, "ttt_mlp_momentum_fwd")
    return Z, W1o, W2o, S1o, S2o


def ttt_mlp_bwd(Q, K, V, eta, W1, W2, gamma, beta, dZ, b, eps=1e-6, dW1_T=None, dW2_T=None, stream=None):
    """Backward of ttt_mlp_fwd: the gradients of <dZ, Z> + <dW1_T, W1_T> + <dW2_T, W2_T>.
    dZ [B,H,T,d] f32; dW1_T [B,H,d,h], dW2_T [B,H,h,d] f32 or None.  Returns a dict:
    dQ, dK, dV, deta, dW1, dW2 (per unit), dgamma, dbeta [B,H,d] and the per-mini-batch
    states W1_ckpt [B,H,T/b,d,h], W2_ckpt [B,H,T/b,h,d]."""
    dt = _qkv(Q, K, V)
    B, H, T, d = Q.shape
    h = W1.shape[-1]
    _shaped(eta, "eta", (B, H, T))
    _shaped(W1, "W1", (H, d, h))
    _shaped(W2, "W2", (H, h, d))
    _shaped(dZ, "dZ", (B, H, T, d))
    for n, t in (("gamma", gamma), ("beta", beta)):
        _shaped(t, n, (H, d))
    if dW1_T is not None:
        _shaped(dW1_T, "dW1_T", (B, H, d, h))
    if dW2_T is not None:
        _shaped(dW2_T, "dW2_T", (B, H, h, d))
    if b <= 0 or T % b:
        raise ValueError("T must be a multiple of b")
    dev = Q.device
    out = {n: torch.empty(B, H, T, d, device=dev) for n in ("dQ", "dK", "dV")}
    out["deta"] = torch.empty(B, H, T, device=dev)
    out["dW1"] = torch.empty(B, H, d, h, device=dev)
    out["dW2"] = torch.empty(B, H, h, d, device=dev)
    out["dgamma"] = torch.empty(B, H, d, device=dev)
    out["dbeta"] = torch.empty(B, H, d, device=dev)
    out["W1_ckpt"] = torch.empty(B, H, T // b, d, h, device=dev)
    out["W2_ckpt"] = torch.empty(B, H, T // b, h, d, device=dev)
    o = {k: _ptr(v) for k, v in out.items()}
    with torch.cuda.device(dev):
        st = _lib.load().ttt_mlp_bwd(
            _ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(W1), _ptr(W2), _ptr(gamma), _ptr(beta),
            float(eps), _ptr(dZ), _ptr(dW1_T), _ptr(dW2_T), B, H, T, d, h, int(b), o["dQ"], o["dK"],
            o["dV"], o["deta"], o["dW1"], o["dW2"], o["dgamma"], o["dbeta"], o["W1_ckpt"], o["W2_ckpt"],
            _stream(stream, dev))
    check(st, "ttt_mlp_bwd")
    return out


def ttt_linear_ln_bwd_noalloc(Q, K, V, eta, W0, dZ, b, gamma, beta, eps=1e-6, dW_T=None, out=None,
                              stream=None):
    """The backward of ttt_linear_ln_fwd for callers that must not allocate device
    memory: the states its reverse pass reads back stay in the library's own fixed
    array (B*H*T/b <= TTT_NOALLOC_BWD_MAX_STATES), so no W_ckpt is returned.  Pass
    preallocated outputs in `out` (dQ, dK, dV, deta, dW0, dgamma, dbeta) to keep the
    call free of allocation on this side too.  Calls whose kernels overlap on the
    GPU share that array and race; the first call on a device looks its address up
    and should come before any stream capture."""
    dt = _qkv(Q, K, V)
    B, H, T, d = Q.shape
    _shaped(eta, "eta", (B, H, T))
    _shaped(W0, "W0", (H, d, d))
    _shaped(dZ, "dZ", (B, H, T, d))
    for n, t in (("gamma", gamma), ("beta", beta)):
        _shaped(t, n, (H, d))
    if dW_T is not None:
        _shaped(dW_T, "dW_T", (B, H, d, d))
    if b <= 0 or T % b:
        raise ValueError("T must be a multiple of b")
    dev = Q.device
    shapes = {"dQ": (B, H, T, d), "dK": (B, H, T, d), "dV": (B, H, T, d), "deta": (B, H, T),
              "dW0": (B, H, d, d), "dgamma": (B, H, d), "dbeta": (B, H, d)}
    out = dict(out or {})
    for n, shp in shapes.items():
        out[n] = _out(out.get(n), shp, dev, n)
    o = {k: _ptr(v) for k, v in out.items()}
    with torch.cuda.device(dev):
        st = _lib.load().ttt_linear_ln_bwd_noalloc(
            _ptr(Q), _ptr(K), _ptr(V), dt, _ptr(eta), _ptr(W0), _ptr(gamma), _ptr(beta), float(eps),
            _ptr(dZ), _ptr(dW_T), B, H, T, d, int(b), o["dQ"], o["dK"], o["dV"], o["deta"], o["dW0"],
            o["dgamma"], o["dbeta"], _stream(stream, dev))
    check(st, "ttt_linear_ln_bwd_noalloc")
    return out


def _decode_args(q, k, v, eta, W, W_base, z):
    for n, t in (("q", q), ("k", k), ("v", v)):
        _cuda(t, n)
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in _QKV_DTYPES:
        raise TypeError("q, k, v must share one dtype, float32 or bfloat16")
    if not (q.shape == k.shape == v.shape) or q.dim() != 3:
        raise ValueError("q, k, v must have the same shape [B, H, d]")
    B, H, d = q.shape
    _cuda(eta, "eta", torch.float32)
    if tuple(eta.shape) != (B, H):
        raise ValueError(f"eta must have shape {(B, H)}")
    for n, t in (("W", W), ("W_base", W_base)):
        _cuda(t, n, torch.float32)
        if tuple(t.shape) != (B, H, d, d):
            raise ValueError(f"{n} must have shape {(B, H, d, d)}")
    z = _out(z, (B, H, d), q.device, "z")
    return _QKV_DTYPES[q.dtype], B, H, d, z


def ttt_linear_decode(q, k, v, eta, W, W_base, b, pos, z=None, stream=None):
    """One primal-form decode step of TTT-Linear (see include/ttt.h).  q, k, v [B,H,d],
    eta [B,H]; W and W_base [B,H,d,d] f32 are updated in place.  Returns z [B,H,d] f32."""
    dt, B, H, d, z = _decode_args(q, k, v, eta, W, W_base, z)
    with torch.cuda.device(q.device):
        st = _lib.load().ttt_linear_decode(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(eta), _ptr(W),
                                           _ptr(W_base), B, H, d, int(b), int(pos), _ptr(z),
                                           _stream(stream, q.device))
    check(st, "ttt_linear_decode")
    return z


def ttt_linear_ln_decode(q, k, v, eta, W, W_base, gamma, beta, b, pos, eps=1e-6, z=None, stream=None):
    """One primal-form decode step of TTT-Linear with LN + residual; gamma, beta [H,d] f32."""
    dt, B, H, d, z = _decode_args(q, k, v, eta, W, W_base, z)
    for n, t in (("gamma", gamma), ("beta", beta)):
        _shaped(t, n, (H, d))
    with torch.cuda.device(q.device):
        st = _lib.load().ttt_linear_ln_decode(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(eta), _ptr(W),
                                              _ptr(W_base), _ptr(gamma), _ptr(beta), float(eps), B, H,
                                              d, int(b), int(pos), _ptr(z), _stream(stream, q.device))
    check(st, "ttt_linear_ln_decode")
    return z


def _momentum_args(B, H, d, alpha, lam, S):
    for n, t in (("alpha", alpha), ("lam", lam)):
        _cuda(t, n, torch.float32)
        if tuple(t.shape) != (B, H):
            raise ValueError(f"{n} must have shape {(B, H)}")
    _cuda(S, "S", torch.float32)
    if tuple(S.shape) != (B, H, d, d):
        raise ValueError(f"S must have shape {(B, H, d, d)}")


def ttt_linear_momentum_decode(q, k, v, eta, alpha, lam, W, W_base, S, b, pos, z=None, stream=None):
    """One decode step of TTT-Linear with the momentum and decay update (see
    include/ttt.h): alpha, lam [B,H] f32; W, W_base and the momentum S [B,H,d,d] f32
    are updated in place (S starts at zero).  Returns z [B,H,d] f32."""
    dt, B, H, d, z = _decode_args(q, k, v, eta, W, W_base, z)
    _momentum_args(B, H, d, alpha, lam, S)
    with torch.cuda.device(q.device):
        st = _lib.load().ttt_linear_momentum_decode(
            _ptr(q), _ptr(k), _ptr(v), dt, _ptr(eta), _ptr(alpha), _ptr(lam), _ptr(W), _ptr(W_base),
            _ptr(S), B, H, d, int(b), int(pos), _ptr(z), _stream(stream, q.device))
    check(st, "ttt_linear_momentum_decode")
    return z


def ttt_linear_ln_momentum_decode(q, k, v, eta, alpha, lam, W, W_base, S, gamma, beta, b, pos, eps=1e-6,
                                  z=None, stream=None):
    """The momentum and decay decode step of TTT-Linear with LN + residual."""
    dt, B, H, d, z = _decode_args(q, k, v, eta, W, W_base, z)
    _momentum_args(B, H, d, alpha, lam, S)
    for n, t in (("gamma", gamma), ("beta", beta)):
        _shaped(t, n, (H, d))
    with torch.cuda.device(q.device):
        st = _lib.load().ttt_linear_ln_momentum_decode(
            _ptr(q), _ptr(k), _ptr(v), dt, _ptr(eta), _ptr(alpha), _ptr(lam), _ptr(W), _ptr(W_base),
            _ptr(S), _ptr(gamma), _ptr(beta), float(eps), B, H, d, int(b), int(pos), _ptr(z),
            _stream(stream, q.device))
    check(st, "ttt_linear_ln_momentum_decode")
    return z


def ttt_mlp_decode(q, k, v, eta, W1, W2, W1_base, W2_base, gamma, beta, b, pos, eps=1e-6, z=None,
                   stream=None):
    """One primal-form decode step of TTT-MLP.  W1, W1_base [B,H,d,hidden] and W2, W2_base
    [B,H,hidden,d] f32 are updated in place; gamma, beta [H,d].  Returns z [B,H,d] f32."""
    dt, B, H, d, hidden, z = _mlp_decode_args(q, k, v, eta, W1, W2, W1_base, W2_base, gamma, beta, z)
    with torch.cuda.device(q.device):
        st = _lib.load().ttt_mlp_decode(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(eta),
                                        _ptr(W1), _ptr(W2), _ptr(W1_base), _ptr(W2_base), _ptr(gamma),
                                        _ptr(beta), float(eps), B, H, d, hidden, int(b), int(pos), _ptr(z),
                                        _stream(stream, q.device))
    check(st, "ttt_mlp_decode")
    return z


def ttt_mlp_momentum_decode(q, k, v, eta, alpha, lam, W1, W2, W1_base, W2_base, S1, S2, gamma, beta, b,
                            pos, eps=1e-6, z=None, stream=None):
    """The TTT-MLP decode step with the momentum and decay update: alpha, lam [B,H] f32;
    the momenta S1 (like W1) and S2 (like W2) start at zero and are updated in place."""
    dt, B, H, d, hidden, z = _mlp_decode_args(q, k, v, eta, W1, W2, W1_base, W2_base, gamma, beta, z)
    for n, t in (("alpha", alpha), ("lam", lam)):
        _cuda(t, n, torch.float32)
        if tuple(t.shape) != (B, H):
            raise ValueError(f"{n} must have shape {(B, H)}")
    for n, t, ref in (("S1", S1, W1), ("S2", S2, W2)):
        _cuda(t, n, torch.float32)
        if t.shape != ref.shape:
            raise ValueError(f"{n} must have shape {tuple(ref.shape)}")
    with torch.cuda.device(q.device):
        st = _lib.load().ttt_mlp_momentum_decode(
            _ptr(q), _ptr(k), _ptr(v), dt, _ptr(eta), _ptr(alpha), _ptr(lam), _ptr(W1), _ptr(W2),
            _ptr(W1_base), _ptr(W2_base), _ptr(S1), _ptr(S2), _ptr(gamma), _ptr(beta), float(eps), B, H,
            d, hidden, int(b), int(pos), _ptr(z), _stream(stream, q.device))
    check(st, "ttt_mlp_momentum_decode")
    return z


def _mlp_decode_args(q, k, v, eta, W1, W2, W1_base, W2_base, gamma, beta, z):
    for n, t in (("q", q), ("k", k), ("v", v)):
        _cuda(t, n)
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in _QKV_DTYPES:
        raise TypeError("q, k, v must share one dtype, float32 or bfloat16")
    if not (q.shape == k.shape == v.shape) or q.dim() != 3:
        raise ValueError("q, k, v must have the same shape [B, H, d]")
    B, H, d = q.shape
    hidden = W1.shape[-1]
    _shaped(eta, "eta", (B, H))
    for n, t, shp in (("W1", W1, (B, H, d, hidden)), ("W1_base", W1_base, (B, H, d, hidden)),
                      ("W2", W2, (B, H, hidden, d)), ("W2_base", W2_base, (B, H, hidden, d))):
        _cuda(t, n, torch.float32)
        if tuple(t.shape) != shp:
            raise ValueError(f"{n} must have shape {shp}")
    for n, t in (("gamma", gamma), ("beta", beta)):
        _shaped(t, n, (H, d))
    z = _out(z, (B, H, d), q.device, "z")
    return _QKV_DTYPES[q.dtype], B, H, d, hidden, z


def set_path(path: int) -> int:
    """Select the kernel path (TTT_PATH_AUTO / _SIMT / _TC); returns the previous one."""
    prev = _lib.load().ttt_set_path(int(path))
    if prev < 0:
        raise TTTError(prev, "ttt_set_path")
    return prev


def last_device_status(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(_lib.load().ttt_last_device_status(ctypes_stream(s)))


def launch_count() -> int:
    return int(_lib.load().ttt_launch_count())


def debug_inject_timeout(on: bool) -> bool:
    """Test hook: while on, tensor-core launches run their bounded-wait expiry path
    (see ``ttt_debug_inject_timeout`` in include/ttt.h).  Returns the previous setting."""
    return bool(_lib.load().ttt_debug_inject_timeout(1 if on else 0))
