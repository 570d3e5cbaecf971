"""The C ABI without a GPU: the library loads, exports what include/ttt.h declares,
and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

from test_sequence_modeling_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "ttt.h")).read()
    return sorted(set(re.findall(r"TTT_API\s+[\w\s\*]*?\b(ttt_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from test_sequence_modeling_b200.build import build
    build()
    return L.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.SIGNATURES), "binding signatures out of sync with the header"


def test_status_strings(lib):
    for s in (0, -1, -2, -3, -4, -5):
        assert L.status_string(s)
    assert L.status_string(12345) == "unknown status"


def test_set_path(lib):
    prev = lib.ttt_set_path(L.TTT_PATH_SIMT)
    assert prev in (0, 1, 2)
    assert lib.ttt_set_path(prev) == L.TTT_PATH_SIMT
    assert lib.ttt_set_path(7) == L.TTT_ERR_ARG


# Fake, never-dereferenced device addresses: every call below fails validation,
# which runs before any CUDA call.
A = 0x100000


def _ptrs(n, step=1 << 30, base=A):
    return [base + i * step for i in range(n)]


def linear(lib, **kw):
    q, k, v, eta, w0, z, wo = _ptrs(7)
    a = dict(Q=q, K=k, V=v, dt=L.TTT_BF16, eta=eta, W0=w0, B=2, H=3, T=64, d=64, b=16, Z=z, W=wo)
    a.update(kw)
    return lib.ttt_linear_fwd(a["Q"], a["K"], a["V"], a["dt"], a["eta"], a["W0"], a["B"], a["H"],
                              a["T"], a["d"], a["b"], a["Z"], a["W"], None)


def ln(lib, **kw):
    q, k, v, eta, w0, g, bt, z, wo = _ptrs(9)
    a = dict(Q=q, K=k, V=v, dt=L.TTT_BF16, eta=eta, W0=w0, g=g, bt=bt, eps=1e-6, B=2, H=3, T=64,
             d=64, b=16, Z=z, W=wo)
    a.update(kw)
    return lib.ttt_linear_ln_fwd(a["Q"], a["K"], a["V"], a["dt"], a["eta"], a["W0"], a["g"], a["bt"],
                                 a["eps"], a["B"], a["H"], a["T"], a["d"], a["b"], a["Z"], a["W"], None)


def mlp(lib, **kw):
    q, k, v, eta, w1, w2, g, bt, z, w1o, w2o = _ptrs(11)
    a = dict(Q=q, K=k, V=v, dt=L.TTT_BF16, eta=eta, W1=w1, W2=w2, g=g, bt=bt, eps=1e-6, B=2, H=3,
             T=64, d=64, h=256, b=16, Z=z, W1o=w1o, W2o=w2o)
    a.update(kw)
    return lib.ttt_mlp_fwd(a["Q"], a["K"], a["V"], a["dt"], a["eta"], a["W1"], a["W2"], a["g"],
                           a["bt"], a["eps"], a["B"], a["H"], a["T"], a["d"], a["h"], a["b"], a["Z"],
                           a["W1o"], a["W2o"], None)


@pytest.mark.parametrize("fn", [linear, ln, mlp])
def test_argument_errors(lib, fn):
    n0 = lib.ttt_launch_count()
    assert fn(lib, T=60) == L.TTT_ERR_ARG                # T % b != 0
    assert fn(lib, b=0) == L.TTT_ERR_ARG
    assert fn(lib, B=-1) == L.TTT_ERR_ARG
    assert fn(lib, dt=5) == L.TTT_ERR_ARG                # unknown dtype
    assert fn(lib, d=32) == L.TTT_ERR_UNSUPPORTED
    assert fn(lib, b=128, T=128) == L.TTT_ERR_UNSUPPORTED
    assert fn(lib, Q=None) == L.TTT_ERR_ARG
    assert fn(lib, Z=None) == L.TTT_ERR_ARG
    assert fn(lib, Q=A + 8) == L.TTT_ERR_ALIGN
    assert fn(lib, eta=A + 4) == L.TTT_ERR_ALIGN
    assert fn(lib, Z=A + (3 << 30) + 64) == L.TTT_ERR_ARG  # Z overlaps V
    assert fn(lib, B=0) == L.TTT_OK                      # empty: nothing to do, no CUDA call
    assert fn(lib, H=0) == L.TTT_OK
    assert lib.ttt_launch_count() == n0, "a rejected call launched a kernel"


@pytest.mark.parametrize("fn", [linear, ln, mlp])
def test_tensor_core_path_refuses_cases_it_has_no_kernel_for(lib, fn):
    """Under TTT_PATH_TC a well-formed forward the tensor cores do not take (fp32
    inputs; b != 16) is refused on the host, before any CUDA call."""
    n0 = lib.ttt_launch_count()
    prev = lib.ttt_set_path(L.TTT_PATH_TC)
    try:
        assert fn(lib, dt=L.TTT_F32) == L.TTT_ERR_UNSUPPORTED
        assert fn(lib, b=8) == L.TTT_ERR_UNSUPPORTED
        assert fn(lib, B=0) == L.TTT_OK  # empty: nothing to do on any path
    finally:
        lib.ttt_set_path(prev)
    assert lib.ttt_launch_count() == n0, "a refused call launched a kernel"


def test_ln_specific_errors(lib):
    assert ln(lib, eps=0.0) == L.TTT_ERR_ARG
    assert ln(lib, eps=float("nan")) == L.TTT_ERR_ARG
    assert ln(lib, g=None) == L.TTT_ERR_ARG


def test_mlp_specific_errors(lib):
    assert mlp(lib, h=128) == L.TTT_ERR_UNSUPPORTED
    assert mlp(lib, h=0) == L.TTT_ERR_ARG
    assert mlp(lib, b=32, T=64) == L.TTT_ERR_UNSUPPORTED
    assert mlp(lib, W2o=None) == L.TTT_ERR_ARG
    assert mlp(lib, W2o=A + (9 << 30) + 16) == L.TTT_ERR_ARG  # W2_out overlaps W1_out


def test_python_binding_rejects_cpu_tensors():
    import torch
    import test_sequence_modeling_b200 as ttt
    x = torch.zeros(1, 1, 16, 64)
    with pytest.raises(ValueError, match="CUDA"):
        ttt.ttt_linear_fwd(x, x, x, torch.zeros(1, 1, 16), torch.zeros(1, 64, 64), 16)


def decode(lib, ln=False, **kw):
    q, k, v, eta, w, wb, z, g, bt = _ptrs(9)
    a = dict(q=q, k=k, v=v, dt=L.TTT_BF16, eta=eta, W=w, Wb=wb, g=g, bt=bt, eps=1e-6, B=2, H=3,
             d=64, b=16, pos=0, z=z)
    a.update(kw)
    if ln:
        return lib.ttt_linear_ln_decode(a["q"], a["k"], a["v"], a["dt"], a["eta"], a["W"], a["Wb"],
                                        a["g"], a["bt"], a["eps"], a["B"], a["H"], a["d"], a["b"],
                                        a["pos"], a["z"], None)
    return lib.ttt_linear_decode(a["q"], a["k"], a["v"], a["dt"], a["eta"], a["W"], a["Wb"], a["B"],
                                 a["H"], a["d"], a["b"], a["pos"], a["z"], None)


@pytest.mark.parametrize("ln", [False, True])
def test_decode_argument_errors(lib, ln):
    n0 = lib.ttt_launch_count()
    assert decode(lib, ln, pos=16) == L.TTT_ERR_ARG       # pos outside the mini-batch
    assert decode(lib, ln, pos=-1) == L.TTT_ERR_ARG
    assert decode(lib, ln, b=0) == L.TTT_ERR_ARG
    assert decode(lib, ln, dt=3) == L.TTT_ERR_ARG
    assert decode(lib, ln, d=32) == L.TTT_ERR_UNSUPPORTED
    assert decode(lib, ln, q=None) == L.TTT_ERR_ARG
    assert decode(lib, ln, Wb=None) == L.TTT_ERR_ARG
    assert decode(lib, ln, W=A + 8) == L.TTT_ERR_ALIGN
    assert decode(lib, ln, Wb=A + (6 << 30)) == L.TTT_ERR_ARG  # W_base overlaps z
    assert decode(lib, ln, W=A + (4 << 30) + 1024, Wb=A + (4 << 30) + 4096) == L.TTT_ERR_ARG
    assert decode(lib, ln, B=0) == L.TTT_OK
    if ln:
        assert decode(lib, ln, eps=0.0) == L.TTT_ERR_ARG
        assert decode(lib, ln, g=None) == L.TTT_ERR_ARG
    assert lib.ttt_launch_count() == n0, "a rejected call launched a kernel"


def momentum(lib, ln=False, **kw):
    q, k, v, eta, al, lm, w, wb, s, z, g, bt = _ptrs(12)
    a = dict(q=q, k=k, v=v, dt=L.TTT_BF16, eta=eta, al=al, lm=lm, W=w, Wb=wb, S=s, g=g, bt=bt,
             eps=1e-6, B=2, H=3, d=64, b=16, pos=0, z=z)
    a.update(kw)
    head = (a["q"], a["k"], a["v"], a["dt"], a["eta"], a["al"], a["lm"], a["W"], a["Wb"], a["S"])
    tail = (a["B"], a["H"], a["d"], a["b"], a["pos"], a["z"], None)
    if ln:
        return lib.ttt_linear_ln_momentum_decode(*head, a["g"], a["bt"], a["eps"], *tail)
    return lib.ttt_linear_momentum_decode(*head, *tail)


@pytest.mark.parametrize("ln", [False, True])
def test_momentum_decode_argument_errors(lib, ln):
    n0 = lib.ttt_launch_count()
    assert momentum(lib, ln, pos=16) == L.TTT_ERR_ARG
    assert momentum(lib, ln, d=32) == L.TTT_ERR_UNSUPPORTED
    assert momentum(lib, ln, al=None) == L.TTT_ERR_ARG
    assert momentum(lib, ln, lm=None) == L.TTT_ERR_ARG
    assert momentum(lib, ln, S=None) == L.TTT_ERR_ARG
    assert momentum(lib, ln, S=A + 8) == L.TTT_ERR_ALIGN
    assert momentum(lib, ln, al=A + 4) == L.TTT_ERR_ALIGN
    w, s = _ptrs(12)[6], _ptrs(12)[8]
    assert momentum(lib, ln, S=w + 1024) == L.TTT_ERR_ARG    # S overlaps W
    assert momentum(lib, ln, W=s + 4096) == L.TTT_ERR_ARG    # W overlaps S
    assert momentum(lib, ln, lm=s + 64) == L.TTT_ERR_ARG     # lambda inside S
    assert momentum(lib, ln, B=0) == L.TTT_OK
    if ln:
        assert momentum(lib, ln, g=None) == L.TTT_ERR_ARG
    assert lib.ttt_launch_count() == n0, "a rejected call launched a kernel"


def test_mlp_momentum_decode_argument_errors(lib):
    n0 = lib.ttt_launch_count()
    q, k, v, eta, al, lm, w1, w2, w1b, w2b, s1, s2, z, g, bt = _ptrs(15)

    def call(**kw):
        a = dict(q=q, k=k, v=v, dt=L.TTT_BF16, eta=eta, al=al, lm=lm, w1=w1, w2=w2, w1b=w1b, w2b=w2b,
                 s1=s1, s2=s2, g=g, bt=bt, eps=1e-6, B=2, H=3, d=64, h=256, b=16, pos=0, z=z)
        a.update(kw)
        return lib.ttt_mlp_momentum_decode(a["q"], a["k"], a["v"], a["dt"], a["eta"], a["al"], a["lm"],
                                           a["w1"], a["w2"], a["w1b"], a["w2b"], a["s1"], a["s2"],
                                           a["g"], a["bt"], a["eps"], a["B"], a["H"], a["d"], a["h"],
                                           a["b"], a["pos"], a["z"], None)

    assert call(pos=16) == L.TTT_ERR_ARG
    assert call(h=128) == L.TTT_ERR_UNSUPPORTED
    assert call(s1=None) == L.TTT_ERR_ARG
    assert call(lm=None) == L.TTT_ERR_ARG
    assert call(s2=A + 8) == L.TTT_ERR_ALIGN
    assert call(s2=s1 + 4096) == L.TTT_ERR_ARG        # the two momenta overlap
    assert call(s1=w2 + 1024) == L.TTT_ERR_ARG        # S1 overlaps W2
    assert call(al=s2 + 64) == L.TTT_ERR_ARG          # alpha inside S2
    assert call(B=0) == L.TTT_OK
    assert lib.ttt_launch_count() == n0, "a rejected call launched a kernel"


def test_mlp_decode_argument_errors(lib):
    n0 = lib.ttt_launch_count()
    q, k, v, eta, w1, w2, w1b, w2b, z, g, bt = _ptrs(11)

    def call(**kw):
        a = dict(q=q, k=k, v=v, dt=L.TTT_BF16, eta=eta, w1=w1, w2=w2, w1b=w1b, w2b=w2b, g=g, bt=bt,
                 eps=1e-6, B=2, H=3, d=64, h=256, b=16, pos=0, z=z)
        a.update(kw)
        return lib.ttt_mlp_decode(a["q"], a["k"], a["v"], a["dt"], a["eta"], a["w1"], a["w2"], a["w1b"],
                                  a["w2b"], a["g"], a["bt"], a["eps"], a["B"], a["H"], a["d"], a["h"],
                                  a["b"], a["pos"], a["z"], None)

    assert call(pos=16) == L.TTT_ERR_ARG
    assert call(h=0) == L.TTT_ERR_ARG
    assert call(h=128) == L.TTT_ERR_UNSUPPORTED
    assert call(d=32) == L.TTT_ERR_UNSUPPORTED
    assert call(eps=-1.0) == L.TTT_ERR_ARG
    assert call(w2b=None) == L.TTT_ERR_ARG
    assert call(w1=A + 4) == L.TTT_ERR_ALIGN
    assert call(w2b=w1b + 4096) == L.TTT_ERR_ARG      # the two bases overlap
    assert call(B=0) == L.TTT_OK
    assert lib.ttt_launch_count() == n0, "a rejected call launched a kernel"


def bwd(lib, ln=False, **kw):
    q, k, v, eta, w0, dz, dwt, dq, dk, dv, de, dw0, ck, g, bt, dg, db = _ptrs(17)
    a = dict(q=q, k=k, v=v, dt=L.TTT_BF16, eta=eta, w0=w0, dz=dz, dwt=dwt, B=2, H=3, T=64, d=64, b=16,
             dq=dq, dk=dk, dv=dv, de=de, dw0=dw0, ck=ck, g=g, bt=bt, dg=dg, db=db, eps=1e-6)
    a.update(kw)
    if ln:
        return lib.ttt_linear_ln_bwd(a["q"], a["k"], a["v"], a["dt"], a["eta"], a["w0"], a["g"], a["bt"],
                                     a["eps"], a["dz"], a["dwt"], a["B"], a["H"], a["T"], a["d"], a["b"],
                                     a["dq"], a["dk"], a["dv"], a["de"], a["dw0"], a["dg"], a["db"],
                                     a["ck"], None)
    return lib.ttt_linear_bwd(a["q"], a["k"], a["v"], a["dt"], a["eta"], a["w0"], a["dz"], a["dwt"],
                              a["B"], a["H"], a["T"], a["d"], a["b"], a["dq"], a["dk"], a["dv"], a["de"],
                              a["dw0"], a["ck"], None)


@pytest.mark.parametrize("ln", [False, True])
def test_backward_argument_errors(lib, ln):
    n0 = lib.ttt_launch_count()
    p = _ptrs(17)
    assert bwd(lib, ln, b=32) == L.TTT_ERR_UNSUPPORTED      # mini-batch above 16
    assert bwd(lib, ln, d=32) == L.TTT_ERR_UNSUPPORTED
    assert bwd(lib, ln, T=40) == L.TTT_ERR_ARG              # T not a multiple of b
    assert bwd(lib, ln, b=0) == L.TTT_ERR_ARG
    assert bwd(lib, ln, dt=7) == L.TTT_ERR_ARG
    assert bwd(lib, ln, dz=None) == L.TTT_ERR_ARG
    assert bwd(lib, ln, ck=None) == L.TTT_ERR_ARG
    assert bwd(lib, ln, dw0=None) == L.TTT_ERR_ARG
    assert bwd(lib, ln, dq=A + 4) == L.TTT_ERR_ALIGN
    assert bwd(lib, ln, dwt=A + 8) == L.TTT_ERR_ALIGN
    assert bwd(lib, ln, dk=p[7] + 4096) == L.TTT_ERR_ARG    # dK overlaps dQ
    assert bwd(lib, ln, ck=p[5] + 64) == L.TTT_ERR_ARG      # W_ckpt overlaps dZ
    assert bwd(lib, ln, de=p[6] + 16) == L.TTT_ERR_ARG      # deta overlaps dW_T
    assert bwd(lib, ln, B=0) == L.TTT_OK
    if ln:
        assert bwd(lib, ln, eps=0.0) == L.TTT_ERR_ARG
        assert bwd(lib, ln, dg=None) == L.TTT_ERR_ARG
        assert bwd(lib, ln, db=p[15] + 16) == L.TTT_ERR_ARG  # dbeta overlaps dgamma
    assert lib.ttt_launch_count() == n0, "a rejected call launched a kernel"


def momentum_fwd(lib, ln=False, **kw):
    q, k, v, eta, al, lm, w0, z, wo, so, g, bt = _ptrs(12)
    a = dict(q=q, k=k, v=v, dt=L.TTT_BF16, eta=eta, al=al, lm=lm, w0=w0, g=g, bt=bt, eps=1e-6, B=2, H=3,
             T=64, d=64, b=16, z=z, wo=wo, so=so)
    a.update(kw)
    head = (a["q"], a["k"], a["v"], a["dt"], a["eta"], a["al"], a["lm"], a["w0"])
    tail = (a["B"], a["H"], a["T"], a["d"], a["b"], a["z"], a["wo"], a["so"], None)
    if ln:
        return lib.ttt_linear_ln_momentum_fwd(*head, a["g"], a["bt"], a["eps"], *tail)
    return lib.ttt_linear_momentum_fwd(*head, *tail)


@pytest.mark.parametrize("ln", [False, True])
def test_momentum_forward_argument_errors(lib, ln):
    n0 = lib.ttt_launch_count()
    p = _ptrs(12)
    assert momentum_fwd(lib, ln, b=32) == L.TTT_ERR_UNSUPPORTED
    assert momentum_fwd(lib, ln, d=128) == L.TTT_ERR_UNSUPPORTED
    assert momentum_fwd(lib, ln, T=40) == L.TTT_ERR_ARG
    assert momentum_fwd(lib, ln, al=None) == L.TTT_ERR_ARG
    assert momentum_fwd(lib, ln, so=None) == L.TTT_ERR_ARG
    assert momentum_fwd(lib, ln, lm=A + 4) == L.TTT_ERR_ALIGN
    assert momentum_fwd(lib, ln, so=p[8] + 256) == L.TTT_ERR_ARG    # S_out overlaps W_out
    assert momentum_fwd(lib, ln, z=p[4] + 16) == L.TTT_ERR_ARG      # Z overlaps alpha
    assert momentum_fwd(lib, ln, B=0) == L.TTT_OK
    if ln:
        assert momentum_fwd(lib, ln, eps=-1.0) == L.TTT_ERR_ARG
        assert momentum_fwd(lib, ln, bt=None) == L.TTT_ERR_ARG
    assert lib.ttt_launch_count() == n0, "a rejected call launched a kernel"


@pytest.mark.parametrize("ln", [False, True])
def test_momentum_forward_tensor_core_path_refuses_other_cases(lib, ln):
    """Under TTT_PATH_TC a well-formed call the dual form does not take (fp32 inputs,
    b < 16) is refused on the host, before any CUDA call (fake pointers)."""
    n0 = lib.ttt_launch_count()
    prev = lib.ttt_set_path(L.TTT_PATH_TC)
    try:
        assert momentum_fwd(lib, ln, dt=L.TTT_F32) == L.TTT_ERR_UNSUPPORTED
        assert momentum_fwd(lib, ln, b=8) == L.TTT_ERR_UNSUPPORTED
        assert momentum_fwd(lib, ln, T=36, b=8) == L.TTT_ERR_ARG  # argument errors come first
    finally:
        lib.ttt_set_path(prev)
    assert lib.ttt_launch_count() == n0, "a refused call launched a kernel"


def test_noalloc_backward_checks_sizes_before_any_cuda_call(lib):
    """ttt_linear_ln_bwd_noalloc rejects a call whose states exceed its built-in
    array, and malformed sizes, on the host (fake pointers are never touched)."""
    p = _ptrs(14)

    def call(B, H, T, b=16, d=64, eps=1e-6, dt=L.TTT_BF16):
        return lib.ttt_linear_ln_bwd_noalloc(p[0], p[1], p[2], dt, p[3], p[4], p[5], p[6], eps, p[7],
                                             None, B, H, T, d, b, p[8], p[9], p[10], p[11], p[12],
                                             p[13], p[13] + (1 << 29), None)

    cap = L.TTT_NOALLOC_BWD_MAX_STATES
    assert call(4, 32, 16 * cap // 128 + 16) == L.TTT_ERR_UNSUPPORTED  # one mini-batch too many
    assert call(cap + 1, 1, 16) == L.TTT_ERR_UNSUPPORTED
    assert call(2, 3, 40) == L.TTT_ERR_ARG                  # T % b != 0
    assert call(2, 3, 48, eps=0.0) == L.TTT_ERR_ARG
    assert call(2, 3, 48, dt=7) == L.TTT_ERR_ARG
    assert call(2, 3, 48, d=32) == L.TTT_ERR_UNSUPPORTED
    assert call(2, 3, 64, b=32) == L.TTT_ERR_UNSUPPORTED
    assert call(0, 3, 48) == L.TTT_OK                       # no units: nothing to do


def test_host_forward_workspace_size_and_argument_checks(lib):
    """ttt_fwd_host: the workspace query on the host, and every argument error
    (variant, chunks, workspace size and alignment, the forward's own rules)
    rejected before any copy or launch (fake pointers are never touched)."""
    ws_bytes = lib.ttt_fwd_host_workspace_bytes
    B, H, T, d = 2, 3, 64, 64
    n_ln = ws_bytes(L.TTT_VARIANT_LINEAR_LN, L.TTT_BF16, B, H, T, d, 0)
    # Q, K, V bf16, eta, Z, W_out, W0, gamma, beta, each rounded up to 256 bytes.
    up = lambda x: (x + 255) // 256 * 256
    elems = B * H * T * d
    expect = 3 * up(elems * 2) + up(B * H * T * 4) + up(elems * 4) + up(B * H * d * d * 4) + \
        up(H * d * d * 4) + 2 * up(H * d * 4)
    assert n_ln == expect
    assert ws_bytes(L.TTT_VARIANT_LINEAR, L.TTT_F32, B, H, T, d, 0) == \
        3 * up(elems * 4) + up(B * H * T * 4) + up(elems * 4) + up(B * H * d * d * 4) + up(H * d * d * 4)
    n_mlp = ws_bytes(L.TTT_VARIANT_MLP, L.TTT_BF16, B, H, T, d, 256)
    assert n_mlp == 3 * up(elems * 2) + up(B * H * T * 4) + up(elems * 4) + 2 * up(B * H * d * 256 * 4) + \
        2 * up(H * d * 256 * 4) + 2 * up(H * d * 4)
    assert ws_bytes(7, L.TTT_BF16, B, H, T, d, 0) == 0
    assert ws_bytes(L.TTT_VARIANT_LINEAR, 5, B, H, T, d, 0) == 0
    assert ws_bytes(L.TTT_VARIANT_MLP, L.TTT_BF16, B, H, T, d, 0) == 0
    assert ws_bytes(L.TTT_VARIANT_LINEAR, L.TTT_BF16, -1, H, T, d, 0) == 0

    p = _ptrs(12)
    ws = p[11] + (1 << 30)  # 256-byte aligned fake device address

    def call(variant=L.TTT_VARIANT_LINEAR_LN, B=B, T=T, b=16, chunks=4, wsp=ws, wsn=n_ln, eps=1e-6, g=p[6]):
        return lib.ttt_fwd_host(variant, p[0], p[1], p[2], L.TTT_BF16, p[3], p[4], None, g, p[7], eps,
                                B, H, T, d, 0, b, p[8], p[9], None, wsp, wsn, chunks, None)

    n0 = lib.ttt_launch_count()
    assert call(variant=9) == L.TTT_ERR_ARG
    assert call(chunks=0) == L.TTT_ERR_ARG
    assert call(wsp=None) == L.TTT_ERR_ARG
    assert call(wsn=n_ln - 1) == L.TTT_ERR_ARG
    assert call(wsp=ws + 16) == L.TTT_ERR_ALIGN
    assert call(T=40) == L.TTT_ERR_ARG                       # T % b != 0
    assert call(eps=0.0) == L.TTT_ERR_ARG
    assert call(g=None) == L.TTT_ERR_ARG                     # LN without gamma
    assert call(B=0) == L.TTT_OK                             # no units: nothing to do
    assert lib.ttt_launch_count() == n0, "a rejected call launched a kernel"
