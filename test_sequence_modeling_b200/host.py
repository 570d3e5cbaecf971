"""Host-resident inputs and outputs: the forward over batch chunks on three CUDA
streams, so that the copy of chunk i+1 to the device, the forward of chunk i and
the copy of chunk i-1 back overlap (the (batch, head) units are independent, and
a batch chunk is a contiguous slice of every [B, ...] tensor).

Every computation runs in the CUDA kernels of libttt.so through the binding in
``ttt``; this module only moves memory and orders streams.  Host tensors should be
pinned (``Tensor.pin_memory()``) for the copies to be asynchronous.
"""
from __future__ import annotations

import torch

from . import ttt


class HostForward:
    """Reusable device buffers and streams for one workload shape.

    ``variant`` is "linear", "linear_ln" or "mlp"; ``Q`` (any tensor of the
    [B, H, T, d] shape and dtype of the inputs), ``W_shapes`` (the per-unit shapes
    of the final states) and ``param_shapes`` (the per-head inputs) fix the
    buffers.  ``run`` takes host tensors and fills host outputs; it returns after
    enqueueing, with ``done`` (a CUDA event) recorded after the last copy back.
    """

    def __init__(self, variant, Q, W_shapes, param_shapes, chunks=4, device="cuda"):
        self.variant = variant
        self.device = torch.device(device)
        B, H, T, d = Q.shape
        self.B, self.chunks = B, max(1, min(chunks, B))
        bounds = [round(i * B / self.chunks) for i in range(self.chunks + 1)]
        self.slices = [(bounds[i], bounds[i + 1]) for i in range(self.chunks) if bounds[i + 1] > bounds[i]]
        dev = self.device
        self.d_qkv = [torch.empty(Q.shape, dtype=Q.dtype, device=dev) for _ in range(3)]
        self.d_eta = torch.empty(B, H, T, dtype=torch.float32, device=dev)
        self.d_Z = torch.empty(B, H, T, d, dtype=torch.float32, device=dev)
        self.d_W = [torch.empty((B,) + tuple(s), dtype=torch.float32, device=dev) for s in W_shapes]
        self.d_params = [torch.empty(tuple(s), dtype=torch.float32, device=dev) for s in param_shapes]
        self.s_in, self.s_run, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        self.done = torch.cuda.Event()

    def run(self, Q, K, V, eta, params, b, eps, Z, W_outs, after=None):
        """params: the per-head inputs on the host (W0; or W0, gamma, beta; or W1,
        W2, gamma, beta), copied with the first chunk.  Z, W_outs: host outputs.
        ``after``: an event the first copy waits for (the start of a timed region).
        The first copy also waits for the previous call's last copy back, so that
        back-to-back calls never overwrite device buffers still in use."""
        dq, dk, dv = self.d_qkv
        P = self.d_params
        for i, (b0, b1) in enumerate(self.slices):
            with torch.cuda.stream(self.s_in):
                if i == 0:
                    self.s_in.wait_event(self.done)  # no-op before the first call
                    if after is not None:
                        self.s_in.wait_event(after)
                    for dst, src in zip(self.d_params, params):
                        dst.copy_(src, non_blocking=True)
                for dst, src in ((dq, Q), (dk, K), (dv, V), (self.d_eta, eta)):
                    dst[b0:b1].copy_(src[b0:b1], non_blocking=True)
                loaded = torch.cuda.Event()
                loaded.record(self.s_in)
            self.s_run.wait_event(loaded)
            Zs, Ws = self.d_Z[b0:b1], [w[b0:b1] for w in self.d_W]
            args = (dq[b0:b1], dk[b0:b1], dv[b0:b1], self.d_eta[b0:b1])
            if self.variant == "linear":
                ttt.ttt_linear_fwd(*args, P[0], b, Z=Zs, W_out=Ws[0], stream=self.s_run)
            elif self.variant == "linear_ln":
                ttt.ttt_linear_ln_fwd(*args, P[0], P[1], P[2], b, eps, Z=Zs, W_out=Ws[0], stream=self.s_run)
            else:
                ttt.ttt_mlp_fwd(*args, P[0], P[1], P[2], P[3], b, eps, Z=Zs, W1_out=Ws[0], W2_out=Ws[1],
                                stream=self.s_run)
            computed = torch.cuda.Event()
            computed.record(self.s_run)
            self.s_out.wait_event(computed)
            with torch.cuda.stream(self.s_out):
                Z[b0:b1].copy_(Zs, non_blocking=True)
                for h, dw in zip(W_outs, Ws):
                    h[b0:b1].copy_(dw, non_blocking=True)
        self.done.record(self.s_out)
        return self.done
