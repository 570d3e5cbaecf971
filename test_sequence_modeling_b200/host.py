"""Host-resident inputs and outputs: a reusable device workspace and stream for
``ttt_fwd_host`` (C ABI), which copies batch chunks in, runs the forward and copies
them back with the copy of chunk i+1 in, the forward of chunk i and the copy of
chunk i-1 out overlapped (the (batch, head) units are independent, and a batch
chunk is a contiguous slice of every [B, ...] tensor).

Every computation and copy is enqueued by libttt.so; this module only allocates
the workspace and orders the call on its stream.  Host tensors should be pinned
(``Tensor.pin_memory()``) for the copies to be asynchronous.
"""
from __future__ import annotations

import torch

from . import ttt


class HostForward:
    """Device workspace and stream for one workload shape.

    ``variant`` is "linear", "linear_ln" or "mlp"; ``Q`` (any tensor of the
    [B, H, T, d] shape and dtype of the inputs) and ``hidden`` (TTT-MLP) fix the
    workspace size.  ``run`` takes host tensors and fills host outputs; it returns
    after enqueueing, with ``done`` (a CUDA event) recorded after the last copy back.
    """

    def __init__(self, variant, Q, W_shapes=None, param_shapes=None, chunks=4, device="cuda"):
        self.variant = variant
        self.device = torch.device(device)
        self.chunks = chunks
        hidden = tuple(W_shapes[0])[-1] if variant == "mlp" and W_shapes else 0
        nbytes = ttt.fwd_host_workspace_bytes(variant, tuple(Q.shape), Q.dtype, hidden)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.stream = torch.cuda.Stream(self.device)
        self.done = torch.cuda.Event()

    def run(self, Q, K, V, eta, params, b, eps, Z, W_outs, after=None):
        """params: the per-head inputs on the host (W0; or W0, gamma, beta; or W1,
        W2, gamma, beta).  Z, W_outs: host outputs.  ``after``: an event the call
        waits for (the start of a timed region).  Calls are ordered on this object's
        stream, so back-to-back calls never overwrite a workspace still in use."""
        if after is not None:
            self.stream.wait_event(after)
        ttt.ttt_fwd_host(self.variant, Q, K, V, eta, list(params), b, eps, Z, list(W_outs), self.workspace,
                         chunks=self.chunks, stream=self.stream)
        self.done.record(self.stream)
        return self.done
