"""``MoELayer``: the user-facing call of the routed MoE layer forward.

Holds the layer's weights (device tensors) and per-batch-size workspaces, and
runs the whole layer through the C ABI's ``moe_forward``.  All arithmetic
happens in the library's CUDA kernels.  ``forward_graphed`` /
``forward_host`` replay a CUDA graph of the layer captured once per batch size
(static input/output buffers), which removes the per-call launch cost that
dominates small decode batches.
"""

from __future__ import annotations

from typing import Dict, Optional

import torch

from . import binding as B


class _Graphed:
    """One captured layer call for a fixed T: static x / y buffers + graph."""

    def __init__(self, layer: "MoELayer", T: int):
        dev = layer.w13.device
        self.x = torch.zeros(T, layer.d, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(T, layer.d, dtype=torch.bfloat16, device=dev)
        self.ws = B.workspace(layer.shape(T), dev)
        shape = layer.shape(T)
        # One eager call first: first-use set-up (kernel attributes, driver
        # entry points) must not happen under capture.
        B.moe_forward(self.x, layer.w_g, layer.bias, layer.w13, layer.w2, self.y, shape,
                      self.ws)
        torch.cuda.current_stream(dev).synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            B.moe_forward(self.x, layer.w_g, layer.bias, layer.w13, layer.w2, self.y, shape,
                          self.ws)


class MoELayer:
    """Routed MoE layer: router W_g (d, E) fp32 [+ bias (E,)], experts w13
    (E, 2f, d) bf16 (gate rows then up rows) and w2 (E, d, f) bf16, top-k.
    ``R`` > 1 also computes the virtual expert-parallel layout."""

    def __init__(self, w_g: torch.Tensor, bias: Optional[torch.Tensor],
                 w13: torch.Tensor, w2: torch.Tensor, k: int, R: int = 0):
        B.load_library()
        self.w_g, self.bias, self.w13, self.w2 = w_g, bias, w13, w2
        self.d, self.E = int(w_g.shape[0]), int(w_g.shape[1])
        self.f = int(w2.shape[2])
        self.k, self.R = int(k), int(R)
        self._ws: Dict[int, torch.Tensor] = {}
        self._graphs: Dict[int, _Graphed] = {}
        self._last_ws: Optional[torch.Tensor] = None

    def shape(self, T: int) -> B.MoEShape:
        return B.MoEShape.of(T, self.d, self.E, self.k, self.f, self.R)

    def workspace(self, T: int) -> torch.Tensor:
        if T not in self._ws:
            self._ws[T] = B.workspace(self.shape(T), self.w13.device)
        return self._ws[T]

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                idx_out=None, w_out=None, counts_out=None, stream=None) -> torch.Tensor:
        """Eager call: y = MoE(x) for a device tensor x (T, d) bf16."""
        T = int(x.shape[0])
        y = out if out is not None else torch.empty_like(x)
        ws = self.workspace(T)
        self._last_ws = ws
        B.moe_forward(x, self.w_g, self.bias, self.w13, self.w2, y, self.shape(T), ws,
                      idx_out=idx_out, w_out=w_out, counts_out=counts_out, stream=stream)
        return y

    __call__ = forward

    def graphed(self, T: int) -> _Graphed:
        if T not in self._graphs:
            self._graphs[T] = _Graphed(self, T)
        return self._graphs[T]

    def forward_graphed(self, x: torch.Tensor, out: Optional[torch.Tensor] = None):
        """Copy x into the T-sized static buffer and replay the captured layer.
        Returns ``out`` (filled) or the static output buffer."""
        g = self.graphed(int(x.shape[0]))
        g.x.copy_(x, non_blocking=True)
        g.graph.replay()
        self._last_ws = g.ws
        if out is not None:
            out.copy_(g.y, non_blocking=True)
            return out
        return g.y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor) -> torch.Tensor:
        """Host-to-host call: pinned x (T, d) in, pinned y (T, d) out.  The
        copies and the graph replay are queued on the current stream; the
        caller synchronises before reading y_host."""
        g = self.graphed(int(x_host.shape[0]))
        g.x.copy_(x_host, non_blocking=True)
        g.graph.replay()
        y_host.copy_(g.y, non_blocking=True)
        self._last_ws = g.ws
        return y_host

    def check(self, stream=None) -> int:
        """Synchronises and returns (and clears) the last call's error word."""
        return B.moe_check(self._last_ws, stream) if self._last_ws is not None else B.MOE_OK
