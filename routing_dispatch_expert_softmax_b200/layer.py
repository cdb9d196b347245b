"""``MoELayer``: the user-facing call of the routed MoE layer forward.

Holds the layer's weights (device tensors) and per-batch-size workspaces, and
runs the whole layer through the C ABI's ``moe_forward`` (``moe_forward_eplb``
once ``rebalance`` has adopted a replica plan).  All arithmetic
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
        self.ws = layer._new_workspace(T)
        # One eager call first: first-use set-up (kernel attributes, driver
        # entry points) must not happen under capture.
        layer._call(self.x, self.y, self.ws)
        torch.cuda.current_stream(dev).synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            layer._call(self.x, self.y, self.ws)


class MoELayer:
    """Routed MoE layer: router W_g (d, E) fp32 [+ bias (E,)], experts w13
    (E, 2f, d) bf16 (gate rows then up rows) and w2 (E, d, f) bf16, top-k.
    ``R`` > 1 also computes the virtual expert-parallel layout.

    FP8 experts: pass w13 / w2 as uint8 E4M3 codes of the same shapes with
    ``w13_scale`` (E, 2f) and ``w2_scale`` (E, d) fp32 row scales; the layer
    then runs moe_forward_fp8 (batches of up to 256 tokens)."""

    def __init__(self, w_g: torch.Tensor, bias: Optional[torch.Tensor],
                 w13: torch.Tensor, w2: torch.Tensor, k: int, R: int = 0,
                 w13_scale: Optional[torch.Tensor] = None,
                 w2_scale: Optional[torch.Tensor] = None):
        B.load_library()
        if (w13_scale is None) != (w2_scale is None):
            raise ValueError("FP8 experts need both w13_scale and w2_scale")
        self.w_g, self.bias, self.w13, self.w2 = w_g, bias, w13, w2
        self.w13_scale, self.w2_scale = w13_scale, w2_scale
        self.fp8 = w13_scale is not None
        self.d, self.E = int(w_g.shape[0]), int(w_g.shape[1])
        self.f = int(w2.shape[2])
        self.k, self.R = int(k), int(R)
        self._ws: Dict[int, torch.Tensor] = {}
        self._graphs: Dict[int, _Graphed] = {}
        self._last_ws: Optional[torch.Tensor] = None
        self._eplb: Optional[dict] = None

    def shape(self, T: int) -> B.MoEShape:
        return B.MoEShape.of(T, self.d, self.E, self.k, self.f, self.R)

    def _new_workspace(self, T: int) -> torch.Tensor:
        if self._eplb is None:
            return B.workspace(self.shape(T), self.w13.device)
        return B.workspace_eplb(self.shape(T), self._eplb["E_phys"], self.w13.device)

    def workspace(self, T: int) -> torch.Tensor:
        if T not in self._ws:
            self._ws[T] = self._new_workspace(T)
        return self._ws[T]

    def _call(self, x, y, ws, idx_out=None, w_out=None, counts_out=None, stream=None):
        shape = self.shape(int(x.shape[0]))
        if self.fp8:
            B.moe_forward_fp8(x, self.w_g, self.bias, self.w13, self.w13_scale, self.w2,
                              self.w2_scale, y, shape, ws, idx_out=idx_out, w_out=w_out,
                              counts_out=counts_out, stream=stream)
        elif self._eplb is None:
            B.moe_forward(x, self.w_g, self.bias, self.w13, self.w2, y, shape, ws,
                          idx_out=idx_out, w_out=w_out, counts_out=counts_out, stream=stream)
        else:
            p = self._eplb
            B.moe_forward_eplb(x, self.w_g, self.bias, p["w13"], p["w2"], y, shape, p["off"],
                               p["phys"], p["E_phys"], ws, idx_out=idx_out, w_out=w_out,
                               counts_out=counts_out, stream=stream)

    def rebalance(self, load, n_redundant: int):
        """Adopt an EPLB-style replica plan built from per-expert ``load``
        (e.g. counts gathered over a window of calls): n_redundant extra
        copies of the busiest experts, placed on max(R, 1) virtual ranks.
        The physical weights are laid out once here; later calls run
        moe_forward_eplb, whose ``counts_out`` then has E + n_redundant
        entries (rows per physical expert).  Returns the plan
        (phys_to_logical, rep_offsets, rep_phys) as CPU int32 tensors."""
        if self.fp8:
            raise NotImplementedError("replica plans run on bf16 experts only")
        dev = self.w13.device
        p2l, off, phys = B.moe_eplb_plan(load, self.E, max(self.R, 1), n_redundant)
        sel = p2l.long().to(dev)
        self._eplb = dict(E_phys=self.E + int(n_redundant),
                          w13=self.w13.index_select(0, sel).contiguous(),
                          w2=self.w2.index_select(0, sel).contiguous(),
                          off=off.to(dev), phys=phys.to(dev))
        self._ws.clear()
        self._graphs.clear()
        return p2l, off, phys

    @property
    def physical_experts(self) -> int:
        return self.E if self._eplb is None else self._eplb["E_phys"]

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                idx_out=None, w_out=None, counts_out=None, stream=None) -> torch.Tensor:
        """Eager call: y = MoE(x) for a device tensor x (T, d) bf16."""
        T = int(x.shape[0])
        y = out if out is not None else torch.empty_like(x)
        ws = self.workspace(T)
        self._last_ws = ws
        self._call(x, y, ws, idx_out=idx_out, w_out=w_out, counts_out=counts_out,
                   stream=stream)
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
