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

import numpy as np
import torch

from . import binding as B


class LoadWindow:
    """Per-expert load over the last ``window`` layer calls, and the rule that
    decides when to re-plan the replicas.

    "vLLM Expert Parallel deployment" (EPLB section): the balancer works from
    the load of a window of recent steps (window_size) and re-plans at a fixed
    step interval (step_interval), adding a configured number of extra expert
    copies.  "Serving MoE models with expert parallelism on 8xH200", section
    "Routing imbalance": the imbalance factor is the busiest device's load over
    the mean, and about 1.3 is where acting pays.  Readings taken: a re-plan
    is considered every ``step_interval`` recorded calls, and adopted when the
    window's imbalance factor over the current placement exceeds
    ``threshold``; the window restarts after a re-plan (its counts described
    the old placement).

    Each call's per-(physical-)expert row counts are written by the layer's
    own routing kernel into one slot of a device ring of ``window`` rows (the
    ``counts_out`` of the layer call), so recording costs no extra work on the
    device; only a re-plan decision copies the ring to the host."""

    def __init__(self, n_experts: int, window: int, device):
        if window < 1:
            raise ValueError("window must be >= 1")
        self.window = int(window)
        self.ring = torch.zeros(self.window, int(n_experts), dtype=torch.int32, device=device)
        self.calls = 0

    def next_slot(self) -> torch.Tensor:
        """The ring row the next call writes its counts into."""
        slot = self.ring[self.calls % self.window]
        self.calls += 1
        return slot

    def reset(self, n_experts: Optional[int] = None):
        if n_experts is not None and n_experts != self.ring.shape[1]:
            self.ring = torch.zeros(self.window, int(n_experts), dtype=torch.int32,
                                    device=self.ring.device)
        else:
            self.ring.zero_()
        self.calls = 0

    def load(self) -> np.ndarray:
        """Rows per expert summed over the recorded calls in the window
        (int64, on the host)."""
        n = min(self.calls, self.window)
        return self.ring[:n].cpu().numpy().astype(np.int64).sum(axis=0)


def imbalance_factor(load, R: int) -> float:
    """Busiest rank's rows over the mean per rank, rank r owning experts
    [r*P/R, (r+1)*P/R) of the P entries of ``load`` ("Serving MoE models with
    expert parallelism on 8xH200", section "Routing imbalance")."""
    load = np.asarray(load, dtype=np.int64)
    R = max(int(R), 1)
    per = load.reshape(R, -1).sum(axis=1)
    mean = per.mean()
    return float(per.max() / mean) if mean > 0 else 0.0


class _Graphed:
    """One captured layer call for a fixed T: static x / y / counts buffers +
    graph."""

    def __init__(self, layer: "MoELayer", T: int):
        dev = layer.w13.device
        self.x = torch.zeros(T, layer.d, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(T, layer.d, dtype=torch.bfloat16, device=dev)
        self.counts = torch.zeros(layer.physical_experts, dtype=torch.int32, device=dev)
        self.ws = layer._new_workspace(T)
        # One eager call first: first-use set-up (kernel attributes, driver
        # entry points) must not happen under capture.
        layer._call(self.x, self.y, self.ws, counts_out=self.counts)
        torch.cuda.current_stream(dev).synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            layer._call(self.x, self.y, self.ws, counts_out=self.counts)


class _GraphedHost:
    """One captured host-to-host layer call for a fixed T and fixed page-locked
    x_host / y_host buffers: a library copy of x_host into a static device
    buffer, then the layer writing its result straight into y_host (the
    combine stores across the bus), with no copy-engine step on either side.
    Keeps references to both host buffers, whose addresses the graph holds."""

    def __init__(self, layer: "MoELayer", T: int, x_host: torch.Tensor, y_host: torch.Tensor):
        dev = layer.w13.device
        self.x_host, self.y_host = x_host, y_host
        self.x = torch.zeros(T, layer.d, dtype=torch.bfloat16, device=dev)
        self.counts = torch.zeros(layer.physical_experts, dtype=torch.int32, device=dev)
        self.ws = layer._new_workspace(T)
        layer._call_from_host(self.x, x_host, y_host, self.ws, self.counts)
        torch.cuda.current_stream(dev).synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            layer._call_from_host(self.x, x_host, y_host, self.ws, self.counts)


class MoELayer:
    """Routed MoE layer: router W_g (d, E) fp32 [+ bias (E,)], experts w13
    (E, 2f, d) bf16 (gate rows then up rows) and w2 (E, d, f) bf16, top-k.
    ``R`` > 1 also computes the virtual expert-parallel layout.

    FP8 experts: pass w13 / w2 as uint8 E4M3 codes of the same shapes with
    ``w13_scale`` (E, 2f) and ``w2_scale`` (E, d) fp32 row scales; the layer
    then runs moe_forward_fp8 (bf16 activations), or with
    ``fp8_activations=True`` moe_forward_w8a8 (activations quantised to E4M3
    too, both GEMM operands one byte)."""

    def __init__(self, w_g: torch.Tensor, bias: Optional[torch.Tensor],
                 w13: torch.Tensor, w2: torch.Tensor, k: int, R: int = 0,
                 w13_scale: Optional[torch.Tensor] = None,
                 w2_scale: Optional[torch.Tensor] = None,
                 fp8_activations: bool = False):
        B.load_library()
        if (w13_scale is None) != (w2_scale is None):
            raise ValueError("FP8 experts need both w13_scale and w2_scale")
        if fp8_activations and w13_scale is None:
            raise ValueError("FP8 activations need FP8 experts (w13_scale, w2_scale)")
        self.w_g, self.bias, self.w13, self.w2 = w_g, bias, w13, w2
        self.w13_scale, self.w2_scale = w13_scale, w2_scale
        self.fp8 = w13_scale is not None
        self.w8a8 = bool(fp8_activations)
        self.d, self.E = int(w_g.shape[0]), int(w_g.shape[1])
        self.f = int(w2.shape[2])
        self.k, self.R = int(k), int(R)
        self._ws: Dict[int, torch.Tensor] = {}
        self._graphs: Dict[int, _Graphed] = {}
        self._host_graphs: Dict[tuple, _GraphedHost] = {}
        self._host_refused: set = set()
        self._last_ws: Optional[torch.Tensor] = None
        self._eplb: Optional[dict] = None
        self._auto: Optional[dict] = None

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
            fwd = B.moe_forward_w8a8 if self.w8a8 else B.moe_forward_fp8
            fwd(x, self.w_g, self.bias, self.w13, self.w13_scale, self.w2, self.w2_scale, y,
                shape, ws, idx_out=idx_out, w_out=w_out, counts_out=counts_out, stream=stream)
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
                          off=off.to(dev), phys=phys.to(dev), p2l=p2l.numpy().astype(np.int64))
        self._ws.clear()
        self._graphs.clear()
        self._host_graphs.clear()
        return p2l, off, phys

    @property
    def physical_experts(self) -> int:
        return self.E if self._eplb is None else self._eplb["E_phys"]

    def enable_auto_rebalance(self, n_redundant: int, window: int = 1000,
                              step_interval: int = 3000, threshold: float = 1.3):
        """Keep a load window over the layer's calls and re-plan the replicas
        by it (see ``LoadWindow``): every ``step_interval`` calls, if the
        busiest of max(R, 1) ranks carries more than ``threshold`` times the
        mean rows of the window, adopt ``rebalance(load, n_redundant)``.
        The defaults are the example settings of the vLLM EPLB configuration
        and the ~1.3 of the routing-imbalance discussion."""
        if self.fp8:
            raise NotImplementedError("replica plans run on bf16 experts only")
        if step_interval < 1 or threshold < 1.0:
            raise ValueError("step_interval >= 1 and threshold >= 1 required")
        self._auto = dict(window=LoadWindow(self.physical_experts, window, self.w13.device),
                          n_redundant=int(n_redundant), step_interval=int(step_interval),
                          threshold=float(threshold), since=0, replans=0, last_factor=None)

    @property
    def load_window(self) -> Optional[LoadWindow]:
        return None if self._auto is None else self._auto["window"]

    def logical_load(self) -> np.ndarray:
        """The window's rows per logical expert (replicas summed)."""
        load = self._auto["window"].load()
        if self._eplb is None:
            return load
        out = np.zeros(self.E, dtype=np.int64)
        np.add.at(out, self._eplb["p2l"], load)
        return out

    def _after_call(self):
        """Counts one recorded call; at each interval decides on a re-plan."""
        a = self._auto
        a["since"] += 1
        if a["since"] < a["step_interval"]:
            return
        a["since"] = 0
        factor = imbalance_factor(a["window"].load(), max(self.R, 1))
        a["last_factor"] = factor
        if factor > a["threshold"]:
            self.rebalance(self.logical_load(), a["n_redundant"])
            a["replans"] += 1
            a["window"].reset(self.physical_experts)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                idx_out=None, w_out=None, counts_out=None, stream=None) -> torch.Tensor:
        """Eager call: y = MoE(x) for a device tensor x (T, d) bf16."""
        T = int(x.shape[0])
        y = out if out is not None else torch.empty_like(x)
        ws = self.workspace(T)
        self._last_ws = ws
        slot = self._auto["window"].next_slot() if self._auto is not None else None
        self._call(x, y, ws, idx_out=idx_out, w_out=w_out,
                   counts_out=slot if slot is not None else counts_out, stream=stream)
        if slot is not None:
            if counts_out is not None:
                counts_out.copy_(slot)
            self._after_call()
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
        self._record_graphed(g)
        if out is not None:
            out.copy_(g.y, non_blocking=True)
            return out
        return g.y

    # host-buffer graphs kept per layer (each holds a workspace)
    _MAX_HOST_GRAPHS = 8
    # the in-place path up to this many bytes per buffer; above it the copy
    # engines move x and y faster than the copy kernel and the combine's
    # stores across the bus (same-box A/B, us per step: T = 64 135 vs 141,
    # T = 256 244 vs 302, T = 1 46 vs 57; prefill T = 8192 1966 vs 1939)
    _HOST_DIRECT_MAX_BYTES = 4 << 20

    def _call_from_host(self, x_dev, x_host, y_host, ws, counts):
        B.moe_copy(x_dev, x_host)
        self._call(x_dev, y_host, ws, counts_out=counts)

    def _host_direct(self, x_host: torch.Tensor, y_host: torch.Tensor) -> bool:
        """Whether forward_host can read x_host and write y_host in place:
        page-locked, contiguous, 16-byte aligned bf16 buffers of at most
        _HOST_DIRECT_MAX_BYTES, and a layer call that accepts a host y (not
        the replica-plan path)."""
        ok = self._eplb is None and x_host.numel() * 2 <= self._HOST_DIRECT_MAX_BYTES
        for t in (x_host, y_host):
            ok = ok and (t.device.type == "cpu" and t.dtype == torch.bfloat16 and
                         t.is_contiguous() and t.is_pinned() and t.data_ptr() % 16 == 0)
        return ok and tuple(x_host.shape) == tuple(y_host.shape) == (x_host.shape[0], self.d)

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor) -> torch.Tensor:
        """Host-to-host call: pinned x (T, d) in, pinned y (T, d) out, queued
        on the current stream; the caller synchronises before reading
        y_host.  For page-locked buffers the captured graph starts with a
        library copy of x_host (chained to the router without a copy-engine
        step) and the combine writes y_host directly; graphs are kept per
        (T, x_host, y_host) buffer triple, the most recent few.  Other (and
        larger) buffers go through copies to and from a device-side graph."""
        T = int(x_host.shape[0])
        key = (T, x_host.data_ptr(), y_host.data_ptr())
        if key not in self._host_refused and self._host_direct(x_host, y_host):
            g = self._host_graphs.pop(key, None)
            if g is None:
                try:
                    g = _GraphedHost(self, T, x_host, y_host)
                except B.MoEError as err:
                    # the library refused a host buffer (before any launch or
                    # capture): these buffers take the copy path from now on
                    if err.status != B.MOE_ERR_INVALID_ARG:
                        raise
                    self._host_refused.add(key)
            if g is not None:
                self._host_graphs[key] = g  # most recent last
                while len(self._host_graphs) > self._MAX_HOST_GRAPHS:
                    self._host_graphs.pop(next(iter(self._host_graphs)))
                g.graph.replay()
                self._last_ws = g.ws
                self._record_graphed(g)
                return y_host
        g = self.graphed(T)
        g.x.copy_(x_host, non_blocking=True)
        g.graph.replay()
        y_host.copy_(g.y, non_blocking=True)
        self._last_ws = g.ws
        self._record_graphed(g)
        return y_host

    def _record_graphed(self, g: _Graphed):
        if self._auto is not None:
            self._auto["window"].next_slot().copy_(g.counts, non_blocking=True)
            self._after_call()

    def check(self, stream=None) -> int:
        """Synchronises and returns (and clears) the last call's error word."""
        return B.moe_check(self._last_ws, stream) if self._last_ws is not None else B.MOE_OK
