"""``MoELayer``: the user-facing call of the routed MoE layer forward.

Holds the layer's weights (device tensors) and a workspace, and runs the
whole layer through the C ABI's ``moe_forward``.  All arithmetic happens in
the library's CUDA kernels.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


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
        self._ws = None
        self._ws_T = -1

    def shape(self, T: int) -> B.MoEShape:
        return B.MoEShape.of(T, self.d, self.E, self.k, self.f, self.R)

    def workspace(self, T: int) -> torch.Tensor:
        if self._ws is None or T > self._ws_T:
            self._ws = B.workspace(self.shape(T), self.w13.device)
            self._ws_T = T
        return self._ws

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                idx_out=None, w_out=None, counts_out=None, stream=None) -> torch.Tensor:
        T = int(x.shape[0])
        y = out if out is not None else torch.empty_like(x)
        # The workspace layout depends on T, so it is sized for this T.
        shape = self.shape(T)
        ws = self.workspace(T) if T == self._ws_T else self._fresh(T)
        B.moe_forward(x, self.w_g, self.bias, self.w13, self.w2, y, shape, ws,
                      idx_out=idx_out, w_out=w_out, counts_out=counts_out, stream=stream)
        return y

    def _fresh(self, T: int) -> torch.Tensor:
        self._ws = B.workspace(self.shape(T), self.w13.device)
        self._ws_T = T
        return self._ws

    __call__ = forward

    def check(self, stream=None) -> int:
        return B.moe_check(self._ws, stream) if self._ws is not None else B.MOE_OK
