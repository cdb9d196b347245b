"""moe_dispatch_noalloc: dispatch for callers that cannot allocate.

Some callers cannot hand the library a workspace: their device memory is a
fixed pool set up before serving starts, or they are a plugin that receives
its inputs and outputs and may not call an allocator.  moe_dispatch_noalloc
serves them by keeping its scratch in a fixed device array inside the
library.  This test calls it through the C ABI and checks that its results
equal moe_dispatch's (which uses a caller workspace) on two calls in a row,
with different shapes, so the second call runs on the scratch the first one
left behind.  Routing tables and the gathered rows must match bit for bit.

This file is collected last on purpose; it passes alone in a fresh process as
well as after the rest of the suite.
"""

import ctypes

import numpy as np
import pytest
import torch

import routing_dispatch_expert_softmax_b200 as moe
from routing_dispatch_expert_softmax_b200 import binding as B
from routing_dispatch_expert_softmax_b200 import workloads as wl
from routing_dispatch_expert_softmax_b200.binding import MoEShape

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _outputs(T, d, E, k, R):
    z = lambda *s: torch.full(s, -3, dtype=torch.int32, device=DEV)
    return dict(counts=z(E), offsets=z(E + 1), perm=z(T * k), row_of=z(T, k),
                x_perm=torch.zeros(T * k, d, dtype=torch.bfloat16, device=DEV),
                send=z(R, R) if R > 1 else None, roff=z(R + 1) if R > 1 else None)


def _routing(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    L = torch.randn(T, E, generator=g)
    return torch.topk(L, k, dim=1).indices.to(torch.int32)  # distinct experts per token


@pytest.mark.parametrize("calls", [[(300, 256, 64, 8, 8), (64, 2048, 128, 8, 0)]])
def test_noalloc_dispatch_matches_workspace_dispatch(calls):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    for n, (T, d, E, k, R) in enumerate(calls):
        idx = _routing(T, E, k, 10 + n).to(DEV)
        x = wl.make_hidden(wl.MoEConfig("x", T=T, d=d, E=E, k=k, f=64), DEV, n)
        shape = MoEShape.of(T, d, E, k, 64, R)
        ref = _outputs(T, d, E, k, R)
        ws = moe.workspace(shape)
        moe.moe_dispatch(idx, x, ref["counts"], ref["offsets"], ref["perm"], ref["row_of"],
                         ref["x_perm"], shape, ws, ref["send"], ref["roff"])
        got = _outputs(T, d, E, k, R)
        moe.moe_dispatch_noalloc(idx, x, got["counts"], got["offsets"], got["perm"],
                                 got["row_of"], got["x_perm"], shape, got["send"], got["roff"])
        torch.cuda.synchronize()
        assert moe.moe_check(ws) == moe.MOE_OK
        for name in ref:
            if ref[name] is not None:
                assert torch.equal(got[name], ref[name]), (n, name)
        assert int(got["offsets"][-1]) == T * k


def test_noalloc_dispatch_rejects_shapes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = B.load_library()
    big = MoEShape.of(1 << 20, 64, 256, 8, 64, 0)
    p = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected before launch
    st = lib.moe_dispatch_noalloc(p, p, ctypes.byref(big), p, p, p, p, p, None, None, None)
    assert st == moe.MOE_ERR_UNSUPPORTED
    torch.ones(1, device=DEV).sum().item()
