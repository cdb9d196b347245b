"""moe_dispatch_noalloc: dispatch for callers that cannot allocate.

Some callers cannot hand the library a workspace: their device memory is a
fixed pool set up before serving starts, or they are a plugin that receives
its inputs and outputs and may not call an allocator.  moe_dispatch_noalloc
serves them by keeping its scratch in a fixed device array inside the
library.  These tests call it through the C ABI and check that its results
equal moe_dispatch's (which uses a caller workspace) and the oracle's on two
calls in a row, with different shapes, so the second call runs on the scratch
the first one left behind; routing tables and the gathered rows must match
bit for bit.  They also check that a warmed-up call changes neither the free
device memory nor PyTorch's allocation count, that an empty batch zeroes the
tables, and what an out-of-range expert id does (it is left out of the
counts, so offsets[E] comes out below T*k).

This file is collected last on purpose; it passes alone in a fresh process as
well as after the rest of the suite.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
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
        # and against the oracle's dispatch of the same ids
        idx_h = idx.cpu().numpy()
        ref_counts = oracle.expert_counts(idx_h, E)
        ref_perm, ref_row_of = oracle.dispatch_rows(idx_h, E)
        np.testing.assert_array_equal(got["counts"].cpu().numpy(), ref_counts)
        np.testing.assert_array_equal(got["offsets"].cpu().numpy(),
                                      oracle.expert_offsets(ref_counts))
        np.testing.assert_array_equal(got["perm"].cpu().numpy(), ref_perm)
        np.testing.assert_array_equal(got["row_of"].cpu().numpy(), ref_row_of)
        assert torch.equal(got["x_perm"], x[torch.from_numpy(ref_perm).long().to(DEV)])
        if R > 1:
            S, ro = oracle.virtual_ep_layout(idx_h, E, R)
            np.testing.assert_array_equal(got["send"].cpu().numpy(), S)
            np.testing.assert_array_equal(got["roff"].cpu().numpy(), ro)


def _noalloc(idx, x, out, shape):
    moe.moe_dispatch_noalloc(idx, x, out["counts"], out["offsets"], out["perm"],
                             out["row_of"], out["x_perm"], shape, out["send"], out["roff"])


def test_noalloc_dispatch_allocates_nothing():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    T, d, E, k, R = 256, 512, 64, 4, 4
    idx = _routing(T, E, k, 3).to(DEV)
    x = wl.make_hidden(wl.MoEConfig("x", T=T, d=d, E=E, k=k, f=64), DEV, 2)
    shape = MoEShape.of(T, d, E, k, 64, R)
    out = _outputs(T, d, E, k, R)
    _noalloc(idx, x, out, shape)  # warm-up: kernels loaded, scratch address looked up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    _noalloc(idx, x, out, shape)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0, (free0, free1)


def test_noalloc_dispatch_empty_batch_zeroes_tables():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    E, R = 16, 4
    shape = MoEShape.of(0, 64, E, 2, 64, R)
    counts = torch.full((E,), 5, dtype=torch.int32, device=DEV)
    offsets = torch.full((E + 1,), 5, dtype=torch.int32, device=DEV)
    send = torch.full((R, R), 5, dtype=torch.int32, device=DEV)
    roff = torch.full((R + 1,), 5, dtype=torch.int32, device=DEV)
    moe.moe_dispatch_noalloc(None, None, counts, offsets, None, None, None, shape, send, roff)
    torch.cuda.synchronize()
    for t in (counts, offsets, send, roff):
        assert int(t.abs().sum()) == 0


def test_noalloc_dispatch_leaves_out_of_range_ids_uncounted():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    T, d, E, k = 50, 64, 8, 2
    idx = _routing(T, E, k, 4)
    idx[7, 1] = E + 3  # out of range: never dereferenced, not counted
    shape = MoEShape.of(T, d, E, k, 64)
    x = wl.make_hidden(wl.MoEConfig("x", T=T, d=d, E=E, k=k, f=64), DEV, 1)
    out = _outputs(T, d, E, k, 0)
    _noalloc(idx.to(DEV), x, out, shape)
    torch.cuda.synchronize()
    valid = idx.numpy().reshape(-1)
    valid = valid[valid < E]
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), oracle.expert_counts(valid, E))
    assert int(out["offsets"][-1]) == T * k - 1
    torch.ones(1, device=DEV).sum().item()  # the context is still healthy


def test_noalloc_dispatch_rejects_shapes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = B.load_library()
    big = MoEShape.of(1 << 20, 64, 256, 8, 64, 0)
    p = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected before launch
    st = lib.moe_dispatch_noalloc(p, p, ctypes.byref(big), p, p, p, p, p, None, None, None)
    assert st == moe.MOE_ERR_UNSUPPORTED
    torch.ones(1, device=DEV).sum().item()
