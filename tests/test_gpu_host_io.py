"""Host-buffer input and output of the layer: moe_copy (a library kernel that
copies between device memory and page-locked host memory) and the layer calls
whose y is page-locked host memory (the combine writes it across the bus),
as MoELayer.forward_host uses them.  Every result is compared bit for bit with
the device-only path; pageable host memory is refused before any launch."""

import ctypes

import pytest
import torch

import routing_dispatch_expert_softmax_b200 as moe
from routing_dispatch_expert_softmax_b200 import binding as B
from routing_dispatch_expert_softmax_b200 import workloads as wl
from routing_dispatch_expert_softmax_b200.binding import MoEShape

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("nbytes", [16, 4096 + 16, 3 << 20])
def test_copy_between_device_and_pinned_host(nbytes):
    g = torch.Generator().manual_seed(nbytes)
    src_host = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=g).pin_memory()
    dev = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    dev2 = torch.empty_like(dev)
    back = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
    moe.moe_copy(dev, src_host)          # host -> device
    moe.moe_copy(dev2, dev)              # device -> device
    moe.moe_copy(back, dev2)             # device -> host
    torch.cuda.synchronize()
    assert torch.equal(dev.cpu(), src_host)
    assert torch.equal(back, src_host)


def test_pageable_host_memory_is_refused_before_any_launch():
    lib = B.load_library()
    pageable = torch.zeros(1024, dtype=torch.uint8)          # not page-locked
    addr = pageable.data_ptr() + (-pageable.data_ptr()) % 16
    dev = torch.zeros(1024, dtype=torch.uint8, device=DEV)
    st = ctypes.c_void_p(int(torch.cuda.current_stream().cuda_stream))
    assert lib.moe_copy(ctypes.c_void_p(dev.data_ptr()), ctypes.c_void_p(addr), 512,
                        st) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_copy(ctypes.c_void_p(addr), ctypes.c_void_p(dev.data_ptr()), 512,
                        st) == B.MOE_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.count_nonzero(pageable) == 0
    # the layer's y: a pageable host y is refused too
    cfg = wl.TINY
    t = wl.make_layer(cfg, DEV, 0)
    shape = MoEShape.from_config(cfg)
    y_pageable = torch.zeros(cfg.T * cfg.d + 16, dtype=torch.bfloat16)
    yaddr = y_pageable.data_ptr() + (-y_pageable.data_ptr()) % 16
    ws = moe.workspace(shape)
    p = lambda x: ctypes.c_void_p(x.data_ptr())
    status = lib.moe_forward(p(t["x"]), p(t["w_g"]), p(t["bias"]) if t["bias"] is not None
                             else None, p(t["w13"]), p(t["w2"]), ctypes.byref(shape),
                             ctypes.c_void_p(yaddr), None, None, None, p(ws), st)
    assert status == B.MOE_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.count_nonzero(y_pageable) == 0
    with pytest.raises(ValueError, match="pinned"):
        moe.moe_copy(dev, pageable)


@pytest.mark.parametrize("cfg", [wl.QWEN3_30B_A3B_DECODE.with_T(8),
                                 wl.QWEN3_30B_A3B_DECODE.with_T(64),
                                 wl.MoEConfig("host-ragged", T=37, d=320, E=6, k=3, f=128)],
                         ids=["T8", "T64", "ragged"])
def test_forward_with_pinned_y_equals_device_y(cfg):
    t = wl.make_layer(cfg, DEV, 0)
    shape = MoEShape.from_config(cfg)
    y_dev = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_forward(t["x"], t["w_g"], t["bias"], t["w13"], t["w2"], y_dev, shape,
                    moe.workspace(shape))
    y_host = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.bfloat16).pin_memory()
    moe.moe_forward(t["x"], t["w_g"], t["bias"], t["w13"], t["w2"], y_host, shape,
                    moe.workspace(shape))
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_dev.cpu())


def test_forward_host_direct_and_copy_paths_agree():
    """MoELayer.forward_host: page-locked buffers take the graph that copies
    x by a library kernel and writes y in place (one graph per buffer pair);
    pageable buffers take device copies; both give the eager call's bits, for
    the bf16 and the W8A8 layer, and a replay re-reads x_host."""
    cfg = wl.QWEN3_30B_A3B_DECODE.with_T(64)
    t = wl.make_layer(cfg, DEV, 0)
    layer = moe.MoELayer(t["w_g"], t["bias"], t["w13"], t["w2"], cfg.k)
    y_ref = layer(t["x"]).cpu()
    x_pinned = t["x"].cpu().pin_memory()
    y_pinned = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory()
    layer.forward_host(x_pinned, y_pinned)
    torch.cuda.synchronize()
    assert torch.equal(y_pinned, y_ref)
    assert len(layer._host_graphs) == 1
    x_page, y_page = t["x"].cpu(), torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16)
    layer.forward_host(x_page, y_page)
    torch.cuda.synchronize()
    assert torch.equal(y_page, y_ref)
    assert len(layer._host_graphs) == 1
    # new contents in the same pinned buffers: the graph reads them again
    x2 = wl.make_hidden(cfg, DEV, 7)
    y2_ref = layer(x2).cpu()
    x_pinned.copy_(x2.cpu())
    layer.forward_host(x_pinned, y_pinned)
    torch.cuda.synchronize()
    assert torch.equal(y_pinned, y2_ref)
    assert layer.check() == moe.MOE_OK
    # buffers above the in-place limit (4 MB each) keep the copy path
    big = 1100  # 1100 x 2048 bf16 = 4.5 MB
    x_big = torch.zeros(big, cfg.d, dtype=torch.bfloat16).pin_memory()
    assert not layer._host_direct(x_big, torch.empty_like(x_big).pin_memory())
    assert layer._host_direct(x_pinned, y_pinned)
    # the W8A8 layer
    from routing_dispatch_expert_softmax_b200 import workloads
    c13, s13, c2, s2 = workloads.make_experts_fp8(cfg, DEV, 0)
    layer8 = moe.MoELayer(t["w_g"], t["bias"], c13, c2, cfg.k, w13_scale=s13, w2_scale=s2,
                          fp8_activations=True)
    y8_ref = layer8(t["x"]).cpu()
    layer8.forward_host(x_pinned.copy_(t["x"].cpu()), y_pinned)
    torch.cuda.synchronize()
    assert torch.equal(y_pinned, y8_ref)
    assert layer8.check() == moe.MOE_OK
