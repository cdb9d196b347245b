"""Thin ctypes binding of ``libmoe_b200.so`` (the C ABI in ``include/moe.h``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (PyTorch supplies device memory and
streams; the layer calls' y and moe_copy's operands may also be pinned host
tensors); the functions keep the C names and raise :class:`MoEError` on a
non-zero status.  There is no fallback: if the library is missing or the
device is not an sm_100 GPU, calls raise.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_NAME = "libmoe_b200.so"
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), LIB_NAME)

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_TIMEOUT = 4
MOE_ERR_DEVICE_CHECK = 5

# Every symbol include/moe.h declares.
EXPORTS = ("moe_error_string", "moe_version", "moe_workspace_size", "moe_router",
           "moe_topk", "moe_dispatch", "moe_ffn", "moe_combine", "moe_forward",
           "moe_forward_staged", "moe_selftest_bounded_wait", "moe_check",
           "moe_dispatch_noalloc", "moe_eplb_plan", "moe_eplb_remap",
           "moe_workspace_size_eplb", "moe_forward_eplb", "moe_dispatch_dedup",
           "moe_ffn_fp8", "moe_forward_fp8", "moe_forward_fp8_staged", "moe_ep_recv_experts",
           "moe_ffn_w8a8", "moe_forward_w8a8", "moe_forward_w8a8_staged",
           "moe_quantise_rows_e4m3", "moe_copy")


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {moe_error_string(status)}")


class MoEShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("f", ctypes.c_int32), ("R", ctypes.c_int32)]

    @classmethod
    def of(cls, T, d, E, k, f, R=0) -> "MoEShape":
        return cls(int(T), int(d), int(E), int(k), int(f), int(R))

    @classmethod
    def from_config(cls, cfg) -> "MoEShape":
        return cls.of(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.R)


_lib = None
_P = ctypes.c_void_p
_S = ctypes.POINTER(MoEShape)


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads the library once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{LIB_NAME} is not built (expected at {path}); run "
            "`python -m routing_dispatch_expert_softmax_b200.build`")
    lib = ctypes.CDLL(path)
    lib.moe_error_string.restype = ctypes.c_char_p
    lib.moe_error_string.argtypes = [ctypes.c_int]
    lib.moe_version.restype = ctypes.c_int
    lib.moe_version.argtypes = []
    lib.moe_workspace_size.restype = ctypes.c_size_t
    lib.moe_workspace_size.argtypes = [_S]
    lib.moe_router.restype = ctypes.c_int
    lib.moe_router.argtypes = [_P, _P, _P, _S, _P, _P, _P]
    lib.moe_topk.restype = ctypes.c_int
    lib.moe_topk.argtypes = [_P, _S, _P, _P, _P]
    lib.moe_dispatch.restype = ctypes.c_int
    lib.moe_dispatch.argtypes = [_P, _P, _S, _P, _P, _P, _P, _P, _P, _P, _P, _P]
    lib.moe_ffn.restype = ctypes.c_int
    lib.moe_ffn.argtypes = [_P, _P, _P, _P, _S, _P, _P, _P]
    lib.moe_combine.restype = ctypes.c_int
    lib.moe_combine.argtypes = [_P, _P, _P, _S, _P, _P]
    lib.moe_forward.restype = ctypes.c_int
    lib.moe_forward.argtypes = [_P, _P, _P, _P, _P, _S, _P, _P, _P, _P, _P, _P]
    lib.moe_forward_staged.restype = ctypes.c_int
    lib.moe_forward_staged.argtypes = [_P, _P, _P, _P, _P, _S, _P, _P, _P, _P]
    lib.moe_dispatch_noalloc.restype = ctypes.c_int
    lib.moe_dispatch_noalloc.argtypes = [_P, _P, _S, _P, _P, _P, _P, _P, _P, _P, _P]
    lib.moe_check.restype = ctypes.c_int
    lib.moe_check.argtypes = [_P, _P]
    lib.moe_selftest_bounded_wait.restype = ctypes.c_int
    lib.moe_selftest_bounded_wait.argtypes = [ctypes.c_longlong, _P, _P]
    _i32 = ctypes.c_int32
    lib.moe_eplb_plan.restype = ctypes.c_int
    lib.moe_eplb_plan.argtypes = [_P, _i32, _i32, _i32, _P, _P, _P]
    lib.moe_eplb_remap.restype = ctypes.c_int
    lib.moe_eplb_remap.argtypes = [_P, _S, _P, _P, _i32, _P, _P, _P]
    lib.moe_workspace_size_eplb.restype = ctypes.c_size_t
    lib.moe_workspace_size_eplb.argtypes = [_S, _i32]
    lib.moe_dispatch_dedup.restype = ctypes.c_int
    lib.moe_dispatch_dedup.argtypes = [_P, _P, _S, _P, _P, _P, _P, _P, _P, _P, _P]
    lib.moe_ep_recv_experts.restype = ctypes.c_int
    lib.moe_ep_recv_experts.argtypes = [_P, _i32, _i32, _i32, _P, _P]
    lib.moe_forward_eplb.restype = ctypes.c_int
    lib.moe_forward_eplb.argtypes = [_P, _P, _P, _P, _P, _S, _P, _P, _i32, _P, _P, _P, _P,
                                     _P, _P]
    lib.moe_ffn_fp8.restype = ctypes.c_int
    lib.moe_ffn_fp8.argtypes = [_P, _P, _P, _P, _P, _P, _S, _P, _P, _P]
    lib.moe_forward_fp8.restype = ctypes.c_int
    lib.moe_forward_fp8.argtypes = [_P, _P, _P, _P, _P, _P, _P, _S, _P, _P, _P, _P, _P, _P]
    lib.moe_forward_fp8_staged.restype = ctypes.c_int
    lib.moe_forward_fp8_staged.argtypes = [_P, _P, _P, _P, _P, _P, _P, _S, _P, _P, _P, _P]
    lib.moe_ffn_w8a8.restype = ctypes.c_int
    lib.moe_ffn_w8a8.argtypes = [_P, _P, _P, _P, _P, _P, _S, _P, _P, _P]
    lib.moe_forward_w8a8.restype = ctypes.c_int
    lib.moe_forward_w8a8.argtypes = [_P, _P, _P, _P, _P, _P, _P, _S, _P, _P, _P, _P, _P, _P]
    lib.moe_forward_w8a8_staged.restype = ctypes.c_int
    lib.moe_forward_w8a8_staged.argtypes = [_P, _P, _P, _P, _P, _P, _P, _S, _P, _P, _P, _P]
    lib.moe_quantise_rows_e4m3.restype = ctypes.c_int
    lib.moe_quantise_rows_e4m3.argtypes = [_P, ctypes.c_int64, ctypes.c_int32, _P, _P, _P]
    lib.moe_copy.restype = ctypes.c_int
    lib.moe_copy.argtypes = [_P, _P, ctypes.c_int64, _P]
    _lib = lib
    return lib


def moe_error_string(status: int) -> str:
    return load_library().moe_error_string(int(status)).decode()


def moe_version() -> int:
    return load_library().moe_version()


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _ptr_dev_or_pinned(t: Optional[torch.Tensor], dtype=None, name="tensor"):
    """A CUDA tensor, or a page-locked CPU tensor the device addresses
    directly (the calls that accept host memory check it again)."""
    if isinstance(t, torch.Tensor) and t.device.type == "cpu":
        if not t.is_pinned():
            raise ValueError(f"{name} must be a CUDA tensor or page-locked (pinned) host memory")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return ctypes.c_void_p(t.data_ptr())
    return _ptr(t, dtype, name)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(stream.cuda_stream))


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


def moe_workspace_size(shape: MoEShape) -> int:
    return int(load_library().moe_workspace_size(ctypes.byref(shape)))


def workspace(shape: MoEShape, device="cuda") -> torch.Tensor:
    """A zeroed uint8 workspace of moe_workspace_size(shape) bytes (torch's
    allocator returns 512-byte aligned blocks, above the 256 required)."""
    n = moe_workspace_size(shape)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_router(x, w_g, bias, logits, shape: MoEShape, ws, stream=None):
    _check(load_library().moe_router(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_g, torch.float32, "w_g"),
        _ptr(bias, torch.float32, "bias"), ctypes.byref(shape),
        _ptr(logits, torch.float32, "logits"), _ptr(ws, torch.uint8, "ws"), _stream(stream)),
        "moe_router")


def moe_topk(logits, idx, w, shape: MoEShape, stream=None):
    _check(load_library().moe_topk(
        _ptr(logits, torch.float32, "logits"), ctypes.byref(shape),
        _ptr(idx, torch.int32, "idx"), _ptr(w, torch.float32, "w"), _stream(stream)),
        "moe_topk")


def moe_dispatch(idx, x, counts, offsets, perm, row_of, x_perm, shape: MoEShape, ws,
                 send_counts=None, rank_offsets=None, stream=None):
    _check(load_library().moe_dispatch(
        _ptr(idx, torch.int32, "idx"), _ptr(x, torch.bfloat16, "x"), ctypes.byref(shape),
        _ptr(counts, torch.int32, "counts"), _ptr(offsets, torch.int32, "offsets"),
        _ptr(perm, torch.int32, "perm"), _ptr(row_of, torch.int32, "row_of"),
        _ptr(x_perm, torch.bfloat16, "x_perm"),
        _ptr(send_counts, torch.int32, "send_counts"),
        _ptr(rank_offsets, torch.int32, "rank_offsets"),
        _ptr(ws, torch.uint8, "ws"), _stream(stream)), "moe_dispatch")


def moe_dispatch_noalloc(idx, x, counts, offsets, perm, row_of, x_perm, shape: MoEShape,
                         send_counts=None, rank_offsets=None, stream=None):
    """moe_dispatch for callers that cannot allocate: the scratch is the
    library's own fixed device array, so no workspace is passed (calls must
    not overlap on the GPU)."""
    _check(load_library().moe_dispatch_noalloc(
        _ptr(idx, torch.int32, "idx"), _ptr(x, torch.bfloat16, "x"), ctypes.byref(shape),
        _ptr(counts, torch.int32, "counts"), _ptr(offsets, torch.int32, "offsets"),
        _ptr(perm, torch.int32, "perm"), _ptr(row_of, torch.int32, "row_of"),
        _ptr(x_perm, torch.bfloat16, "x_perm"),
        _ptr(send_counts, torch.int32, "send_counts"),
        _ptr(rank_offsets, torch.int32, "rank_offsets"), _stream(stream)),
        "moe_dispatch_noalloc")


def moe_ffn(x_perm, offsets, w13, w2, z, shape: MoEShape, ws, stream=None):
    _check(load_library().moe_ffn(
        _ptr(x_perm, torch.bfloat16, "x_perm"), _ptr(offsets, torch.int32, "offsets"),
        _ptr(w13, torch.bfloat16, "w13"), _ptr(w2, torch.bfloat16, "w2"),
        ctypes.byref(shape), _ptr(z, torch.bfloat16, "z"), _ptr(ws, torch.uint8, "ws"),
        _stream(stream)), "moe_ffn")


def moe_combine(z, row_of, w, y, shape: MoEShape, stream=None):
    _check(load_library().moe_combine(
        _ptr(z, torch.bfloat16, "z"), _ptr(row_of, torch.int32, "row_of"),
        _ptr(w, torch.float32, "w"), ctypes.byref(shape), _ptr(y, torch.bfloat16, "y"),
        _stream(stream)), "moe_combine")


def moe_forward(x, w_g, bias, w13, w2, y, shape: MoEShape, ws, idx_out=None, w_out=None,
                counts_out=None, stream=None):
    _check(load_library().moe_forward(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_g, torch.float32, "w_g"),
        _ptr(bias, torch.float32, "bias"), _ptr(w13, torch.bfloat16, "w13"),
        _ptr(w2, torch.bfloat16, "w2"), ctypes.byref(shape),
        _ptr_dev_or_pinned(y, torch.bfloat16, "y"),
        _ptr(idx_out, torch.int32, "idx_out"), _ptr(w_out, torch.float32, "w_out"),
        _ptr(counts_out, torch.int32, "counts_out"), _ptr(ws, torch.uint8, "ws"),
        _stream(stream)), "moe_forward")


def moe_dispatch_dedup(idx, x, send_counts, rank_offsets, token_of, slot_mask, shape: MoEShape,
                       ws, rank_row_of=None, x_dedup=None, stream=None):
    """Token-deduplicated per-rank dispatch (uint32 slot masks are passed as
    int32 tensors of the same bits)."""
    _check(load_library().moe_dispatch_dedup(
        _ptr(idx, torch.int32, "idx"), _ptr(x, torch.bfloat16, "x"), ctypes.byref(shape),
        _ptr(send_counts, torch.int32, "send_counts"),
        _ptr(rank_offsets, torch.int32, "rank_offsets"), _ptr(token_of, torch.int32, "token_of"),
        _ptr(slot_mask, torch.int32, "slot_mask"), _ptr(rank_row_of, torch.int32, "rank_row_of"),
        _ptr(x_dedup, torch.bfloat16, "x_dedup"), _ptr(ws, torch.uint8, "ws"),
        _stream(stream)), "moe_dispatch_dedup")


def moe_ep_recv_experts(recv_counts, R: int, E_loc: int, N: int, expert_of_row, stream=None):
    """Local expert of each row an expert-parallel rank received (rows ordered
    by source rank, then local expert)."""
    _check(load_library().moe_ep_recv_experts(
        _ptr(recv_counts, torch.int32, "recv_counts"), int(R), int(E_loc), int(N),
        _ptr(expert_of_row, torch.int32, "expert_of_row"), _stream(stream)),
        "moe_ep_recv_experts")


def moe_eplb_plan(load, E: int, R: int, n_redundant: int):
    """Replica plan on the host: returns (phys_to_logical, rep_offsets,
    rep_phys) as int32 CPU tensors.  ``load``: E per-expert loads."""
    load = torch.as_tensor(load, dtype=torch.int64).contiguous()
    if load.device.type != "cpu" or load.numel() != E:
        raise ValueError("load: E int64 values on the host")
    P = E + n_redundant
    p2l = torch.empty(max(P, 1), dtype=torch.int32)
    off = torch.empty(E + 1, dtype=torch.int32)
    phys = torch.empty(max(P, 1), dtype=torch.int32)
    _check(load_library().moe_eplb_plan(load.data_ptr(), E, R, n_redundant, p2l.data_ptr(),
                                        off.data_ptr(), phys.data_ptr()), "moe_eplb_plan")
    return p2l[:P], off, phys[:P]


def moe_eplb_remap(idx, rep_offsets, rep_phys, E_phys: int, idx_phys, shape: MoEShape, ws,
                   stream=None):
    _check(load_library().moe_eplb_remap(
        _ptr(idx, torch.int32, "idx"), ctypes.byref(shape),
        _ptr(rep_offsets, torch.int32, "rep_offsets"), _ptr(rep_phys, torch.int32, "rep_phys"),
        E_phys, _ptr(idx_phys, torch.int32, "idx_phys"), _ptr(ws, torch.uint8, "ws"),
        _stream(stream)), "moe_eplb_remap")


def moe_workspace_size_eplb(shape: MoEShape, E_phys: int) -> int:
    return int(load_library().moe_workspace_size_eplb(ctypes.byref(shape), E_phys))


def workspace_eplb(shape: MoEShape, E_phys: int, device="cuda") -> torch.Tensor:
    n = moe_workspace_size_eplb(shape, E_phys)
    if n == 0:
        raise ValueError("invalid shape or E_phys for moe_forward_eplb")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_forward_eplb(x, w_g, bias, w13_phys, w2_phys, y, shape: MoEShape, rep_offsets,
                     rep_phys, E_phys: int, ws, idx_out=None, w_out=None, counts_out=None,
                     stream=None):
    _check(load_library().moe_forward_eplb(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_g, torch.float32, "w_g"),
        _ptr(bias, torch.float32, "bias"), _ptr(w13_phys, torch.bfloat16, "w13_phys"),
        _ptr(w2_phys, torch.bfloat16, "w2_phys"), ctypes.byref(shape),
        _ptr(rep_offsets, torch.int32, "rep_offsets"), _ptr(rep_phys, torch.int32, "rep_phys"),
        E_phys, _ptr(y, torch.bfloat16, "y"), _ptr(idx_out, torch.int32, "idx_out"),
        _ptr(w_out, torch.float32, "w_out"), _ptr(counts_out, torch.int32, "counts_out"),
        _ptr(ws, torch.uint8, "ws"), _stream(stream)), "moe_forward_eplb")


MOE_STAGE_EVENTS = 6
STAGE_NAMES = ("router", "topk+dispatch+gather", "expert GEMM1+SwiGLU",
               "expert GEMM2", "combine")


def _event_handle(ev) -> int:
    try:
        return int(ev.cuda_event)
    except Exception:
        return 0


def _event_array(events, st):
    if len(events) != MOE_STAGE_EVENTS:
        raise ValueError(f"need {MOE_STAGE_EVENTS} events")
    handles = []
    for ev in events:
        if ev is None:
            handles.append(None)
            continue
        if not _event_handle(ev):
            ev.record(st)  # torch creates the CUDA event at its first record
        handles.append(ctypes.c_void_p(_event_handle(ev)))
    return (ctypes.c_void_p * MOE_STAGE_EVENTS)(*handles)


def moe_forward_staged(x, w_g, bias, w13, w2, y, shape: MoEShape, ws, events, stream=None):
    """``events``: MOE_STAGE_EVENTS torch.cuda.Event objects (or None entries)
    recorded at the stage boundaries on the launch stream."""
    st = torch.cuda.current_stream() if stream is None else stream
    arr = _event_array(events, st)
    _check(load_library().moe_forward_staged(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_g, torch.float32, "w_g"),
        _ptr(bias, torch.float32, "bias"), _ptr(w13, torch.bfloat16, "w13"),
        _ptr(w2, torch.bfloat16, "w2"), ctypes.byref(shape), _ptr(y, torch.bfloat16, "y"),
        _ptr(ws, torch.uint8, "ws"), arr, _stream(st)), "moe_forward_staged")


def moe_ffn_fp8(x_perm, offsets, w13, w13_scale, w2, w2_scale, z, shape: MoEShape, ws,
                stream=None):
    """Expert FFNs with E4M3 expert weights (uint8 codes) and fp32 row scales."""
    _check(load_library().moe_ffn_fp8(
        _ptr(x_perm, torch.bfloat16, "x_perm"), _ptr(offsets, torch.int32, "offsets"),
        _ptr(w13, torch.uint8, "w13"), _ptr(w13_scale, torch.float32, "w13_scale"),
        _ptr(w2, torch.uint8, "w2"), _ptr(w2_scale, torch.float32, "w2_scale"),
        ctypes.byref(shape), _ptr(z, torch.bfloat16, "z"), _ptr(ws, torch.uint8, "ws"),
        _stream(stream)), "moe_ffn_fp8")


def moe_forward_fp8(x, w_g, bias, w13, w13_scale, w2, w2_scale, y, shape: MoEShape, ws,
                    idx_out=None, w_out=None, counts_out=None, stream=None):
    """The whole layer with E4M3 expert weights and fp32 row scales."""
    _check(load_library().moe_forward_fp8(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_g, torch.float32, "w_g"),
        _ptr(bias, torch.float32, "bias"), _ptr(w13, torch.uint8, "w13"),
        _ptr(w13_scale, torch.float32, "w13_scale"), _ptr(w2, torch.uint8, "w2"),
        _ptr(w2_scale, torch.float32, "w2_scale"), ctypes.byref(shape),
        _ptr_dev_or_pinned(y, torch.bfloat16, "y"), _ptr(idx_out, torch.int32, "idx_out"),
        _ptr(w_out, torch.float32, "w_out"), _ptr(counts_out, torch.int32, "counts_out"),
        _ptr(ws, torch.uint8, "ws"), _stream(stream)), "moe_forward_fp8")


def moe_ffn_w8a8(x_perm, offsets, w13, w13_scale, w2, w2_scale, z, shape: MoEShape, ws,
                 stream=None):
    """Expert FFNs with E4M3 weights and E4M3 activations (the rows of x_perm
    and the SwiGLU output quantised with power-of-two row scales)."""
    _check(load_library().moe_ffn_w8a8(
        _ptr(x_perm, torch.bfloat16, "x_perm"), _ptr(offsets, torch.int32, "offsets"),
        _ptr(w13, torch.uint8, "w13"), _ptr(w13_scale, torch.float32, "w13_scale"),
        _ptr(w2, torch.uint8, "w2"), _ptr(w2_scale, torch.float32, "w2_scale"),
        ctypes.byref(shape), _ptr(z, torch.bfloat16, "z"), _ptr(ws, torch.uint8, "ws"),
        _stream(stream)), "moe_ffn_w8a8")


def moe_forward_w8a8(x, w_g, bias, w13, w13_scale, w2, w2_scale, y, shape: MoEShape, ws,
                     idx_out=None, w_out=None, counts_out=None, stream=None):
    """The whole layer with E4M3 expert weights and E4M3 activations."""
    _check(load_library().moe_forward_w8a8(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_g, torch.float32, "w_g"),
        _ptr(bias, torch.float32, "bias"), _ptr(w13, torch.uint8, "w13"),
        _ptr(w13_scale, torch.float32, "w13_scale"), _ptr(w2, torch.uint8, "w2"),
        _ptr(w2_scale, torch.float32, "w2_scale"), ctypes.byref(shape),
        _ptr_dev_or_pinned(y, torch.bfloat16, "y"), _ptr(idx_out, torch.int32, "idx_out"),
        _ptr(w_out, torch.float32, "w_out"), _ptr(counts_out, torch.int32, "counts_out"),
        _ptr(ws, torch.uint8, "ws"), _stream(stream)), "moe_forward_w8a8")


def moe_forward_w8a8_staged(x, w_g, bias, w13, w13_scale, w2, w2_scale, y, shape: MoEShape,
                            ws, events, stream=None):
    """moe_forward_w8a8 with the stage events of moe_forward_staged."""
    st = torch.cuda.current_stream() if stream is None else stream
    arr = _event_array(events, st)
    _check(load_library().moe_forward_w8a8_staged(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_g, torch.float32, "w_g"),
        _ptr(bias, torch.float32, "bias"), _ptr(w13, torch.uint8, "w13"),
        _ptr(w13_scale, torch.float32, "w13_scale"), _ptr(w2, torch.uint8, "w2"),
        _ptr(w2_scale, torch.float32, "w2_scale"), ctypes.byref(shape),
        _ptr(y, torch.bfloat16, "y"), _ptr(ws, torch.uint8, "ws"), arr, _stream(st)),
        "moe_forward_w8a8_staged")


def moe_quantise_rows_e4m3(a, codes, scales, stream=None):
    """E4M3 codes (uint8, a's shape) and power-of-two row scales (fp32) of a
    2-D bf16 tensor."""
    rows, cols = int(a.shape[0]), int(a.shape[1])
    _check(load_library().moe_quantise_rows_e4m3(
        _ptr(a, torch.bfloat16, "a"), rows, cols, _ptr(codes, torch.uint8, "codes"),
        _ptr(scales, torch.float32, "scales"), _stream(stream)), "moe_quantise_rows_e4m3")


def moe_copy(dst, src, stream=None):
    """Copies src's bytes into dst by a library kernel (either may be a pinned
    host tensor); a multiple of 16 bytes, 16-byte aligned."""
    nbytes = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() < nbytes:
        raise ValueError("dst is smaller than src")
    _check(load_library().moe_copy(_ptr_dev_or_pinned(dst, None, "dst"),
                                   _ptr_dev_or_pinned(src, None, "src"), nbytes,
                                   _stream(stream)), "moe_copy")


def moe_forward_fp8_staged(x, w_g, bias, w13, w13_scale, w2, w2_scale, y, shape: MoEShape, ws,
                           events, stream=None):
    """moe_forward_fp8 with the stage events of moe_forward_staged."""
    st = torch.cuda.current_stream() if stream is None else stream
    arr = _event_array(events, st)
    _check(load_library().moe_forward_fp8_staged(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_g, torch.float32, "w_g"),
        _ptr(bias, torch.float32, "bias"), _ptr(w13, torch.uint8, "w13"),
        _ptr(w13_scale, torch.float32, "w13_scale"), _ptr(w2, torch.uint8, "w2"),
        _ptr(w2_scale, torch.float32, "w2_scale"), ctypes.byref(shape),
        _ptr(y, torch.bfloat16, "y"), _ptr(ws, torch.uint8, "ws"), arr, _stream(st)),
        "moe_forward_fp8_staged")


def moe_selftest_bounded_wait(limit_ns: int, ws, stream=None):
    _check(load_library().moe_selftest_bounded_wait(
        int(limit_ns), _ptr(ws, torch.uint8, "ws"), _stream(stream)),
        "moe_selftest_bounded_wait")


def moe_check(ws, stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error word."""
    return int(load_library().moe_check(_ptr(ws, torch.uint8, "ws"), _stream(stream)))
