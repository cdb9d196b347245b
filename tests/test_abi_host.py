"""Host-side tests of the C ABI: the library loads, exports every symbol the
header declares, sizes workspaces, and rejects bad arguments before any
launch.  None of these calls reaches a kernel, so they are safe anywhere."""

import ctypes
import os
import re

import pytest
import torch

import routing_dispatch_expert_softmax_b200 as moe
from routing_dispatch_expert_softmax_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    return B.load_library()


def _declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", src)))


def test_header_declares_what_the_binding_knows():
    assert _declared_functions() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_version_and_error_strings(lib):
    assert moe.moe_version() == 105
    for code in range(6):
        assert moe.moe_error_string(code).startswith("MOE_")
    assert "unknown" in moe.moe_error_string(99)


VALID = dict(T=64, d=256, E=8, k=2, f=512, R=0)


@pytest.mark.parametrize("bad", [
    dict(T=-1), dict(T=(1 << 20) + 1), dict(d=0), dict(d=96), dict(d=16448),
    dict(E=0), dict(E=1025), dict(k=0), dict(k=9), dict(k=33, E=64),
    dict(f=0), dict(f=100), dict(R=-1), dict(R=3), dict(R=65),
])
def test_workspace_size_rejects_invalid_shapes(lib, bad):
    s = dict(VALID, **bad)
    assert moe.moe_workspace_size(B.MoEShape.of(**s)) == 0


def test_workspace_size_grows_with_T(lib):
    sizes = [moe.moe_workspace_size(B.MoEShape.of(**dict(VALID, T=t))) for t in (0, 1, 64, 4096)]
    assert all(s > 0 for s in sizes)
    assert sizes == sorted(sizes)
    assert moe.moe_workspace_size(B.MoEShape.of(**dict(VALID, E=8, R=4))) > 0


def _raw(lib, name, *args):
    return getattr(lib, name)(*args)


def _P(v):
    return ctypes.c_void_p(v)


A16 = 1 << 20          # an aligned fake address (never dereferenced)
MIS = (1 << 20) + 2    # misaligned


def test_bad_arguments_are_rejected_before_launch(lib):
    s = ctypes.byref(B.MoEShape.of(**VALID))
    bad_shape = ctypes.byref(B.MoEShape.of(**dict(VALID, k=0)))
    INV = B.MOE_ERR_INVALID_ARG
    # moe_router: null / misaligned x, null logits, invalid shape
    assert _raw(lib, "moe_router", None, _P(A16), None, s, _P(A16), _P(A16), None) == INV
    assert _raw(lib, "moe_router", _P(MIS), _P(A16), None, s, _P(A16), _P(A16), None) == INV
    assert _raw(lib, "moe_router", _P(A16), _P(A16), None, s, None, _P(A16), None) == INV
    assert _raw(lib, "moe_router", _P(A16), _P(A16), None, s, _P(A16), None, None) == INV
    assert _raw(lib, "moe_router", _P(A16), _P(A16), None, bad_shape, _P(A16), _P(A16),
                None) == INV
    # moe_topk
    assert _raw(lib, "moe_topk", None, s, _P(A16), _P(A16), None) == INV
    assert _raw(lib, "moe_topk", _P(A16 + 1), s, _P(A16), _P(A16), None) == INV
    # moe_dispatch: send_counts without R > 1, misaligned workspace
    args = [_P(A16)] * 2
    assert _raw(lib, "moe_dispatch", *args, s, *[_P(A16)] * 5, _P(A16), None, _P(A16),
                None) == INV
    assert _raw(lib, "moe_dispatch", *args, s, *[_P(A16)] * 5, None, None, _P(A16 + 16),
                None) == INV
    # moe_ffn: misaligned weights, null workspace
    assert _raw(lib, "moe_ffn", _P(A16), _P(A16), _P(MIS), _P(A16), s, _P(A16), _P(A16),
                None) == INV
    assert _raw(lib, "moe_ffn", _P(A16), _P(A16), _P(A16), _P(A16), s, _P(A16), None,
                None) == INV
    # moe_combine
    assert _raw(lib, "moe_combine", _P(A16), None, _P(A16), s, _P(A16), None) == INV
    # moe_forward: null workspace, misaligned y
    assert _raw(lib, "moe_forward", *[_P(A16)] * 5, s, _P(A16), None, None, None, None,
                None) == INV
    assert _raw(lib, "moe_forward", *[_P(A16)] * 5, s, _P(MIS), None, None, None, _P(A16),
                None) == INV
    # self-test limits
    assert _raw(lib, "moe_selftest_bounded_wait", ctypes.c_longlong(0), _P(A16), None) == INV
    assert _raw(lib, "moe_selftest_bounded_wait", ctypes.c_longlong(2 * 10 ** 9), _P(A16),
                None) == INV
    assert _raw(lib, "moe_check", _P(A16 + 8), None) == INV
    # moe_copy: sizes not a multiple of 16, misaligned or null pointers
    assert _raw(lib, "moe_copy", _P(A16), _P(A16), ctypes.c_int64(24), None) == INV
    assert _raw(lib, "moe_copy", _P(A16), _P(A16), ctypes.c_int64(-16), None) == INV
    assert _raw(lib, "moe_copy", _P(A16 + 4), _P(A16), ctypes.c_int64(32), None) == INV
    assert _raw(lib, "moe_copy", None, _P(A16), ctypes.c_int64(32), None) == INV
    assert _raw(lib, "moe_copy", None, None, ctypes.c_int64(0), None) == B.MOE_OK
    # dedup dispatch: needs R >= 2 and a workspace
    s_r4 = ctypes.byref(B.MoEShape.of(**dict(VALID, R=4)))
    assert _raw(lib, "moe_dispatch_dedup", _P(A16), None, s, _P(A16), _P(A16), _P(A16),
                _P(A16), None, None, _P(A16), None) == INV
    assert _raw(lib, "moe_dispatch_dedup", _P(A16), None, s_r4, _P(A16), _P(A16), _P(A16),
                _P(A16), None, None, None, None) == INV
    assert _raw(lib, "moe_dispatch_dedup", _P(A16), None, s_r4, _P(A16), _P(A16), _P(A16),
                _P(A16), None, _P(A16), _P(A16), None) == INV   # x_dedup without x
    # EPLB: fewer physical than logical experts, misaligned plan, null workspace
    assert _raw(lib, "moe_eplb_remap", _P(A16), s, _P(A16), _P(A16), VALID["E"] - 1, _P(A16),
                _P(A16), None) == INV
    assert _raw(lib, "moe_eplb_remap", _P(A16), s, _P(A16 + 2), _P(A16), VALID["E"], _P(A16),
                _P(A16), None) == INV
    assert _raw(lib, "moe_forward_eplb", *[_P(A16)] * 5, s, _P(A16), _P(A16), VALID["E"] + 8,
                _P(A16), None, None, None, None, None) == INV
    assert _raw(lib, "moe_forward_eplb", *[_P(A16)] * 5, s, _P(A16), _P(A16), 1025,
                _P(A16), None, None, None, _P(A16), None) == INV


def test_fp8_calls_reject_before_launch(lib):
    s = ctypes.byref(B.MoEShape.of(**VALID))
    INV = B.MOE_ERR_INVALID_ARG
    ws = _P(A16)
    # moe_ffn_fp8(x_perm, offsets, w13, w13_scale, w2, w2_scale, s, z, ws, stream)
    assert _raw(lib, "moe_ffn_fp8", _P(A16), _P(A16), _P(A16), None, _P(A16), _P(A16), s,
                _P(A16), ws, None) == INV                       # null w13 scales
    assert _raw(lib, "moe_ffn_fp8", _P(A16), _P(A16), _P(A16 + 8), _P(A16), _P(A16), _P(A16),
                s, _P(A16), ws, None) == INV                    # codes not 16-byte aligned
    assert _raw(lib, "moe_ffn_fp8", _P(A16), _P(A16), _P(A16), _P(A16), _P(A16), _P(A16 + 2),
                s, _P(A16), ws, None) == INV                    # misaligned w2 scales
    # moe_forward_fp8(x, w_g, bias, w13, w13_scale, w2, w2_scale, s, y, idx, w, counts, ws, st)
    fwd = [_P(A16), _P(A16), None, _P(A16), _P(A16), _P(A16), _P(A16)]
    assert _raw(lib, "moe_forward_fp8", *fwd[:6], None, s, _P(A16), None, None, None, ws,
                None) == INV                                    # null w2 scales
    assert _raw(lib, "moe_forward_fp8", *fwd, s, _P(A16), None, None, None, None, None) == INV
    s0 = ctypes.byref(B.MoEShape.of(**dict(VALID, T=0)))
    assert _raw(lib, "moe_forward_fp8", *[None] * 7, s0, None, None, None, None, ws,
                None) == B.MOE_OK


def test_w8a8_calls_reject_before_launch(lib):
    s = ctypes.byref(B.MoEShape.of(**VALID))
    INV = B.MOE_ERR_INVALID_ARG
    ws = _P(A16)
    # moe_ffn_w8a8(x_perm, offsets, w13, w13_scale, w2, w2_scale, s, z, ws, stream)
    assert _raw(lib, "moe_ffn_w8a8", _P(A16), _P(A16), _P(A16), None, _P(A16), _P(A16), s,
                _P(A16), ws, None) == INV                       # null w13 scales
    assert _raw(lib, "moe_ffn_w8a8", _P(A16), _P(A16), _P(A16 + 8), _P(A16), _P(A16),
                _P(A16), s, _P(A16), ws, None) == INV           # codes not 16-byte aligned
    fwd = [_P(A16), _P(A16), None, _P(A16), _P(A16), _P(A16), _P(A16)]
    assert _raw(lib, "moe_forward_w8a8", *fwd[:6], None, s, _P(A16), None, None, None, ws,
                None) == INV                                    # null w2 scales
    assert _raw(lib, "moe_forward_w8a8", *fwd, s, _P(A16), None, None, None, None,
                None) == INV                                    # null workspace
    s0 = ctypes.byref(B.MoEShape.of(**dict(VALID, T=0)))
    assert _raw(lib, "moe_forward_w8a8", *[None] * 7, s0, None, None, None, None, ws,
                None) == B.MOE_OK
    # moe_quantise_rows_e4m3(a, rows, cols, codes, scales, stream)
    assert _raw(lib, "moe_quantise_rows_e4m3", _P(A16), 4, 24, _P(A16), _P(A16),
                None) == INV                                    # cols not a multiple of 16
    assert _raw(lib, "moe_quantise_rows_e4m3", _P(A16), -1, 32, _P(A16), _P(A16),
                None) == INV                                    # negative rows
    assert _raw(lib, "moe_quantise_rows_e4m3", _P(A16), 4, 32, _P(A16 + 4), _P(A16),
                None) == INV                                    # misaligned codes
    assert _raw(lib, "moe_quantise_rows_e4m3", None, 0, 32, None, None, None) == B.MOE_OK


def test_empty_batch_is_a_no_op(lib):
    s0 = ctypes.byref(B.MoEShape.of(**dict(VALID, T=0)))
    # T = 0 launches nothing, so even null activation pointers are accepted.
    assert _raw(lib, "moe_router", None, None, None, s0, None, None, None) == B.MOE_OK
    assert _raw(lib, "moe_topk", None, s0, None, None, None) == B.MOE_OK
    assert _raw(lib, "moe_combine", None, None, None, s0, None, None) == B.MOE_OK
    assert _raw(lib, "moe_forward", *[None] * 5, s0, None, None, None, None, _P(A16),
                None) == B.MOE_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_no_cpu_fallback_without_a_gpu(lib):
    s = ctypes.byref(B.MoEShape.of(**VALID))
    # Valid arguments but no device: the library refuses, it never computes on the CPU.
    assert _raw(lib, "moe_topk", _P(A16), s, _P(A16), _P(A16), None) == B.MOE_ERR_CUDA
    assert _raw(lib, "moe_forward", *[_P(A16)] * 5, s, _P(A16), None, None, None, _P(A16),
                None) == B.MOE_ERR_CUDA
    assert _raw(lib, "moe_forward_fp8", *[_P(A16)] * 7, s, _P(A16), None, None, None,
                _P(A16), None) == B.MOE_ERR_CUDA
    assert _raw(lib, "moe_forward_w8a8", *[_P(A16)] * 7, s, _P(A16), None, None, None,
                _P(A16), None) == B.MOE_ERR_CUDA
    assert _raw(lib, "moe_quantise_rows_e4m3", _P(A16), 4, 32, _P(A16), _P(A16),
                None) == B.MOE_ERR_CUDA
    assert _raw(lib, "moe_copy", _P(A16), _P(A16 + 64), ctypes.c_int64(32),
                None) == B.MOE_ERR_CUDA


def test_binding_refuses_cpu_tensors(lib):
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        moe.moe_combine(x, x, x, x, B.MoEShape.of(4, 64, 8, 1, 64))


# ---------------------------------------------------------------- EPLB plan (host code)
def test_eplb_plan_matches_oracle_on_random_loads(lib):
    import numpy as np

    import oracle
    rng = np.random.default_rng(11)
    for _ in range(200):
        R = int(rng.choice([1, 2, 4, 8]))
        E = R * int(rng.integers(1, 17))
        rd = R * int(rng.integers(0, 4))
        load = (rng.zipf(1.2, E).clip(max=1000) * int(rng.integers(1, 50))).tolist()
        if rng.random() < 0.2:
            load = [int(rng.integers(0, 3))] * E  # all ties
        want = [a.tolist() for a in oracle.eplb_plan(load, rd, R)]
        got = [a.tolist() for a in moe.moe_eplb_plan(load, E, R, rd)]
        assert got == want, (load, rd, R)


def test_eplb_plan_rejects_bad_arguments(lib):
    import numpy as np
    load = np.ones(8, dtype=np.int64)
    out = [np.zeros(16, dtype=np.int32) for _ in range(3)]
    INV = B.MOE_ERR_INVALID_ARG

    def call(E, R, rd, lo=load):
        return lib.moe_eplb_plan(lo.ctypes.data, E, R, rd, out[0].ctypes.data,
                                 out[1].ctypes.data, out[2].ctypes.data)
    assert call(8, 4, 4) == B.MOE_OK
    assert call(8, 3, 0) == INV          # 8 slots on 3 ranks
    assert call(8, 4, -4) == INV
    assert call(0, 1, 0) == INV
    assert call(8, 65, 57) == INV        # R above 64
    assert call(1024, 1, 8) == INV       # more than 1024 physical experts
    neg = load.copy()
    neg[3] = -1
    assert call(8, 4, 4, neg) == INV
    assert lib.moe_eplb_plan(None, 8, 4, 4, out[0].ctypes.data, out[1].ctypes.data,
                             out[2].ctypes.data) == INV


def test_eplb_workspace_size(lib):
    s = B.MoEShape.of(**VALID)
    assert moe.moe_workspace_size_eplb(s, VALID["E"] + 8) >= moe.moe_workspace_size(s)
    assert moe.moe_workspace_size_eplb(s, VALID["E"] - 1) == 0
    assert moe.moe_workspace_size_eplb(s, 1025) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_plain_c_client_builds_links_and_runs(lib, tmp_path):
    import shutil
    import subprocess

    import numpy as np

    import oracle
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    pkg = os.path.dirname(B.LIB_PATH)
    exe = str(tmp_path / "abi_from_c")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I",
                    os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_from_c.c"),
                    "-L", pkg, "-l:" + os.path.basename(B.LIB_PATH), "-Wl,-rpath," + pkg,
                    "-o", exe], check=True, capture_output=True, text=True)
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")  # no device: nothing may launch
    out = subprocess.run([exe], check=True, capture_output=True, text=True, env=env,
                         timeout=120).stdout
    f = dict(kv.split("=", 1) for kv in out.split()[:6])
    assert int(f["version"]) == moe.moe_version()
    assert int(f["ws"]) == moe.moe_workspace_size(B.MoEShape.of(**VALID))
    assert int(f["plan"]) == B.MOE_OK
    p2l, _, _ = oracle.eplb_plan(np.array([9, 1, 1, 1, 1, 1, 1, 1]), 2, 2)  # (load, n_redundant, R)
    assert int(f["p2l0"]) == int(p2l[0])
    assert int(f["forward"]) == B.MOE_ERR_CUDA
    assert int(f["bad"]) == B.MOE_ERR_INVALID_ARG
    assert "MOE_ERR_CUDA" in out
