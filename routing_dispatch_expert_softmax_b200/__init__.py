"""B200-native (sm_100a) routed mixture-of-experts layer forward.

The layer of the expert-parallel serving pages -- router gate, top-k expert
selection, dispatch into per-expert rows, SwiGLU expert GEMMs, gate-weighted
combine -- as hand-written CUDA kernels behind a C ABI (``include/moe.h``,
``libmoe_b200.so``).  This package is the thin Python binding over it.
"""

from .binding import (EXPORTS, MOE_STAGE_EVENTS, STAGE_NAMES, MOE_ERR_CUDA, MOE_ERR_DEVICE_CHECK,  # noqa: F401
                      MOE_ERR_INVALID_ARG, MOE_ERR_TIMEOUT, MOE_ERR_UNSUPPORTED,
                      MOE_OK, MoEError, MoEShape, load_library, moe_check,
                      moe_combine, moe_dispatch, moe_dispatch_noalloc, moe_error_string, moe_ffn,
                      moe_forward, moe_forward_staged, moe_router, moe_selftest_bounded_wait,
                      moe_topk, moe_version,
                      moe_workspace_size, workspace, moe_eplb_plan, moe_eplb_remap,
                      moe_workspace_size_eplb, workspace_eplb, moe_forward_eplb,
                      moe_dispatch_dedup, moe_ffn_fp8, moe_forward_fp8,
                      moe_forward_fp8_staged, moe_ep_recv_experts, moe_ffn_w8a8,
                      moe_forward_w8a8, moe_forward_w8a8_staged, moe_quantise_rows_e4m3,
                      moe_copy)
from .layer import MoELayer  # noqa: F401
