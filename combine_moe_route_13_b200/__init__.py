"""Single-GPU MoE expert layer for B200 (sm_100a): route -> dispatch -> grouped
SwiGLU expert MLP -> combine, as hand-written CUDA kernels behind the C ABI in
include/moe.h (libmoe.so), and its expert-parallel form over W GPUs
(include/moe_ep.h). This package is the thin Python binding; ep.py holds the
host-side setup of an expert-parallel group."""
from ._binding import *  # noqa: F401,F403
from ._binding import (LIB, LIB_PATH, EXPORTS, MoeConfig, MoeError, MoeLayerAux,  # noqa: F401
                       alloc_route_outputs, alloc_workspace, layer_views, make_config,
                       shared_row0, quantize_fp8, fp8_views, MoeEp, MoeEpAux, make_ep,
                       ep_views)
