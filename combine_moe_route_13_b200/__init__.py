"""Single-GPU MoE expert layer for B200 (sm_100a): route -> dispatch -> grouped
SwiGLU expert MLP -> combine, as hand-written CUDA kernels behind the C ABI in
include/moe.h (libmoe.so). This package is the thin Python binding."""
from ._binding import *  # noqa: F401,F403
from ._binding import (LIB, LIB_PATH, EXPORTS, MoeConfig, MoeError, MoeLayerAux,  # noqa: F401
                       alloc_route_outputs, alloc_workspace, layer_views, make_config,
                       shared_row0, quantize_fp8, fp8_views)
