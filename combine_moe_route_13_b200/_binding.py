"""ctypes binding of libmoe.so: the C entry points under the same names.

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels. torch tensors supply device memory and the stream; each
function checks dtype, device and contiguity, passes raw pointers and raises
MoeError on a non-OK status. There is no fallback: if the library is missing
or fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LIBRARY selects another build of the same library: a file name inside
# this package (libmoe_check.so, the bounds-checked build) or an absolute path.
LIB_PATH = os.path.join(HERE, os.environ.get("MOE_LIBRARY", "") or "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_DEVICE_INPUT = 6
MOE_F32 = 0
MOE_BF16 = 1
MOE_FLAG_NONE = 0
MOE_FLAG_OVERLAP = 1

# every symbol declared in include/moe.h
EXPORTS = ("moe_capacity", "moe_max_rows", "moe_check_config", "moe_route_workspace_bytes",
           "moe_workspace_bytes", "moe_workspace_init", "moe_route_topk", "moe_dispatch",
           "moe_expert_mlp", "moe_combine", "moe_layer_forward", "moe_get_device_status",
           "moe_status_string", "moe_version", "moe_route_topk_noalloc", "moe_combine_wait",
           "moe_route_topk_biased", "moe_router_logits", "moe_layer_forward_x",
           "moe_fp8_scale_bytes", "moe_quantize_fp8", "moe_dispatch_fp8", "moe_expert_mlp_fp8",
           "moe_layer_forward_fp8", "moe_debug_bounds_failures") + (
    # include/moe_ep.h
           "moe_ep_recv_rows", "moe_ep_symmetric_bytes", "moe_ep_workspace_bytes", "moe_ep_check",
           "moe_ep_aux", "moe_ep_symmetric_init", "moe_ep_route", "moe_ep_dispatch",
           "moe_ep_expert_mlp", "moe_ep_combine", "moe_ep_layer_forward", "moe_ep_sym_alloc",
           "moe_ep_sym_free", "moe_ipc_get_handle", "moe_ipc_open", "moe_ipc_close",
           "moe_ep_dispatch_fp8", "moe_ep_expert_mlp_fp8", "moe_ep_layer_forward_fp8",
           "moe_ep_workspace_init")


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("K", ctypes.c_int32), ("F", ctypes.c_int32), ("S", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("row_align", ctypes.c_int32),
                ("act_dtype", ctypes.c_int32), ("n_shared", ctypes.c_int32)]

    def __repr__(self):
        return ("MoeConfig(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")")


class MoeLayerAux(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "topk_idx", "expert_counts", "overflow", "expert_offsets", "segment_offsets",
        "token_slot", "row_src", "totals", "topk_w", "xp", "h", "y", "logits",
        "xq", "xs", "hq", "hs")]


class MoeEp(ctypes.Structure):
    _fields_ = [("world", ctypes.c_int32), ("rank", ctypes.c_int32), ("epoch", ctypes.c_uint32),
                ("timeout_us", ctypes.c_uint32), ("flags", ctypes.c_uint32)]


MOE_EP_TILE_SIGNAL = 1
MOE_EP_REMOTE_FIRST = 2


class MoeEpAux(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "topk_idx", "expert_counts", "overflow", "expert_offsets", "segment_offsets",
        "token_slot", "row_src", "totals", "topk_w", "counts_all", "flags", "send_dst_row",
        "recv_offsets", "recv_counts", "xr", "h", "y", "h_shared", "y_shared",
        "xq", "xs", "hq", "hs", "recv_split", "y_ready")]


_P = ctypes.c_void_p
_CFG = ctypes.POINTER(MoeConfig)
_EP = ctypes.POINTER(MoeEp)
_SZ = ctypes.c_size_t


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run "
                          "`python combine_moe_route_13_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "moe_capacity": (ctypes.c_int32, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_double]),
        "moe_max_rows": (ctypes.c_int64, [_CFG]),
        "moe_check_config": (ctypes.c_int, [_CFG]),
        "moe_route_workspace_bytes": (ctypes.c_size_t, [_CFG]),
        "moe_workspace_bytes": (ctypes.c_size_t, [_CFG, ctypes.c_uint32]),
        "moe_workspace_init": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
        "moe_route_topk": (ctypes.c_int, [_CFG] + [_P] * 10 + [_P, ctypes.c_size_t, _P]),
        "moe_dispatch": (ctypes.c_int, [_CFG, _P, _P, _P, _P]),
        "moe_expert_mlp": (ctypes.c_int, [_CFG] + [_P] * 7 + [_P, ctypes.c_size_t, _P]),
        "moe_combine": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P]),
        "moe_layer_forward": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, ctypes.c_uint32, _P,
                                             ctypes.c_size_t, ctypes.POINTER(MoeLayerAux), _P]),
        "moe_get_device_status": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int), _P]),
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_version": (ctypes.c_int32, []),
        "moe_debug_bounds_failures": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32),
                                                     ctypes.POINTER(ctypes.c_uint32),
                                                     ctypes.c_int32]),
        "moe_route_topk_noalloc": (ctypes.c_int, [_CFG] + [_P] * 10 + [_P]),
        "moe_combine_wait": (ctypes.c_int, [_CFG, _P, _P, _P, _P, ctypes.c_uint32, _P,
                                            ctypes.c_uint32, _P, ctypes.c_size_t, _P]),
        "moe_route_topk_biased": (ctypes.c_int, [_CFG] + [_P] * 11 + [_P, ctypes.c_size_t, _P]),
        "moe_router_logits": (ctypes.c_int, [_CFG, _P, _P, _P, _P, ctypes.c_size_t, _P]),
        "moe_layer_forward_x": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, ctypes.c_uint32,
                                               _P, ctypes.c_size_t, ctypes.POINTER(MoeLayerAux),
                                               _P]),
        "moe_fp8_scale_bytes": (ctypes.c_int64, [ctypes.c_int64, ctypes.c_int64]),
        "moe_quantize_fp8": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int64, _P, _P, _P]),
        "moe_dispatch_fp8": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P]),
        "moe_expert_mlp_fp8": (ctypes.c_int, [_CFG] + [_P] * 11 + [_P, ctypes.c_size_t, _P]),
        "moe_layer_forward_fp8": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P,
                                                 ctypes.c_uint32, _P, ctypes.c_size_t,
                                                 ctypes.POINTER(MoeLayerAux), _P]),
        "moe_ep_recv_rows": (ctypes.c_int64, [_CFG, ctypes.c_int32]),
        "moe_ep_symmetric_bytes": (_SZ, [_CFG, ctypes.c_int32]),
        "moe_ep_workspace_bytes": (_SZ, [_CFG, ctypes.c_int32]),
        "moe_ep_check": (ctypes.c_int, [_CFG, _EP]),
        "moe_ep_aux": (ctypes.c_int, [_CFG, _EP, _P, _P, ctypes.POINTER(MoeEpAux)]),
        "moe_ep_symmetric_init": (ctypes.c_int, [_CFG, ctypes.c_int32, _P, _SZ, _P]),
        "moe_ep_workspace_init": (ctypes.c_int, [_CFG, ctypes.c_int32, _P, _SZ, _P]),
        "moe_ep_route": (ctypes.c_int, [_CFG, _EP, _P, _P, _P, _P, _SZ, _P]),
        "moe_ep_dispatch": (ctypes.c_int, [_CFG, _EP, _P, _P, _P, _P, _SZ, _P]),
        "moe_ep_expert_mlp": (ctypes.c_int, [_CFG, _EP, _P, _P, _P, _P, _P, _P, _SZ, _P]),
        "moe_ep_combine": (ctypes.c_int, [_CFG, _EP, _P, _P, _P, _P, _SZ, _P]),
        "moe_ep_layer_forward": (ctypes.c_int, [_CFG, _EP, _P, _P, _P, _P, _P, _P, _P,
                                                ctypes.POINTER(MoeEpAux), _P, _SZ, _P]),
        "moe_ep_dispatch_fp8": (ctypes.c_int, [_CFG, _EP, _P, _P, _P, _P, _SZ, _P]),
        "moe_ep_expert_mlp_fp8": (ctypes.c_int, [_CFG, _EP, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
        "moe_ep_layer_forward_fp8": (ctypes.c_int, [_CFG, _EP, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                                    ctypes.POINTER(MoeEpAux), _P, _SZ, _P]),
        "moe_ep_sym_alloc": (ctypes.c_int, [_SZ, ctypes.POINTER(ctypes.c_void_p)]),
        "moe_ep_sym_free": (ctypes.c_int, [_P]),
        "moe_ipc_get_handle": (ctypes.c_int, [_P, ctypes.c_char_p]),
        "moe_ipc_open": (ctypes.c_int, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_void_p)]),
        "moe_ipc_close": (ctypes.c_int, [_P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


LIB = _load()


def status_string(code: int) -> str:
    return LIB.moe_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != MOE_OK:
        raise MoeError(code, where)


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None, dtype=None, name="tensor") -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def make_config(T, H, E, K, F, S, capacity, row_align=128, act="bf16", n_shared=0) -> MoeConfig:
    return MoeConfig(int(T), int(H), int(E), int(K), int(F), int(S), int(capacity),
                     int(row_align), MOE_F32 if act in ("f32", torch.float32, MOE_F32) else MOE_BF16,
                     int(n_shared))


def shared_row0(cfg: MoeConfig) -> int:
    """First row of the shared expert in xp / h / y (the rows before it are routed)."""
    return moe_max_rows(cfg) - cfg.n_shared * cfg.T


def act_dtype(cfg: MoeConfig) -> torch.dtype:
    return torch.float32 if cfg.act_dtype == MOE_F32 else torch.bfloat16


# ---------------------------------------------------------------- entry points

def moe_capacity(T: int, K: int, E: int, cf: float) -> int:
    return int(LIB.moe_capacity(T, K, E, float(cf)))


def moe_max_rows(cfg: MoeConfig) -> int:
    return int(LIB.moe_max_rows(ctypes.byref(cfg)))


def moe_check_config(cfg: MoeConfig) -> int:
    return int(LIB.moe_check_config(ctypes.byref(cfg)))


def moe_route_workspace_bytes(cfg: MoeConfig) -> int:
    return int(LIB.moe_route_workspace_bytes(ctypes.byref(cfg)))


def moe_workspace_bytes(cfg: MoeConfig, flags: int = MOE_FLAG_NONE) -> int:
    return int(LIB.moe_workspace_bytes(ctypes.byref(cfg), flags))


def moe_workspace_init(ws: torch.Tensor, stream=None):
    _check(LIB.moe_workspace_init(_ptr(ws, name="ws"), ws.numel() * ws.element_size(),
                                  _stream(stream)), "moe_workspace_init")


def moe_route_topk(cfg, logits, topk_idx, topk_w, expert_counts, overflow, expert_offsets,
                   segment_offsets, token_slot, row_src, totals, ws, stream=None):
    i32 = torch.int32
    _check(LIB.moe_route_topk(
        ctypes.byref(cfg), _ptr(logits, torch.float32, "logits"), _ptr(topk_idx, i32, "topk_idx"),
        _ptr(topk_w, torch.float32, "topk_w"), _ptr(expert_counts, i32, "expert_counts"),
        _ptr(overflow, i32, "overflow"), _ptr(expert_offsets, i32, "expert_offsets"),
        _ptr(segment_offsets, i32, "segment_offsets"), _ptr(token_slot, i32, "token_slot"),
        _ptr(row_src, i32, "row_src"), _ptr(totals, i32, "totals"), _ptr(ws, name="ws"),
        ws.numel() * ws.element_size(), _stream(stream)), "moe_route_topk")


def moe_route_topk_biased(cfg, logits, sel_bias, topk_idx, topk_w, expert_counts, overflow,
                          expert_offsets, segment_offsets, token_slot, row_src, totals, ws,
                          stream=None):
    i32 = torch.int32
    _check(LIB.moe_route_topk_biased(
        ctypes.byref(cfg), _ptr(logits, torch.float32, "logits"),
        _ptr(sel_bias, torch.float32, "sel_bias"), _ptr(topk_idx, i32, "topk_idx"),
        _ptr(topk_w, torch.float32, "topk_w"), _ptr(expert_counts, i32, "expert_counts"),
        _ptr(overflow, i32, "overflow"), _ptr(expert_offsets, i32, "expert_offsets"),
        _ptr(segment_offsets, i32, "segment_offsets"), _ptr(token_slot, i32, "token_slot"),
        _ptr(row_src, i32, "row_src"), _ptr(totals, i32, "totals"), _ptr(ws, name="ws"),
        ws.numel() * ws.element_size(), _stream(stream)), "moe_route_topk_biased")


def moe_router_logits(cfg, x, w_g, logits, ws, stream=None):
    dt = act_dtype(cfg)
    _check(LIB.moe_router_logits(ctypes.byref(cfg), _ptr(x, dt, "x"), _ptr(w_g, dt, "w_g"),
                                 _ptr(logits, torch.float32, "logits"), _ptr(ws, name="ws"),
                                 ws.numel() * ws.element_size(), _stream(stream)),
           "moe_router_logits")


def moe_layer_forward_x(cfg, x, w_g, sel_bias, w_gu, w_d, out, ws, flags=MOE_FLAG_NONE,
                        stream=None):
    """The layer from hidden states (router projection included); returns a
    MoeLayerAux like moe_layer_forward, with the logits' address."""
    dt = act_dtype(cfg)
    aux = MoeLayerAux()
    _check(LIB.moe_layer_forward_x(
        ctypes.byref(cfg), _ptr(x, dt, "x"), _ptr(w_g, dt, "w_g"),
        _ptr(sel_bias, torch.float32, "sel_bias"), _ptr(w_gu, dt, "w_gu"), _ptr(w_d, dt, "w_d"),
        _ptr(out, dt, "out"), flags, _ptr(ws, name="ws"), ws.numel() * ws.element_size(),
        ctypes.byref(aux), _stream(stream)), "moe_layer_forward_x")
    return aux


def moe_route_topk_noalloc(cfg, logits, topk_idx, topk_w, expert_counts, overflow,
                           expert_offsets, segment_offsets, token_slot, row_src, totals,
                           stream=None):
    """moe_route_topk without a workspace (for callers that cannot allocate):
    the scratch is a fixed 1 MiB device array inside the library."""
    i32 = torch.int32
    _check(LIB.moe_route_topk_noalloc(
        ctypes.byref(cfg), _ptr(logits, torch.float32, "logits"), _ptr(topk_idx, i32, "topk_idx"),
        _ptr(topk_w, torch.float32, "topk_w"), _ptr(expert_counts, i32, "expert_counts"),
        _ptr(overflow, i32, "overflow"), _ptr(expert_offsets, i32, "expert_offsets"),
        _ptr(segment_offsets, i32, "segment_offsets"), _ptr(token_slot, i32, "token_slot"),
        _ptr(row_src, i32, "row_src"), _ptr(totals, i32, "totals"), _stream(stream)),
        "moe_route_topk_noalloc")


def moe_dispatch(cfg, x, token_slot, xp, stream=None):
    dt = act_dtype(cfg)
    _check(LIB.moe_dispatch(ctypes.byref(cfg), _ptr(x, dt, "x"),
                            _ptr(token_slot, torch.int32, "token_slot"), _ptr(xp, dt, "xp"),
                            _stream(stream)), "moe_dispatch")


def moe_expert_mlp(cfg, xp, expert_offsets, expert_counts, w_gu, w_d, h, y, ws, stream=None):
    dt = act_dtype(cfg)
    _check(LIB.moe_expert_mlp(
        ctypes.byref(cfg), _ptr(xp, dt, "xp"), _ptr(expert_offsets, torch.int32, "expert_offsets"),
        _ptr(expert_counts, torch.int32, "expert_counts"), _ptr(w_gu, dt, "w_gu"),
        _ptr(w_d, dt, "w_d"), _ptr(h, dt, "h"), _ptr(y, dt, "y"), _ptr(ws, name="ws"),
        ws.numel() * ws.element_size(), _stream(stream)), "moe_expert_mlp")


def moe_combine(cfg, y, token_slot, topk_w, out, stream=None):
    dt = act_dtype(cfg)
    _check(LIB.moe_combine(ctypes.byref(cfg), _ptr(y, dt, "y"),
                           _ptr(token_slot, torch.int32, "token_slot"),
                           _ptr(topk_w, torch.float32, "topk_w"), _ptr(out, dt, "out"),
                           _stream(stream)), "moe_combine")


def moe_combine_wait(cfg, y, token_slot, topk_w, row_ready, ready_target, out, ws,
                     timeout_us=2_000_000, stream=None):
    dt = act_dtype(cfg)
    _check(LIB.moe_combine_wait(
        ctypes.byref(cfg), _ptr(y, dt, "y"), _ptr(token_slot, torch.int32, "token_slot"),
        _ptr(topk_w, torch.float32, "topk_w"), _ptr(row_ready, (torch.int32, torch.uint32), "row_ready"),
        int(ready_target), _ptr(out, dt, "out"), int(timeout_us), _ptr(ws, name="ws"),
        ws.numel() * ws.element_size(), _stream(stream)), "moe_combine_wait")


def ready_target(cfg: MoeConfig) -> int:
    """Counter value at which a 128-row block of y is final (the down GEMM's N tiles)."""
    return (cfg.H + 255) // 256


def moe_layer_forward(cfg, logits, x, w_gu, w_d, out, ws, flags=MOE_FLAG_NONE, stream=None):
    """Runs the fused layer; returns a MoeLayerAux with the workspace pointers of
    the intermediates (see layer_views)."""
    dt = act_dtype(cfg)
    aux = MoeLayerAux()
    _check(LIB.moe_layer_forward(
        ctypes.byref(cfg), _ptr(logits, torch.float32, "logits"), _ptr(x, dt, "x"),
        _ptr(w_gu, dt, "w_gu"), _ptr(w_d, dt, "w_d"), _ptr(out, dt, "out"), flags,
        _ptr(ws, name="ws"), ws.numel() * ws.element_size(), ctypes.byref(aux), _stream(stream)),
        "moe_layer_forward")
    return aux


def moe_get_device_status(ws, stream=None) -> int:
    st = ctypes.c_int(0)
    _check(LIB.moe_get_device_status(_ptr(ws, name="ws"), ctypes.byref(st), _stream(stream)),
           "moe_get_device_status")
    return int(st.value)


def moe_version() -> int:
    return int(LIB.moe_version())


def moe_debug_bounds_failures(reset: bool = False):
    """(failures, first failing source line) of the bounds-checked build;
    raises MoeError(MOE_ERR_UNSUPPORTED) on the release build."""
    n, line = ctypes.c_uint32(0), ctypes.c_uint32(0)
    _check(LIB.moe_debug_bounds_failures(ctypes.byref(n), ctypes.byref(line), int(bool(reset))),
           "moe_debug_bounds_failures")
    return int(n.value), int(line.value)


# ---------------------------------------------------------------- fp8 block-scaled path

U8 = torch.uint8


def moe_fp8_scale_bytes(rows: int, cols: int) -> int:
    return int(LIB.moe_fp8_scale_bytes(int(rows), int(cols)))


def moe_quantize_fp8(src, codes, scales, stream=None):
    """Block-quantise a [rows, cols] bf16 tensor into codes (uint8, same shape) and scales."""
    rows, cols = src.shape
    _check(LIB.moe_quantize_fp8(_ptr(src, torch.bfloat16, "src"), rows, cols,
                                _ptr(codes, U8, "codes"), _ptr(scales, U8, "scales"),
                                _stream(stream)), "moe_quantize_fp8")


def quantize_fp8(src: torch.Tensor, stream=None):
    """Allocate and fill (codes, scales) for a bf16 tensor viewed as [-1, last dim]."""
    m = src.reshape(-1, src.shape[-1])
    codes = torch.empty(m.shape, dtype=U8, device=src.device)
    scales = torch.empty(max(moe_fp8_scale_bytes(*m.shape), 16), dtype=U8, device=src.device)
    moe_quantize_fp8(m, codes, scales, stream)
    return codes.view(src.shape), scales


def moe_dispatch_fp8(cfg, x, token_slot, xq, xs, stream=None):
    _check(LIB.moe_dispatch_fp8(ctypes.byref(cfg), _ptr(x, torch.bfloat16, "x"),
                                _ptr(token_slot, torch.int32, "token_slot"), _ptr(xq, U8, "xq"),
                                _ptr(xs, U8, "xs"), _stream(stream)), "moe_dispatch_fp8")


def moe_expert_mlp_fp8(cfg, xq, xs, expert_offsets, expert_counts, wq_gu, ws_gu, wq_d, ws_d,
                       hq, hs, y, ws, stream=None):
    i32 = torch.int32
    _check(LIB.moe_expert_mlp_fp8(
        ctypes.byref(cfg), _ptr(xq, U8, "xq"), _ptr(xs, U8, "xs"),
        _ptr(expert_offsets, i32, "expert_offsets"), _ptr(expert_counts, i32, "expert_counts"),
        _ptr(wq_gu, U8, "wq_gu"), _ptr(ws_gu, U8, "ws_gu"), _ptr(wq_d, U8, "wq_d"),
        _ptr(ws_d, U8, "ws_d"), _ptr(hq, U8, "hq"), _ptr(hs, U8, "hs"),
        _ptr(y, torch.bfloat16, "y"), _ptr(ws, name="ws"), ws.numel() * ws.element_size(),
        _stream(stream)), "moe_expert_mlp_fp8")


def moe_layer_forward_fp8(cfg, logits, x, wq_gu, ws_gu, wq_d, ws_d, out, ws,
                          flags=MOE_FLAG_NONE, stream=None):
    aux = MoeLayerAux()
    _check(LIB.moe_layer_forward_fp8(
        ctypes.byref(cfg), _ptr(logits, torch.float32, "logits"), _ptr(x, torch.bfloat16, "x"),
        _ptr(wq_gu, U8, "wq_gu"), _ptr(ws_gu, U8, "ws_gu"), _ptr(wq_d, U8, "wq_d"),
        _ptr(ws_d, U8, "ws_d"), _ptr(out, torch.bfloat16, "out"), flags, _ptr(ws, name="ws"),
        ws.numel() * ws.element_size(), ctypes.byref(aux), _stream(stream)),
        "moe_layer_forward_fp8")
    return aux


def fp8_views(cfg: MoeConfig, ws: torch.Tensor, aux: MoeLayerAux) -> dict:
    """torch views of the fp8 intermediates moe_layer_forward_fp8 left in ws."""
    base = ws.data_ptr()
    R = moe_max_rows(cfg)

    def view(ptr, nbytes, shape):
        off = ptr - base
        return ws[off:off + nbytes].view(shape)

    return {"xq": view(aux.xq, R * cfg.H, (R, cfg.H)),
            "xs": view(aux.xs, moe_fp8_scale_bytes(R, cfg.H), (-1,)),
            "hq": view(aux.hq, R * cfg.F, (R, cfg.F)),
            "hs": view(aux.hs, moe_fp8_scale_bytes(R, cfg.F), (-1,))}


# ---------------------------------------------------------------- conveniences

def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zeroed byte workspace (torch allocations are 256-byte aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def alloc_route_outputs(cfg: MoeConfig, device="cuda") -> dict:
    i32 = dict(dtype=torch.int32, device=device)
    R = moe_max_rows(cfg)
    return {
        "topk_idx": torch.empty(cfg.T, cfg.K, **i32),
        "topk_w": torch.empty(cfg.T, cfg.K, dtype=torch.float32, device=device),
        "expert_counts": torch.empty(cfg.E, **i32),
        "overflow": torch.empty(cfg.E, **i32),
        "expert_offsets": torch.empty(cfg.E + 1, **i32),
        "segment_offsets": torch.empty(cfg.S + 1, **i32),
        "token_slot": torch.empty(cfg.T, cfg.K, **i32),
        "row_src": torch.empty(max(R, 1), **i32),
        "totals": torch.empty(4, **i32),
    }


def layer_views(cfg: MoeConfig, ws: torch.Tensor, aux: MoeLayerAux) -> dict:
    """torch views of the intermediates that moe_layer_forward left in ws."""
    base = ws.data_ptr()
    R = moe_max_rows(cfg)
    dt = act_dtype(cfg)
    es = 4 if dt == torch.float32 else 2

    def view(ptr, nbytes, dtype, shape):
        if ptr is None:   # not produced by this entry point (xp / h of the fp8 layer)
            return None
        off = ptr - base
        return ws[off:off + nbytes].view(dtype).view(shape)

    TK = cfg.T * cfg.K
    return {
        "topk_idx": view(aux.topk_idx, TK * 4, torch.int32, (cfg.T, cfg.K)),
        "topk_w": view(aux.topk_w, TK * 4, torch.float32, (cfg.T, cfg.K)),
        "expert_counts": view(aux.expert_counts, cfg.E * 4, torch.int32, (cfg.E,)),
        "overflow": view(aux.overflow, cfg.E * 4, torch.int32, (cfg.E,)),
        "expert_offsets": view(aux.expert_offsets, (cfg.E + 1) * 4, torch.int32, (cfg.E + 1,)),
        "segment_offsets": view(aux.segment_offsets, (cfg.S + 1) * 4, torch.int32, (cfg.S + 1,)),
        "token_slot": view(aux.token_slot, TK * 4, torch.int32, (cfg.T, cfg.K)),
        "row_src": view(aux.row_src, R * 4, torch.int32, (R,)),
        "totals": view(aux.totals, 16, torch.int32, (4,)),
        "xp": view(aux.xp, R * cfg.H * es, dt, (R, cfg.H)),
        "h": view(aux.h, R * cfg.F * es, dt, (R, cfg.F)),
        "y": view(aux.y, R * cfg.H * es, dt, (R, cfg.H)),
        "logits": view(aux.logits, TK // max(cfg.K, 1) * cfg.E * 4, torch.float32, (cfg.T, cfg.E)),
    }


# ---------------------------------------------------------------- expert parallelism (moe_ep.h)

def make_ep(world: int, rank: int, epoch: int, timeout_us: int = 0, flags: int = 0) -> MoeEp:
    return MoeEp(int(world), int(rank), int(epoch), int(timeout_us), int(flags))


def _addr(buf, name) -> int:
    """Device address of a CUDA tensor, or an address given as an int (a
    region mapped by moe_ipc_open or allocated by moe_ep_sym_alloc)."""
    if isinstance(buf, int):
        return buf
    return _ptr(buf, name=name)


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def moe_ep_recv_rows(cfg: MoeConfig, world: int) -> int:
    return int(LIB.moe_ep_recv_rows(ctypes.byref(cfg), int(world)))


def moe_ep_symmetric_bytes(cfg: MoeConfig, world: int) -> int:
    return int(LIB.moe_ep_symmetric_bytes(ctypes.byref(cfg), int(world)))


def moe_ep_workspace_bytes(cfg: MoeConfig, world: int) -> int:
    return int(LIB.moe_ep_workspace_bytes(ctypes.byref(cfg), int(world)))


def moe_ep_check(cfg: MoeConfig, ep: MoeEp) -> int:
    return int(LIB.moe_ep_check(ctypes.byref(cfg), ctypes.byref(ep)))


def moe_ep_aux(cfg, ep, sym, ws) -> MoeEpAux:
    aux = MoeEpAux()
    _check(LIB.moe_ep_aux(ctypes.byref(cfg), ctypes.byref(ep), _addr(sym, "sym"),
                          _ptr(ws, name="ws"), ctypes.byref(aux)), "moe_ep_aux")
    return aux


def moe_ep_symmetric_init(cfg, world, sym, sym_bytes=None, stream=None):
    n = _nbytes(sym) if sym_bytes is None else int(sym_bytes)
    _check(LIB.moe_ep_symmetric_init(ctypes.byref(cfg), int(world), _addr(sym, "sym"), n,
                                     _stream(stream)), "moe_ep_symmetric_init")


def moe_ep_workspace_init(cfg, world, ws, stream=None):
    _check(LIB.moe_ep_workspace_init(ctypes.byref(cfg), int(world), _ptr(ws, name="ws"),
                                     _nbytes(ws), _stream(stream)), "moe_ep_workspace_init")


def _peers(peers):
    return _ptr(peers, torch.int64, "peers")


def moe_ep_route(cfg, ep, logits, sym, peers, ws, stream=None):
    _check(LIB.moe_ep_route(ctypes.byref(cfg), ctypes.byref(ep),
                            _ptr(logits, torch.float32, "logits"), _addr(sym, "sym"),
                            _peers(peers), _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)),
           "moe_ep_route")


def moe_ep_dispatch(cfg, ep, x, sym, peers, ws, stream=None):
    _check(LIB.moe_ep_dispatch(ctypes.byref(cfg), ctypes.byref(ep), _ptr(x, act_dtype(cfg), "x"),
                               _addr(sym, "sym"), _peers(peers), _ptr(ws, name="ws"), _nbytes(ws),
                               _stream(stream)), "moe_ep_dispatch")


def moe_ep_expert_mlp(cfg, ep, x, w_gu_local, w_d_local, sym, peers, ws, stream=None):
    """x: this rank's tokens, read only for the shared expert (None without one)."""
    dt = act_dtype(cfg)
    _check(LIB.moe_ep_expert_mlp(ctypes.byref(cfg), ctypes.byref(ep), _ptr(x, dt, "x"),
                                 _ptr(w_gu_local, dt, "w_gu_local"), _ptr(w_d_local, dt, "w_d_local"),
                                 _addr(sym, "sym"), _peers(peers), _ptr(ws, name="ws"),
                                 _nbytes(ws), _stream(stream)), "moe_ep_expert_mlp")


def moe_ep_combine(cfg, ep, sym, peers, out, ws, stream=None):
    _check(LIB.moe_ep_combine(ctypes.byref(cfg), ctypes.byref(ep), _addr(sym, "sym"),
                              _peers(peers), _ptr(out, act_dtype(cfg), "out"), _ptr(ws, name="ws"),
                              _nbytes(ws), _stream(stream)), "moe_ep_combine")


def moe_ep_layer_forward(cfg, ep, logits, x, w_gu_local, w_d_local, sym, peers, out, ws,
                         stream=None) -> MoeEpAux:
    dt = act_dtype(cfg)
    aux = MoeEpAux()
    _check(LIB.moe_ep_layer_forward(
        ctypes.byref(cfg), ctypes.byref(ep), _ptr(logits, torch.float32, "logits"),
        _ptr(x, dt, "x"), _ptr(w_gu_local, dt, "w_gu_local"), _ptr(w_d_local, dt, "w_d_local"),
        _addr(sym, "sym"), _peers(peers), _ptr(out, dt, "out"), ctypes.byref(aux),
        _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)), "moe_ep_layer_forward")
    return aux


def moe_ep_dispatch_fp8(cfg, ep, x, sym, peers, ws, stream=None):
    _check(LIB.moe_ep_dispatch_fp8(ctypes.byref(cfg), ctypes.byref(ep),
                                   _ptr(x, torch.bfloat16, "x"), _addr(sym, "sym"), _peers(peers),
                                   _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)),
           "moe_ep_dispatch_fp8")


def moe_ep_expert_mlp_fp8(cfg, ep, wq_gu_local, ws_gu_local, wq_d_local, ws_d_local, sym, peers,
                          ws, stream=None):
    _check(LIB.moe_ep_expert_mlp_fp8(
        ctypes.byref(cfg), ctypes.byref(ep), _ptr(wq_gu_local, U8, "wq_gu_local"),
        _ptr(ws_gu_local, U8, "ws_gu_local"), _ptr(wq_d_local, U8, "wq_d_local"),
        _ptr(ws_d_local, U8, "ws_d_local"), _addr(sym, "sym"), _peers(peers), _ptr(ws, name="ws"),
        _nbytes(ws), _stream(stream)), "moe_ep_expert_mlp_fp8")


def moe_ep_layer_forward_fp8(cfg, ep, logits, x, wq_gu_local, ws_gu_local, wq_d_local,
                             ws_d_local, sym, peers, out, ws, stream=None) -> MoeEpAux:
    aux = MoeEpAux()
    _check(LIB.moe_ep_layer_forward_fp8(
        ctypes.byref(cfg), ctypes.byref(ep), _ptr(logits, torch.float32, "logits"),
        _ptr(x, torch.bfloat16, "x"), _ptr(wq_gu_local, U8, "wq_gu_local"),
        _ptr(ws_gu_local, U8, "ws_gu_local"), _ptr(wq_d_local, U8, "wq_d_local"),
        _ptr(ws_d_local, U8, "ws_d_local"), _addr(sym, "sym"), _peers(peers),
        _ptr(out, torch.bfloat16, "out"), ctypes.byref(aux), _ptr(ws, name="ws"), _nbytes(ws),
        _stream(stream)), "moe_ep_layer_forward_fp8")
    return aux


def ep_local_fp8_weights(wq, sf, world: int, E: int, rows_per_expert: int, cols: int,
                         n_shared: int = 0) -> list:
    """Each rank's slice of weights quantised by quantize_fp8 over all E experts
    ([E + n_shared, rows_per_expert, cols] codes and their blocked scales):
    (codes, scales) per rank, with the shared expert (the last one, held by
    every rank) appended when n_shared = 1. rows_per_expert must be a multiple
    of 128 (the scale row blocks), so that each expert's scales are one
    contiguous byte range."""
    El = E // world
    per = rows_per_expert // 128 * ((cols // 128 + 3) // 4) * 512   # scale bytes per expert
    out = []
    for r in range(world):
        q, f = wq[r * El:(r + 1) * El], sf[r * El * per:(r + 1) * El * per]
        if n_shared:
            q = torch.cat([q, wq[E:E + 1]]).contiguous()
            f = torch.cat([f, sf[E * per:(E + 1) * per]]).contiguous()
        out.append((q, f))
    return out


def moe_ep_sym_alloc(nbytes: int) -> int:
    p = ctypes.c_void_p()
    _check(LIB.moe_ep_sym_alloc(int(nbytes), ctypes.byref(p)), "moe_ep_sym_alloc")
    return int(p.value)


def moe_ep_sym_free(addr: int):
    _check(LIB.moe_ep_sym_free(int(addr)), "moe_ep_sym_free")


def moe_ipc_get_handle(addr: int) -> bytes:
    buf = ctypes.create_string_buffer(64)
    _check(LIB.moe_ipc_get_handle(int(addr), buf), "moe_ipc_get_handle")
    return buf.raw


def moe_ipc_open(handle: bytes) -> int:
    if len(handle) != 64:
        raise ValueError("a CUDA IPC handle has 64 bytes")
    p = ctypes.c_void_p()
    _check(LIB.moe_ipc_open(handle, ctypes.byref(p)), "moe_ipc_open")
    return int(p.value)


def moe_ipc_close(addr: int):
    _check(LIB.moe_ipc_close(int(addr)), "moe_ipc_close")


def ep_views(cfg: MoeConfig, world: int, sym: torch.Tensor, ws: torch.Tensor,
             aux: MoeEpAux) -> dict:
    """torch views of one rank's intermediates (sym and ws given as tensors)."""
    El = cfg.E // world
    R = moe_ep_recv_rows(cfg, world)
    dt = act_dtype(cfg)
    es = 4 if dt == torch.float32 else 2
    TK = cfg.T * cfg.K
    Rl = moe_max_rows(make_config(cfg.T, cfg.H, cfg.E, cfg.K, cfg.F, cfg.S, cfg.capacity,
                                  cfg.row_align, cfg.act_dtype))   # the routed rows

    def view(buf, ptr, nbytes, dtype, shape):
        off = ptr - buf.data_ptr()
        assert 0 <= off and off + nbytes <= _nbytes(buf)
        return buf[off:off + nbytes].view(dtype).view(shape)

    i32 = torch.int32
    return {
        "topk_idx": view(ws, aux.topk_idx, TK * 4, i32, (cfg.T, cfg.K)),
        "topk_w": view(ws, aux.topk_w, TK * 4, torch.float32, (cfg.T, cfg.K)),
        "expert_counts": view(ws, aux.expert_counts, cfg.E * 4, i32, (cfg.E,)),
        "overflow": view(ws, aux.overflow, cfg.E * 4, i32, (cfg.E,)),
        "expert_offsets": view(ws, aux.expert_offsets, (cfg.E + 1) * 4, i32, (cfg.E + 1,)),
        "segment_offsets": view(ws, aux.segment_offsets, (cfg.S + 1) * 4, i32, (cfg.S + 1,)),
        "token_slot": view(ws, aux.token_slot, TK * 4, i32, (cfg.T, cfg.K)),
        "row_src": view(ws, aux.row_src, Rl * 4, i32, (Rl,)),
        "totals": view(ws, aux.totals, 16, i32, (4,)),
        "send_dst_row": view(ws, aux.send_dst_row, cfg.E * 4, i32, (cfg.E,)),
        "recv_offsets": view(ws, aux.recv_offsets, (El + 1) * 4, i32, (El + 1,)),
        "recv_counts": view(ws, aux.recv_counts, El * 4, i32, (El,)),
        "counts_all": view(sym, aux.counts_all, world * cfg.E * 4, i32, (world, cfg.E)),
        "flags": view(sym, aux.flags, 3 * world * 4, i32, (3, world)),
        "xr": view(sym, aux.xr, R * cfg.H * es, dt, (R, cfg.H)),
        "h": view(ws, aux.h, R * cfg.F * es, dt, (R, cfg.F)),
        "y": view(sym, aux.y, R * cfg.H * es, dt, (R, cfg.H)),
        "h_shared": view(ws, aux.h_shared, cfg.T * cfg.F * es, dt, (cfg.T, cfg.F))
        if aux.h_shared else None,
        "y_shared": view(ws, aux.y_shared, cfg.T * cfg.H * es, dt, (cfg.T, cfg.H))
        if aux.y_shared else None,
        "xq": view(sym, aux.xq, R * cfg.H, U8, (R, cfg.H)) if aux.xq else None,
        "xs": view(sym, aux.xs, moe_fp8_scale_bytes(R, cfg.H), U8, (-1,)) if aux.xs else None,
        "hq": view(ws, aux.hq, R * cfg.F, U8, (R, cfg.F)) if aux.hq else None,
        "hs": view(ws, aux.hs, moe_fp8_scale_bytes(R, cfg.F), U8, (-1,)) if aux.hs else None,
        "recv_split": view(ws, aux.recv_split, El * (world + 1) * 4, i32, (El, world + 1)),
        "y_ready": view(sym, aux.y_ready, 2 * ((R + 127) // 128) * 4, i32, (2, (R + 127) // 128)),
    }
