"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/*.h declares, and its host-only functions (capacity,
sizes, validation, status strings) behave as documented."""
import ctypes
import glob
import os
import re

import pytest

import combine_moe_route_13_b200 as M
from oracle import moe_oracle as O
import workloads as W

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
HEADER = os.path.join(INCLUDE, "moe.h")


def declared_functions():
    names = set()
    for h in sorted(glob.glob(os.path.join(INCLUDE, "*.h"))):
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 30
    lib = ctypes.CDLL(M.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(M.EXPORTS) == names


def test_version():
    assert M.moe_version() == 10200


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_capacity_matches_oracle(name):
    w = W.WORKLOADS[name]
    assert M.moe_capacity(w.T, w.K, w.E, w.cf) == O.capacity(w.T, w.K, w.E, w.cf)


def test_capacity_edge_cases():
    assert M.moe_capacity(10, 3, 4, 1.0) == 8
    assert M.moe_capacity(10, 3, 4, -1.0) == 10
    assert M.moe_capacity(0, 3, 4, 1.0) == 0
    assert M.moe_capacity(-1, 3, 4, 1.0) == -1
    assert M.moe_capacity(10, 0, 4, 1.0) == -1


def cfg_of(w, **kw):
    C = O.capacity(w.T, w.K, w.E, w.cf)
    d = dict(T=w.T, H=w.H, E=w.E, K=w.K, F=w.F, S=w.S, capacity=C, row_align=w.row_align, act=w.act)
    d.update(kw)
    return M.make_config(**d)


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_sizes_match_oracle(name):
    w = W.WORKLOADS[name]
    cfg = cfg_of(w)
    C = cfg.capacity
    assert M.moe_max_rows(cfg) == O.max_rows(w.T, w.K, w.E, C, w.row_align)
    assert M.moe_check_config(cfg) == M.MOE_OK
    R = M.moe_max_rows(cfg)
    s = 4 if w.act == "f32" else 2
    need = R * (2 * w.H + w.F) * s
    assert M.moe_workspace_bytes(cfg) >= need
    assert 256 < M.moe_route_workspace_bytes(cfg) < M.moe_workspace_bytes(cfg)


@pytest.mark.parametrize("name", ["tiny", "mixtral", "dsv3", "kimi"])
def test_sizes_with_a_shared_expert(name):
    # moe.h: the shared expert's T rows start at the routed bound rounded up to
    # 128 and R_max grows by them; routed sizes are unchanged.
    w = W.WORKLOADS[name]
    base = cfg_of(w)
    cfg = cfg_of(w, n_shared=1)
    R_r = O.max_rows(w.T, w.K, w.E, base.capacity, w.row_align)
    R_sh = -(-R_r // 128) * 128
    assert M.moe_max_rows(base) == R_r
    assert M.moe_max_rows(cfg) == R_sh + w.T
    assert M.shared_row0(cfg) == R_sh and M.shared_row0(base) == R_r
    assert M.moe_check_config(cfg) == M.MOE_OK
    assert M.moe_workspace_bytes(cfg) >= M.moe_workspace_bytes(base) + w.T * (2 * w.H + w.F) * (
        4 if w.act == "f32" else 2)


def test_n_shared_other_than_0_or_1_is_invalid():
    cfg = cfg_of(W.WORKLOADS["tiny"], n_shared=2)
    assert M.moe_check_config(cfg) == M.MOE_ERR_INVALID_ARG
    cfg.n_shared = -1
    assert M.moe_max_rows(cfg) == -1


def test_config_struct_matches_header():
    # the ctypes mirror of moe_config_t has the header's fields in order
    src = open(HEADER).read()
    body = re.search(r"typedef struct \{(.*?)\} moe_config_t;", src, re.S).group(1)
    names = re.findall(r"\b([A-Za-z_]+)\s*[,;]", body)
    assert [n for n, _ in M.MoeConfig._fields_] == names
    assert ctypes.sizeof(M.MoeConfig) == 4 * len(names)


@pytest.mark.parametrize("field,value,code", [
    ("K", 0, M.MOE_ERR_INVALID_ARG), ("K", 9, M.MOE_ERR_INVALID_ARG),      # K > E
    ("S", 3, M.MOE_ERR_INVALID_ARG),                                       # E % S != 0
    ("capacity", -1, M.MOE_ERR_INVALID_ARG), ("row_align", 0, M.MOE_ERR_INVALID_ARG),
    ("T", -5, M.MOE_ERR_INVALID_ARG), ("act_dtype", 7, M.MOE_ERR_INVALID_ARG),
    ("H", 4100, M.MOE_ERR_UNSUPPORTED),                                    # bf16 GEMM needs H % 64
    ("F", 100, M.MOE_ERR_UNSUPPORTED), ("row_align", 4096, M.MOE_ERR_UNSUPPORTED),
])
def test_invalid_configs_are_rejected(field, value, code):
    cfg = cfg_of(W.WORKLOADS["mixtral"])
    setattr(cfg, field, value)
    assert M.moe_check_config(cfg) == code


def test_too_many_experts_unsupported():
    cfg = M.make_config(T=16, H=64, E=2048, K=2, F=64, S=1, capacity=4)
    assert M.moe_check_config(cfg) == M.MOE_ERR_UNSUPPORTED
    cfg = M.make_config(T=16, H=64, E=64, K=33, F=64, S=1, capacity=4)
    assert M.moe_check_config(cfg) == M.MOE_ERR_UNSUPPORTED


def test_entry_points_reject_bad_arguments_before_any_launch():
    lib = M.LIB
    cfg = cfg_of(W.WORKLOADS["tiny"])
    nul = None
    # null config
    assert lib.moe_dispatch(None, nul, nul, nul, nul) == M.MOE_ERR_INVALID_ARG
    # null buffers
    assert lib.moe_dispatch(ctypes.byref(cfg), nul, nul, nul, nul) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(ctypes.byref(cfg), nul, nul, nul, nul, nul) == M.MOE_ERR_INVALID_ARG
    # a missing or misaligned workspace
    fake = ctypes.c_void_p(0x10000)
    args = [ctypes.byref(cfg)] + [fake] * 10 + [None, 0, None]
    assert lib.moe_route_topk(*args) == M.MOE_ERR_WORKSPACE
    args = [ctypes.byref(cfg)] + [fake] * 10 + [ctypes.c_void_p(0x10010), 1 << 30, None]
    assert lib.moe_route_topk(*args) == M.MOE_ERR_WORKSPACE
    small = M.moe_route_workspace_bytes(cfg) - 256
    args = [ctypes.byref(cfg)] + [fake] * 10 + [fake, small, None]
    assert lib.moe_route_topk(*args) == M.MOE_ERR_WORKSPACE
    # layer: flags that are not defined
    assert lib.moe_layer_forward(ctypes.byref(cfg), fake, fake, fake, fake, fake, 7, fake,
                                 1 << 40, None, None) == M.MOE_ERR_UNSUPPORTED
    assert lib.moe_workspace_init(None, 0, None) == M.MOE_ERR_WORKSPACE
    st = ctypes.c_int(0)
    assert lib.moe_get_device_status(None, ctypes.byref(st), None) == M.MOE_ERR_INVALID_ARG


def test_overlap_flag_needs_bf16_and_128_row_alignment():
    lib = M.LIB
    fake = ctypes.c_void_p(0x10000)
    for A, act in ((1, "bf16"), (64, "bf16"), (128, "f32")):
        cfg = M.make_config(T=256, H=128, E=8, K=2, F=128, S=2, capacity=64, row_align=A, act=act)
        assert lib.moe_layer_forward(ctypes.byref(cfg), fake, fake, fake, fake, fake,
                                     M.MOE_FLAG_OVERLAP, fake, 1 << 40, None, None) == M.MOE_ERR_UNSUPPORTED
    cfg = M.make_config(T=256, H=128, E=8, K=2, F=128, S=2, capacity=64, row_align=1)
    assert lib.moe_combine_wait(ctypes.byref(cfg), fake, fake, fake, fake, 1, fake, 10, fake,
                                256, None) == M.MOE_ERR_UNSUPPORTED
    cfg.row_align = 128
    assert lib.moe_combine_wait(ctypes.byref(cfg), fake, fake, fake, None, 1, fake, 10, fake,
                                256, None) == M.MOE_ERR_INVALID_ARG


def test_status_strings():
    for code in range(7):
        s = M.status_string(code)
        assert s and s != "unknown status"
    assert M.status_string(99) == "unknown status"


def test_fp8_scale_bytes():
    assert M.moe_fp8_scale_bytes(1, 128) == 512
    assert M.moe_fp8_scale_bytes(128, 512) == 512
    assert M.moe_fp8_scale_bytes(128, 640) == 1024
    assert M.moe_fp8_scale_bytes(129, 7168) == 2 * 14 * 512
    assert M.moe_fp8_scale_bytes(0, 128) == 0
    assert M.moe_fp8_scale_bytes(10, 100) == -1 and M.moe_fp8_scale_bytes(-1, 128) == -1


@pytest.mark.parametrize("kw,code", [
    (dict(act="f32"), M.MOE_ERR_UNSUPPORTED),
    (dict(H=4224), M.MOE_ERR_UNSUPPORTED),          # H % 256 != 0
    (dict(F=14400), M.MOE_ERR_UNSUPPORTED),         # F % 128 != 0
    (dict(row_align=64), M.MOE_ERR_UNSUPPORTED),
    (dict(E=640, K=2, S=8), M.MOE_ERR_UNSUPPORTED),
])
def test_fp8_configs_outside_the_kernels_are_rejected(kw, code):
    w = W.WORKLOADS["mixtral"]
    cfg = cfg_of(w, **kw)
    fake = ctypes.c_void_p(0x10000)
    assert M.LIB.moe_layer_forward_fp8(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake, fake,
                                       0, fake, 1 << 40, None, None) == code
    assert M.LIB.moe_dispatch_fp8(ctypes.byref(cfg), fake, fake, fake, fake, None) == code


def test_fp8_entry_points_reject_bad_arguments():
    lib = M.LIB
    cfg = cfg_of(W.WORKLOADS["mixtral"])
    fake = ctypes.c_void_p(0x10000)
    assert lib.moe_quantize_fp8(fake, 10, 100, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_quantize_fp8(None, 10, 128, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_quantize_fp8(fake, 0, 128, None, None, None) == M.MOE_OK
    assert lib.moe_dispatch_fp8(ctypes.byref(cfg), None, fake, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_forward_fp8(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake, fake,
                                     M.MOE_FLAG_OVERLAP, fake, 1 << 40, None, None) == M.MOE_ERR_UNSUPPORTED
    assert lib.moe_layer_forward_fp8(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake, fake,
                                     0, fake, 1024, None, None) == M.MOE_ERR_WORKSPACE


@pytest.mark.parametrize("T,b", [(1, 32), (9472, 32), (9473, 64), (18944, 64), (18945, 128),
                                 (131072, 128)])
def test_route_workspace_follows_the_route_block_size(T, b):
    # the route's scratch is ceil(T/b) * E int32 counters, b the tokens of a
    # top-K block: 32 up to 9472 tokens, 64 up to 18944, else 128 (moe.h)
    E = 64
    cfg = M.make_config(T=T, H=64, E=E, K=2, F=64, S=1, capacity=8)
    nblk = -(-T // b)
    assert M.moe_route_workspace_bytes(cfg) == 256 + (-(-(nblk * E * 4) // 256)) * 256
