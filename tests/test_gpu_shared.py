"""GPU parity of the shared expert (n_shared = 1): an expert that every token
uses with weight 1 next to its routed ones, run as one more group of the
grouped GEMMs and added by the combine.

* route: the routed outputs equal the oracle's bit for bit; row_src marks the
  gap before the shared rows with -1 and the shared rows with T*K + t;
* dispatch: the shared rows of xp are x itself, bit for bit;
* expert MLP: routed rows against the oracle per expert, shared rows against
  the oracle's SwiGLU of x with the last expert's weights;
* combine and the whole layer: against the oracle's combine with the shared
  output added (on the GPU's own y), and the whole chain within a relative
  Frobenius error of 1e-2 of the oracle's layer with n_shared = 1.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from oracle import moe_oracle as O
import workloads as W
from _gpu_common import act_np, assert_close_act, assert_route_equal, host, run_route

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    W.WORKLOADS["tiny"].with_(n_shared=1),
    W.small_case(300, 256, 8, 2, 256, 2, 1.0, "bf16", 128, n_shared=1),      # 128-row tiles
    W.small_case(2048, 256, 4, 2, 192, 2, 1.25, "bf16", 1, n_shared=1),      # pair tiles, N tail
    W.small_case(700, 384, 12, 3, 192, 4, 0.8, "bf16", 1, bias="zipf1.2", n_shared=1),
    W.small_case(200, 128, 8, 2, 128, 2, 0.0, "bf16", 16, n_shared=1),       # C = 0: shared only
    W.small_case(333, 128, 16, 4, 128, 8, 1.0, "f32", 4, n_shared=1),
]


def _cfg(wl, C):
    return M.make_config(T=wl.T, H=wl.H, E=wl.E, K=wl.K, F=wl.F, S=wl.S, capacity=C,
                         row_align=wl.row_align, act=wl.act, n_shared=wl.n_shared)


def _check_row_src(rs: np.ndarray, R_r: int, R_sh: int, T: int, K: int):
    assert np.all(rs[R_r:R_sh] == -1)
    assert np.array_equal(rs[R_sh:R_sh + T], T * K + np.arange(T))


def _check_shared_mlp(h, y, x, wl, R_sh, w_gu, w_d):
    """Shared rows of h and y against the oracle's SwiGLU of x with expert E."""
    he, ye = O.expert_mlp_rows(x, w_gu[wl.E], w_d[wl.E], wl.act)
    assert_close_act(h[R_sh:R_sh + wl.T], he, wl.act, "h shared")
    assert_close_act(y[R_sh:R_sh + wl.T], ye, wl.act, "y shared")


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_stage_api_with_shared_expert(cuda_ok, wl):
    C = O.capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = _cfg(wl, C)
    inp = W.make_inputs(wl, seed=wl.T + 1, device=DEV)
    r = run_route(cfg, inp["logits"])
    ref = O.route(inp["logits"].cpu().numpy(), wl.K, C, wl.row_align, wl.S)
    R_r, R = ref["R_max"], M.moe_max_rows(cfg)
    R_sh = M.shared_row0(cfg)
    assert R == R_sh + wl.T and R_sh % 128 == 0 and R_sh >= R_r
    g = host(r)
    assert_route_equal(g, ref, R_r)
    _check_row_src(g["row_src"], R_r, R_sh, wl.T, wl.K)

    dt = wl.torch_act
    xp = torch.zeros(R, wl.H, dtype=dt, device=DEV)
    h = torch.zeros(R, wl.F, dtype=dt, device=DEV)
    y = torch.zeros(R, wl.H, dtype=dt, device=DEV)
    out = torch.empty(wl.T, wl.H, dtype=dt, device=DEV)
    ws = M.alloc_workspace(256)
    M.moe_dispatch(cfg, inp["x"], r["token_slot"], xp)
    M.moe_expert_mlp(cfg, xp, r["expert_offsets"], r["expert_counts"], inp["w_gu"], inp["w_d"],
                     h, y, ws)
    M.moe_combine(cfg, y, r["token_slot"], r["topk_w"], out)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    x_n, xp_n, h_n, y_n = act_np(inp["x"]), act_np(xp), act_np(h), act_np(y)
    w_gu, w_d = act_np(inp["w_gu"]), act_np(inp["w_d"])
    # dispatch: routed rows and the shared copy of x, bit for bit
    kept = ref["row_src"] >= 0
    assert np.array_equal(xp_n[:R_r][kept], O.dispatch(x_n, ref["token_slot"], R_r)[kept])
    assert np.array_equal(xp_n[R_sh:], x_n)
    # routed experts
    h_ref, y_ref = O.expert_mlp(xp_n[:R_r], ref["expert_offsets"], ref["kept"], w_gu[:wl.E],
                                w_d[:wl.E], wl.act)
    assert_close_act(h_n[:R_r][kept], h_ref[kept], wl.act, "h routed")
    assert_close_act(y_n[:R_r][kept], y_ref[kept], wl.act, "y routed")
    _check_shared_mlp(h_n, y_n, x_n, wl, R_sh, w_gu, w_d)
    # combine of the GPU's own y, shared output added
    ref_out = O.combine(y_n, ref["token_slot"], ref["topk_w"], wl.act, y_shared=y_n[R_sh:])
    assert_close_act(act_np(out), ref_out, wl.act, "out")


@pytest.mark.parametrize("overlap", [False, True])
@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_layer_forward_with_shared_expert(cuda_ok, wl, overlap):
    if overlap and (wl.act != "bf16" or wl.row_align % 128):
        pytest.skip("the overlapped combine needs bf16 and 128-row alignment")
    C = O.capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = _cfg(wl, C)
    inp = W.make_inputs(wl, seed=wl.T + 2, device=DEV)
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg))
    out = torch.empty(wl.T, wl.H, dtype=wl.torch_act, device=DEV)
    flags = M.MOE_FLAG_OVERLAP if overlap else M.MOE_FLAG_NONE
    aux = M.moe_layer_forward(cfg, inp["logits"], inp["x"], inp["w_gu"], inp["w_d"], out, ws,
                              flags=flags)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    v = M.layer_views(cfg, ws, aux)
    x_n, w_gu, w_d = act_np(inp["x"]), act_np(inp["w_gu"]), act_np(inp["w_d"])
    ref_out, ref = O.layer_forward(inp["logits"].cpu().numpy(), x_n, w_gu, w_d, wl.K, C,
                                   wl.row_align, wl.S, wl.act, n_shared=1)
    R_r, R_sh = ref["R_max"], M.shared_row0(cfg)
    g = host({k: v[k] for k in ("topk_idx", "topk_w", "expert_counts", "overflow",
                                "expert_offsets", "segment_offsets", "token_slot", "row_src",
                                "totals")})
    assert_route_equal(g, ref, R_r)
    _check_row_src(g["row_src"], R_r, R_sh, wl.T, wl.K)
    xp_n, h_n, y_n, out_n = act_np(v["xp"]), act_np(v["h"]), act_np(v["y"]), act_np(out)
    kept = ref["row_src"] >= 0
    assert np.array_equal(xp_n[:R_r][kept], ref["xp"][kept])
    _, y_ref = O.expert_mlp(xp_n[:R_r], ref["expert_offsets"], ref["kept"], w_gu[:wl.E],
                            w_d[:wl.E], wl.act)
    assert_close_act(y_n[:R_r][kept], y_ref[kept], wl.act, "y routed")
    _check_shared_mlp(h_n, y_n, x_n, wl, R_sh, w_gu, w_d)
    ref_from_gpu_y = O.combine(y_n, ref["token_slot"], ref["topk_w"], wl.act,
                               y_shared=y_n[R_sh:])
    assert_close_act(out_n, ref_from_gpu_y, wl.act, "out")
    gd, rd = O.act_to_f64(out_n, wl.act), O.act_to_f64(ref_out, wl.act)
    fro = np.sqrt(np.sum((gd - rd) ** 2)) / max(np.sqrt(np.sum(rd * rd)), 1e-300)
    assert fro <= 1e-2, f"whole chain: relative Frobenius error {fro:.3e}"
