"""Router projection (logits = x W_g^T, fp32) and the selection-only bias,
through the C ABI, against the CPU oracle.

Logits are floating point: max|err| <= 1e-5 * max|ref| (the fp32 rule).
Routing decisions are compared bit for bit on the same fp32 logits (the
GPU's), so that both sides take each decision in the same precision.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from oracle import moe_oracle as O
import workloads as W
from _gpu_common import act_np, assert_layer_stages, assert_route_equal, host

pytestmark = pytest.mark.gpu


def _logits_close(got, ref):
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64)).max()
    assert err <= 1e-5 * np.abs(ref).max(), (err, np.abs(ref).max())


@pytest.mark.parametrize("T,H,E,act", [
    (300, 256, 8, "bf16"), (1024, 7168, 256, "bf16"), (513, 512, 384, "bf16"),
    (200, 320, 17, "bf16"), (4096, 4096, 8, "bf16"), (64, 128, 8, "f32"), (77, 96, 5, "f32")])
def test_router_logits(cuda_ok, T, H, E, act):
    wl = W.small_case(T, H, E, 2, 64, 1, 1.0, act, 128)
    inp = W.make_inputs(wl, seed=T + E, device="cuda", weights=False, router=True)
    cfg = M.make_config(T, H, E, 2, 64, 1, 64, 128, act)
    logits = torch.full((T, E), float("nan"), device="cuda")
    ws = M.alloc_workspace(256)
    M.moe_router_logits(cfg, inp["x"], inp["w_g"], logits, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    ref = O.router_logits(act_np(inp["x"]), act_np(inp["w_g"]), act)
    _logits_close(logits.cpu().numpy(), ref)


@pytest.mark.parametrize("T,E,K,S,cf,A", [(1000, 64, 6, 8, 1.0, 128), (513, 384, 8, 16, 1.25, 128),
                                          (300, 17, 3, 1, 0.8, 1)])
def test_route_with_selection_bias(cuda_ok, T, E, K, S, cf, A):
    g = torch.Generator().manual_seed(T + E)
    lg = torch.randn(T, E, generator=g)
    bias = torch.randn(E, generator=g) * 0.5
    C = O.capacity(T, K, E, cf)
    cfg = M.make_config(T, 64, E, K, 64, S, C, A, "bf16")
    out = M.alloc_route_outputs(cfg)
    ws = M.alloc_workspace(M.moe_route_workspace_bytes(cfg))
    M.moe_route_topk_biased(cfg, lg.cuda(), bias.cuda(), out["topk_idx"], out["topk_w"],
                            out["expert_counts"], out["overflow"], out["expert_offsets"],
                            out["segment_offsets"], out["token_slot"], out["row_src"],
                            out["totals"], ws)
    ref = O.route(lg.numpy(), K, C, A, S, sel_bias=bias.numpy())
    assert_route_equal(host(out), ref, ref["R_max"])
    plain = O.route(lg.numpy(), K, C, A, S)
    assert not np.array_equal(plain["topk_idx"], ref["topk_idx"])   # the bias mattered


@pytest.mark.parametrize("wl", [
    W.small_case(600, 512, 16, 4, 256, 4, 1.25, "bf16", 128),
    W.small_case(300, 256, 8, 2, 128, 2, 1.0, "bf16", 1),
    W.small_case(64, 128, 8, 2, 256, 2, 1.25, "f32", 1),
], ids=lambda w: w.name)
@pytest.mark.parametrize("biased", [False, True])
def test_layer_forward_from_hidden_states(cuda_ok, wl, biased):
    inp = W.make_inputs(wl, seed=3, device="cuda", router=True)
    C = M.moe_capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = M.make_config(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align, wl.act)
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg))
    out = torch.empty(wl.T, wl.H, dtype=wl.torch_act, device="cuda")
    bias = inp["sel_bias"] if biased else None
    aux = M.moe_layer_forward_x(cfg, inp["x"], inp["w_g"], bias, inp["w_gu"], inp["w_d"], out, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    v = M.layer_views(cfg, ws, aux)
    gpu_logits = v["logits"].cpu().numpy()
    _logits_close(gpu_logits, O.router_logits(act_np(inp["x"]), act_np(inp["w_g"]), wl.act))
    r = O.route(gpu_logits, wl.K, C, wl.row_align, wl.S,
                sel_bias=bias.cpu().numpy() if biased else None)
    xp = O.dispatch(act_np(inp["x"]), r["token_slot"], r["R_max"])
    h, y = O.expert_mlp(xp, r["expert_offsets"], r["kept"], act_np(inp["w_gu"]),
                        act_np(inp["w_d"]), wl.act)
    ref_out = O.combine(y, r["token_slot"], r["topk_w"], wl.act)
    r.update(xp=xp, h=h, y=y)
    assert_route_equal(host({k: v[k] for k in ("topk_idx", "topk_w", "expert_counts", "overflow",
                                                "expert_offsets", "segment_offsets", "token_slot",
                                                "row_src", "totals")}), r, r["R_max"])
    assert_layer_stages({"xp": act_np(v["xp"]), "y": act_np(v["y"])}, act_np(out),
                        act_np(inp["x"]), act_np(inp["w_gu"]), act_np(inp["w_d"]), r, ref_out,
                        wl.act)
