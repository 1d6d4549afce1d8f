"""Parity at the workloads' full sizes, through moe_layer_forward (the call and
launch configuration bench.py times).

* route outputs: compared with the oracle in full, bit for bit;
* dispatch: every kept row of xp equals its source token row (a property that
  holds at any size, checked on the device in full);
* expert MLP: h and y rows of sampled experts (the fullest, the emptiest
  non-empty one and random ones; first, last and random rows of each) against
  the oracle's SwiGLU on the same xp rows;
* combine: sampled tokens against the oracle's weighted sum of the GPU's y rows.

DeepSeek-V3 and Kimi-K2 also run with their shared expert (n_shared = 1): its
rows of h and y are sampled like an expert's, from x, and the combine adds
them.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from oracle import moe_oracle as O
import workloads as W
from _gpu_common import act_np, assert_close_act, assert_route_equal, host

pytestmark = pytest.mark.gpu
ROUTE_KEYS = ("topk_idx", "topk_w", "expert_counts", "overflow", "expert_offsets",
              "segment_offsets", "token_slot", "row_src", "totals")


@pytest.mark.parametrize("name,n_shared", [("mixtral", 0), ("dsv3", 0), ("skewed", 0),
                                           ("kimi", 0), ("dsv3", 1), ("kimi", 1)])
def test_workload_full_size(cuda_ok, name, n_shared):
    wl = W.WORKLOADS[name].with_(n_shared=n_shared)
    dev = torch.device("cuda")
    C = M.moe_capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = M.make_config(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align, wl.act,
                        n_shared=n_shared)
    inp = W.make_inputs(wl, seed=0, device=dev)
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg), dev)
    out = torch.empty(wl.T, wl.H, dtype=wl.torch_act, device=dev)
    aux = M.moe_layer_forward(cfg, inp["logits"], inp["x"], inp["w_gu"], inp["w_d"], out, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    v = M.layer_views(cfg, ws, aux)

    # route, in full
    ref = O.route(inp["logits"].cpu().numpy(), wl.K, C, wl.row_align, wl.S)
    R_max = ref["R_max"]
    assert_route_equal(host({k: v[k] for k in ROUTE_KEYS}), ref, R_max)

    R_sh = M.shared_row0(cfg)
    if n_shared:   # the shared rows' ids, in full
        assert torch.all(v["row_src"][R_max:R_sh] == -1)
        assert torch.equal(v["row_src"][R_sh:].cpu(),
                           torch.arange(wl.T, dtype=torch.int32) + wl.T * wl.K)

    # dispatch, in full on the device: xp[row] == x[row_src[row] // K]
    rs = v["row_src"][:R_max]
    rows = torch.nonzero(rs >= 0).squeeze(1)
    assert rows.numel() == int(ref["totals"][1])
    src_tok = (rs[rows] // wl.K).long()
    assert torch.equal(v["xp"][rows].view(torch.int16), inp["x"][src_tok].view(torch.int16))

    # expert MLP on sampled experts and rows
    rng = np.random.default_rng(0)
    kept = np.minimum(ref["expert_counts"], C)
    off = ref["expert_offsets"]
    nonempty = np.nonzero(kept)[0]
    experts = {int(nonempty[np.argmax(kept[nonempty])]), int(nonempty[np.argmin(kept[nonempty])])}
    experts |= set(int(e) for e in rng.choice(nonempty, min(6, len(nonempty)), replace=False))
    for e in sorted(experts):
        n = int(kept[e])
        pick = np.unique(np.concatenate([np.arange(min(4, n)), np.arange(max(0, n - 4), n),
                                         rng.integers(0, n, 8)]))
        rws = off[e] + pick
        xp_rows = act_np(v["xp"][torch.from_numpy(rws).to(dev)])
        he, ye = O.expert_mlp_rows(xp_rows, act_np(inp["w_gu"][e]), act_np(inp["w_d"][e]), wl.act)
        idx = torch.from_numpy(rws).to(dev)
        assert_close_act(act_np(v["h"][idx]), he, wl.act, f"h[e={e}]")
        assert_close_act(act_np(v["y"][idx]), ye, wl.act, f"y[e={e}]")
    if n_shared:   # the shared expert's rows: first, last and random tokens, from x
        tk = np.unique(np.concatenate([[0, 1, wl.T - 1], rng.integers(0, wl.T, 13)]))
        he, ye = O.expert_mlp_rows(act_np(inp["x"][torch.from_numpy(tk).to(dev)]),
                                   act_np(inp["w_gu"][wl.E]), act_np(inp["w_d"][wl.E]), wl.act)
        idx = torch.from_numpy(R_sh + tk).to(dev)
        assert_close_act(act_np(v["h"][idx]), he, wl.act, "h[shared]")
        assert_close_act(act_np(v["y"][idx]), ye, wl.act, "y[shared]")

    # combine on sampled tokens, from the GPU's y
    toks = np.unique(np.concatenate([[0, wl.T - 1], rng.integers(0, wl.T, 254)]))
    slot = ref["token_slot"][toks]
    need = np.unique(slot[slot >= 0])
    remap = np.full(max(int(slot.max()) + 1, 1), -1, dtype=np.int64)
    remap[need] = np.arange(len(need))
    slot_sub = np.where(slot >= 0, remap[np.maximum(slot, 0)], -1).astype(np.int32)
    y_sub = act_np(v["y"][torch.from_numpy(need).to(dev)]) if len(need) else \
        np.zeros((1, wl.H), np.uint16)
    y_sh = act_np(v["y"][torch.from_numpy(R_sh + toks).to(dev)]) if n_shared else None
    ref_out = O.combine(y_sub, slot_sub, ref["topk_w"][toks], wl.act, y_shared=y_sh)
    got = act_np(out[torch.from_numpy(toks).to(dev)])
    assert_close_act(got, ref_out, wl.act, "out")
    del inp, ws, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("mode", ["bf16", "bf16_overlap", "fp8"])
def test_layer_is_deterministic_run_to_run(cuda_ok, mode):
    # no atomics on any output path: two runs of the whole layer on the same
    # inputs give the same bits (catches races in the scans, scatter and tiles)
    wl = W.WORKLOADS["skewed"]
    dev = torch.device("cuda")
    C = M.moe_capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = M.make_config(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align, wl.act)
    inp = W.make_inputs(wl, seed=3, device=dev)
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg), dev)
    outs = []
    if mode == "fp8":
        gq, gs = M.quantize_fp8(inp["w_gu"])
        dq, ds = M.quantize_fp8(inp["w_d"])
    for _ in range(2):
        out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev)
        ws.zero_()
        if mode == "fp8":
            M.moe_layer_forward_fp8(cfg, inp["logits"], inp["x"], gq, gs, dq, ds, out, ws)
        else:
            flags = M.MOE_FLAG_OVERLAP if mode == "bf16_overlap" else M.MOE_FLAG_NONE
            M.moe_layer_forward(cfg, inp["logits"], inp["x"], inp["w_gu"], inp["w_d"], out, ws,
                                flags=flags)
        assert M.moe_get_device_status(ws) == M.MOE_OK
        outs.append(out.view(torch.int16).clone())
    assert torch.equal(outs[0], outs[1])
