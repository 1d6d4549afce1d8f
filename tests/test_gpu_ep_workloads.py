"""Expert-parallel layer at the workloads' full per-rank sizes, W ranks
emulated on one device (the launch configuration `bench.py --ep-emulate W`
times): every rank's route bit for bit against the oracle, the exchanged
counts and the layout bit for bit against the oracle's plan, sampled received
rows bit for bit against the senders' token rows, and every rank's output
bit for bit equal to the one-rank library layer over all E experts (which the
one-rank tests check against the oracle)."""
import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from combine_moe_route_13_b200.ep import EpOnOneDevice
from oracle import moe_oracle as O
from oracle import moe_oracle_ep as P
import workloads as W
from _gpu_common import act_np, assert_route_equal, host

pytestmark = pytest.mark.gpu
ROUTE_KEYS = ("topk_idx", "topk_w", "expert_counts", "overflow", "expert_offsets",
              "segment_offsets", "token_slot", "row_src", "totals")


@pytest.mark.parametrize("name,world", [("mixtral", 2), ("dsv3", 8), ("skewed", 4)])
def test_workload_full_size_ep(cuda_ok, name, world):
    wl = W.WORKLOADS[name]
    dev = torch.device("cuda")
    C = M.moe_capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = M.make_config(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align, wl.act)
    full = W.make_inputs(wl, seed=0, device=dev)
    inps = [full] + [W.make_inputs(wl, seed=r, device=dev, weights=False) for r in range(1, world)]
    El = wl.E // world
    emu = EpOnOneDevice(cfg, world, dev)
    outs = [torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev) for _ in range(world)]
    emu.forward([i["logits"] for i in inps], [i["x"] for i in inps],
                [full["w_gu"][r * El:(r + 1) * El] for r in range(world)],
                [full["w_d"][r * El:(r + 1) * El] for r in range(world)], outs)
    torch.cuda.synchronize()
    routes = []
    for r in range(world):
        assert emu.status(r) == M.MOE_OK
        ref = O.route(inps[r]["logits"].cpu().numpy(), wl.K, C, wl.row_align, wl.S)
        assert_route_equal(host({k: emu.views(r)[k] for k in ROUTE_KEYS}), ref, ref["R_max"])
        routes.append(ref)
    counts_all = np.stack([r["expert_counts"] for r in routes])
    rng = np.random.default_rng(0)
    for d in range(world):
        v = emu.views(d)
        plan = P.ep_plan(counts_all, C, wl.row_align, d)
        assert np.array_equal(v["counts_all"].cpu().numpy(), counts_all)
        for k in ("send_dst_row", "recv_offsets", "recv_counts"):
            assert np.array_equal(v[k].cpu().numpy(), plan[k]), (d, k)
        # sampled received rows: the sender's token row, bit for bit
        xr = v["xr"]
        for s in range(world):
            r = routes[s]
            pairs = np.argwhere(r["token_slot"] >= 0)
            mine = [(t, k) for t, k in pairs if r["topk_idx"][t, k] // El == d]
            if not mine:
                continue
            send = P.ep_plan(counts_all, C, wl.row_align, s)["send_dst_row"]
            for i in rng.choice(len(mine), min(24, len(mine)), replace=False):
                t, k = mine[i]
                e = int(r["topk_idx"][t, k])
                row = int(send[e]) + int(r["token_slot"][t, k]) - int(r["expert_offsets"][e])
                assert torch.equal(xr[row], inps[s]["x"][t]), (d, s, t, k)
    # every rank's output equals the one-rank layer of its tokens over all E experts
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg), dev)
    ref_out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev)
    for r in range(world):
        M.moe_layer_forward(cfg, inps[r]["logits"], inps[r]["x"], full["w_gu"], full["w_d"],
                            ref_out, ws)
        assert M.moe_get_device_status(ws) == M.MOE_OK
        g, w = act_np(outs[r]), act_np(ref_out)
        assert np.array_equal(g, w), f"rank {r}: {(g != w).sum()} elements differ"
    del emu, full, inps, outs, ws
    torch.cuda.empty_cache()
