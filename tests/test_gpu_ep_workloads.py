"""Expert-parallel layer at the workloads' full per-rank sizes, W ranks
emulated on one device (the launch configuration `bench.py --ep-emulate W
[--ep-tiles]` times), untagged and tile-signalled: every rank's route bit for bit against the oracle, the exchanged
counts and the layout bit for bit against the oracle's plan, sampled received
rows bit for bit against the senders' token rows, and every rank's output
bit for bit equal to the one-rank library layer over all E experts (which the
one-rank tests check against the oracle). Sampled tokens of every rank are
also checked against the oracle directly, token by token: the owners' y rows
of their kept assignments against the oracle's SwiGLU of the token row with
that expert's weights, the token's output against the oracle's weighted sum
of those GPU y rows, and against the oracle's own chain by relative Frobenius
error (the tolerances of the one-rank layer tests)."""
import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from combine_moe_route_13_b200.ep import EpOnOneDevice
from oracle import moe_oracle as O
from oracle import moe_oracle_ep as P
import workloads as W
from _gpu_common import act_np, assert_close_act, assert_route_equal, host

pytestmark = pytest.mark.gpu
ROUTE_KEYS = ("topk_idx", "topk_w", "expert_counts", "overflow", "expert_offsets",
              "segment_offsets", "token_slot", "row_src", "totals")


TILES = M.MOE_EP_TILE_SIGNAL
REMOTE_FIRST = M.MOE_EP_TILE_SIGNAL | M.MOE_EP_REMOTE_FIRST


@pytest.mark.parametrize("name,world,flags", [
    ("mixtral", 2, 0), ("dsv3", 8, 0), ("skewed", 4, 0),
    # the tile-signalled layer (MOE_EP_TILE_SIGNAL) at the same sizes
    ("mixtral", 2, REMOTE_FIRST), ("dsv3", 8, TILES)])
def test_workload_full_size_ep(cuda_ok, name, world, flags):
    wl = W.WORKLOADS[name]
    dev = torch.device("cuda")
    C = M.moe_capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = M.make_config(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align, wl.act)
    full = W.make_inputs(wl, seed=0, device=dev)
    inps = [full] + [W.make_inputs(wl, seed=r, device=dev, weights=False) for r in range(1, world)]
    El = wl.E // world
    emu = EpOnOneDevice(cfg, world, dev, flags=flags)
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
    # sampled tokens against the oracle, one token at a time
    w_gu_h, w_d_h = {}, {}
    for s in range(world):
        r = routes[s]
        toks = rng.choice(wl.T, 6, replace=False)
        g_y, o_y, g_out, o_out, o_chain = [], [], [], [], []
        for t in toks:
            rows_gpu, rows_ref = [], []
            for k in range(wl.K):
                sl = int(r["token_slot"][t, k])
                if sl < 0:
                    continue
                e = int(r["topk_idx"][t, k])
                d = e // El
                send = P.ep_plan(counts_all, C, wl.row_align, s)["send_dst_row"]
                row = int(send[e]) + sl - int(r["expert_offsets"][e])
                if e not in w_gu_h:
                    w_gu_h[e], w_d_h[e] = act_np(full["w_gu"][e]), act_np(full["w_d"][e])
                _, y_ref = O.expert_mlp_rows(act_np(inps[s]["x"][t:t + 1]), w_gu_h[e], w_d_h[e],
                                             wl.act)
                rows_gpu.append(act_np(emu.views(d)["y"][row:row + 1]))
                rows_ref.append(y_ref)
            slot1 = np.full((1, wl.K), -1, np.int32)
            kept_k = [k for k in range(wl.K) if r["token_slot"][t, k] >= 0]
            slot1[0, kept_k] = np.arange(len(kept_k))
            w1 = r["topk_w"][t:t + 1]
            ygpu = np.concatenate(rows_gpu) if rows_gpu else np.zeros((0, wl.H), np.uint16)
            yref = np.concatenate(rows_ref) if rows_ref else np.zeros((0, wl.H), np.uint16)
            g_y.append(ygpu)
            o_y.append(yref)
            g_out.append(act_np(outs[s][t:t + 1]))
            o_out.append(O.combine(ygpu, slot1, w1, wl.act))
            o_chain.append(O.combine(yref, slot1, w1, wl.act))
        assert_close_act(np.concatenate(g_y), np.concatenate(o_y), wl.act, f"rank {s} y")
        assert_close_act(np.concatenate(g_out), np.concatenate(o_out), wl.act, f"rank {s} out")
        g = O.act_to_f64(np.concatenate(g_out), wl.act)
        c = O.act_to_f64(np.concatenate(o_chain), wl.act)
        fro = np.sqrt(np.sum((g - c) ** 2)) / max(np.sqrt(np.sum(c * c)), 1e-300)
        assert fro <= 1e-2, f"rank {s}: whole chain relative Frobenius error {fro:.3e}"
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
