"""GPU parity of the expert-parallel layer with the fp8 payload
(moe_ep_dispatch_fp8, moe_ep_expert_mlp_fp8), W ranks emulated on one device:

* the layout bit for bit against the oracle's plan;
* the received codes and scales bit for bit against the fp8 oracle's
  quantisation of the senders' token rows (every kept row);
* every rank's output bit for bit equal to the one-rank fp8 layer
  (moe_layer_forward_fp8) of its tokens over all E experts, which the fp8
  tests check against the fp8 oracle; and the whole chain within a relative
  Frobenius error of 1e-2 of the fp8 oracle's layer on two ranks;
* at the Mixtral shape with two ranks (untagged, tile-signalled and
  remote-first), bit for bit the one-rank fp8 layer;
* with a shared expert (every rank applies it to its own tokens), bit for bit
  the one-rank fp8 layer with the shared expert.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from combine_moe_route_13_b200.ep import EpOnOneDevice
from oracle import moe_oracle as O
from oracle import moe_oracle_ep as P
from oracle import moe_oracle_fp8 as Q
import workloads as W_
from _gpu_common import act_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def np_u8(t):
    return t.detach().cpu().contiguous().numpy()


def fp8_one_rank(cfg, logits, x, wq):
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg))
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
    M.moe_layer_forward_fp8(cfg, logits, x, *wq, out, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    return out


def run_case(W, T, H, E, K, F, cf, seed, check_rows=True, n_shared=0):
    C = O.capacity(T, K, E, cf)
    cfg = M.make_config(T=T, H=H, E=E, K=K, F=F, S=W, capacity=C, row_align=128, act="bf16",
                        n_shared=n_shared)
    g = torch.Generator().manual_seed(seed)
    logits = [torch.randn(T, E, generator=g).to(DEV) for _ in range(W)]
    xs = [torch.randn(T, H, generator=g).to(torch.bfloat16).to(DEV) for _ in range(W)]
    w_gu = (torch.randn(E + n_shared, 2 * F, H, generator=g) * 0.05).to(torch.bfloat16).to(DEV)
    w_d = (torch.randn(E + n_shared, H, F, generator=g) * 0.05).to(torch.bfloat16).to(DEV)
    gq, gs = M.quantize_fp8(w_gu)
    dq, ds = M.quantize_fp8(w_d)
    loc_gu = M.ep_local_fp8_weights(gq, gs, W, E, 2 * F, H, n_shared)
    loc_d = M.ep_local_fp8_weights(dq, ds, W, E, H, F, n_shared)
    wq = [loc_gu[r] + loc_d[r] for r in range(W)]
    emu = EpOnOneDevice(cfg, W, DEV)
    outs = [torch.full((T, H), float("nan"), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    emu.forward_fp8(logits, xs, wq, outs)
    torch.cuda.synchronize()
    routes = [O.route(l.cpu().numpy(), K, C, 128, W) for l in logits]
    counts_all = np.stack([r["expert_counts"] for r in routes])
    El = E // W
    for r in range(W):
        assert emu.status(r) == M.MOE_OK, M.status_string(emu.status(r))
        v = emu.views(r)
        plan = P.ep_plan(counts_all, C, 128, r)
        for k in ("send_dst_row", "recv_offsets", "recv_counts"):
            assert np.array_equal(v[k].cpu().numpy(), plan[k]), (r, k)
        ref = fp8_one_rank(cfg, logits[r], xs[r], (gq, gs, dq, ds))
        assert torch.equal(outs[r], ref), f"rank {r}: {(outs[r] != ref).sum().item()} differ"
    if check_rows:   # every kept row's codes and scales at its owner
        R = M.moe_ep_recv_rows(cfg, W)
        for d in range(W):
            v = emu.views(d)
            xq = np_u8(v["xq"])
            xe = Q.scales_from_blocked(np_u8(v["xs"]), R, H // 128)
            for s in range(W):
                r = routes[s]
                send = P.ep_plan(counts_all, C, 128, s)["send_dst_row"]
                tq, te = Q.quantize_rows(O.bf16_bits_to_f64(act_np(xs[s])))
                for t, k in zip(*np.nonzero(r["token_slot"] >= 0)):
                    e = int(r["topk_idx"][t, k])
                    if e // El != d:
                        continue
                    row = int(send[e]) + int(r["token_slot"][t, k]) - int(r["expert_offsets"][e])
                    assert np.array_equal(xq[row], tq[t]) and np.array_equal(xe[row], te[t])
    return cfg, emu, outs, logits, xs, (gq, gs, dq, ds), C


@pytest.mark.parametrize("W,T,H,E,K,F,cf", [
    (2, 256, 256, 8, 2, 256, 1.25),
    (4, 300, 512, 16, 4, 384, 0.5),     # overflow
    (8, 64, 256, 64, 8, 128, 1.5),      # many small experts per owner
    (2, 200, 256, 8, 2, 256, 0.0),      # C = 0
])
def test_ep_fp8_layer(cuda_ok, W, T, H, E, K, F, cf):
    run_case(W, T, H, E, K, F, cf, seed=W * 31 + T)


@pytest.mark.parametrize("W,T,H,E,K,F,cf", [
    (2, 256, 256, 8, 2, 256, 1.25),
    (4, 300, 512, 16, 4, 384, 0.5),     # overflow: the shared expert still reaches every token
])
def test_ep_fp8_layer_with_a_shared_expert(cuda_ok, W, T, H, E, K, F, cf):
    # every rank runs the shared expert on its own tokens, quantised with the
    # dispatch's arithmetic: bit for bit the one-rank fp8 layer with a shared expert
    run_case(W, T, H, E, K, F, cf, seed=W * 37 + T, n_shared=1)


def test_ep_fp8_chain_against_the_fp8_oracle(cuda_ok):
    W, T, H, E, K, F = 2, 256, 256, 8, 2, 256
    cfg, emu, outs, logits, xs, (gq, gs, dq, ds), C = run_case(W, T, H, E, K, F, 1.25, seed=5,
                                                               check_rows=False)
    ge = Q.scales_from_blocked(np_u8(gs), E * 2 * F, H // 128).reshape(E, 2 * F, H // 128)
    de = Q.scales_from_blocked(np_u8(ds), E * H, F // 128).reshape(E, H, F // 128)
    for r in range(W):
        ref_out, _ = Q.layer_forward_fp8(logits[r].cpu().numpy(), act_np(xs[r]), np_u8(gq), ge,
                                         np_u8(dq), de, K, C, 128, W)
        g, w = O.bf16_bits_to_f64(act_np(outs[r])), O.bf16_bits_to_f64(ref_out)
        fro = np.linalg.norm(g - w) / np.linalg.norm(w)
        assert fro <= 1e-2, f"rank {r}: relative Frobenius error {fro:.3e}"


@pytest.mark.parametrize("flags", [0, M.MOE_EP_TILE_SIGNAL,
                                   M.MOE_EP_TILE_SIGNAL | M.MOE_EP_REMOTE_FIRST],
                         ids=["untagged", "tiles", "remote_first"])
def test_ep_fp8_mixtral_two_ranks(cuda_ok, flags):
    wl = W_.WORKLOADS["mixtral"]
    W = 2
    dev = torch.device("cuda")
    C = M.moe_capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = M.make_config(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align, wl.act)
    full = W_.make_inputs(wl, seed=0, device=dev)
    inps = [full] + [W_.make_inputs(wl, seed=1, device=dev, weights=False)]
    gq, gs = M.quantize_fp8(full["w_gu"])
    dq, ds = M.quantize_fp8(full["w_d"])
    del full["w_gu"], full["w_d"]
    loc_gu = M.ep_local_fp8_weights(gq, gs, W, wl.E, 2 * wl.F, wl.H)
    loc_d = M.ep_local_fp8_weights(dq, ds, W, wl.E, wl.H, wl.F)
    emu = EpOnOneDevice(cfg, W, dev, flags=flags)
    outs = [torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev) for _ in range(W)]
    emu.forward_fp8([i["logits"] for i in inps], [i["x"] for i in inps],
                    [loc_gu[r] + loc_d[r] for r in range(W)], outs)
    torch.cuda.synchronize()
    for r in range(W):
        assert emu.status(r) == M.MOE_OK
        ref = fp8_one_rank(cfg, inps[r]["logits"], inps[r]["x"], (gq, gs, dq, ds))
        assert torch.equal(outs[r], ref), f"rank {r}"
