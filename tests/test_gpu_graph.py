"""The fused layer captured in a CUDA graph and replayed on new inputs.

A serving loop replays one captured step instead of launching its kernels
again. Every entry point only enqueues work on the caller's stream (no
allocation, no host synchronisation, the counts never leave the device), so
moe_layer_forward, its overlapped form and moe_layer_forward_fp8 can be
captured once and replayed: each replay on new inputs, copied into the
captured input buffers, must give bit for bit what an eager call gives. The
expert-parallel step (W ranks emulated on one device) is captured with the
ranks' device-resident step counters (epoch 0), so that every replay is a new
step.
"""
import pytest
import torch

import combine_moe_route_13_b200 as M
from combine_moe_route_13_b200.ep import EpOnOneDevice
import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _setup(T=512, H=256, E=8, K=2, F=256):
    wl = W.small_case(T, H, E, K, F, 2, 1.25, "bf16", 128)
    C = M.moe_capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = M.make_config(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align, wl.act)
    return wl, cfg, W.make_inputs(wl, seed=3, device=DEV)


def _check_replays(wl, cfg, run, ws_bytes):
    """run(logits, x, out, ws) enqueues one layer; captured once, replayed on
    two new inputs and compared with eager calls."""
    inp = W.make_inputs(wl, seed=3, device=DEV, weights=False)
    logits_s, x_s = inp["logits"].clone(), inp["x"].clone()
    ws = M.alloc_workspace(ws_bytes)
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=DEV)
    run(logits_s, x_s, out, ws)        # eager once: one-time attributes are set outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(logits_s, x_s, out, ws)
    ws_ref = M.alloc_workspace(ws_bytes)
    ref = torch.empty_like(out)
    for seed in (4, 5):
        new = W.make_inputs(wl, seed=seed, device=DEV, weights=False)
        logits_s.copy_(new["logits"])
        x_s.copy_(new["x"])
        g.replay()
        run(new["logits"], new["x"], ref, ws_ref)
        torch.cuda.synchronize()
        assert M.moe_get_device_status(ws) == M.MOE_OK
        assert torch.equal(out, ref), f"replay on seed {seed} differs from the eager call"


@pytest.mark.parametrize("flags", [M.MOE_FLAG_NONE, M.MOE_FLAG_OVERLAP])
def test_layer_forward_in_a_graph(cuda_ok, flags):
    wl, cfg, inp = _setup()
    w_gu, w_d = inp["w_gu"], inp["w_d"]
    _check_replays(wl, cfg,
                   lambda lg, x, out, ws: M.moe_layer_forward(cfg, lg, x, w_gu, w_d, out, ws,
                                                              flags=flags),
                   M.moe_workspace_bytes(cfg, flags))


def test_layer_forward_fp8_in_a_graph(cuda_ok):
    wl, cfg, inp = _setup()
    wq = M.quantize_fp8(inp["w_gu"]) + M.quantize_fp8(inp["w_d"])
    _check_replays(wl, cfg,
                   lambda lg, x, out, ws: M.moe_layer_forward_fp8(cfg, lg, x, *wq, out, ws),
                   M.moe_workspace_bytes(cfg))


@pytest.mark.parametrize("fp8", [False, True])
def test_expert_parallel_step_in_a_graph(cuda_ok, fp8):
    Wn = 2
    wl, cfg, inp = _setup()
    El = wl.E // Wn
    if fp8:
        gq, gs = M.quantize_fp8(inp["w_gu"])
        dq, ds = M.quantize_fp8(inp["w_d"])
        lg = M.ep_local_fp8_weights(gq, gs, Wn, wl.E, 2 * wl.F, wl.H)
        ld = M.ep_local_fp8_weights(dq, ds, Wn, wl.E, wl.H, wl.F)
        wq = [lg[r] + ld[r] for r in range(Wn)]
    else:
        wg = [inp["w_gu"][r * El:(r + 1) * El] for r in range(Wn)]
        wd = [inp["w_d"][r * El:(r + 1) * El] for r in range(Wn)]
    emu = EpOnOneDevice(cfg, Wn, DEV, device_epoch=True)
    first = [W.make_inputs(wl, seed=20 + r, device=DEV, weights=False) for r in range(Wn)]
    logits_s = [f["logits"].clone() for f in first]
    x_s = [f["x"].clone() for f in first]
    outs = [torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=DEV) for _ in range(Wn)]

    def step():
        if fp8:
            emu.forward_fp8(logits_s, x_s, wq, outs)
        else:
            emu.forward(logits_s, x_s, wg, wd, outs)

    step()                            # eager once (step 1 of the counters)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    ws_ref = M.alloc_workspace(M.moe_workspace_bytes(cfg))
    ref = torch.empty_like(outs[0])
    for seed in (30, 40, 50):
        new = [W.make_inputs(wl, seed=seed + r, device=DEV, weights=False) for r in range(Wn)]
        for r in range(Wn):
            logits_s[r].copy_(new[r]["logits"])
            x_s[r].copy_(new[r]["x"])
        g.replay()
        torch.cuda.synchronize()
        for r in range(Wn):
            assert emu.status(r) == M.MOE_OK, M.status_string(emu.status(r))
            if fp8:
                M.moe_layer_forward_fp8(cfg, new[r]["logits"], new[r]["x"], gq, gs, dq, ds, ref,
                                        ws_ref)
            else:
                M.moe_layer_forward(cfg, new[r]["logits"], new[r]["x"], inp["w_gu"], inp["w_d"],
                                    ref, ws_ref)
            torch.cuda.synchronize()
            assert torch.equal(outs[r], ref), f"replay {seed}, rank {r}"
