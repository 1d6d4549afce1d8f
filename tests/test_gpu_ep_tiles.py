"""The tile-signalled expert-parallel layer (MOE_EP_TILE_SIGNAL, include/moe_ep.h;
the producer/consumer of "Mixture-of-Experts acceleration through overlap"),
W ranks emulated on one device:

* every rank's output bit for bit equal to the one-rank layer of its tokens,
  and the first step checked stage by stage against the expert-parallel
  oracle, with and without the remote-first tile order and with a shared
  expert, over several steps (the two banks of ready counters alternate);
* the per-sender row split of every local expert against the oracle's plan,
  and the ready counters of the step's bank: ceil(H/256) on every 128-row
  block of y that holds rows, 0 elsewhere;
* a sender that never dispatches: the owner's gate/up GEMM gives up within its
  bound with MOE_ERR_TIMEOUT (no hang), and the device stays usable;
* a sender that is late: its DISPATCH flag is set from the host (a copy on
  another stream) 0.3 s after the owner's GEMM started waiting for it; the
  GEMM (whose pair CTAs, epilogues and final drain all outlast the wait)
  then finishes and the layer is bit for bit the one-rank layer.
"""
import time

import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from combine_moe_route_13_b200.ep import EpOnOneDevice
from oracle import moe_oracle as O
from oracle import moe_oracle_ep as P
from _gpu_common import act_np
from test_gpu_ep import assert_ep_matches_oracle, local_weights, make_case, one_rank_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"
TILES = M.MOE_EP_TILE_SIGNAL
REMOTE_FIRST = M.MOE_EP_TILE_SIGNAL | M.MOE_EP_REMOTE_FIRST


def _cfg(W, T, H, E, K, F, cf, n_shared=0):
    C = O.capacity(T, K, E, cf)
    return M.make_config(T=T, H=H, E=E, K=K, F=F, S=W, capacity=C, row_align=128, act="bf16",
                         n_shared=n_shared), C


def _step(emu, cfg, W, logits, xs, w_gu, w_d):
    outs = [torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
            for _ in range(W)]
    emu.forward([l.to(DEV) for l in logits], [x.to(DEV) for x in xs],
                local_weights(w_gu, W, cfg.E, cfg.n_shared),
                local_weights(w_d, W, cfg.E, cfg.n_shared), outs)
    torch.cuda.synchronize()
    return outs


CASES = [
    # W, T, H, E, K, F, cf, n_shared: experts of 2-4 M tiles whose tiles mix senders
    (2, 1024, 256, 8, 2, 256, 1.25, 0),
    (4, 640, 512, 16, 4, 384, 1.0, 0),
    (2, 700, 256, 8, 3, 256, 0.8, 1),    # overflow, a shared expert
    (8, 128, 256, 64, 8, 128, 1.5, 0),   # eight senders inside one pair tile
    (8, 64, 256, 64, 8, 128, 1.5, 0),    # small experts: 128-row one-CTA tiles
    (2, 0, 256, 8, 2, 256, 1.25, 0),     # empty batch on every rank
    (2, 200, 256, 8, 2, 256, 0.0, 0),    # C = 0: every assignment dropped
]


@pytest.mark.parametrize("flags", [TILES, REMOTE_FIRST], ids=["tiles", "remote_first"])
@pytest.mark.parametrize("W,T,H,E,K,F,cf,n_shared", CASES)
def test_tile_signalled_layer(cuda_ok, flags, W, T, H, E, K, F, cf, n_shared):
    cfg, C = _cfg(W, T, H, E, K, F, cf, n_shared)
    emu = EpOnOneDevice(cfg, W, DEV, flags=flags)
    El = E // W
    for step in range(3):
        logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, "bf16", seed=500 + 11 * step + W,
                                          n_shared=n_shared)
        outs = _step(emu, cfg, W, logits, xs, w_gu, w_d)
        for r in range(W):
            assert emu.status(r) == M.MOE_OK, (step, r, M.status_string(emu.status(r)))
            ref = one_rank_layer(cfg, logits[r], xs[r], w_gu, w_d)
            g, w = act_np(outs[r]), act_np(ref)
            assert np.array_equal(g, w), f"step {step} rank {r}: {(g != w).sum()} differ"
        counts_all = np.stack([emu.views(r)["expert_counts"].cpu().numpy() for r in range(W)])
        for d in range(W):
            v = emu.views(d)
            plan = P.ep_plan(counts_all, C, 128, d)
            split = v["recv_split"].cpu().numpy()
            assert np.array_equal(split[:, :W], plan["block_row"] - plan["recv_offsets"][:El, None])
            assert np.array_equal(split[:, W], plan["recv_counts"])
            # this step's bank: every block holding rows reached ceil(H/256)
            bank = v["y_ready"][emu.epoch & 1].cpu().numpy()
            used = np.zeros_like(bank, dtype=bool)
            for j in range(El):
                lo, n = int(plan["recv_offsets"][j]), int(plan["recv_counts"][j])
                if n:
                    used[lo // 128:(lo + n + 127) // 128] = True
            assert np.all(bank[used] == (H + 255) // 256), (step, d)
            assert np.all(bank[~used] == 0), (step, d)
        if step == 0 and n_shared == 0:
            assert_ep_matches_oracle(emu, outs, logits, xs, w_gu, w_d, K, C, 128, W, "bf16", W)


def test_owner_gemm_times_out_when_a_sender_never_dispatches(cuda_ok):
    W, T, H, E, K, F = 2, 1024, 256, 8, 2, 256
    cfg, C = _cfg(W, T, H, E, K, F, 1.25)
    emu = EpOnOneDevice(cfg, W, DEV, timeout_us=50_000, flags=TILES)
    logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, "bf16", seed=77)
    wg, wd = local_weights(w_gu, W, E, 0), local_weights(w_d, W, E, 0)
    emu.epoch += 1
    for r in range(W):
        M.moe_ep_route(cfg, emu.ep(r), logits[r].to(DEV), emu.sym[r], emu.peers, emu.ws[r])
    # rank 1 never dispatches: owner 0's tiles holding rank 1's rows wait for it
    M.moe_ep_dispatch(cfg, emu.ep(0), xs[0].to(DEV), emu.sym[0], emu.peers, emu.ws[0])
    torch.cuda.synchronize()
    assert emu.status(0) == M.MOE_OK
    t0 = time.perf_counter()
    M.moe_ep_expert_mlp(cfg, emu.ep(0), None, wg[0], wd[0], emu.sym[0], emu.peers, emu.ws[0])
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert emu.status(0) == M.MOE_ERR_TIMEOUT
    assert elapsed < 5.0, elapsed
    f1 = emu.views(1)["flags"].cpu().numpy()
    assert f1[2, 0] == 0            # no Y flag raised for a step that timed out
    # the device is still usable: a fresh group runs a correct step
    emu2 = EpOnOneDevice(cfg, W, DEV, flags=TILES)
    outs = _step(emu2, cfg, W, logits, xs, w_gu, w_d)
    for r in range(W):
        assert emu2.status(r) == M.MOE_OK
        assert torch.equal(outs[r], one_rank_layer(cfg, logits[r], xs[r], w_gu, w_d))


def test_owner_gemm_waits_for_a_late_sender(cuda_ok):
    W, T, H, E, K, F = 2, 1024, 256, 8, 2, 256
    cfg, C = _cfg(W, T, H, E, K, F, 1.25)
    emu = EpOnOneDevice(cfg, W, DEV, flags=TILES)
    logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, "bf16", seed=78)
    wg, wd = local_weights(w_gu, W, E, 0), local_weights(w_d, W, E, 0)
    _step(emu, cfg, W, logits, xs, w_gu, w_d)     # one whole step first (warm)
    s_gemm, s_copy = torch.cuda.Stream(), torch.cuda.Stream()
    emu.epoch += 1
    ep = emu.epoch
    outs = [torch.empty(T, H, dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    with torch.cuda.stream(s_gemm):
        for r in range(W):
            M.moe_ep_route(cfg, emu.ep(r), logits[r].to(DEV), emu.sym[r], emu.peers, emu.ws[r])
        for r in range(W):
            M.moe_ep_dispatch(cfg, emu.ep(r), xs[r].to(DEV), emu.sym[r], emu.peers, emu.ws[r])
    torch.cuda.synchronize()
    flag = emu.views(0)["flags"][1, 1:2]          # owner 0's DISPATCH flag of sender 1
    assert int(flag.item()) == ep
    flag.fill_(ep - 1)                            # rank 1 is late
    torch.cuda.synchronize()
    late = torch.tensor([ep], dtype=torch.int32).pin_memory()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s_gemm):
        start.record()
        M.moe_ep_expert_mlp(cfg, emu.ep(0), None, wg[0], wd[0], emu.sym[0], emu.peers,
                            emu.ws[0])
        end.record()
    time.sleep(0.3)                               # the GEMM is running and waiting
    with torch.cuda.stream(s_copy):               # a copy engine raises the flag
        flag.copy_(late, non_blocking=True)
    torch.cuda.synchronize()
    assert emu.status(0) == M.MOE_OK
    assert start.elapsed_time(end) >= 250.0       # it did wait for the late sender
    with torch.cuda.stream(s_gemm):
        M.moe_ep_expert_mlp(cfg, emu.ep(1), None, wg[1], wd[1], emu.sym[1], emu.peers,
                            emu.ws[1])
        for r in range(W):
            M.moe_ep_combine(cfg, emu.ep(r), emu.sym[r], emu.peers, outs[r], emu.ws[r])
    torch.cuda.synchronize()
    for r in range(W):
        assert emu.status(r) == M.MOE_OK
        assert torch.equal(outs[r], one_rank_layer(cfg, logits[r], xs[r], w_gu, w_d))


@pytest.mark.parametrize("flags", [TILES, REMOTE_FIRST], ids=["tiles", "remote_first"])
def test_tile_signalled_layer_over_many_steps(cuda_ok, flags):
    # sixteen steps on the same inputs: the two banks of ready counters and the
    # step-numbered flags alternate and wrap, and every step's output is bit for
    # bit the first one's, which is the one-rank layer's
    W, T, H, E, K, F = 4, 640, 512, 16, 4, 384
    cfg, C = _cfg(W, T, H, E, K, F, 1.0)
    emu = EpOnOneDevice(cfg, W, DEV, flags=flags)
    logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, "bf16", seed=4242)
    first = _step(emu, cfg, W, logits, xs, w_gu, w_d)
    for r in range(W):
        assert emu.status(r) == M.MOE_OK
        assert torch.equal(first[r], one_rank_layer(cfg, logits[r], xs[r], w_gu, w_d)), r
    for step in range(1, 16):
        outs = _step(emu, cfg, W, logits, xs, w_gu, w_d)
        for r in range(W):
            assert emu.status(r) == M.MOE_OK, (step, r)
            assert torch.equal(outs[r], first[r]), (step, r)
