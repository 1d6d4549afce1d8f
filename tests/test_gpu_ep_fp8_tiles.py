"""The tile-signalled expert-parallel layer with the fp8 payload
(MOE_EP_TILE_SIGNAL with moe_ep_dispatch_fp8 / moe_ep_expert_mlp_fp8; the
producer/consumer of "Mixture-of-Experts acceleration through overlap" on the
fp8 block-scaled grouped GEMM), W ranks emulated on one device:

* every rank's output bit for bit equal to the one-rank fp8 layer of its
  tokens (which the fp8 tests check against the fp8 oracle), over several
  steps, with and without the remote-first tile order and with a shared
  expert; the first step's chain within a relative Frobenius error of 1e-2 of
  the fp8 oracle's layer;
* the ready counters of the step's bank: ceil(H/256) on every 128-row block
  of y that holds rows, 0 elsewhere;
* a sender that never dispatches: the owner's fp8 gate/up GEMM gives up within
  its bound with MOE_ERR_TIMEOUT (no hang) and the device stays usable;
* a sender that is late: its DISPATCH flag is set from the host 0.3 s after
  the owner's GEMM started waiting for it; the GEMM then finishes and the
  layer is bit for bit the one-rank fp8 layer.
"""
import time

import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from combine_moe_route_13_b200.ep import EpOnOneDevice
from oracle import moe_oracle as O
from oracle import moe_oracle_ep as P
from oracle import moe_oracle_fp8 as Q
from _gpu_common import act_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
TILES = M.MOE_EP_TILE_SIGNAL
REMOTE_FIRST = M.MOE_EP_TILE_SIGNAL | M.MOE_EP_REMOTE_FIRST


def np_u8(t):
    return t.detach().cpu().contiguous().numpy()


def _case(W, T, H, E, K, F, cf, seed, n_shared=0):
    """Config, per-rank logits and tokens, the fp8 weights over all experts and
    each rank's local slice of them."""
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
    wq_local = [loc_gu[r] + loc_d[r] for r in range(W)]
    return cfg, C, logits, xs, (gq, gs, dq, ds), wq_local


def fp8_one_rank(cfg, logits, x, wq):
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg))
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
    M.moe_layer_forward_fp8(cfg, logits, x, *wq, out, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    return out


def _step(emu, cfg, W, logits, xs, wq_local):
    outs = [torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
            for _ in range(W)]
    emu.forward_fp8(logits, xs, wq_local, outs)
    torch.cuda.synchronize()
    return outs


CASES = [
    # W, T, H, E, K, F, cf, n_shared
    (2, 1024, 256, 8, 2, 256, 1.25, 0),   # 256-row CTA-pair tiles mixing senders
    (4, 640, 512, 16, 4, 384, 1.0, 0),
    (2, 700, 256, 8, 3, 256, 0.8, 1),     # overflow, a shared expert
    (8, 64, 256, 64, 8, 128, 1.5, 0),     # small experts: 128-row one-CTA tiles
    (2, 0, 256, 8, 2, 256, 1.25, 0),      # empty batch on every rank
    (2, 200, 256, 8, 2, 256, 0.0, 0),     # C = 0: every assignment dropped
]


@pytest.mark.parametrize("flags", [TILES, REMOTE_FIRST], ids=["tiles", "remote_first"])
@pytest.mark.parametrize("W,T,H,E,K,F,cf,n_shared", CASES)
def test_tile_signalled_fp8_layer(cuda_ok, flags, W, T, H, E, K, F, cf, n_shared):
    emu = None
    El = E // W
    for step in range(3):
        cfg, C, logits, xs, wq, wq_local = _case(W, T, H, E, K, F, cf, 900 + 13 * step + W,
                                                  n_shared)
        if emu is None:
            emu = EpOnOneDevice(cfg, W, DEV, flags=flags)
        outs = _step(emu, cfg, W, logits, xs, wq_local)
        for r in range(W):
            assert emu.status(r) == M.MOE_OK, (step, r, M.status_string(emu.status(r)))
            ref = fp8_one_rank(cfg, logits[r], xs[r], wq)
            assert torch.equal(outs[r], ref), \
                f"step {step} rank {r}: {(outs[r] != ref).sum().item()} differ"
        counts_all = np.stack([emu.views(r)["expert_counts"].cpu().numpy() for r in range(W)])
        for d in range(W):
            v = emu.views(d)
            plan = P.ep_plan(counts_all, C, 128, d)
            bank = v["y_ready"][emu.epoch & 1].cpu().numpy()
            used = np.zeros_like(bank, dtype=bool)
            for j in range(El):
                lo, n = int(plan["recv_offsets"][j]), int(plan["recv_counts"][j])
                if n:
                    used[lo // 128:(lo + n + 127) // 128] = True
            assert np.all(bank[used] == (H + 255) // 256), (step, d)
            assert np.all(bank[~used] == 0), (step, d)
        if step == 0 and n_shared == 0 and T > 0 and C > 0:
            gq, gs, dq, ds = wq
            ge = Q.scales_from_blocked(np_u8(gs), E * 2 * F, H // 128).reshape(E, 2 * F, H // 128)
            de = Q.scales_from_blocked(np_u8(ds), E * H, F // 128).reshape(E, H, F // 128)
            for r in range(W):
                ref_out, _ = Q.layer_forward_fp8(logits[r].cpu().numpy(), act_np(xs[r]),
                                                 np_u8(gq), ge, np_u8(dq), de, K, C, 128, W)
                g, w = O.bf16_bits_to_f64(act_np(outs[r])), O.bf16_bits_to_f64(ref_out)
                fro = np.linalg.norm(g - w) / max(np.linalg.norm(w), 1e-30)
                assert fro <= 1e-2, f"rank {r}: relative Frobenius error {fro:.3e}"


def test_fp8_owner_gemm_times_out_when_a_sender_never_dispatches(cuda_ok):
    W, T, H, E, K, F = 2, 1024, 256, 8, 2, 256
    cfg, C, logits, xs, wq, wq_local = _case(W, T, H, E, K, F, 1.25, 77)
    emu = EpOnOneDevice(cfg, W, DEV, timeout_us=50_000, flags=TILES)
    emu.epoch += 1
    for r in range(W):
        M.moe_ep_route(cfg, emu.ep(r), logits[r], emu.sym[r], emu.peers, emu.ws[r])
    # rank 1 never dispatches: owner 0's tiles holding rank 1's rows wait for it
    M.moe_ep_dispatch_fp8(cfg, emu.ep(0), xs[0], emu.sym[0], emu.peers, emu.ws[0])
    torch.cuda.synchronize()
    assert emu.status(0) == M.MOE_OK
    t0 = time.perf_counter()
    M.moe_ep_expert_mlp_fp8(cfg, emu.ep(0), *wq_local[0], emu.sym[0], emu.peers, emu.ws[0])
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert emu.status(0) == M.MOE_ERR_TIMEOUT
    assert elapsed < 5.0, elapsed
    assert emu.views(1)["flags"].cpu().numpy()[2, 0] == 0   # no Y flag for a timed-out step
    # the device is still usable: a fresh group runs a correct step
    emu2 = EpOnOneDevice(cfg, W, DEV, flags=TILES)
    outs = _step(emu2, cfg, W, logits, xs, wq_local)
    for r in range(W):
        assert emu2.status(r) == M.MOE_OK
        assert torch.equal(outs[r], fp8_one_rank(cfg, logits[r], xs[r], wq))


def test_fp8_owner_gemm_waits_for_a_late_sender(cuda_ok):
    W, T, H, E, K, F = 2, 1024, 256, 8, 2, 256
    cfg, C, logits, xs, wq, wq_local = _case(W, T, H, E, K, F, 1.25, 78)
    emu = EpOnOneDevice(cfg, W, DEV, flags=TILES)
    _step(emu, cfg, W, logits, xs, wq_local)      # one whole step first (warm)
    s_gemm, s_copy = torch.cuda.Stream(), torch.cuda.Stream()
    emu.epoch += 1
    ep = emu.epoch
    outs = [torch.empty(T, H, dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    with torch.cuda.stream(s_gemm):
        for r in range(W):
            M.moe_ep_route(cfg, emu.ep(r), logits[r], emu.sym[r], emu.peers, emu.ws[r])
        for r in range(W):
            M.moe_ep_dispatch_fp8(cfg, emu.ep(r), xs[r], emu.sym[r], emu.peers, emu.ws[r])
    torch.cuda.synchronize()
    flag = emu.views(0)["flags"][1, 1:2]          # owner 0's DISPATCH flag of sender 1
    assert int(flag.item()) == ep
    flag.fill_(ep - 1)                            # rank 1 is late
    torch.cuda.synchronize()
    late = torch.tensor([ep], dtype=torch.int32).pin_memory()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s_gemm):
        start.record()
        M.moe_ep_expert_mlp_fp8(cfg, emu.ep(0), *wq_local[0], emu.sym[0], emu.peers, emu.ws[0])
        end.record()
    time.sleep(0.3)                               # the GEMM is running and waiting
    with torch.cuda.stream(s_copy):               # a copy engine raises the flag
        flag.copy_(late, non_blocking=True)
    torch.cuda.synchronize()
    assert emu.status(0) == M.MOE_OK
    assert start.elapsed_time(end) >= 250.0       # it did wait for the late sender
    with torch.cuda.stream(s_gemm):
        M.moe_ep_expert_mlp_fp8(cfg, emu.ep(1), *wq_local[1], emu.sym[1], emu.peers, emu.ws[1])
        for r in range(W):
            M.moe_ep_combine(cfg, emu.ep(r), emu.sym[r], emu.peers, outs[r], emu.ws[r])
    torch.cuda.synchronize()
    for r in range(W):
        assert emu.status(r) == M.MOE_OK
        assert torch.equal(outs[r], fp8_one_rank(cfg, logits[r], xs[r], wq))


@pytest.mark.parametrize("flags", [TILES, REMOTE_FIRST], ids=["tiles", "remote_first"])
def test_tile_signalled_fp8_layer_over_many_steps(cuda_ok, flags):
    # as the bf16 test: sixteen steps on the same inputs, every step bit for bit
    # the first, which is the one-rank fp8 layer
    W, T, H, E, K, F = 4, 640, 512, 16, 4, 384
    cfg, C, logits, xs, wq, wq_local = _case(W, T, H, E, K, F, 1.0, 4243)
    emu = EpOnOneDevice(cfg, W, DEV, flags=flags)
    first = _step(emu, cfg, W, logits, xs, wq_local)
    for r in range(W):
        assert emu.status(r) == M.MOE_OK
        assert torch.equal(first[r], fp8_one_rank(cfg, logits[r], xs[r], wq)), r
    for step in range(1, 16):
        outs = _step(emu, cfg, W, logits, xs, wq_local)
        for r in range(W):
            assert emu.status(r) == M.MOE_OK, (step, r)
            assert torch.equal(outs[r], first[r]), (step, r)
