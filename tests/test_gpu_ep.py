"""GPU parity of the expert-parallel layer (include/moe_ep.h) against the
expert-parallel oracle, with W ranks emulated on one device
(EpOnOneDevice: every rank's buffers are separate allocations reached
through the same peer table the kernels use across GPUs).

* per rank: route bit for bit; the exchanged counts table, send_dst_row,
  recv_offsets and recv_counts bit for bit; the received rows of xr bit for
  bit; y against the oracle's SwiGLU of the GPU's own received rows (tolerance
  of the one-rank tests); out against the oracle's weighted sum of the GPU's
  own y rows, and the whole chain against the oracle's layer (relative
  Frobenius error 1e-2, as in the one-rank layer tests);
* out bit for bit equal to the one-rank library layer (moe_layer_forward)
  of the same rank's tokens over all E experts;
* several steps in a row (epochs), empty and fully dropped batches, E/W < K;
* a shared expert on every rank's own tokens (its GEMM runs before the wait
  for the peers' rows): its y against the oracle, out bit for bit equal to
  the one-rank layer with the shared expert;
* a wait that runs out: rank 0 alone, its peer never publishing, ends with
  MOE_ERR_TIMEOUT within the bound instead of hanging.
"""
import time

import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from combine_moe_route_13_b200.ep import EpOnOneDevice
from oracle import moe_oracle as O
from oracle import moe_oracle_ep as P
from _gpu_common import act_np, assert_close_act, assert_route_equal, host

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROUTE_KEYS = ("topk_idx", "topk_w", "expert_counts", "overflow", "expert_offsets",
              "segment_offsets", "token_slot", "row_src", "totals")


def make_case(W, T, H, E, K, F, act, seed, bias=0.0, n_shared=0):
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if act == "bf16" else torch.float32
    logits = [torch.randn(T, E, generator=g) + bias * torch.log(torch.arange(1, E + 1).float())
              for _ in range(W)]
    xs = [torch.randn(T, H, generator=g).to(dt) for _ in range(W)]
    w_gu = (torch.randn(E + n_shared, 2 * F, H, generator=g) * 0.05).to(dt)
    w_d = (torch.randn(E + n_shared, H, F, generator=g) * 0.05).to(dt)
    return logits, xs, w_gu, w_d


def local_weights(w, W, E, n_shared, dev=DEV):
    """Each rank's experts, then the shared expert (every rank holds it)."""
    El = E // W
    w = w.to(dev)
    if not n_shared:
        return [w[r * El:(r + 1) * El] for r in range(W)]
    return [torch.cat([w[r * El:(r + 1) * El], w[E:E + 1]]).contiguous() for r in range(W)]


def run_ep(cfg, W, logits, xs, w_gu, w_d, emu=None):
    emu = emu or EpOnOneDevice(cfg, W, DEV)
    dt = M.act_dtype(cfg)
    outs = [torch.full((cfg.T, cfg.H), float("nan"), dtype=dt, device=DEV) for _ in range(W)]
    emu.forward([l.to(DEV) for l in logits], [x.to(DEV) for x in xs],
                local_weights(w_gu, W, cfg.E, cfg.n_shared),
                local_weights(w_d, W, cfg.E, cfg.n_shared), outs)
    torch.cuda.synchronize()
    return emu, outs


def one_rank_layer(cfg, logits, x, w_gu, w_d):
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg))
    out = torch.empty(cfg.T, cfg.H, dtype=M.act_dtype(cfg), device=DEV)
    M.moe_layer_forward(cfg, logits.to(DEV), x.to(DEV), w_gu.to(DEV), w_d.to(DEV), out, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    return out


CASES = [
    # W, T, H, E, K, F, cf, A, act, bias
    (2, 256, 256, 8, 2, 256, 1.25, 128, "bf16", 0.0),
    (4, 300, 512, 16, 4, 384, 0.5, 128, "bf16", -2.4),   # overflow, skewed experts
    (8, 64, 256, 64, 8, 128, 1.5, 128, "bf16", 0.0),     # many small experts per owner
    (4, 50, 256, 8, 4, 128, 2.0, 128, "bf16", 0.0),      # E/W = 2 < K
    (2, 100, 128, 8, 2, 256, 1.25, 1, "f32", 0.0),       # fp32: CUDA-core GEMM, compact rows
    (4, 90, 64, 8, 3, 96, 0.7, 4, "f32", -2.4),
    (2, 0, 256, 8, 2, 256, 1.25, 128, "bf16", 0.0),      # empty batch on every rank
    (2, 200, 256, 8, 2, 256, 0.0, 128, "bf16", 0.0),     # C = 0: every assignment dropped
]


@pytest.mark.parametrize("W,T,H,E,K,F,cf,A,act,bias", CASES)
def test_ep_layer_matches_oracle(cuda_ok, W, T, H, E, K, F, cf, A, act, bias):
    C = O.capacity(T, K, E, cf)
    S = W
    cfg = M.make_config(T=T, H=H, E=E, K=K, F=F, S=S, capacity=C, row_align=A, act=act)
    logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, act, seed=W * 1000 + T, bias=bias)
    emu, outs = run_ep(cfg, W, logits, xs, w_gu, w_d)
    assert_ep_matches_oracle(emu, outs, logits, xs, w_gu, w_d, K, C, A, S, act, W)


def assert_ep_matches_oracle(emu, outs, logits, xs, w_gu, w_d, K, C, A, S, act, W):
    """Every rank of an emulated step against the expert-parallel oracle: route,
    counts table and layout bit for bit, received rows bit for bit, y against
    the oracle's SwiGLU of the GPU's own received rows, out against the
    oracle's weighted sum of the GPU's own y rows, and the whole chain by
    relative Frobenius error."""
    E = w_gu.shape[0]
    for r in range(W):
        assert emu.status(r) == M.MOE_OK, f"rank {r}: {M.status_string(emu.status(r))}"
    np_act = act_np
    ref_outs, inter = P.ep_layer_forward([l.numpy() for l in logits], [np_act(x) for x in xs],
                                         np_act(w_gu), np_act(w_d), K, C, A, S, act, W)
    El = E // W
    ys = []
    for r in range(W):
        v = emu.views(r)
        ref = inter[r]
        assert_route_equal(host({k: v[k] for k in ROUTE_KEYS}), ref, ref["R_max"])
        for k in ("counts_all", "send_dst_row", "recv_offsets", "recv_counts"):
            assert np.array_equal(v[k].cpu().numpy(), ref[k]), (r, k)
        xr = np_act(v["xr"])
        y = np_act(v["y"])
        ys.append(y)
        for j in range(El):
            lo, n = int(ref["recv_offsets"][j]), int(ref["recv_counts"][j])
            if n == 0:
                continue
            assert np.array_equal(xr[lo:lo + n], ref["xr"][lo:lo + n]), (r, j)
            _, y_ref = O.expert_mlp_rows(xr[lo:lo + n], np_act(w_gu[r * El + j]),
                                         np_act(w_d[r * El + j]), act)
            assert_close_act(y[lo:lo + n], y_ref, act, f"y rank {r} expert {j}")
    # combine of the GPU's own y rows (owners' rows, found by the plan), and the chain
    for r in range(W):
        ref = inter[r]
        sizes = [y.shape[0] for y in ys]
        base = np.concatenate([[0], np.cumsum(sizes)[:-1]])
        slot = ref["token_slot"]
        cat = np.full(slot.shape, -1, dtype=np.int64)
        for t, k in zip(*np.nonzero(slot >= 0)):
            e = int(ref["topk_idx"][t, k])
            row = int(ref["send_dst_row"][e]) + int(slot[t, k]) - int(ref["expert_offsets"][e])
            cat[t, k] = base[e // El] + row
        want = O.combine(np.concatenate(ys), cat, ref["topk_w"], act)
        got = np_act(outs[r])
        assert_close_act(got, want, act, f"out rank {r}")
        # the whole chain (two bf16 roundings, y's and out's, compound): relative
        # Frobenius error, as in the one-rank layer tests
        g, w = O.act_to_f64(got, act), O.act_to_f64(ref_outs[r], act)
        if np.any(w):
            fro = np.linalg.norm(g - w) / np.linalg.norm(w)
            assert fro <= 1e-2, f"chain rank {r}: relative Frobenius error {fro:.3e}"
        else:
            assert not np.any(g)


@pytest.mark.parametrize("W,T,H,E,K,F,cf,A,act", [
    (2, 512, 256, 8, 2, 256, 1.25, 128, "bf16"),
    (4, 300, 512, 16, 4, 384, 0.5, 128, "bf16"),
    (8, 128, 256, 64, 8, 128, 1.5, 128, "bf16"),
    (2, 100, 128, 8, 2, 256, 1.25, 1, "f32"),
])
def test_ep_equals_one_rank_layer_over_several_steps(cuda_ok, W, T, H, E, K, F, cf, A, act):
    C = O.capacity(T, K, E, cf)
    cfg = M.make_config(T=T, H=H, E=E, K=K, F=F, S=W, capacity=C, row_align=A, act=act)
    emu = None
    for step in range(3):
        logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, act, seed=step * 7 + W)
        emu, outs = run_ep(cfg, W, logits, xs, w_gu, w_d, emu)
        assert emu.epoch == step + 1
        for r in range(W):
            assert emu.status(r) == M.MOE_OK
            ref = one_rank_layer(cfg, logits[r], xs[r], w_gu, w_d)
            g, w = act_np(outs[r]), act_np(ref)
            if not np.array_equal(g, w):
                bad = np.argwhere(g != w)
                raise AssertionError(f"step {step} rank {r}: {len(bad)} elements differ, "
                                     f"first {bad[:3].tolist()}")


@pytest.mark.parametrize("W,T,H,E,K,F,cf,A", [
    (2, 100, 128, 8, 2, 256, 1.25, 1),
    (4, 90, 64, 8, 3, 96, 0.7, 4),
])
def test_ep_fp32_with_a_shared_expert(cuda_ok, W, T, H, E, K, F, cf, A):
    # fp32: the shared expert runs on the CUDA-core grouped GEMM over the rank's
    # own tokens; against the oracle and bit for bit the one-rank fp32 layer
    C = O.capacity(T, K, E, cf)
    cfg = M.make_config(T=T, H=H, E=E, K=K, F=F, S=W, capacity=C, row_align=A, act="f32",
                        n_shared=1)
    logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, "f32", seed=W * 13 + T, n_shared=1)
    emu, outs = run_ep(cfg, W, logits, xs, w_gu, w_d)
    ref_outs, _ = P.ep_layer_forward([l.numpy() for l in logits], [act_np(x) for x in xs],
                                     act_np(w_gu), act_np(w_d), K, C, A, W, "f32", W, n_shared=1)
    for r in range(W):
        assert emu.status(r) == M.MOE_OK
        assert_close_act(act_np(outs[r]), ref_outs[r], "f32", f"out rank {r}")
        ref = one_rank_layer(cfg, logits[r], xs[r], w_gu, w_d)
        assert torch.equal(outs[r], ref), f"rank {r}: {(outs[r] != ref).sum().item()} differ"


def test_ep_layer_forward_one_rank(cuda_ok):
    # the fused entry point with W = 1 (no peers): the one-rank layer, bit for bit
    T, H, E, K, F = 384, 256, 8, 2, 256
    C = O.capacity(T, K, E, 1.25)
    cfg = M.make_config(T=T, H=H, E=E, K=K, F=F, S=2, capacity=C, row_align=128, act="bf16")
    logits, xs, w_gu, w_d = make_case(1, T, H, E, K, F, "bf16", seed=3)
    sym = torch.zeros(M.moe_ep_symmetric_bytes(cfg, 1), dtype=torch.uint8, device=DEV)
    ws = M.alloc_workspace(M.moe_ep_workspace_bytes(cfg, 1))
    peers = torch.tensor([sym.data_ptr()], dtype=torch.int64, device=DEV)
    M.moe_ep_symmetric_init(cfg, 1, sym)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
    for epoch in (1, 2):
        M.moe_ep_layer_forward(cfg, M.make_ep(1, 0, epoch), logits[0].to(DEV), xs[0].to(DEV),
                               w_gu.to(DEV), w_d.to(DEV), sym, peers, out, ws)
        assert M.moe_get_device_status(ws) == M.MOE_OK
        ref = one_rank_layer(cfg, logits[0], xs[0], w_gu, w_d)
        assert torch.equal(out, ref)


def test_a_peer_that_never_publishes_times_out(cuda_ok):
    W, T, H, E, K, F = 2, 64, 256, 8, 2, 256
    C = O.capacity(T, K, E, 1.25)
    cfg = M.make_config(T=T, H=H, E=E, K=K, F=F, S=2, capacity=C, row_align=128, act="bf16")
    emu = EpOnOneDevice(cfg, W, DEV, timeout_us=2000)
    logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, "bf16", seed=9)
    emu.epoch = 1
    ep = emu.ep(0)
    out = torch.zeros(T, H, dtype=torch.bfloat16, device=DEV)
    wg, wd = w_gu[:E // W].to(DEV), w_d[:E // W].to(DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    # rank 0 alone: rank 1 never publishes its counts, dispatches or signals
    M.moe_ep_route(cfg, ep, logits[0].to(DEV), emu.sym[0], emu.peers, emu.ws[0])
    M.moe_ep_dispatch(cfg, ep, xs[0].to(DEV), emu.sym[0], emu.peers, emu.ws[0])
    M.moe_ep_expert_mlp(cfg, ep, None, wg, wd, emu.sym[0], emu.peers, emu.ws[0])
    M.moe_ep_combine(cfg, ep, emu.sym[0], emu.peers, out, emu.ws[0])
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert emu.status(0) == M.MOE_ERR_TIMEOUT
    assert elapsed < 5.0          # one 2 ms wait, the later ones give up at once
    v = emu.views(0)
    # after the timeout nothing was sent and no flag of rank 0 was raised anywhere
    for r in range(W):
        f = emu.views(r)["flags"].cpu().numpy()
        assert f[1, 0] == 0 and f[2, 0] == 0
    assert int(v["recv_counts"].sum()) == 0


@pytest.mark.parametrize("W,T,H,E,K,F,cf", [
    (2, 256, 256, 8, 2, 256, 1.25),
    (4, 300, 512, 16, 4, 384, 0.5),     # overflow: some tokens keep only the shared term
    (8, 64, 256, 64, 8, 128, 1.5),
    (2, 200, 256, 8, 2, 256, 0.0),      # C = 0: the shared expert alone
])
def test_ep_shared_expert(cuda_ok, W, T, H, E, K, F, cf):
    C = O.capacity(T, K, E, cf)
    cfg = M.make_config(T=T, H=H, E=E, K=K, F=F, S=W, capacity=C, row_align=128, act="bf16",
                        n_shared=1)
    logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, "bf16", seed=T + E, n_shared=1)
    emu, outs = run_ep(cfg, W, logits, xs, w_gu, w_d)
    ref_outs, inter = P.ep_layer_forward([l.numpy() for l in logits], [act_np(x) for x in xs],
                                         act_np(w_gu), act_np(w_d), K, C, 128, W, "bf16", W,
                                         n_shared=1)
    for r in range(W):
        assert emu.status(r) == M.MOE_OK
        v = emu.views(r)
        # the shared expert's y on this rank's tokens against the oracle's SwiGLU
        _, y_ref = O.expert_mlp_rows(act_np(xs[r]), act_np(w_gu[E]), act_np(w_d[E]), "bf16")
        assert_close_act(act_np(v["y_shared"]), y_ref, "bf16", f"y_shared rank {r}")
        # bit for bit the one-rank layer with the shared expert
        ref = one_rank_layer(cfg, logits[r], xs[r], w_gu, w_d)
        g, w = act_np(outs[r]), act_np(ref)
        assert np.array_equal(g, w), f"rank {r}: {(g != w).sum()} elements differ"
        gd, rd = O.act_to_f64(g, "bf16"), O.act_to_f64(ref_outs[r], "bf16")
        fro = np.linalg.norm(gd - rd) / np.linalg.norm(rd)
        assert fro <= 1e-2, f"chain rank {r}: relative Frobenius error {fro:.3e}"


def test_ep_random_sweep(cuda_ok):
    # seeded random shapes: ranks, experts per rank, K, capacity factor, alignment,
    # dtype; every rank bit for bit the one-rank layer, layout bit for bit the oracle's
    rng = np.random.default_rng(2024)
    for case in range(16):
        W = int(rng.choice([2, 3, 4, 8]))
        El = int(rng.integers(1, 9))
        E = W * El
        K = int(rng.integers(1, min(E, 8) + 1))
        act = "bf16" if rng.random() < 0.75 else "f32"
        H = int(rng.choice([128, 256, 384])) if act == "bf16" else int(rng.choice([64, 96, 128]))
        F = int(rng.choice([128, 192, 256]))
        T = int(rng.integers(1, 200))
        cf = float(rng.choice([0.3, 0.8, 1.0, 1.5, 4.0]))
        A = int(rng.choice([1, 8, 128])) if act == "f32" else 128
        C = O.capacity(T, K, E, cf)
        cfg = M.make_config(T=T, H=H, E=E, K=K, F=F, S=W, capacity=C, row_align=A, act=act)
        logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, act, seed=case,
                                          bias=float(rng.choice([0.0, -2.4])))
        emu, outs = run_ep(cfg, W, logits, xs, w_gu, w_d)
        counts_all = np.stack([O.route(l.numpy(), K, C, A, W)["expert_counts"] for l in logits])
        for r in range(W):
            assert emu.status(r) == M.MOE_OK, (case, r)
            v = emu.views(r)
            plan = P.ep_plan(counts_all, C, A, r)
            for k in ("send_dst_row", "recv_offsets", "recv_counts"):
                assert np.array_equal(v[k].cpu().numpy(), plan[k]), (case, r, k)
            ref = one_rank_layer(cfg, logits[r], xs[r], w_gu, w_d)
            assert torch.equal(outs[r], ref), (case, W, T, E, K, act, A, r)


def test_a_rank_that_leaves_between_steps_times_the_others_out(cuda_ok):
    # two good steps, then rank 1 stops taking part: rank 0's next step records
    # MOE_ERR_TIMEOUT within its bound, and nothing of rank 0 reaches rank 1
    W, T, H, E, K, F = 2, 96, 256, 8, 2, 256
    C = O.capacity(T, K, E, 1.25)
    cfg = M.make_config(T=T, H=H, E=E, K=K, F=F, S=2, capacity=C, row_align=128, act="bf16")
    emu = EpOnOneDevice(cfg, W, DEV, timeout_us=5000)
    emu_out = None
    for step in range(2):
        logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, "bf16", seed=50 + step)
        emu, emu_out = run_ep(cfg, W, logits, xs, w_gu, w_d, emu)
        for r in range(W):
            assert emu.status(r) == M.MOE_OK
            assert torch.equal(emu_out[r], one_rank_layer(cfg, logits[r], xs[r], w_gu, w_d))
    emu.epoch += 1
    ep = emu.ep(0)
    logits, xs, w_gu, w_d = make_case(W, T, H, E, K, F, "bf16", seed=99)
    wg, wd = local_weights(w_gu, W, E, 0), local_weights(w_d, W, E, 0)
    # a sentinel the timed-out combine must leave in place (include/moe_ep.h:
    # after a timeout the rank reads nothing from its peers and `out` is untouched)
    out = torch.full((T, H), 7.0, dtype=torch.bfloat16, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    M.moe_ep_route(cfg, ep, logits[0].to(DEV), emu.sym[0], emu.peers, emu.ws[0])
    M.moe_ep_dispatch(cfg, ep, xs[0].to(DEV), emu.sym[0], emu.peers, emu.ws[0])
    M.moe_ep_expert_mlp(cfg, ep, None, wg[0], wd[0], emu.sym[0], emu.peers, emu.ws[0])
    M.moe_ep_combine(cfg, ep, emu.sym[0], emu.peers, out, emu.ws[0])
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    # a further step of the timed-out rank (its status word still holds the
    # timeout: reading it would reset it) publishes nothing into its peer
    M.moe_ep_route(cfg, M.make_ep(W, 0, emu.epoch + 1, 5000),
                   logits[0].to(DEV), emu.sym[0], emu.peers, emu.ws[0])
    torch.cuda.synchronize()
    assert emu.status(0) == M.MOE_ERR_TIMEOUT
    assert emu.status(1) == M.MOE_OK
    f1 = emu.views(1)["flags"].cpu().numpy()
    assert f1[0, 0] == emu.epoch          # rank 0's counts of the timed-out step did arrive
    assert f1[1, 0] == emu.epoch - 1 and f1[2, 0] == emu.epoch - 1   # nothing after that
    assert torch.all(out == 7.0)
