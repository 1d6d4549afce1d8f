"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Integer outputs (routing indices, counts, overflow, offsets, the permutation,
the dispatched rows) must match bit for bit; router weights within 2e-6
relative; expert MLP and combine outputs within max|err| <= 1e-2 * rms(ref)
for bf16 and max|err| <= 1e-5 * max|ref| for fp32.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from oracle import moe_oracle as O
import workloads as W
from _gpu_common import (act_np, assert_close_act, assert_layer_stages, assert_route_equal,
                         cfg_for, host, run_route)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def logits_for(T, E, kind, seed):
    g = torch.Generator().manual_seed(seed)
    if kind == "tied":
        return W.tied_logits(T, E, 3, g)
    lg = torch.randn(T, E, generator=g)
    if kind == "zipf":
        lg += 2.0 * torch.log(torch.arange(1, E + 1, dtype=torch.float64) ** -1.2).float()
    if kind == "bias":
        lg += torch.randn(E, generator=g) * 0.1
    if kind == "hot":
        lg[:, 0] += 2.0
    return lg


ROUTE_CASES = [
    # T, E, K, S, cf, A, logits
    (64, 8, 2, 2, 1.25, 1, "normal"),
    (300, 8, 2, 8, 1.25, 128, "normal"),
    (1000, 17, 5, 1, 0.7, 4, "normal"),
    (1024, 256, 8, 8, 1.5, 128, "bias"),
    (4097, 64, 6, 8, 1.0, 128, "zipf"),
    (513, 384, 8, 16, 1.25, 128, "normal"),
    (200, 1024, 32, 4, 2.0, 8, "normal"),
    (256, 32, 32, 4, 1.0, 1, "normal"),
    (300, 12, 3, 3, 1.0, 1, "tied"),
    (128, 8, 2, 2, 0.0, 1, "normal"),
    (100, 8, 1, 1, -1.0, 1, "normal"),
    (0, 8, 2, 2, 1.0, 4, "normal"),
    (5000, 1, 1, 1, 1.0, 128, "normal"),
    (777, 40, 4, 5, 0.9, 32, "hot"),
]


@pytest.mark.parametrize("T,E,K,S,cf,A,kind", ROUTE_CASES)
def test_route_bit_exact(cuda_ok, T, E, K, S, cf, A, kind):
    C = O.capacity(T, K, E, cf)
    lg = logits_for(T, E, kind, T * 7 + E)
    cfg = cfg_for(T, 64, E, K, 64, S, C, A, "bf16")
    gpu = host(run_route(cfg, lg.to(DEV)))
    ref = O.route(lg.numpy(), K, C, A, S)
    assert_route_equal(gpu, ref, ref["R_max"])


def test_route_is_deterministic(cuda_ok):
    T, E, K, S, A = 4096, 64, 6, 8, 128
    lg = logits_for(T, E, "zipf", 3).to(DEV)
    cfg = cfg_for(T, 64, E, K, 64, S, O.capacity(T, K, E, 1.0), A, "bf16")
    a, b = host(run_route(cfg, lg)), host(run_route(cfg, lg))
    for k in a:
        assert np.array_equal(a[k], b[k]), k


@pytest.mark.parametrize("act", ["bf16", "f32"])
@pytest.mark.parametrize("T,H,E,K,S,cf,A", [
    (300, 256, 8, 2, 2, 1.0, 128), (1000, 128, 17, 5, 1, 0.7, 4), (64, 7168, 4, 2, 2, 1.0, 1),
    (333, 7168, 32, 8, 8, 0.5, 1),        # 14 KB rows, K = 8, half the assignments dropped
    (4096, 4096, 32, 8, 4, 1.0, 128),     # 8 KB (bf16) / 16 KB (f32) rows, several tokens per block
    (4133, 7168, 64, 8, 8, 0.5, 1),       # a ragged token tail
    (4096, 4096, 16, 10, 2, 0.1, 128),    # most tokens lose every assignment
])
def test_dispatch_bit_exact(cuda_ok, act, T, H, E, K, S, cf, A):
    C = O.capacity(T, K, E, cf)
    lg = logits_for(T, E, "hot", 11)
    cfg = cfg_for(T, H, E, K, 64, S, C, A, act)
    r = run_route(cfg, lg.to(DEV))
    dt = torch.float32 if act == "f32" else torch.bfloat16
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(5)).to(dt).to(DEV)
    R = M.moe_max_rows(cfg)
    xp = torch.full((R, H), 7, dtype=x.dtype, device=DEV)    # sentinel in unwritten rows
    M.moe_dispatch(cfg, x, r["token_slot"], xp)
    torch.cuda.synchronize()
    ref = O.dispatch(act_np(x), r["token_slot"].cpu().numpy(), R)
    rs = r["row_src"].cpu().numpy()[:R]
    kept = rs >= 0
    assert np.array_equal(act_np(xp)[kept], ref[kept])
    # rows no slot points at are left untouched
    untouched = act_np(xp)[~kept]
    sentinel = act_np(torch.full((1, H), 7, dtype=x.dtype))
    assert np.all(untouched == sentinel)


@pytest.mark.parametrize("act,K", [("bf16", 1), ("bf16", 2), ("bf16", 4), ("bf16", 8),
                                   ("f32", 1), ("f32", 2)])
def test_round_trip_identity_experts_bit_exact(cuda_ok, act, K):
    # y := xp (identity experts), weights summing to 1 in binary (K = 1, or equal
    # logits so that w = 1/K), no drops: combine(dispatch(x)) == x bit for bit.
    # Exact only while every partial sum k*x/K is exact in the fp32 accumulator:
    # any K <= 32 for bf16 rows (8 significant bits), K <= 2 for fp32 rows.
    T, H, E, S = 513, 512, 8, 2
    g = torch.Generator().manual_seed(2)
    lg = torch.randn(T, E, generator=g) - 10.0
    for t in range(T):   # K experts per token share the largest logit
        lg[t, torch.randperm(E, generator=g)[:K]] = 1.0
    cfg = cfg_for(T, H, E, K, 64, S, T, 8, act)
    r = run_route(cfg, lg.to(DEV))
    w = r["topk_w"].cpu()
    assert torch.all(w == 1.0 / K)
    dt = torch.float32 if act == "f32" else torch.bfloat16
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(3)).to(dt).to(DEV)
    xp = torch.zeros(M.moe_max_rows(cfg), H, dtype=dt, device=DEV)
    out = torch.empty_like(x)
    M.moe_dispatch(cfg, x, r["token_slot"], xp)
    M.moe_combine(cfg, xp, r["token_slot"], r["topk_w"], out)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16) if dt == torch.bfloat16 else out.view(torch.int32),
                       x.view(torch.int16) if dt == torch.bfloat16 else x.view(torch.int32))


@pytest.mark.parametrize("act", ["bf16", "f32"])
@pytest.mark.parametrize("T,H,E,K,cf", [(300, 256, 8, 2, 1.0), (777, 1024, 40, 6, 0.8),
                                        (50, 7168, 384, 8, 1.25), (64, 128, 8, 2, 0.0)])
def test_combine_matches_explicit_weighted_sum(cuda_ok, act, T, H, E, K, cf):
    C = O.capacity(T, K, E, cf)
    lg = logits_for(T, E, "hot", 13)
    cfg = cfg_for(T, H, E, K, 64, 1, C, 16, act)
    r = run_route(cfg, lg.to(DEV))
    R = M.moe_max_rows(cfg)
    dt = torch.float32 if act == "f32" else torch.bfloat16
    y = torch.randn(max(R, 1), H, generator=torch.Generator().manual_seed(4)).to(dt).to(DEV)
    out = torch.empty(T, H, dtype=dt, device=DEV)
    M.moe_combine(cfg, y, r["token_slot"], r["topk_w"], out)
    torch.cuda.synchronize()
    ref = O.combine(act_np(y), r["token_slot"].cpu().numpy(), r["topk_w"].cpu().numpy(), act)
    assert_close_act(act_np(out), ref, act, "combine")
    if C == 0:
        assert torch.all(out == 0)


MLP_CASES = [
    # T, H, E, K, F, S, cf, A, logits
    (256, 256, 4, 2, 256, 2, 1.25, 128, "normal"),
    (300, 320, 6, 2, 192, 3, 1.0, 1, "normal"),        # N tails, tiles straddling experts
    (1000, 512, 16, 4, 128, 4, 0.5, 128, "hot"),       # overflow
    (130, 128, 2, 1, 64, 1, -1.0, 8, "normal"),
    (600, 256, 8, 2, 384, 8, 2.0, 128, "zipf"),        # empty experts
    (128, 64, 64, 8, 64, 8, 2.0, 16, "normal"),        # many tiny experts
    (1200, 1024, 8, 2, 1024, 2, 1.25, 128, "normal"),  # several M and N tiles per expert
    # >= 192 rows per expert: 256-row tiles on CTA pairs
    (2048, 256, 4, 2, 192, 2, 1.25, 1, "normal"),      # pair tiles straddling experts, N tail
    (1500, 320, 6, 2, 256, 3, 1.0, 128, "zipf"),       # odd 128-row blocks, small experts
    (3000, 512, 12, 2, 320, 4, 2.0, 128, "hot"),       # one hot expert over many pair tiles
]


def _run_mlp(T, H, E, K, F, S, cf, A, kind, act):
    C = O.capacity(T, K, E, cf)
    lg = logits_for(T, E, kind, T + H + F)
    cfg = cfg_for(T, H, E, K, F, S, C, A, act)
    wl = W.small_case(T, H, E, K, F, S, cf, act, A)
    inp = W.make_inputs(wl, seed=T + E, device=DEV)
    r = run_route(cfg, lg.to(DEV))
    R = M.moe_max_rows(cfg)
    dt = wl.torch_act
    xp = torch.zeros(R, H, dtype=dt, device=DEV)
    h = torch.zeros(R, F, dtype=dt, device=DEV)
    y = torch.zeros(R, H, dtype=dt, device=DEV)
    ws = M.alloc_workspace(256)
    M.moe_dispatch(cfg, inp["x"], r["token_slot"], xp)
    M.moe_expert_mlp(cfg, xp, r["expert_offsets"], r["expert_counts"], inp["w_gu"], inp["w_d"],
                     h, y, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    return cfg, r, inp, xp, h, y


@pytest.mark.parametrize("T,H,E,K,F,S,cf,A,kind", MLP_CASES)
def test_expert_mlp_bf16(cuda_ok, T, H, E, K, F, S, cf, A, kind):
    cfg, r, inp, xp, h, y = _run_mlp(T, H, E, K, F, S, cf, A, kind, "bf16")
    off = r["expert_offsets"].cpu().numpy()
    kept = np.minimum(r["expert_counts"].cpu().numpy(), cfg.capacity)
    xp_n, h_n, y_n = act_np(xp), act_np(h), act_np(y)
    w_gu, w_d = act_np(inp["w_gu"]), act_np(inp["w_d"])
    rows = np.concatenate([np.arange(off[e], off[e] + kept[e]) for e in range(E)] + [np.zeros(0, int)])
    ref_h = np.zeros((len(rows), F), np.uint16)
    ref_y = np.zeros((len(rows), H), np.uint16)
    p = 0
    for e in range(E):
        n = int(kept[e])
        if n:
            he, ye = O.expert_mlp_rows(xp_n[off[e]:off[e] + n], w_gu[e], w_d[e], O.ACT_BF16)
            ref_h[p:p + n], ref_y[p:p + n] = he, ye
            p += n
    assert_close_act(h_n[rows], ref_h, O.ACT_BF16, "h")
    assert_close_act(y_n[rows], ref_y, O.ACT_BF16, "y")


def test_expert_mlp_f32_tiny(cuda_ok):
    w = W.WORKLOADS["tiny"]
    cfg, r, inp, xp, h, y = _run_mlp(w.T, w.H, w.E, w.K, w.F, w.S, w.cf, 1, "normal", "f32")
    ref_h, ref_y = O.expert_mlp(act_np(xp), r["expert_offsets"].cpu().numpy(),
                                np.minimum(r["expert_counts"].cpu().numpy(), cfg.capacity),
                                act_np(inp["w_gu"]), act_np(inp["w_d"]), O.ACT_F32)
    rs = r["row_src"].cpu().numpy()[:M.moe_max_rows(cfg)]
    kept = rs >= 0
    assert_close_act(act_np(h)[kept], ref_h[kept], O.ACT_F32, "h")
    assert_close_act(act_np(y)[kept], ref_y[kept], O.ACT_F32, "y")


def _layer(wl, C, seed=0):
    inp = W.make_inputs(wl, seed=seed, device=DEV)
    cfg = cfg_for(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align, wl.act)
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg))
    out = torch.empty(wl.T, wl.H, dtype=wl.torch_act, device=DEV)
    aux = M.moe_layer_forward(cfg, inp["logits"], inp["x"], inp["w_gu"], inp["w_d"], out, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    return cfg, inp, out, M.layer_views(cfg, ws, aux)


@pytest.mark.parametrize("wl", [
    W.WORKLOADS["tiny"],
    W.small_case(512, 256, 8, 2, 256, 2, 1.25, "bf16", 128),
    W.small_case(700, 384, 12, 3, 192, 4, 0.8, "bf16", 1, bias="zipf1.2"),
    W.small_case(300, 128, 16, 4, 128, 8, 1.0, "f32", 4),
], ids=lambda w: w.name)
def test_layer_forward_end_to_end(cuda_ok, wl):
    C = O.capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg, inp, out, v = _layer(wl, C)
    ref_out, ref = O.layer_forward(inp["logits"].cpu().numpy(), act_np(inp["x"]),
                                   act_np(inp["w_gu"]), act_np(inp["w_d"]), wl.K, C,
                                   wl.row_align, wl.S, wl.act)
    assert_route_equal(host({k: v[k] for k in ("topk_idx", "topk_w", "expert_counts", "overflow",
                                                "expert_offsets", "segment_offsets", "token_slot",
                                                "row_src", "totals")}), ref, ref["R_max"])
    assert_layer_stages({"xp": act_np(v["xp"]), "y": act_np(v["y"])}, act_np(out),
                        act_np(inp["x"]), act_np(inp["w_gu"]), act_np(inp["w_d"]), ref, ref_out,
                        wl.act)


def test_empty_batch(cuda_ok):
    wl = W.small_case(0, 128, 8, 2, 128, 2, 1.0, "bf16", 128)
    cfg, inp, out, v = _layer(wl, 0)
    assert v["totals"].cpu().tolist() == [0, 0, 0, 0]
    assert torch.all(v["expert_counts"] == 0)
    assert torch.all(v["row_src"] == -1)


@pytest.mark.parametrize("act", ["bf16", "f32"])
@pytest.mark.parametrize("T,H,K", [(257, 256, 2), (257, 7168, 8), (4099, 4096, 8)])
def test_dispatch_shared_expert_rows(cuda_ok, act, T, H, K):
    # with a shared expert the piecewise dispatch also copies every token to its
    # shared row shared_row0 + t: one more destination per token
    E, S, A = 16, 4, 128
    C = O.capacity(T, K, E, 0.75)
    cfg = M.make_config(T=T, H=H, E=E, K=K, F=64, S=S, capacity=C, row_align=A, act=act,
                        n_shared=1)
    r = run_route(cfg, logits_for(T, E, "zipf", 31).to(DEV))
    dt = torch.float32 if act == "f32" else torch.bfloat16
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(8)).to(dt).to(DEV)
    R = M.moe_max_rows(cfg)
    xp = torch.full((R, H), 5, dtype=dt, device=DEV)
    M.moe_dispatch(cfg, x, r["token_slot"], xp)
    torch.cuda.synchronize()
    r0 = M.shared_row0(cfg)
    assert r0 + T <= R
    assert np.array_equal(act_np(xp[r0:r0 + T]), act_np(x))          # the shared rows
    ts = r["token_slot"].cpu().numpy()
    ref = O.dispatch(act_np(x), ts, r0)
    kept = np.zeros(r0, bool)
    kept[ts[ts >= 0]] = True
    assert np.array_equal(act_np(xp[:r0])[kept], ref[kept])          # the routed rows
    assert np.all(act_np(xp[:r0])[~kept] == act_np(torch.full((1, H), 5, dtype=dt)))


@pytest.mark.parametrize("T,H,K", [(300, 256, 2), (4096, 4096, 8)])
def test_out_of_range_slots_are_treated_as_dropped(cuda_ok, T, H, K):
    # caller-supplied tables: entries beyond the routed rows (or below -1) must
    # not be written or read; the kernels treat them as dropped assignments
    E, S, A = 8, 2, 8
    C = O.capacity(T, K, E, 1.0)
    cfg = cfg_for(T, H, E, K, 64, S, C, A, "bf16")
    r = run_route(cfg, logits_for(T, E, "normal", 21).to(DEV))
    R = M.moe_max_rows(cfg)
    slot = r["token_slot"].clone()
    bad = torch.zeros_like(slot, dtype=torch.bool)
    bad[::7, 0] = True
    slot[bad] = torch.tensor([R, R + 5, 1 << 30, -7], dtype=torch.int32,
                             device=DEV).repeat(int(bad.sum()) // 4 + 1)[:int(bad.sum())]
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16).to(DEV)
    guard = 64
    xp_full = torch.full((R + guard, H), 3, dtype=torch.bfloat16, device=DEV)
    M.moe_dispatch(cfg, x, slot, xp_full[:R])
    torch.cuda.synchronize()
    assert torch.all(xp_full[R:] == 3)                         # nothing past the buffer
    ref_slot = slot.cpu().numpy().copy()
    ref_slot[(ref_slot < 0) | (ref_slot >= R)] = -1
    ref = O.dispatch(act_np(x), ref_slot, R)
    kept = np.zeros(R, bool)
    kept[ref_slot[ref_slot >= 0]] = True
    assert np.array_equal(act_np(xp_full[:R])[kept], ref[kept])
    y = torch.randn(R, H, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16).to(DEV)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
    M.moe_combine(cfg, y, slot, r["topk_w"], out)
    torch.cuda.synchronize()
    ref_out = O.combine(act_np(y), ref_slot, r["topk_w"].cpu().numpy(), O.ACT_BF16)
    assert_close_act(act_np(out), ref_out, O.ACT_BF16, "combine with dropped entries")


def _random_route_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        E = int(rng.choice([1, 2, 3, 8, 16, 40, 64, 96, 256, 384, 1024]))
        K = int(rng.integers(1, min(E, 32) + 1))
        divisors = [d for d in (1, 2, 3, 4, 8, 16) if E % d == 0]
        S = int(rng.choice(divisors))
        T = int(rng.choice([0, 1, 7, 127, 128, 129, 500, 1000, 3001]))
        A = int(rng.choice([1, 2, 8, 16, 128]))
        cf = float(rng.choice([-1.0, 0.0, 0.3, 0.75, 1.0, 1.25, 2.0]))
        kind = str(rng.choice(["normal", "zipf", "hot", "tied"]))
        cases.append((T, E, K, S, cf, A, kind))
    return cases


@pytest.mark.parametrize("T,E,K,S,cf,A,kind", _random_route_cases(40, 2024))
def test_route_random_sweep(cuda_ok, T, E, K, S, cf, A, kind):
    # seeded random sweep over (T, E, K, S, A, cf, logit kind), overflow and cf -> 0 included
    C = O.capacity(T, K, E, cf)
    lg = logits_for(T, E, kind, T * 3 + E * 5 + K)
    cfg = cfg_for(T, 64, E, K, 64, S, C, A, "bf16")
    gpu = host(run_route(cfg, lg.to(DEV)))
    ref = O.route(lg.numpy(), K, C, A, S)
    assert_route_equal(gpu, ref, ref["R_max"])


def test_expert_mlp_rejects_out_of_range_offsets(cuda_ok):
    # a caller offsets table pointing an expert past the buffer: the GEMMs record
    # MOE_ERR_DEVICE_INPUT, skip that expert and compute the others as before
    cfg, r, inp, xp, h, y = _run_mlp(1200, 256, 8, 2, 256, 2, 1.25, 128, "normal", "bf16")
    R = M.moe_max_rows(cfg)
    bad = r["expert_offsets"].clone()
    bad[3] = R + 4096
    h2, y2 = torch.zeros_like(h), torch.zeros_like(y)
    ws = M.alloc_workspace(256)
    M.moe_expert_mlp(cfg, xp, bad, r["expert_counts"], inp["w_gu"], inp["w_d"], h2, y2, ws)
    assert M.moe_get_device_status(ws) == M.MOE_ERR_DEVICE_INPUT
    off = r["expert_offsets"].cpu().numpy()
    kept = np.minimum(r["expert_counts"].cpu().numpy(), cfg.capacity)
    for e in range(8):
        if e == 3 or kept[e] == 0:
            continue
        sl = slice(int(off[e]), int(off[e]) + int(kept[e]))
        assert torch.equal(y2[sl].view(torch.int16), y[sl].view(torch.int16)), e
