"""GPU parity of the fp8 block-scaled path against the fp8 oracle.

* quantisation (weights, and the dispatch of token rows): codes and scale
  bytes bit for bit;
* the gate/up GEMM: h's codes and scales against the oracle's quantisation of
  h computed from the same (bit-identical) fp8 operands.  h is quantised from
  fp32 values that the GPU and the oracle reach by different summation orders,
  so a code may land one step apart where h sits next to a rounding boundary
  (and a scale where a block's amax sits next to a power of two): at most
  1e-3 of the codes may differ, by one step only, and 1e-3 of the scales by one;
* the down GEMM: y against the oracle's y from the GPU's own h codes and
  scales, within the bf16 tolerance (1e-2 * rms + one bf16 step);
* the layer: route bit for bit, dispatch bit for bit, the combine against the
  oracle's combine of the GPU's y, and the whole chain within a relative
  Frobenius error of 1e-2 of the oracle's fp8 layer.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from oracle import moe_oracle as O
from oracle import moe_oracle_fp8 as Q
import workloads as W
from _gpu_common import act_np, assert_close_act, assert_route_equal, host, run_route

pytestmark = pytest.mark.gpu
DEV = "cuda"


def np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy()


def _adversarial_matrix(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    v = torch.randn(rows, cols, generator=g) * torch.exp2(torch.randint(-30, 30, (rows, 1), generator=g).float())
    v[0, :128] = 0.0                                     # an all-zero block
    if rows > 2:
        v[1, :128] = 448.0 * 2.0 ** -3                   # amax exactly on a power-of-two boundary
        v[2, 5] = -448.0 * 2.0 ** 4
    return v.to(torch.bfloat16)


@pytest.mark.parametrize("rows,cols", [(1, 128), (300, 256), (128, 384), (1000, 1024), (77, 7168)])
def test_quantize_bit_exact(cuda_ok, rows, cols):
    src = _adversarial_matrix(rows, cols, rows + cols)
    codes, scales = M.quantize_fp8(src.to(DEV))
    torch.cuda.synchronize()
    q, p = Q.quantize_rows(O.bf16_bits_to_f64(act_np(src)))
    assert np.array_equal(np_u8(codes), q)
    assert np.array_equal(Q.scales_from_blocked(np_u8(scales), rows, cols // 128), p)


def _cfg(T, H, E, K, F, S, C, A=128):
    return M.make_config(T=T, H=H, E=E, K=K, F=F, S=S, capacity=C, row_align=A, act="bf16")


def _logits(T, E, kind, seed):
    g = torch.Generator().manual_seed(seed)
    lg = torch.randn(T, E, generator=g)
    if kind == "zipf":
        lg += 2.0 * torch.log(torch.arange(1, E + 1, dtype=torch.float64) ** -1.2).float()
    if kind == "hot":
        lg[:, 0] += 2.0
    return lg


@pytest.mark.parametrize("T,H,E,K,cf", [(300, 256, 8, 2, 1.0), (1000, 1024, 17, 5, 0.7),
                                        (64, 7168, 4, 2, 1.0)])
def test_dispatch_fp8_bit_exact(cuda_ok, T, H, E, K, cf):
    C = O.capacity(T, K, E, cf)
    cfg = _cfg(T, H, E, K, 256, 1, C)
    r = run_route(cfg, _logits(T, E, "hot", 3).to(DEV))
    R = M.moe_max_rows(cfg)
    x = (torch.randn(T, H, generator=torch.Generator().manual_seed(4)) * 3).to(torch.bfloat16)
    xq = torch.zeros(R, H, dtype=torch.uint8, device=DEV)
    xs = torch.zeros(M.moe_fp8_scale_bytes(R, H), dtype=torch.uint8, device=DEV)
    M.moe_dispatch_fp8(cfg, x.to(DEV), r["token_slot"], xq, xs)
    torch.cuda.synchronize()
    slot = r["token_slot"].cpu().numpy()
    ref_q, ref_p = Q.dispatch_fp8(act_np(x), slot, R)
    kept = r["row_src"].cpu().numpy()[:R] >= 0
    assert np.array_equal(np_u8(xq)[kept], ref_q[kept])
    assert np.all(np_u8(xq)[~kept] == 0)                  # unwritten rows untouched
    got_p = Q.scales_from_blocked(np_u8(xs), R, H // 128)
    assert np.array_equal(got_p[kept], ref_p[kept])


def _weights_fp8(E, F, H, seed):
    g = torch.Generator().manual_seed(seed)
    w_gu = (torch.randn(E, 2 * F, H, generator=g) * 0.02).to(torch.bfloat16)
    w_d = (torch.randn(E, H, F, generator=g) * 0.02).to(torch.bfloat16)
    gq, gs = M.quantize_fp8(w_gu.to(DEV))
    dq, ds = M.quantize_fp8(w_d.to(DEV))
    torch.cuda.synchronize()
    ge = Q.scales_from_blocked(np_u8(gs), E * 2 * F, H // 128).reshape(E, 2 * F, H // 128)
    de = Q.scales_from_blocked(np_u8(ds), E * H, F // 128).reshape(E, H, F // 128)
    return (gq, gs, dq, ds), (np_u8(gq), ge, np_u8(dq), de)


def assert_h_close(hq_gpu, he_gpu, hq_ref, he_ref, what):
    """Codes and scales equal except at rounding boundaries (see the module doc)."""
    n = hq_ref.size
    if n == 0:
        return
    scale_diff = he_gpu != he_ref
    assert scale_diff.mean() <= 1e-3 + 1.0 / max(he_ref.size, 1), f"{what}: {scale_diff.sum()} scales differ"
    assert np.all(np.abs(he_gpu - he_ref) <= 1), f"{what}: a scale differs by more than one"
    same_scale_rows = ~np.repeat(scale_diff, 128, axis=1)
    a, b = hq_gpu[same_scale_rows].astype(np.int64), hq_ref[same_scale_rows].astype(np.int64)
    # codes of equal sign are ordered by magnitude: one step apart = codes differ by 1
    diff = a != b
    assert diff.mean() <= 1e-3, f"{what}: {diff.sum()} of {diff.size} codes differ"
    va = Q.e4m3_decode(a[diff].astype(np.uint8))
    vb = Q.e4m3_decode(b[diff].astype(np.uint8))
    one_step = (np.abs(a[diff] - b[diff]) == 1) | ((np.abs(va) + np.abs(vb)) <= 2.0 ** -9)
    assert np.all(one_step), f"{what}: codes more than one step apart"


MLP_CASES = [
    # T, H, E, K, F, S, cf, logits
    (300, 256, 8, 2, 256, 2, 1.0, "normal"),
    (1000, 512, 16, 4, 384, 4, 0.5, "hot"),       # overflow
    (600, 256, 8, 2, 384, 8, 2.0, "zipf"),        # empty experts
    (128, 256, 64, 8, 128, 8, 2.0, "normal"),     # many tiny experts
    (1200, 1024, 8, 2, 1024, 2, 1.25, "normal"),  # several M and N tiles per expert
    # >= 192 rows per expert: 256-row CTA-pair tiles, several per expert
    (2048, 256, 4, 2, 256, 2, 1.25, "normal"),    # ragged last tile per expert
    (1500, 512, 6, 2, 384, 3, 1.0, "zipf"),       # skewed experts, some at capacity
    (3000, 256, 12, 2, 256, 4, 2.0, "hot"),       # one hot expert over many tiles
]


@pytest.mark.parametrize("T,H,E,K,F,S,cf,kind", MLP_CASES)
def test_expert_mlp_fp8(cuda_ok, T, H, E, K, F, S, cf, kind):
    C = O.capacity(T, K, E, cf)
    cfg = _cfg(T, H, E, K, F, S, C)
    r = run_route(cfg, _logits(T, E, kind, T + F).to(DEV))
    R = M.moe_max_rows(cfg)
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(T)).to(torch.bfloat16).to(DEV)
    (gq, gs, dq, ds), (gq_n, ge, dq_n, de) = _weights_fp8(E, F, H, T + 1)
    xq = torch.zeros(R, H, dtype=torch.uint8, device=DEV)
    xs = torch.zeros(M.moe_fp8_scale_bytes(R, H), dtype=torch.uint8, device=DEV)
    hq = torch.zeros(R, F, dtype=torch.uint8, device=DEV)
    hs = torch.zeros(M.moe_fp8_scale_bytes(R, F), dtype=torch.uint8, device=DEV)
    y = torch.zeros(R, H, dtype=torch.bfloat16, device=DEV)
    ws = M.alloc_workspace(256)
    M.moe_dispatch_fp8(cfg, x, r["token_slot"], xq, xs)
    M.moe_expert_mlp_fp8(cfg, xq, xs, r["expert_offsets"], r["expert_counts"], gq, gs, dq, ds,
                         hq, hs, y, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    off = r["expert_offsets"].cpu().numpy()
    kept = np.minimum(r["expert_counts"].cpu().numpy(), C)
    xq_n, hq_n, y_n = np_u8(xq), np_u8(hq), act_np(y)
    xe = Q.scales_from_blocked(np_u8(xs), R, H // 128)
    he_all = Q.scales_from_blocked(np_u8(hs), R, F // 128)
    for e in range(E):
        n = int(kept[e])
        if n == 0:
            continue
        sl = slice(int(off[e]), int(off[e]) + n)
        rq, re_, _, _ = Q.expert_mlp_fp8_rows(xq_n[sl], xe[sl], gq_n[e], ge[e], dq_n[e], de[e])
        assert_h_close(hq_n[sl], he_all[sl], rq, re_, f"h[e={e}]")
        y_ref = Q.down_fp8_rows(hq_n[sl], he_all[sl], dq_n[e], de[e])
        assert_close_act(y_n[sl], y_ref, O.ACT_BF16, f"y[e={e}]")


@pytest.mark.parametrize("wl", [
    W.small_case(512, 256, 8, 2, 256, 2, 1.25, "bf16", 128),
    W.small_case(700, 512, 12, 3, 384, 4, 0.8, "bf16", 128, bias="zipf1.2"),
    W.small_case(200, 256, 8, 2, 128, 2, 0.0, "bf16", 128),          # C = 0: nothing kept
    W.small_case(1024, 512, 4, 2, 256, 2, 1.25, "bf16", 128),        # 512 rows per expert
], ids=lambda w: w.name)
def test_layer_forward_fp8(cuda_ok, wl):
    C = O.capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = _cfg(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align)
    inp = W.make_inputs(wl, seed=wl.T, device=DEV)
    (gq, gs, dq, ds), (gq_n, ge, dq_n, de) = _weights_fp8(wl.E, wl.F, wl.H, wl.T + 5)
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg))
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=DEV)
    aux = M.moe_layer_forward_fp8(cfg, inp["logits"], inp["x"], gq, gs, dq, ds, out, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    v = M.layer_views(cfg, ws, aux)
    f = M.fp8_views(cfg, ws, aux)
    x_n = act_np(inp["x"])
    ref_out, ref = Q.layer_forward_fp8(inp["logits"].cpu().numpy(), x_n, gq_n, ge, dq_n, de,
                                       wl.K, C, wl.row_align, wl.S)
    R = ref["R_max"]
    g = host({k: v[k] for k in ("topk_idx", "topk_w", "expert_counts", "overflow",
                                "expert_offsets", "segment_offsets", "token_slot", "row_src",
                                "totals")})
    assert_route_equal(g, ref, R)
    kept = ref["row_src"] >= 0
    assert np.array_equal(np_u8(f["xq"])[kept], ref["xq"][kept])
    assert np.array_equal(Q.scales_from_blocked(np_u8(f["xs"]), R, wl.H // 128)[kept],
                          ref["x_exp"][kept])
    hq_n = np_u8(f["hq"])
    he = Q.scales_from_blocked(np_u8(f["hs"]), R, wl.F // 128)
    assert_h_close(hq_n[kept], he[kept], ref["hq"][kept], ref["h_exp"][kept], "h")
    y_n = act_np(v["y"])
    off = ref["expert_offsets"]
    for e in range(wl.E):
        n = int(ref["kept"][e])
        if n:
            sl = slice(int(off[e]), int(off[e]) + n)
            assert_close_act(y_n[sl], Q.down_fp8_rows(hq_n[sl], he[sl], dq_n[e], de[e]),
                             O.ACT_BF16, f"y[e={e}]")
    out_n = act_np(out)
    assert_close_act(out_n, O.combine(y_n, ref["token_slot"], ref["topk_w"], O.ACT_BF16),
                     O.ACT_BF16, "out")
    gd, rd = O.bf16_bits_to_f64(out_n), O.bf16_bits_to_f64(ref_out)
    if np.any(rd):
        fro = np.linalg.norm(gd - rd) / np.linalg.norm(rd)
        assert fro <= 1e-2, f"whole chain: relative Frobenius error {fro:.3e}"
    else:
        assert not np.any(gd)


@pytest.mark.parametrize("corruption", ["past_the_buffer", "off_a_128_row_block"])
def test_expert_mlp_fp8_rejects_bad_offsets(cuda_ok, corruption):
    # the fp8 GEMMs read scale chunks per 128 rows with untiled bulk copies, so a
    # caller offsets table is checked first: an expert whose rows leave the
    # buffer or start off a 128-row block is skipped and reported
    T, H, E, K, F, S = 1200, 256, 8, 2, 256, 2
    C = O.capacity(T, K, E, 1.25)
    cfg = _cfg(T, H, E, K, F, S, C)
    r = run_route(cfg, _logits(T, E, "normal", 31).to(DEV))
    R = M.moe_max_rows(cfg)
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(32)).to(torch.bfloat16).to(DEV)
    (gq, gs, dq, ds), _ = _weights_fp8(E, F, H, 33)
    xq = torch.zeros(R, H, dtype=torch.uint8, device=DEV)
    xs = torch.zeros(M.moe_fp8_scale_bytes(R, H), dtype=torch.uint8, device=DEV)
    M.moe_dispatch_fp8(cfg, x, r["token_slot"], xq, xs)

    def run(offsets):
        hq = torch.zeros(R, F, dtype=torch.uint8, device=DEV)
        hs = torch.zeros(M.moe_fp8_scale_bytes(R, F), dtype=torch.uint8, device=DEV)
        y = torch.zeros(R, H, dtype=torch.bfloat16, device=DEV)
        ws = M.alloc_workspace(256)
        M.moe_expert_mlp_fp8(cfg, xq, xs, offsets, r["expert_counts"], gq, gs, dq, ds, hq, hs, y, ws)
        return y, M.moe_get_device_status(ws)

    y_ok, st = run(r["expert_offsets"])
    assert st == M.MOE_OK
    bad = r["expert_offsets"].clone()
    bad[5] = R + 4096 if corruption == "past_the_buffer" else bad[5] + 8
    y_bad, st = run(bad)
    assert st == M.MOE_ERR_DEVICE_INPUT
    off = r["expert_offsets"].cpu().numpy()
    kept = np.minimum(r["expert_counts"].cpu().numpy(), C)
    for e in range(E):
        if e == 5 or kept[e] == 0:
            continue
        sl = slice(int(off[e]), int(off[e]) + int(kept[e]))
        assert torch.equal(y_bad[sl].view(torch.int16), y_ok[sl].view(torch.int16)), e


def test_layer_forward_fp8_with_shared_expert(cuda_ok):
    # the shared expert (n_shared = 1) on the fp8 path: its rows of xq are the
    # tokens' quantisation, its h / y rows follow the fp8 oracle, and the
    # combine adds its output with weight 1
    wl = W.small_case(700, 512, 8, 2, 256, 2, 1.25, "bf16", 128, n_shared=1)
    C = O.capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = M.make_config(T=wl.T, H=wl.H, E=wl.E, K=wl.K, F=wl.F, S=wl.S, capacity=C,
                        row_align=wl.row_align, act="bf16", n_shared=1)
    inp = W.make_inputs(wl, seed=77, device=DEV)
    (gq, gs, dq, ds), (gq_n, ge, dq_n, de) = _weights_fp8(wl.E + 1, wl.F, wl.H, 78)
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg))
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=DEV)
    aux = M.moe_layer_forward_fp8(cfg, inp["logits"], inp["x"], gq, gs, dq, ds, out, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    v, f = M.layer_views(cfg, ws, aux), M.fp8_views(cfg, ws, aux)
    x_n = act_np(inp["x"])
    ref_out, ref = Q.layer_forward_fp8(inp["logits"].cpu().numpy(), x_n, gq_n, ge, dq_n, de,
                                       wl.K, C, wl.row_align, wl.S, n_shared=1)
    R_r, R_sh, Rt = ref["R_max"], M.shared_row0(cfg), M.moe_max_rows(cfg)
    assert Rt == R_sh + wl.T
    xq_n, hq_n, y_n = np_u8(f["xq"]), np_u8(f["hq"]), act_np(v["y"])
    xe = Q.scales_from_blocked(np_u8(f["xs"]), Rt, wl.H // 128)
    he = Q.scales_from_blocked(np_u8(f["hs"]), Rt, wl.F // 128)
    kept = ref["row_src"] >= 0
    assert np.array_equal(xq_n[:R_r][kept], ref["xq"][kept])
    tq, te = Q.quantize_rows(O.bf16_bits_to_f64(x_n))
    assert np.array_equal(xq_n[R_sh:], tq) and np.array_equal(xe[R_sh:], te)
    assert_h_close(hq_n[R_sh:], he[R_sh:], ref["hq_shared"], ref["h_exp_shared"], "h shared")
    assert_close_act(y_n[R_sh:], Q.down_fp8_rows(hq_n[R_sh:], he[R_sh:], dq_n[wl.E], de[wl.E]),
                     O.ACT_BF16, "y shared")
    assert_h_close(hq_n[:R_r][kept], he[:R_r][kept], ref["hq"][kept], ref["h_exp"][kept], "h")
    got = O.combine(y_n, ref["token_slot"], ref["topk_w"], O.ACT_BF16, y_shared=y_n[R_sh:])
    assert_close_act(act_np(out), got, O.ACT_BF16, "out")
    gd, rd = O.bf16_bits_to_f64(act_np(out)), O.bf16_bits_to_f64(ref_out)
    assert np.linalg.norm(gd - rd) / np.linalg.norm(rd) <= 1e-2
