"""fp8 parity at the workloads' full sizes, through moe_layer_forward_fp8 (the call
and launch configuration `bench.py --fp8` times).

* route outputs in full, bit for bit;
* dispatch: sampled kept rows' codes and scales bit for bit against the
  oracle's quantisation of their token rows;
* weights: the sampled experts' codes and scales bit for bit against the
  oracle's quantisation;
* expert MLP: sampled rows of sampled experts (the fullest, the emptiest
  non-empty one and a random one): h within the rounding-boundary allowance of
  test_gpu_fp8, y against the oracle's down GEMM of the GPU's own h;
* combine: sampled tokens against the oracle's weighted sum of the GPU's y.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from oracle import moe_oracle as O
from oracle import moe_oracle_fp8 as Q
import workloads as W
from _gpu_common import act_np, assert_close_act, assert_route_equal, host
from test_gpu_fp8 import assert_h_close, np_u8

pytestmark = pytest.mark.gpu
ROUTE_KEYS = ("topk_idx", "topk_w", "expert_counts", "overflow", "expert_offsets",
              "segment_offsets", "token_slot", "row_src", "totals")


def _expert_scales(buf, e, rows_per_expert, cols):
    """Scale exponents of expert e's rows of a weight matrix quantised as
    [E * rows_per_expert, cols] (its row blocks are contiguous chunks)."""
    KB = cols // 128
    per = rows_per_expert // 128 * (-(-KB // 4)) * 512   # the expert's chunks are contiguous
    return Q.scales_from_blocked(np_u8(buf[e * per:(e + 1) * per]), rows_per_expert, KB)


@pytest.mark.parametrize("name,n_shared", [("mixtral", 0), ("dsv3", 0), ("skewed", 0),
                                           ("kimi", 0), ("dsv3", 1)])
def test_workload_full_size_fp8(cuda_ok, name, n_shared):
    wl = W.WORKLOADS[name].with_(n_shared=n_shared)
    dev = torch.device("cuda")
    C = M.moe_capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = M.make_config(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align, wl.act,
                        n_shared=n_shared)
    inp = W.make_inputs(wl, seed=0, device=dev)
    gq, gs = M.quantize_fp8(inp["w_gu"])
    dq, ds = M.quantize_fp8(inp["w_d"])
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg), dev)
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev)
    aux = M.moe_layer_forward_fp8(cfg, inp["logits"], inp["x"], gq, gs, dq, ds, out, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    v = M.layer_views(cfg, ws, aux)
    f = M.fp8_views(cfg, ws, aux)
    H, F, K = wl.H, wl.F, wl.K

    ref = O.route(inp["logits"].cpu().numpy(), K, C, wl.row_align, wl.S)
    R = ref["R_max"]
    assert_route_equal(host({k: v[k] for k in ROUTE_KEYS}), ref, R)

    rng = np.random.default_rng(0)
    rs = ref["row_src"]
    kept_rows = np.nonzero(rs >= 0)[0]
    xs_all = Q.scales_from_blocked(np_u8(f["xs"]), R, H // 128)
    # dispatch on sampled rows
    pick = np.unique(np.concatenate([kept_rows[:4], kept_rows[-4:],
                                     rng.choice(kept_rows, min(56, len(kept_rows)), replace=False)]))
    toks = rs[pick] // K
    q_ref, p_ref = Q.quantize_rows(O.bf16_bits_to_f64(act_np(inp["x"][torch.from_numpy(toks).to(dev)])))
    idx = torch.from_numpy(pick).to(dev)
    assert np.array_equal(np_u8(f["xq"][idx]), q_ref)
    assert np.array_equal(xs_all[pick], p_ref)

    kept = np.minimum(ref["expert_counts"], C)
    off = ref["expert_offsets"]
    nonempty = np.nonzero(kept)[0]
    experts = {int(nonempty[np.argmax(kept[nonempty])]), int(nonempty[np.argmin(kept[nonempty])]),
               int(rng.choice(nonempty))}
    hs_all = Q.scales_from_blocked(np_u8(f["hs"]), R, F // 128)
    if n_shared:
        experts.add(wl.E)   # the shared expert: its rows are the tokens, from shared_row0 on
    R_sh = M.shared_row0(cfg)
    Rt = M.moe_max_rows(cfg)
    if n_shared:
        hs_all = Q.scales_from_blocked(np_u8(f["hs"]), Rt, F // 128)
        xs_all = Q.scales_from_blocked(np_u8(f["xs"]), Rt, H // 128)
    for e in sorted(experts):
        # the expert's weights: codes and scales against the oracle's quantisation
        wgu = O.bf16_bits_to_f64(act_np(inp["w_gu"][e]))
        wd = O.bf16_bits_to_f64(act_np(inp["w_d"][e]))
        gq_ref, ge_ref = Q.quantize_rows(wgu)
        dq_ref, de_ref = Q.quantize_rows(wd)
        assert np.array_equal(np_u8(gq[e]), gq_ref)
        assert np.array_equal(_expert_scales(gs, e, 2 * F, H), ge_ref)
        assert np.array_equal(np_u8(dq[e]), dq_ref)
        assert np.array_equal(_expert_scales(ds, e, H, F), de_ref)
        n = int(kept[e]) if e < wl.E else wl.T
        first = off[e] if e < wl.E else R_sh
        rows = first + np.unique(np.concatenate([np.arange(min(3, n)), np.arange(max(0, n - 3), n),
                                                  rng.integers(0, n, 6)]))
        ridx = torch.from_numpy(rows).to(dev)
        xq_rows = np_u8(f["xq"][ridx])
        if e == wl.E:   # the shared expert's dispatch: the tokens' own quantisation
            tq, te = Q.quantize_rows(O.bf16_bits_to_f64(act_np(inp["x"][ridx - R_sh])))
            assert np.array_equal(xq_rows, tq) and np.array_equal(xs_all[rows], te)
        hq_ref, he_ref, _, _ = Q.expert_mlp_fp8_rows(xq_rows, xs_all[rows], gq_ref, ge_ref, dq_ref,
                                                     de_ref)
        hq_rows = np_u8(f["hq"][ridx])
        assert_h_close(hq_rows, hs_all[rows], hq_ref, he_ref, f"h[e={e}]")
        y_ref = Q.down_fp8_rows(hq_rows, hs_all[rows], dq_ref, de_ref)
        assert_close_act(act_np(v["y"][ridx]), y_ref, O.ACT_BF16, f"y[e={e}]")

    # combine on sampled tokens, from the GPU's y
    toks = np.unique(np.concatenate([[0, wl.T - 1], rng.integers(0, wl.T, 126)]))
    slot = ref["token_slot"][toks]
    need = np.unique(slot[slot >= 0])
    remap = np.full(max(int(slot.max()) + 1, 1), -1, dtype=np.int64)
    remap[need] = np.arange(len(need))
    slot_sub = np.where(slot >= 0, remap[np.maximum(slot, 0)], -1).astype(np.int32)
    y_sub = act_np(v["y"][torch.from_numpy(need).to(dev)])
    y_sh = act_np(v["y"][torch.from_numpy(R_sh + toks).to(dev)]) if n_shared else None
    ref_out = O.combine(y_sub, slot_sub, ref["topk_w"][toks], O.ACT_BF16, y_shared=y_sh)
    assert_close_act(act_np(out[torch.from_numpy(toks).to(dev)]), ref_out, O.ACT_BF16, "out")
    del inp, ws, out, gq, gs, dq, ds
    torch.cuda.empty_cache()
