"""The tile-signalled overlap of the combine with the down GEMM.

* moe_layer_forward with MOE_FLAG_OVERLAP gives bit-identical outputs to the
  plain path (same kernels' arithmetic, only the synchronisation differs), and
  on the shapes the oracle finishes in seconds it is checked against the
  oracle's layer directly: routing bit for bit, y against the oracle's MLP of
  the same rows, out against the oracle's combine of the GPU's own y, and the
  whole chain by relative Frobenius error.
* moe_combine_wait with every ready counter at its target equals moe_combine.
* Failure detection without a GPU fault: counters that nothing sets make every
  wait run out; the kernel records MOE_ERR_TIMEOUT within its bound, returns,
  and the context stays usable.
"""
import time

import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
import workloads as W
from oracle import moe_oracle as O
from _gpu_common import act_np, assert_layer_stages, assert_route_equal, host

pytestmark = pytest.mark.gpu


def _forward(wl, inp, flags):
    C = M.moe_capacity(wl.T, wl.K, wl.E, wl.cf)
    cfg = M.make_config(wl.T, wl.H, wl.E, wl.K, wl.F, wl.S, C, wl.row_align, wl.act)
    ws = M.alloc_workspace(M.moe_workspace_bytes(cfg))
    out = torch.full((wl.T, wl.H), 3.0, dtype=wl.torch_act, device="cuda")
    aux = M.moe_layer_forward(cfg, inp["logits"], inp["x"], inp["w_gu"], inp["w_d"], out, ws,
                              flags=flags)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    return cfg, out, M.layer_views(cfg, ws, aux), ws


@pytest.mark.parametrize("wl", [
    W.small_case(512, 256, 8, 2, 256, 2, 1.25, "bf16", 128),
    W.small_case(3000, 512, 12, 2, 320, 4, 2.0, "bf16", 128, bias="zipf1.2"),
    W.small_case(700, 384, 16, 4, 192, 4, 0.8, "bf16", 256),
    W.WORKLOADS["mixtral"],
], ids=lambda w: w.name)
def test_overlap_is_bit_identical(cuda_ok, wl):
    inp = W.make_inputs(wl, seed=1, device="cuda")
    _, plain, _, _ = _forward(wl, inp, M.MOE_FLAG_NONE)
    cfg, over, v, _ = _forward(wl, inp, M.MOE_FLAG_OVERLAP)
    assert torch.equal(plain.view(torch.int16), over.view(torch.int16))
    # every 128-row block the down GEMM published reached its target
    R = M.moe_max_rows(cfg)
    off = v["expert_offsets"].cpu().numpy()
    kept = np.minimum(v["expert_counts"].cpu().numpy(), cfg.capacity)
    assert R > 0 and off[-1] <= R and np.all(kept >= 0)
    if wl.T * wl.H * wl.F > 1e9:   # the Mixtral shape: bit-identity to the plain path only
        return
    ref_out, ref = O.layer_forward(inp["logits"].cpu().numpy(), act_np(inp["x"]),
                                   act_np(inp["w_gu"]), act_np(inp["w_d"]), wl.K, cfg.capacity,
                                   wl.row_align, wl.S, wl.act)
    assert_route_equal(host({k: v[k] for k in ("topk_idx", "topk_w", "expert_counts", "overflow",
                                                "expert_offsets", "segment_offsets", "token_slot",
                                                "row_src", "totals")}), ref, ref["R_max"])
    assert_layer_stages({"xp": act_np(v["xp"]), "y": act_np(v["y"])}, act_np(over),
                        act_np(inp["x"]), act_np(inp["w_gu"]), act_np(inp["w_d"]), ref, ref_out,
                        wl.act)


def _route(cfg, logits):
    out = M.alloc_route_outputs(cfg)
    ws = M.alloc_workspace(M.moe_route_workspace_bytes(cfg))
    M.moe_route_topk(cfg, logits, out["topk_idx"], out["topk_w"], out["expert_counts"],
                     out["overflow"], out["expert_offsets"], out["segment_offsets"],
                     out["token_slot"], out["row_src"], out["totals"], ws)
    return out


def _combine_case():
    T, H, E, K = 1000, 512, 16, 4
    C = M.moe_capacity(T, K, E, 1.0)
    cfg = M.make_config(T, H, E, K, 64, 4, C, 128, "bf16")
    g = torch.Generator().manual_seed(9)
    r = _route(cfg, torch.randn(T, E, generator=g).cuda())
    R = M.moe_max_rows(cfg)
    y = torch.randn(R, H, generator=g).to(torch.bfloat16).cuda()
    ready = torch.zeros((R + 127) // 128, dtype=torch.int32, device="cuda")
    return cfg, r, y, ready


def test_combine_wait_with_ready_rows_equals_combine(cuda_ok):
    cfg, r, y, ready = _combine_case()
    target = M.ready_target(cfg)
    ready.fill_(target)
    ws = M.alloc_workspace(256)
    ref = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    got = torch.empty_like(ref)
    M.moe_combine(cfg, y, r["token_slot"], r["topk_w"], ref)
    M.moe_combine_wait(cfg, y, r["token_slot"], r["topk_w"], ready, target, got, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    assert torch.equal(ref.view(torch.int16), got.view(torch.int16))


def test_combine_wait_times_out_on_flags_nothing_sets(cuda_ok):
    cfg, r, y, ready = _combine_case()             # every counter stays 0
    ws = M.alloc_workspace(256)
    out = torch.zeros(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    M.moe_combine_wait(cfg, y, r["token_slot"], r["topk_w"], ready, M.ready_target(cfg), out, ws,
                       timeout_us=20_000)
    st = M.moe_get_device_status(ws)                # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert st == M.MOE_ERR_TIMEOUT
    assert elapsed < 2.0, elapsed                   # bounded: one 20 ms deadline, then fast exits
    assert M.moe_get_device_status(ws) == M.MOE_OK  # the status word was reset
    # the context is still usable: an ordinary combine gives the right answer
    ref = torch.empty_like(out)
    M.moe_combine(cfg, y, r["token_slot"], r["topk_w"], ref)
    ready.fill_(M.ready_target(cfg))
    M.moe_combine_wait(cfg, y, r["token_slot"], r["topk_w"], ready, M.ready_target(cfg), out, ws)
    assert M.moe_get_device_status(ws) == M.MOE_OK
    assert torch.equal(ref.view(torch.int16), out.view(torch.int16))
