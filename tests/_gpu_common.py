"""Helpers of the GPU parity tests: run the C ABI on seeded inputs and compare
with the CPU oracle element by element."""
from __future__ import annotations

import numpy as np
import torch

import combine_moe_route_13_b200 as M
from oracle import moe_oracle as O

ROUTE_KEYS_EXACT = ("topk_idx", "expert_counts", "overflow", "expert_offsets",
                    "segment_offsets", "token_slot", "row_src", "totals")

# Tolerances. Router weights: fp32 expf and division against the float64
# reference, 2e-6 relative. Expert MLP and combine: 1e-2 * rms(ref) (plus the
# bf16 step, see assert_close_act) for bf16 inputs with fp32 accumulation, and
# max|err| <= 1e-5 * max|ref| for fp32.
W_RTOL = 2e-6
BF16_TOL = 1e-2
F32_TOL = 1e-5


def act_np(t: torch.Tensor) -> np.ndarray:
    """Host numpy copy in the oracle's representation (bf16 -> uint16 bits)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def cfg_for(T, H, E, K, F, S, C, A, act):
    return M.make_config(T=T, H=H, E=E, K=K, F=F, S=S, capacity=C, row_align=A, act=act)


def run_route(cfg, logits: torch.Tensor):
    out = M.alloc_route_outputs(cfg, logits.device)
    ws = M.alloc_workspace(M.moe_route_workspace_bytes(cfg), logits.device)
    M.moe_route_topk(cfg, logits, out["topk_idx"], out["topk_w"], out["expert_counts"],
                     out["overflow"], out["expert_offsets"], out["segment_offsets"],
                     out["token_slot"], out["row_src"], out["totals"], ws)
    torch.cuda.synchronize()
    return out


def host(d: dict) -> dict:
    return {k: v.cpu().numpy() for k, v in d.items()}


def assert_route_equal(gpu: dict, ref: dict, R_max: int):
    for k in ROUTE_KEYS_EXACT:
        g = np.asarray(gpu[k])
        r = np.asarray(ref[k])
        if k == "row_src":
            g = g[:R_max]
        assert g.shape == r.shape, (k, g.shape, r.shape)
        if not np.array_equal(g, r):
            bad = np.argwhere(g != r)[:5]
            raise AssertionError(f"{k} differs at {bad.tolist()}: gpu {g[tuple(bad[0])]} ref {r[tuple(bad[0])]}")
    gw = np.asarray(gpu["topk_w"], dtype=np.float64)
    rw = np.asarray(ref["topk_w"], dtype=np.float64)
    if gw.size:
        rel = np.abs(gw - rw) / np.maximum(np.abs(rw), 1e-30)
        assert rel.max() <= W_RTOL, f"topk_w rel err {rel.max()}"


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |v| (2^(e-7) for 2^e <= |v| < 2^(e+1))."""
    _, e = np.frexp(np.abs(v))
    return np.where(v == 0, 2.0 ** -133, np.ldexp(1.0, np.maximum(e - 1, -126) - 7))


def assert_close_act(gpu_act: np.ndarray, ref_act: np.ndarray, act: str, what: str):
    """bf16: |gpu - ref| <= 1e-2 * rms(ref) + ulp_bf16(ref) element-wise, and the
    relative Frobenius error <= 1e-2. The ulp term is the storage format's own
    step: two correctly rounded results of nearly equal real numbers (the GPU's
    fp32 accumulation and the oracle's float64) may land on neighbouring bf16
    values, and for the largest elements of a tensor one bf16 step already
    exceeds 1e-2 * rms.  fp32: max|gpu - ref| <= 1e-5 * max|ref|."""
    g = O.act_to_f64(gpu_act, act)
    r = O.act_to_f64(ref_act, act)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    if r.size == 0:
        return
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    diff = np.abs(g - r)
    if act == O.ACT_BF16:
        rms = np.sqrt(np.mean(r * r))
        allowed = BF16_TOL * rms + bf16_ulp(r)
        worst = np.unravel_index(np.argmax(diff - allowed), diff.shape)
        assert np.all(diff <= allowed), (
            f"{what}: |err| {diff[worst]:.3e} > {allowed[worst]:.3e} at {worst} "
            f"(ref {r[worst]:.4e}, gpu {g[worst]:.4e}, rms {rms:.3e})")
        fro = np.sqrt(np.sum(diff * diff)) / max(np.sqrt(np.sum(r * r)), 1e-300)
        assert fro <= BF16_TOL, f"{what}: relative Frobenius error {fro:.3e}"
    else:
        bound = F32_TOL * np.abs(r).max()
        assert diff.max() <= bound, f"{what}: max|err| {diff.max():.3e} > {bound:.3e}"


def assert_layer_stages(gpu: dict, gpu_out: np.ndarray, x: np.ndarray, w_gu: np.ndarray,
                        w_d: np.ndarray, ref: dict, ref_out: np.ndarray, act: str):
    """End-to-end check stage by stage, each against the oracle with the stated
    tolerance: xp bit-exact; y against the oracle's MLP on the same rows; out
    against the oracle's combine of the GPU's own y. (Comparing out with the
    oracle's whole chain element-wise would compound two independent bf16
    roundings, y's and out's.) The whole chain must also agree within a relative
    Frobenius error of 1e-2."""
    kept = ref["row_src"] >= 0
    assert np.array_equal(gpu["xp"][kept], ref["xp"][kept])
    h_ref, y_ref = O.expert_mlp(gpu["xp"], ref["expert_offsets"], ref["kept"], w_gu, w_d, act)
    assert_close_act(gpu["y"][kept], y_ref[kept], act, "y")
    out_from_gpu_y = O.combine(gpu["y"], ref["token_slot"], ref["topk_w"], act)
    assert_close_act(gpu_out, out_from_gpu_y, act, "out")
    g = O.act_to_f64(gpu_out, act)
    r = O.act_to_f64(ref_out, act)
    fro = np.sqrt(np.sum((g - r) ** 2)) / max(np.sqrt(np.sum(r * r)), 1e-300)
    assert fro <= 1e-2, f"whole chain: relative Frobenius error {fro:.3e}"
