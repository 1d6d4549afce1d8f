"""CPU oracle for the single-GPU MoE layer: route -> dispatch -> expert MLP -> combine.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its CPU-baseline and reference legs) may import this module.
The CUDA library never imports, links or calls it, and it shares no code,
table or helper with the CUDA library.

Every step is written as its plain definition, in float64 numpy, with library
primitives (a stable sort, a matmul, exp) as single steps.  Sources:

* "Efficient and portable Mixture-of-Experts communication" (pplx-kernels
  page), "Introductie": a router gives a probability distribution, the top-K
  experts are chosen and the output is the weighted average of the expert
  outputs with weights derived from that distribution.  "Dispatch": tokens
  are packed into contiguous per-expert buffers and the position each token
  must return to is recorded.  "Combine": 16-bit expert outputs are gathered
  and the weighted average is taken on the receiving side.
* "Enabling trillion-parameter models on AWS EFA", "Диспетчеризация и
  комбинирование": tokens per expert are counted, an exclusive cumulative sum
  gives the offsets, tokens are packed contiguously at those offsets; the
  grouped GEMM multiplies the packed tokens by their expert's weights
  ("MoE all-to-all через EFA").
* "MoE Expert Parallel Benchmark", Step 2 (table): overflow =
  max(assigned - capacity, 0); effective tokens = sum of (assigned - overflow).
* "Mixture-of-Experts acceleration through overlap": the remote-owner-aligned
  layout, where every tile of the grouped buffer belongs to exactly one owner
  segment.

Readings where the pages are silent (each is listed in the design notes):
capacity C = ceil(cf*T*K/E); the first C assignments of an expert in token
order are kept and the rest overflow; weights are the softmax renormalised over
the K selected logits; ties in the top-K go to the lower expert index; experts
are laid out in ascending index order, owner segment s holding experts
[s*E/S, (s+1)*E/S); every expert's rows start on a multiple of the row
alignment A; the expert MLP is SwiGLU, silu(x Wg^T) * (x Wu^T) then W_d^T, with
w_gu [E,2F,H] (gate rows first) and w_d [E,H,F]; bf16 runs round h and y to
bf16; dropped assignments contribute zero to the combine.

Activation tensors are passed as numpy float32 arrays (fp32 workloads) or as
numpy uint16 arrays holding bf16 bit patterns (bf16 workloads).
"""
from __future__ import annotations

import math

import numpy as np

ACT_F32 = "f32"
ACT_BF16 = "bf16"


# ----------------------------------------------------------------------------
# Number formats
# ----------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns: a bf16 value is the top 16 bits of
    the fp32 with the same sign, exponent and leading mantissa bits."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 to the nearest bf16 (ties to even) and return its bits.

    bf16 keeps 8 significant bits and fp32's exponent range.  For |v| in
    [2^e', 2^(e'+1)) the spacing of bf16 values is 2^(e'-7); below the
    smallest normal (2^-126) the spacing stays 2^-133 (subnormals).  np.rint
    rounds halfway cases to even.  Values at or beyond the overflow threshold
    (max bf16 plus half a spacing) become infinities.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.float64)
    finite = np.isfinite(v)
    m, e = np.frexp(np.where(finite, v, 0.0))        # v = m * 2^e, 0.5 <= |m| < 1
    e_val = e - 1                                    # v in [2^e_val, 2^(e_val+1))
    spacing_exp = np.maximum(e_val - 7, -133)
    q = np.ldexp(1.0, spacing_exp)
    r = np.rint(v / q) * q
    max_bf16 = float.fromhex("0x1.fep127")
    r = np.where(np.abs(r) > max_bf16, np.copysign(np.inf, v), r)
    out[finite] = r[finite]
    out[~finite] = v[~finite]
    f32 = out.astype(np.float32)                     # exact: out is a bf16 value
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def act_to_f64(a: np.ndarray, act: str) -> np.ndarray:
    if act == ACT_BF16:
        return bf16_bits_to_f64(a)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def f64_to_act(v: np.ndarray, act: str) -> np.ndarray:
    if act == ACT_BF16:
        return f64_to_bf16_bits(v)
    return np.asarray(v, dtype=np.float64).astype(np.float32)


# ----------------------------------------------------------------------------
# Capacity and buffer sizes
# ----------------------------------------------------------------------------

def capacity(T: int, K: int, E: int, cf: float) -> int:
    """Per-expert capacity C = ceil(cf * T * K / E).

    The pages fix only that capacity is an expert's per-step limit ("MoE
    Expert Parallel Benchmark", Step 2); the capacity-factor formula is the
    reading taken here.  A negative cf means no limit (C = T: a token picks an
    expert at most once).
    """
    if cf < 0:
        return T
    return int(math.ceil(cf * T * K / E))


def max_rows(T: int, K: int, E: int, C: int, A: int) -> int:
    """Upper bound R_max on the dispatch-buffer rows: at most min(T*K, E*C)
    rows are kept and every expert adds at most A-1 rows of alignment
    padding.  This is the fixed worst-case receive-buffer sizing of the
    pplx-kernels page ("Draagbare kernels"), for one GPU."""
    return min(T * K, E * C) + E * (A - 1)


# ----------------------------------------------------------------------------
# Route: top-K and softmax weights
# ----------------------------------------------------------------------------

def router_logits(x: np.ndarray, w_g: np.ndarray, act: str) -> np.ndarray:
    """The router's linear layer: logits[t,e] = sum_h x[t,h] * w_g[e,h]
    (pplx-kernels page, "Introductie": a small linear layer gives the router's
    distribution), exact float64 sums of the widened inputs, stored as fp32."""
    return (act_to_f64(x, act) @ act_to_f64(w_g, act).T).astype(np.float32)


def route_topk(logits: np.ndarray, K: int, sel_bias: np.ndarray | None = None):
    """Top-K experts per token and their weights.

    Selection orders experts by (fp32 key descending, index ascending) where
    the key is the logit, or the fp32 sum logit + sel_bias[e] when a
    selection-only bias is given; a stable sort of the negated keys realises
    exactly that order.  The weights are the softmax over the K selected
    (unbiased) logits, i.e. the router's probability distribution renormalised
    to the chosen experts (pplx-kernels page, "Introductie"):
    w_k = exp(l_k - m) / sum_j exp(l_j - m) with m the largest selected logit,
    in float64, stored as float32.
    """
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    key = lg if sel_bias is None else lg + np.asarray(sel_bias, dtype=np.float32)[None, :]
    order = np.argsort(-key, axis=1, kind="stable")
    idx = order[:, :K].astype(np.int32)
    sel = np.take_along_axis(lg, idx, axis=1).astype(np.float64)
    ex = np.exp(sel - sel.max(axis=1, keepdims=True))
    w = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    return idx, w


# ----------------------------------------------------------------------------
# Histogram, capacity, overflow
# ----------------------------------------------------------------------------

def expert_histogram(topk_idx: np.ndarray, E: int) -> np.ndarray:
    """cnt_e = number of (token, k) assignments routed to expert e."""
    return np.bincount(np.asarray(topk_idx).reshape(-1), minlength=E).astype(np.int64)[:E]


def capacity_overflow(counts: np.ndarray, C: int):
    """Step 2 of the "MoE Expert Parallel Benchmark" page: overflow_e =
    max(assigned_e - C, 0); effective tokens = sum_e (assigned_e - overflow_e)."""
    counts = np.asarray(counts, dtype=np.int64)
    overflow = np.maximum(counts - C, 0)
    kept = counts - overflow
    return kept, overflow, int(kept.sum()), int(overflow.sum())


# ----------------------------------------------------------------------------
# Owner-aligned offsets and the permutation
# ----------------------------------------------------------------------------

def aligned_offsets(kept: np.ndarray, A: int, S: int):
    """Exclusive scan of the kept counts, each rounded up to the row
    alignment A: off[0] = 0, off[e+1] = off[e] + ceil(kept_e / A) * A
    (the cumulative sum of the EFA page's "Диспетчеризация и комбинирование",
    with the alignment that makes every expert start a tile boundary, so that
    a tile never spans two owners, as in the remote-owner-aligned layout).
    Owner segment s holds experts [s*E/S, (s+1)*E/S), so its rows start at
    off[s*E/S]."""
    kept = np.asarray(kept, dtype=np.int64)
    E = kept.shape[0]
    padded = ((kept + A - 1) // A) * A
    off = np.zeros(E + 1, dtype=np.int64)
    off[1:] = np.cumsum(padded)
    per = E // S
    seg = off[np.arange(S + 1) * per]
    return off, seg


def positions(topk_idx: np.ndarray, E: int) -> np.ndarray:
    """pos[t,k] = rank of assignment (t,k) among all assignments of its
    expert, in token order.  A stable sort of the flattened expert ids
    (flattened in (t,k) order) groups the assignments by expert and keeps
    token order inside each group; the rank is the place in the group."""
    flat = np.asarray(topk_idx, dtype=np.int64).reshape(-1)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    group_start = np.zeros(E + 1, dtype=np.int64)
    group_start[1:] = np.cumsum(counts)
    pos = np.empty_like(flat)
    pos[order] = np.arange(flat.size) - group_start[flat[order]]
    return pos.reshape(np.asarray(topk_idx).shape)


def permutation(topk_idx: np.ndarray, E: int, C: int, off: np.ndarray, R_max: int):
    """token_slot[t,k] = off_e + pos[t,k] if pos[t,k] < C else -1 (first come,
    first kept); row_src[slot] = t*K + k for every kept assignment, -1 on
    padding rows.  row_src is the return address the pplx-kernels page's
    dispatch stores for the combine ("Dispatch")."""
    idx = np.asarray(topk_idx, dtype=np.int64)
    T, K = idx.shape
    pos = positions(idx, E)
    slot = np.where(pos < C, off[idx] + pos, -1).astype(np.int32)
    row_src = np.full(R_max, -1, dtype=np.int32)
    kept_mask = slot >= 0
    tk = (np.arange(T)[:, None] * K + np.arange(K)[None, :]).astype(np.int32)
    row_src[slot[kept_mask]] = tk[kept_mask]
    return slot, row_src


def route(logits: np.ndarray, K: int, C: int, A: int, S: int, sel_bias: np.ndarray | None = None):
    """Steps a1-a3 together: top-K, histogram, capacity/overflow, offsets and
    the permutation.  Returns a dict of the route outputs."""
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    idx, w = route_topk(lg, K, sel_bias)
    cnt = expert_histogram(idx, E)
    kept, overflow, effective, total_overflow = capacity_overflow(cnt, C)
    off, seg = aligned_offsets(kept, A, S)
    R_max = max_rows(T, K, E, C, A)
    slot, row_src = permutation(idx, E, C, off, R_max)
    totals = np.array([T * K, effective, total_overflow, int(off[E])], dtype=np.int32)
    return {
        "topk_idx": idx, "topk_w": w,
        "expert_counts": cnt.astype(np.int32), "overflow": overflow.astype(np.int32),
        "kept": kept.astype(np.int32),
        "expert_offsets": off.astype(np.int32), "segment_offsets": seg.astype(np.int32),
        "token_slot": slot, "row_src": row_src, "totals": totals, "R_max": R_max,
    }


# ----------------------------------------------------------------------------
# Dispatch
# ----------------------------------------------------------------------------

def dispatch(x: np.ndarray, token_slot: np.ndarray, R_max: int) -> np.ndarray:
    """xp[slot[t,k]] = x[t] (a bit copy) for every kept assignment.  Rows that
    no assignment fills are left as zeros here; their contents are
    unspecified in the layer and never reach an output."""
    x = np.asarray(x)
    xp = np.zeros((R_max,) + x.shape[1:], dtype=x.dtype)
    slot = np.asarray(token_slot)
    t_idx, k_idx = np.nonzero(slot >= 0)
    xp[slot[t_idx, k_idx]] = x[t_idx]
    return xp


# ----------------------------------------------------------------------------
# Expert MLP (grouped SwiGLU)
# ----------------------------------------------------------------------------

def silu(a: np.ndarray) -> np.ndarray:
    """silu(a) = a * sigmoid(a) = a / (1 + exp(-a))."""
    return a / (1.0 + np.exp(-a))


def expert_mlp_rows(xp_rows: np.ndarray, w_gu_e: np.ndarray, w_d_e: np.ndarray, act: str):
    """SwiGLU MLP of one expert on some of its rows.

    g = x Wg^T, u = x Wu^T (float64 sums of exactly widened inputs),
    h = silu(g) * u rounded to the activation dtype, y = h W_d^T rounded to
    the activation dtype.  Wg = w_gu_e[:F], Wu = w_gu_e[F:].
    Returns (h_act, y_act)."""
    F = w_gu_e.shape[0] // 2
    x = act_to_f64(xp_rows, act)
    wg = act_to_f64(w_gu_e[:F], act)
    wu = act_to_f64(w_gu_e[F:], act)
    wd = act_to_f64(w_d_e, act)
    g = x @ wg.T
    u = x @ wu.T
    h = f64_to_act(silu(g) * u, act)
    y = f64_to_act(act_to_f64(h, act) @ wd.T, act)
    return h, y


def expert_mlp(xp: np.ndarray, expert_offsets: np.ndarray, kept: np.ndarray,
               w_gu: np.ndarray, w_d: np.ndarray, act: str):
    """Grouped SwiGLU over every expert's kept rows [off_e, off_e + kept_e).
    Returns (h, y) with the same row count as xp; rows outside any expert's
    kept range are zero."""
    R = xp.shape[0]
    E, twoF, H = w_gu.shape
    F = twoF // 2
    dt = np.uint16 if act == ACT_BF16 else np.float32
    h = np.zeros((R, F), dtype=dt)
    y = np.zeros((R, H), dtype=dt)
    for e in range(E):
        lo, n = int(expert_offsets[e]), int(kept[e])
        if n == 0:
            continue
        he, ye = expert_mlp_rows(xp[lo:lo + n], w_gu[e], w_d[e], act)
        h[lo:lo + n] = he
        y[lo:lo + n] = ye
    return h, y


# ----------------------------------------------------------------------------
# Combine
# ----------------------------------------------------------------------------

def combine(y: np.ndarray, token_slot: np.ndarray, topk_w: np.ndarray, act: str,
            y_shared: np.ndarray | None = None) -> np.ndarray:
    """out[t] = sum over k with slot[t,k] != -1 of w[t,k] * y[slot[t,k]], summed
    in float64 in k order, plus the shared expert's output y_shared[t] (weight
    1) when there is one, rounded once to the activation dtype.  Dropped
    assignments contribute nothing and the remaining weights are not
    renormalised; a token with every assignment dropped (and no shared
    expert) gets zeros."""
    slot = np.asarray(token_slot)
    T, K = slot.shape
    H = y.shape[1]
    acc = np.zeros((T, H), dtype=np.float64)
    w = np.asarray(topk_w, dtype=np.float32).astype(np.float64)
    for k in range(K):
        s = slot[:, k]
        m = s >= 0
        acc[m] += w[m, k][:, None] * act_to_f64(y[s[m]], act)
    if y_shared is not None:
        acc += act_to_f64(y_shared, act)
    return f64_to_act(acc, act)


# ----------------------------------------------------------------------------
# The whole layer
# ----------------------------------------------------------------------------

def layer_forward(logits, x, w_gu, w_d, K: int, C: int, A: int, S: int, act: str,
                  n_shared: int = 0):
    """route -> dispatch -> expert MLP -> combine.  With n_shared = 1 the last
    expert of w_gu / w_d is a shared expert that every token uses with weight 1
    on top of its routed experts (its rows are the tokens themselves).
    Returns (out, intermediates)."""
    E_routed = w_gu.shape[0] - n_shared
    r = route(logits, K, C, A, S)
    xp = dispatch(x, r["token_slot"], r["R_max"])
    h, y = expert_mlp(xp, r["expert_offsets"], r["kept"], w_gu[:E_routed], w_d[:E_routed], act)
    y_sh = None
    if n_shared:
        _, y_sh = expert_mlp_rows(x, w_gu[E_routed], w_d[E_routed], act)
    out = combine(y, r["token_slot"], r["topk_w"], act, y_shared=y_sh)
    r.update(xp=xp, h=h, y=y, y_shared=y_sh)
    return out, r
