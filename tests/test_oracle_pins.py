"""Pins of the CPU oracle to facts outside itself (no GPU needed).

Each test checks the oracle against something it does not compute itself:
values printed on the pages (tests/golden), closed forms, brute force on tiny
inputs written here as plain loops, independent library routines (torch,
scipy), or exact special cases of the layer (identity experts).
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import moe_oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# helpers written from the definitions, independent of the oracle's code
# ----------------------------------------------------------------------------

def brute_topk(row, K):
    """Repeatedly take the largest remaining logit; equal logits go to the
    lower expert index."""
    remaining = list(range(len(row)))
    chosen = []
    for _ in range(K):
        best = remaining[0]
        for e in remaining[1:]:
            if row[e] > row[best]:
                best = e
        chosen.append(best)
        remaining.remove(best)
    return chosen


def brute_permutation(idx, E, C, A, S):
    """Loops over tokens in order with one running counter per expert."""
    T, K = len(idx), len(idx[0])
    cnt = [0] * E
    for t in range(T):
        for k in range(K):
            cnt[idx[t][k]] += 1
    kept = [min(c, C) for c in cnt]
    off = [0]
    for e in range(E):
        pad = kept[e] if kept[e] % A == 0 else kept[e] + (A - kept[e] % A)
        off.append(off[-1] + pad)
    seg = [off[s * (E // S)] for s in range(S + 1)]
    R_max = min(T * K, E * C) + E * (A - 1)
    slot = [[-1] * K for _ in range(T)]
    row_src = [-1] * R_max
    running = [0] * E
    for t in range(T):
        for k in range(K):
            e = idx[t][k]
            p = running[e]
            running[e] += 1
            if p < C:
                slot[t][k] = off[e] + p
                row_src[off[e] + p] = t * K + k
    return cnt, kept, off, seg, slot, row_src


def bf16_bits_of(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

def test_bf16_widening_matches_torch_for_every_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = O.bf16_bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # round trip of every non-NaN pattern (signed zeros included)
    back = O.f64_to_bf16_bits(ours[~nan])
    assert np.array_equal(back, bits[~nan])


def test_bf16_rounding_matches_torch_on_fp32_values():
    # For inputs that are exact fp32 values torch's conversion is a single
    # round-to-nearest-even, so it must agree bit for bit.
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        rng.standard_normal(2000) * 1e-39,                       # bf16 subnormals
        np.array([0.0, -0.0, 3.3895313892515355e38, 3.4e38, -3.4e38, 1e-45]),
    ]).astype(np.float32).astype(np.float64)
    # exact halfway cases between neighbouring bf16 values
    base = O.bf16_bits_to_f64(rng.integers(0x0080, 0x7F00, 5000).astype(np.uint16))
    halfway = base * (1.0 + 2.0 ** -8)
    v = np.concatenate([v, halfway.astype(np.float32).astype(np.float64)])
    ours = O.f64_to_bf16_bits(v)
    ref = bf16_bits_of(torch.from_numpy(v.astype(np.float32)))
    assert np.array_equal(ours, ref)


def test_bf16_rounding_is_single_rounding_from_f64():
    # 1 + 2^-8 + 2^-30 lies just above the midpoint of 1 and 1 + 2^-7, so the
    # nearest bf16 is 1 + 2^-7 (bits 0x3F81); rounding through fp32 first would
    # land on the midpoint and give 1.0.
    assert O.f64_to_bf16_bits(np.array([1 + 2.0 ** -8 + 2.0 ** -30]))[0] == 0x3F81
    assert O.f64_to_bf16_bits(np.array([1 + 2.0 ** -8]))[0] == 0x3F80       # tie -> even
    assert O.f64_to_bf16_bits(np.array([1 + 3 * 2.0 ** -8]))[0] == 0x3F82   # tie -> even
    assert O.f64_to_bf16_bits(np.array([-2.5]))[0] == 0xC020
    assert O.f64_to_bf16_bits(np.array([1e39]))[0] == 0x7F80                # overflow -> inf


# ----------------------------------------------------------------------------
# capacity
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("name,C", [("tiny", 20), ("mixtral", 1280), ("dsv3", 48),
                                    ("skewed", 1536), ("kimi", 854)])
def test_capacity_of_the_workloads(name, C):
    # hand arithmetic: 1.25*64*2/8 = 20; 1.25*4096*2/8 = 1280; 1.5*1024*8/256 = 48;
    # 1.0*16384*6/64 = 1536; 1.25*32768*8/384 = 853.33... -> 854
    w = W.WORKLOADS[name]
    assert O.capacity(w.T, w.K, w.E, w.cf) == C


def test_capacity_rounds_up_and_no_limit():
    assert O.capacity(10, 3, 4, 1.0) == 8       # 7.5 -> 8
    assert O.capacity(10, 3, 4, 0.0) == 0
    assert O.capacity(10, 3, 4, -1.0) == 10     # no limit: C = T


# ----------------------------------------------------------------------------
# top-K and weights
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("E,K", [(1, 1), (3, 2), (8, 2), (8, 8), (17, 5), (64, 6)])
def test_topk_matches_brute_force(E, K):
    g = torch.Generator().manual_seed(E * 100 + K)
    for logits in (torch.randn(40, E, generator=g), W.tied_logits(40, E, 3, g)):
        lg = logits.numpy()
        idx, w = O.route_topk(lg, K)
        for t in range(lg.shape[0]):
            assert list(idx[t]) == brute_topk(list(lg[t]), K)


def test_topk_special_cases():
    g = torch.Generator().manual_seed(5)
    lg = torch.randn(30, 9, generator=g).numpy()
    idx, w = O.route_topk(lg, 9)                        # K = E: a permutation
    assert all(sorted(r) == list(range(9)) for r in idx.tolist())
    idx1, w1 = O.route_topk(lg, 1)                      # K = 1: weight exactly 1
    assert np.all(w1 == 1.0)
    assert np.array_equal(idx1[:, 0], np.argmax(lg, axis=1))
    same = np.zeros((4, 6), dtype=np.float32)           # all equal: lowest indices, w = 1/K
    idx4, w4 = O.route_topk(same, 4)
    assert np.array_equal(idx4, np.tile(np.arange(4), (4, 1)))
    assert np.all(w4 == 0.25)
    signed_zero = np.array([[0.0, -0.0, 0.0]], dtype=np.float32)   # -0 == +0: index decides
    assert list(O.route_topk(signed_zero, 2)[0][0]) == [0, 1]


def test_weights_closed_form_k2():
    g = torch.Generator().manual_seed(7)
    lg = (torch.randn(200, 16, generator=g) * 3).numpy()
    idx, w = O.route_topk(lg, 2)
    l0 = np.take_along_axis(lg, idx[:, :1], 1)[:, 0].astype(np.float64)
    l1 = np.take_along_axis(lg, idx[:, 1:2], 1)[:, 0].astype(np.float64)
    sig = 1.0 / (1.0 + np.exp(l1 - l0))                 # w0 = sigmoid(l0 - l1)
    assert np.allclose(w[:, 0], sig, rtol=1e-7, atol=0)
    assert np.allclose(w[:, 1], 1.0 - sig, rtol=1e-6, atol=1e-12)


def test_weights_are_full_softmax_renormalised():
    g = torch.Generator().manual_seed(8)
    lg = torch.randn(100, 24, generator=g).numpy()
    K = 5
    idx, w = O.route_topk(lg, K)
    p = scipy.special.softmax(lg.astype(np.float64), axis=1)   # the router's distribution
    sel = np.take_along_axis(p, idx, 1)
    ref = sel / sel.sum(axis=1, keepdims=True)
    assert np.allclose(w, ref, rtol=2e-7, atol=0)
    assert np.all(np.diff(w, axis=1) <= 0)                       # descending like the logits


# ----------------------------------------------------------------------------
# histogram, capacity, overflow
# ----------------------------------------------------------------------------

def test_histogram_brute_force():
    g = torch.Generator().manual_seed(9)
    lg = torch.randn(77, 12, generator=g).numpy()
    idx, _ = O.route_topk(lg, 3)
    cnt = O.expert_histogram(idx, 12)
    loop = [0] * 12
    for t in range(77):
        for k in range(3):
            loop[idx[t, k]] += 1
    assert list(cnt) == loop
    assert cnt.sum() == 77 * 3


def test_overflow_matches_page_records():
    rec = json.load(open(os.path.join(GOLDEN, "p5_capacity_records.json")))
    # The skewed record: 1000 assignments, 280 overflow, 720 effective.  Any
    # per-expert split with those totals must give them back; one such split
    # with capacity 250: [530, 250, 120, 100] -> overflow [280, 0, 0, 0].
    kept, overflow, effective, total_overflow = O.capacity_overflow(np.array([530, 250, 120, 100]), 250)
    skewed = rec["records"][2]
    assert total_overflow == skewed["overflow"] and effective == skewed["effective_tokens"]
    assert list(kept) == [250, 250, 120, 100]
    # The two balanced records: 1000 assignments under capacity -> no overflow.
    _, _, eff_b, ov_b = O.capacity_overflow(np.array([250, 250, 250, 250]), 250)
    assert (eff_b, ov_b) == (1000, 0)
    assert eff_b + eff_b + effective == rec["expected"]["total_effective_tokens"]
    assert max(ov_b, total_overflow) == rec["expected"]["max_overflow"]


def test_overflow_definitions_brute_force():
    rng = np.random.default_rng(3)
    for _ in range(50):
        cnt = rng.integers(0, 40, rng.integers(1, 20))
        C = int(rng.integers(0, 45))
        kept, ov, eff, tov = O.capacity_overflow(cnt, C)
        for e in range(len(cnt)):
            assert ov[e] == (cnt[e] - C if cnt[e] > C else 0)
            assert kept[e] + ov[e] == cnt[e]
        assert eff == sum(int(c) - int(o) for c, o in zip(cnt, ov))
        assert tov == sum(int(o) for o in ov)


# ----------------------------------------------------------------------------
# offsets and permutation
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("T,E,K,S,cf,A", [
    (64, 8, 2, 2, 1.25, 1), (64, 8, 2, 2, 1.25, 128), (50, 16, 4, 4, 0.5, 8),
    (33, 6, 6, 3, 1.0, 4), (100, 12, 3, 1, -1.0, 1), (10, 4, 2, 4, 0.0, 16)])
def test_permutation_brute_force(T, E, K, S, cf, A):
    g = torch.Generator().manual_seed(T + E + K)
    lg = torch.randn(T, E, generator=g)
    lg[:, 0] += 1.5                                      # one hot expert, so that overflow occurs
    C = O.capacity(T, K, E, cf)
    r = O.route(lg.numpy(), K, C, A, S)
    cnt, kept, off, seg, slot, row_src = brute_permutation(r["topk_idx"].tolist(), E, C, A, S)
    assert list(r["expert_counts"]) == cnt
    assert list(r["kept"]) == kept
    assert list(r["expert_offsets"]) == off
    assert list(r["segment_offsets"]) == seg
    assert r["token_slot"].tolist() == slot
    assert r["row_src"].tolist() == row_src
    assert r["totals"].tolist() == [T * K, sum(kept), sum(cnt) - sum(kept), off[-1]]


def test_permutation_is_a_bijection_in_owner_order():
    T, E, K, S, A = 300, 16, 4, 4, 8
    g = torch.Generator().manual_seed(11)
    lg = torch.randn(T, E, generator=g) - 0.3 * torch.arange(E)
    C = O.capacity(T, K, E, 1.0)
    r = O.route(lg.numpy(), K, C, A, S)
    slot, row_src, off = r["token_slot"], r["row_src"], r["expert_offsets"]
    kept_tk = [(t, k) for t in range(T) for k in range(K) if slot[t, k] >= 0]
    assert len(kept_tk) == r["totals"][1]
    seen = sorted(int(v) for v in row_src if v >= 0)
    assert seen == sorted(t * K + k for t, k in kept_tk)          # each kept (t,k) exactly once
    for t, k in kept_tk:
        assert row_src[slot[t, k]] == t * K + k
    prev = (-1, -1)                                              # rows sorted by (expert, token)
    for row in range(off[-1]):
        if row_src[row] < 0:
            continue
        t, k = divmod(int(row_src[row]), K)
        e = int(r["topk_idx"][t, k])
        assert off[e] <= row < off[e + 1]
        assert (e, t) > prev
        prev = (e, t)
        s = e // (E // S)                                        # inside its owner segment
        assert r["segment_offsets"][s] <= row < r["segment_offsets"][s + 1]
    assert all(o % A == 0 for o in off)


def test_hand_worked_route_example():
    # T=4, E=4, K=2, S=2, cf=1 -> C = ceil(4*2/4) = 2.
    lg = np.array([[0.5, 2.0, -1.0, 1.0],     # top-2: e1, e3
                   [1.0, 1.0, 0.0, 3.0],      # e3, then the tie e0/e1 goes to e0
                   [0.0, 0.0, 0.0, 0.0],      # e0, e1
                   [-2.0, 4.0, 4.0, 0.0]],    # e1, e2 (tie at 4 -> lower index first)
                  dtype=np.float32)
    C = O.capacity(4, 2, 4, 1.0)
    assert C == 2
    r = O.route(lg, 2, C, 1, 2)
    assert r["topk_idx"].tolist() == [[1, 3], [3, 0], [0, 1], [1, 2]]
    s1, s2 = 1 / (1 + math.exp(-1.0)), 1 / (1 + math.exp(-2.0))
    assert np.allclose(r["topk_w"], [[s1, 1 - s1], [s2, 1 - s2], [0.5, 0.5], [0.5, 0.5]], rtol=1e-7)
    # e0: t1, t2 -> 2; e1: t0, t2, t3 -> 3 (t3 overflows); e2: t3 -> 1; e3: t0, t1 -> 2
    assert r["expert_counts"].tolist() == [2, 3, 1, 2]
    assert r["overflow"].tolist() == [0, 1, 0, 0]
    assert r["expert_offsets"].tolist() == [0, 2, 4, 5, 7]
    assert r["segment_offsets"].tolist() == [0, 4, 7]
    assert r["token_slot"].tolist() == [[2, 5], [6, 0], [1, 3], [-1, 4]]
    assert r["row_src"].tolist() == [3, 4, 0, 5, 7, 1, 2, -1]
    assert r["totals"].tolist() == [8, 7, 1, 7]
    r4 = O.route(lg, 2, C, 4, 2)                          # A = 4: every expert starts at a multiple of 4
    assert r4["expert_offsets"].tolist() == [0, 4, 8, 12, 16]
    assert r4["segment_offsets"].tolist() == [0, 8, 16]
    assert r4["token_slot"].tolist() == [[4, 12], [13, 0], [1, 5], [-1, 8]]
    rs = [-1] * 20
    for row, v in [(0, 3), (1, 4), (4, 0), (5, 5), (8, 7), (12, 1), (13, 2)]:
        rs[row] = v
    assert r4["row_src"].tolist() == rs
    # combine with identity experts: t3 keeps only half of its row (no renormalisation)
    x = np.array([[1, 2], [3, 4], [5, 6], [7, 8]], dtype=np.float32)
    xp = O.dispatch(x, r["token_slot"], r["R_max"])
    out = O.combine(xp, r["token_slot"], r["topk_w"], O.ACT_F32)
    assert np.allclose(out[:3], x[:3], rtol=1e-7)
    assert out[3].tolist() == [3.5, 4.0]


def test_capacity_extremes():
    T, E, K, S = 60, 8, 3, 2
    g = torch.Generator().manual_seed(12)
    lg = torch.randn(T, E, generator=g).numpy()
    r = O.route(lg, K, O.capacity(T, K, E, 100.0), 1, S)         # no drops
    assert r["totals"][2] == 0 and r["totals"][3] == T * K
    assert r["expert_offsets"].tolist() == [0] + list(np.cumsum(O.expert_histogram(r["topk_idx"], E)))
    r0 = O.route(lg, K, 0, 1, S)                                  # C = 0: everything dropped
    assert np.all(r0["token_slot"] == -1) and np.all(r0["row_src"] == -1)
    assert r0["totals"].tolist() == [T * K, 0, T * K, 0]
    x = torch.randn(T, 16, generator=g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    out = O.combine(np.zeros((1, 16), np.uint16), r0["token_slot"], r0["topk_w"], O.ACT_BF16)
    assert np.all(O.bf16_bits_to_f64(out) == 0.0)
    assert x.shape == (T, 16)


# ----------------------------------------------------------------------------
# dispatch + combine round trip, combine = explicit weighted sum
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("act", [O.ACT_F32, O.ACT_BF16])
@pytest.mark.parametrize("K,equal", [(1, False), (2, True), (4, True)])
def test_round_trip_identity_experts(act, K, equal):
    T, E, H = 40, 8, 24
    g = torch.Generator().manual_seed(13)
    lg = torch.zeros(T, E) if equal else torch.randn(T, E, generator=g)
    if equal:  # all logits equal -> w = 1/K exactly; vary which experts by a per-token shift
        lg = torch.zeros(T, E)
    xt = torch.randn(T, H, generator=g)
    x = xt.numpy() if act == O.ACT_F32 else bf16_bits_of(xt)
    r = O.route(lg.numpy(), K, O.capacity(T, K, E, -1.0), 4, 2)
    xp = O.dispatch(x, r["token_slot"], r["R_max"])
    out = O.combine(xp, r["token_slot"], r["topk_w"], act)          # y := xp (identity experts)
    assert out.dtype == x.dtype and np.array_equal(out, x)


def bf16_nearest_bits(s: float) -> int:
    """The bf16 value nearest to the float64 s (ties to the even significand),
    by exact rational arithmetic: |s| = k * 2^(e-8) + r with 128 <= k < 256 (8
    significant bits); normal range only, which the values here stay in."""
    from fractions import Fraction
    import math
    if s == 0.0:
        return 0x8000 if math.copysign(1.0, s) < 0 else 0
    _, e = math.frexp(abs(s))                 # 2^(e-1) <= |s| < 2^e
    q = Fraction(abs(s)) / Fraction(2) ** (e - 8)
    k = math.floor(q)
    rem = q - k
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and k % 2 == 1):
        k += 1
    v = math.ldexp(k, e - 8) * (1.0 if s > 0 else -1.0)
    return int(np.array([v], dtype=np.float32).view(np.uint32)[0] >> 16)


def test_bf16_nearest_bits_by_hand():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties to even -> 1.0 (0x3F80);
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6 -> 1 + 2^-6 (0x3F82);
    # just above the first halfway point rounds up (0x3F81)
    assert bf16_nearest_bits(1.0 + 2 ** -8) == 0x3F80
    assert bf16_nearest_bits(1.0 + 3 * 2 ** -8) == 0x3F82
    assert bf16_nearest_bits(1.0 + 2 ** -8 + 2 ** -40) == 0x3F81
    assert bf16_nearest_bits(-2.0) == 0xC000
    assert bf16_nearest_bits(-0.0) == 0x8000


@pytest.mark.parametrize("act", [O.ACT_F32, O.ACT_BF16])
def test_combine_is_the_explicit_weighted_sum(act):
    T, K, H, R = 12, 3, 5, 40
    rng = np.random.default_rng(14)
    y32 = rng.standard_normal((R, H)).astype(np.float32)
    y = y32 if act == O.ACT_F32 else bf16_bits_of(torch.from_numpy(y32))
    slot = rng.integers(-1, R, (T, K)).astype(np.int32)
    w = rng.random((T, K)).astype(np.float32)
    out = O.combine(y, slot, w, act)
    yv = O.bf16_bits_to_f64(y) if act == O.ACT_BF16 else y.astype(np.float64)
    for t in range(T):
        for j in range(H):
            s = 0.0
            for k in range(K):
                if slot[t, k] >= 0:
                    s += float(w[t, k]) * float(yv[slot[t, k], j])
            if act == O.ACT_F32:
                assert out[t, j] == np.float32(s)
            else:
                assert out[t, j] == bf16_nearest_bits(s), (t, j, s)


# ----------------------------------------------------------------------------
# expert MLP against torch's dense SwiGLU
# ----------------------------------------------------------------------------

def torch_swiglu(x, w_gu, w_d):
    F = w_gu.shape[0] // 2
    g = x @ w_gu[:F].T
    u = x @ w_gu[F:].T
    return torch.nn.functional.silu(g) * u


@pytest.mark.parametrize("act", [O.ACT_F32, O.ACT_BF16])
def test_mlp_single_expert_equals_dense_swiglu(act):
    T, H, F = 37, 48, 80
    g = torch.Generator().manual_seed(15)
    x = torch.randn(T, H, generator=g)
    w_gu = torch.randn(1, 2 * F, H, generator=g) * 0.1
    w_d = torch.randn(1, H, F, generator=g) * 0.1
    if act == O.ACT_BF16:
        x, w_gu, w_d = (t.to(torch.bfloat16) for t in (x, w_gu, w_d))
        to_np = bf16_bits_of
    else:
        to_np = lambda t: t.numpy()  # noqa: E731
    lg = torch.zeros(T, 1).numpy()
    out, r = O.layer_forward(lg, to_np(x), to_np(w_gu), to_np(w_d), 1, T, 1, 1, act)
    h_ref = torch_swiglu(x.double(), w_gu[0].double(), w_d[0].double())
    h = O.act_to_f64(r["h"][:T], act)
    tol = 2 ** -8 if act == O.ACT_BF16 else 2 ** -23
    assert np.allclose(h, h_ref.numpy(), rtol=tol, atol=1e-30)
    y_ref = torch.from_numpy(h) @ w_d[0].double().T                # from the rounded h
    assert np.allclose(O.act_to_f64(out, act), y_ref.numpy(), rtol=tol, atol=1e-30)
    assert np.array_equal(out, r["y"][:T])                         # K = 1, w = 1: out == y


def test_grouped_mlp_uses_each_rows_own_expert():
    # Two experts with different weights; rows routed to e must equal the dense
    # SwiGLU with e's weights (catches an expert-index or offset slip).
    T, H, F, E = 30, 16, 24, 2
    g = torch.Generator().manual_seed(16)
    x = torch.randn(T, H, generator=g)
    w_gu = torch.randn(E, 2 * F, H, generator=g) * 0.2
    w_d = torch.randn(E, H, F, generator=g) * 0.2
    lg = torch.zeros(T, E)
    lg[::3, 1] = 1.0
    out, r = O.layer_forward(lg.numpy(), x.numpy(), w_gu.numpy(), w_d.numpy(), 1, T, 8, 1, O.ACT_F32)
    for t in range(T):
        e = int(r["topk_idx"][t, 0])
        ref = torch_swiglu(x[t:t + 1].double(), w_gu[e].double(), w_d[e].double()) @ w_d[e].double().T
        assert np.allclose(out[t], ref.numpy()[0], rtol=1e-5, atol=1e-7)


def test_planted_mistakes_are_caught(monkeypatch):
    # Plant plausible slips in the oracle and check that the pins above see them.
    T, H, F = 9, 8, 12
    g = torch.Generator().manual_seed(17)
    x = torch.randn(T, H, generator=g)
    w_gu = torch.randn(1, 2 * F, H, generator=g)
    w_d = torch.randn(1, H, F, generator=g)
    ref = torch_swiglu(x.double(), w_gu[0].double(), w_d[0].double()).numpy()

    def mlp_h():
        h, _ = O.expert_mlp_rows(x.numpy(), w_gu[0].numpy(), w_d[0].numpy(), O.ACT_F32)
        return h.astype(np.float64)

    assert np.allclose(mlp_h(), ref, rtol=1e-6)
    monkeypatch.setattr(O, "silu", lambda a: a / (1.0 + np.exp(a)))          # sign slip
    assert not np.allclose(mlp_h(), ref, rtol=1e-3)
    monkeypatch.undo()
    swapped = torch.cat([w_gu[0, F:], w_gu[0, :F]])                           # gate/up swapped
    h_sw, _ = O.expert_mlp_rows(x.numpy(), swapped.numpy(), w_d[0].numpy(), O.ACT_F32)
    assert not np.allclose(h_sw, ref, rtol=1e-3)


# ----------------------------------------------------------------------------
# router projection and the selection-only bias
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("act", [O.ACT_F32, O.ACT_BF16])
def test_router_logits_equal_torch_matmul(act):
    g = torch.Generator().manual_seed(21)
    x = torch.randn(33, 96, generator=g)
    w_g = torch.randn(13, 96, generator=g) / 10
    if act == O.ACT_BF16:
        x, w_g = x.to(torch.bfloat16), w_g.to(torch.bfloat16)
        to_np = bf16_bits_of
    else:
        to_np = lambda t: t.numpy()  # noqa: E731
    got = O.router_logits(to_np(x), to_np(w_g), act)
    ref = (x.double() @ w_g.double().T).float().numpy()     # x W_g^T, not W_g x
    assert got.dtype == np.float32 and got.shape == (33, 13)
    assert np.array_equal(got, ref)


def test_selection_bias_brute_force():
    g = torch.Generator().manual_seed(22)
    lg = torch.randn(60, 12, generator=g).numpy()
    bias = (torch.randn(12, generator=g) * 0.7).numpy().astype(np.float32)
    K = 4
    idx, w = O.route_topk(lg, K, bias)
    for t in range(60):
        keys = [np.float32(lg[t, e]) + np.float32(bias[e]) for e in range(12)]
        assert list(idx[t]) == brute_topk(keys, K)
        sel = [float(lg[t, e]) for e in idx[t]]          # weights from the unbiased logits
        m = max(sel)
        ex = [math.exp(v - m) for v in sel]
        assert np.allclose(w[t], [v / sum(ex) for v in ex], rtol=1e-7)
    # a bias that reorders the experts changes the selection but not how weights are made
    big = np.zeros(12, np.float32)
    big[11] = 100.0
    idx2, w2 = O.route_topk(lg, 1, big)
    assert np.all(idx2[:, 0] == 11) and np.all(w2 == 1.0)
    assert np.array_equal(O.route_topk(lg, K, np.zeros(12, np.float32))[0], O.route_topk(lg, K)[0])


# ----------------------------------------------------------------------------
# shared expert
# ----------------------------------------------------------------------------

def test_shared_expert_adds_a_dense_swiglu_of_every_token():
    # E routed experts with all-dropped routing (C = 0) leave only the shared
    # expert: out must be torch's dense SwiGLU of x with the shared weights.
    T, H, F, E = 21, 16, 24, 3
    g = torch.Generator().manual_seed(31)
    x = torch.randn(T, H, generator=g)
    w_gu = torch.randn(E + 1, 2 * F, H, generator=g) * 0.3
    w_d = torch.randn(E + 1, H, F, generator=g) * 0.3
    lg = torch.randn(T, E, generator=g).numpy()
    out, r = O.layer_forward(lg, x.numpy(), w_gu.numpy(), w_d.numpy(), 2, 0, 1, 1, O.ACT_F32,
                             n_shared=1)
    ref = torch_swiglu(x.double(), w_gu[E].double(), w_d[E].double()) @ w_d[E].double().T
    assert np.allclose(out, ref.numpy(), rtol=1e-5, atol=1e-7)
    # with routing kept, out = routed combine + shared output (the routed part unchanged)
    out2, r2 = O.layer_forward(lg, x.numpy(), w_gu.numpy(), w_d.numpy(), 2, T, 1, 1, O.ACT_F32,
                               n_shared=1)
    routed = O.combine(r2["y"], r2["token_slot"], r2["topk_w"], O.ACT_F32)
    assert np.allclose(out2, routed + r2["y_shared"], rtol=1e-5, atol=1e-6)
    assert not np.allclose(out2, routed, rtol=1e-3)
