"""Pins of the expert-parallel oracle (no GPU needed).

* Every rank's output equals the one-rank layer of that rank's tokens over all
  E experts (the one-rank oracle is pinned on its own in test_oracle_pins).
* The receive layout is rebuilt here by enumeration: walk owner d's local
  experts in order, each from a multiple of A, and within an expert the
  senders in rank order and each sender's kept assignments in token order,
  numbering rows one by one.  The oracle's scans must give the same rows.
* The layout is a bijection: every kept assignment of every sender has its
  own row inside its expert's block of its owner, and nothing else lands there.
* One rank reduces to the one-rank layout.
* Planted mistakes in the plan (senders in the wrong order, a dropped
  alignment) are seen by the pins above.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from oracle import moe_oracle_ep as P


def _inputs(W, T, H, E, K, F, act, seed, bias=0.0, n_shared=0):
    rng = np.random.default_rng(seed)
    logits = [(rng.standard_normal((T, E)) + bias * np.log(np.arange(1, E + 1))).astype(np.float32)
              for _ in range(W)]
    xs = [rng.standard_normal((T, H)).astype(np.float32) for _ in range(W)]
    w_gu = (rng.standard_normal((E + n_shared, 2 * F, H)) * 0.1).astype(np.float32)
    w_d = (rng.standard_normal((E + n_shared, H, F)) * 0.1).astype(np.float32)
    if act == O.ACT_BF16:
        xs = [O.f64_to_bf16_bits(x.astype(np.float64)) for x in xs]
        w_gu = O.f64_to_bf16_bits(w_gu.astype(np.float64))
        w_d = O.f64_to_bf16_bits(w_d.astype(np.float64))
    return logits, xs, w_gu, w_d


def brute_dest_rows(routes, W, E, C, A):
    """dest[(s, t, k)] = (owner, row) by enumeration, without scans."""
    El = E // W
    dest = {}
    ends = []
    for d in range(W):
        row = 0
        for j in range(El):
            e = d * El + j
            row = (row + A - 1) // A * A
            for s in range(W):
                r = routes[s]
                for t in range(r["token_slot"].shape[0]):
                    for k in range(r["token_slot"].shape[1]):
                        if r["topk_idx"][t, k] == e and r["token_slot"][t, k] >= 0:
                            dest[(s, t, k)] = (d, row)
                            row += 1
        ends.append(row)
    return dest, ends


def plan_dest_rows(routes, plans, E, W):
    El = E // W
    dest = {}
    for s in range(W):
        r = routes[s]
        for t, k in zip(*np.nonzero(r["token_slot"] >= 0)):
            e = int(r["topk_idx"][t, k])
            row = int(plans[s]["send_dst_row"][e]) + int(r["token_slot"][t, k]) - int(r["expert_offsets"][e])
            dest[(s, int(t), int(k))] = (e // El, row)
    return dest


CASES = [
    # W, T, E, K, cf, A, bias
    (2, 40, 8, 2, 1.25, 1, 0.0),
    (2, 40, 8, 2, 1.25, 128, 0.0),
    (4, 33, 16, 4, 0.5, 4, -2.4),      # overflow, skewed experts
    (4, 25, 8, 4, 2.0, 8, 0.0),        # E/W = 2 < K
    (3, 17, 9, 3, 1.0, 16, -2.4),
    (8, 12, 64, 8, 1.5, 128, 0.0),     # many experts per owner, most blocks tiny
]


@pytest.mark.parametrize("W,T,E,K,cf,A,bias", CASES)
def test_plan_matches_enumeration(W, T, E, K, cf, A, bias):
    rng = np.random.default_rng(T * E + W)
    logits = [(rng.standard_normal((T, E)) + bias * np.log(np.arange(1, E + 1))).astype(np.float32)
              for _ in range(W)]
    C = O.capacity(T, K, E, cf)
    S = W
    routes = [O.route(lg, K, C, A, S) for lg in logits]
    counts_all = np.stack([r["expert_counts"] for r in routes])
    plans = [P.ep_plan(counts_all, C, A, r) for r in range(W)]
    want, ends = brute_dest_rows(routes, W, E, C, A)
    got = plan_dest_rows(routes, plans, E, W)
    assert got == want
    Rr = P.recv_rows_max(T, K, E, C, A, W)
    El = E // W
    for d in range(W):
        p = plans[d]
        assert np.all(p["recv_offsets"] % A == 0)
        assert int(p["recv_offsets"][El]) == (ends[d] + A - 1) // A * A <= Rr
        rows = sorted(row for (dd, row) in want.values() if dd == d)
        assert len(rows) == len(set(rows)) == int(p["recv_counts"].sum())
        for j in range(El):
            lo, n = int(p["recv_offsets"][j]), int(p["recv_counts"][j])
            mine = [row for (s, t, k), (dd, row) in want.items()
                    if dd == d and routes[s]["topk_idx"][t, k] == d * El + j]
            assert sorted(mine) == list(range(lo, lo + n))
            assert int(p["block_rows"][j].sum()) == n
            assert np.array_equal(p["block_row"][j], lo + np.concatenate([[0], np.cumsum(p["block_rows"][j])[:-1]]))


def test_one_rank_is_the_one_rank_layout():
    rng = np.random.default_rng(5)
    lg = rng.standard_normal((50, 12)).astype(np.float32)
    C = O.capacity(50, 3, 12, 0.8)
    r = O.route(lg, 3, C, 8, 4)
    p = P.ep_plan(r["expert_counts"][None, :], C, 8, 0)
    assert np.array_equal(p["send_dst_row"], r["expert_offsets"][:12])
    assert np.array_equal(p["recv_offsets"], r["expert_offsets"])
    assert np.array_equal(p["recv_counts"], r["kept"])


@pytest.mark.parametrize("act", [O.ACT_F32, O.ACT_BF16])
@pytest.mark.parametrize("W,T,E,K,cf,A,bias", [(2, 24, 8, 2, 1.25, 8, 0.0),
                                                (4, 20, 8, 3, 0.6, 1, -2.4),
                                                (3, 10, 6, 2, 2.0, 4, 0.0)])
def test_every_rank_equals_the_one_rank_layer(act, W, T, E, K, cf, A, bias):
    H, F = 16, 12
    logits, xs, w_gu, w_d = _inputs(W, T, H, E, K, F, act, seed=W * 100 + T, bias=bias)
    C = O.capacity(T, K, E, cf)
    outs, inter = P.ep_layer_forward(logits, xs, w_gu, w_d, K, C, A, W, act, W)
    for r in range(W):
        ref, _ = O.layer_forward(logits[r], xs[r], w_gu, w_d, K, C, A, W, act)
        assert np.array_equal(outs[r], ref), f"rank {r}"
        assert inter[r]["recv_offsets"][-1] <= inter[r]["R_recv"]


@pytest.mark.parametrize("act", [O.ACT_F32, O.ACT_BF16])
def test_shared_expert_every_rank_equals_the_one_rank_layer(act):
    W, T, H, E, K, F = 3, 16, 16, 6, 2, 12
    logits, xs, w_gu, w_d = _inputs(W, T, H, E, K, F, act, seed=77, n_shared=1)
    C = O.capacity(T, K, E, 1.0)
    outs, inter = P.ep_layer_forward(logits, xs, w_gu, w_d, K, C, 4, W, act, W, n_shared=1)
    plain, _ = P.ep_layer_forward(logits, xs, w_gu[:E], w_d[:E], K, C, 4, W, act, W)
    for r in range(W):
        ref, _ = O.layer_forward(logits[r], xs[r], w_gu, w_d, K, C, 4, W, act, n_shared=1)
        assert np.array_equal(outs[r], ref), f"rank {r}"
        assert not np.array_equal(outs[r], plain[r])


def test_planted_mistakes_are_caught():
    W, T, E, K, C, A = 3, 20, 6, 2, 9, 4
    rng = np.random.default_rng(11)
    routes = [O.route(rng.standard_normal((T, E)).astype(np.float32), K, C, A, W) for _ in range(W)]
    counts_all = np.stack([r["expert_counts"] for r in routes])
    want, _ = brute_dest_rows(routes, W, E, C, A)
    real_plan = P.ep_plan

    plans = [real_plan(counts_all[::-1], C, A, W - 1 - r) for r in range(W)]  # senders reversed
    assert plan_dest_rows(routes, plans, E, W) != want
    plans = [real_plan(counts_all, C, 1, r) for r in range(W)]                # alignment dropped
    assert plan_dest_rows(routes, plans, E, W) != want
    plans = [real_plan(counts_all, C + 1000, A, r) for r in range(W)]         # capacity ignored
    assert counts_all.max() > C                                                # some expert overflows
    assert plan_dest_rows(routes, plans, E, W) != want
