"""CPU oracle for the expert-parallel layer: W ranks, each with its own tokens,
rank d owning the experts [d*E/W, (d+1)*E/W).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its CPU-baseline and reference legs) may import this module.
The CUDA library never imports, links or calls it, and it shares no code,
table or helper with the CUDA library.

What the pages fix, and how it is written out here:

* "Enabling trillion-parameter models on AWS EFA", "Буферы отправки и
  получения": before any token moves, the ranks exchange their token counts
  per expert; from them every sender knows where its rows go and every
  receiver knows at which offset each sender's rows arrive.  Inside a node
  the receive buffers are mapped into the peers, which write into them
  directly.  The combine copies the expert outputs back and takes the weighted
  average.
* "Efficient and portable Mixture-of-Experts communication", "Draagbare
  kernels": the number of tokens a rank may send is fixed, which bounds what a
  rank receives for each local expert from each sender, so that every sender
  derives a unique destination address without synchronising with the other
  senders; after receipt the tokens are laid out as the expert GEMM needs.
* "Mixture-of-Experts acceleration through overlap": the
  remote-owner-aligned layout, in which the rows bound for one owner are
  contiguous.

Readings where the pages are silent (listed in the design notes):

* capacity is enforced by each sender on its own batch, as in the one-rank
  layer (the per-sender bound above): a rank's route is exactly the
  one-rank route of its tokens over all E experts;
* the receive layout of owner d is the grouped-GEMM layout of its local
  experts: local expert j's rows start on a multiple of A, and within an
  expert the senders' blocks follow in rank order, each block in the
  sender's own row order (token order);
* the expert output of a row is returned to the token's rank and combined
  there exactly as in the one-rank layer (weights in k order, dropped
  assignments contribute zero);
* a shared expert (n_shared = 1) is held by every rank and applied to the
  rank's own tokens, its output added with weight 1 after the routed terms
  (the pages run it while the dispatch transfers are in flight: "Enabling
  trillion-parameter models on AWS EFA", "Диспетчеризация и комбинирование";
  "Efficient and portable Mixture-of-Experts communication", "Draagbare
  kernels").

Consequence used as the pin: for every rank, the expert-parallel layer equals
the one-rank layer of that rank's tokens over all E experts.

Activation tensors are numpy float32 arrays (fp32) or uint16 bf16 bit
patterns (bf16), as in the one-rank oracle.
"""
from __future__ import annotations

import numpy as np

from oracle import moe_oracle as O


def owner(e: int, E: int, W: int) -> int:
    """Rank that holds expert e: experts are split into W equal consecutive
    ranges, rank d holding [d*E/W, (d+1)*E/W)."""
    return e // (E // W)


def recv_rows_max(T: int, K: int, E: int, C: int, A: int, W: int) -> int:
    """Rows of a receive buffer: every sender contributes at most
    T * min(K, E/W) rows to one owner (a token picks distinct experts) and at
    most C rows per local expert; each local expert's start is rounded up to
    a multiple of A."""
    El = E // W
    c = T if C < 0 else C
    return min(W * T * min(K, El), El * W * c) + El * (A - 1)


def ep_plan(counts_all: np.ndarray, C: int, A: int, rank: int):
    """The layout every rank derives from the exchanged per-expert counts.

    counts_all[s, e] is sender s's count for expert e before capacity;
    kept[s, e] = min(counts_all[s, e], C).  For the owner d of expert e
    (local index j = e - d*E/W):
      recv_counts_d[j]  = sum over senders of kept[s, e]
      recv_offsets_d    = exclusive scan of recv_counts_d, each rounded up to A
      block_row_d[j, s] = recv_offsets_d[j] + sum over s' < s of kept[s', e]
    and rank r sends its kept rows of expert e to owner(e), starting at
      send_dst_row_r[e] = block_row_owner(e)[j, r].
    Returns the arrays of rank `rank` (its sends, and its receive layout)."""
    counts_all = np.asarray(counts_all, dtype=np.int64)
    W, E = counts_all.shape
    El = E // W
    c = counts_all.max(initial=0) if C < 0 else C
    kept = np.minimum(counts_all, c)
    block_row = np.zeros((W, El, W), dtype=np.int64)     # [owner, local expert, sender]
    recv_offsets = np.zeros((W, El + 1), dtype=np.int64)
    recv_counts = np.zeros((W, El), dtype=np.int64)
    for d in range(W):
        row = 0
        for j in range(El):
            e = d * El + j
            recv_offsets[d, j] = row
            n = 0
            for s in range(W):
                block_row[d, j, s] = row + n
                n += int(kept[s, e])
            recv_counts[d, j] = n
            row += (n + A - 1) // A * A
        recv_offsets[d, El] = row
    send_dst_row = np.array([block_row[e // El, e % El, rank] for e in range(E)], dtype=np.int64)
    return {
        "kept_all": kept.astype(np.int32),
        "send_dst_row": send_dst_row.astype(np.int32),
        "recv_offsets": recv_offsets[rank].astype(np.int32),
        "recv_counts": recv_counts[rank].astype(np.int32),
        "block_row": block_row[rank].astype(np.int32),     # [El, W]
        "block_rows": kept[:, rank * El:(rank + 1) * El].T.astype(np.int32),   # [El, W]
    }


def ep_layer_forward(logits, x, w_gu, w_d, K: int, C: int, A: int, S: int, act: str, W: int,
                     n_shared: int = 0):
    """W ranks: logits[r] [T,E], x[r] [T,H]; w_gu [E',2F,H], w_d [E',H,F] with
    E' = E + n_shared (all experts; rank d uses its own E/W routed experts,
    and every rank the shared expert, the last one, on its own tokens).  Steps:
      1. every rank routes its own tokens (the one-rank route);
      2. the per-expert counts are exchanged (counts_all[s] = rank s's counts);
      3. every rank lays out its sends and its receive buffer (ep_plan);
      4. dispatch: rank s writes x_s[t] for each kept (t, k) to row
         send_dst_row_s[e] + (slot - off_s[e]) of owner(e)'s receive buffer;
      5. every owner runs its local experts' SwiGLU on their receive rows;
      6. combine: rank s sums, in k order, w[t,k] times the owner's output
         row of each kept assignment (found by the same address as in 4),
         then adds its shared expert's output with weight 1 (n_shared = 1).
    Returns (outs [W arrays T x H], per-rank intermediates)."""
    E = w_gu.shape[0] - n_shared
    El = E // W
    T = np.asarray(logits[0]).shape[0]
    H = np.asarray(x[0]).shape[1]
    routes = [O.route(logits[r], K, C, A, S) for r in range(W)]
    counts_all = np.stack([r["expert_counts"] for r in routes]).astype(np.int64)
    plans = [ep_plan(counts_all, C, A, r) for r in range(W)]
    Rr = recv_rows_max(T, K, E, C, A, W)
    dt = np.uint16 if act == O.ACT_BF16 else np.float32
    xr = [np.zeros((Rr, H), dtype=dt) for _ in range(W)]

    def dest_row(s, t, k):
        slot = int(routes[s]["token_slot"][t, k])
        e = int(routes[s]["topk_idx"][t, k])
        return owner(e, E, W), int(plans[s]["send_dst_row"][e]) + slot - int(routes[s]["expert_offsets"][e])

    for s in range(W):
        for t, k in zip(*np.nonzero(routes[s]["token_slot"] >= 0)):
            d, row = dest_row(s, t, k)
            xr[d][row] = np.asarray(x[s])[t]
    ys, hs = [], []
    for d in range(W):
        p = plans[d]
        h, y = O.expert_mlp(xr[d], p["recv_offsets"], p["recv_counts"],
                            w_gu[d * El:(d + 1) * El], w_d[d * El:(d + 1) * El], act)
        hs.append(h)
        ys.append(y)
    y_sh = [O.expert_mlp_rows(np.asarray(x[s]), w_gu[E], w_d[E], act)[1] if n_shared else None
            for s in range(W)]
    outs = []
    for s in range(W):
        r = routes[s]
        acc = np.zeros((T, H), dtype=np.float64)
        w = np.asarray(r["topk_w"], dtype=np.float32).astype(np.float64)
        for k in range(K):
            for t in np.nonzero(r["token_slot"][:, k] >= 0)[0]:
                d, row = dest_row(s, t, k)
                acc[t] += w[t, k] * O.act_to_f64(ys[d][row:row + 1], act)[0]
        if n_shared:
            acc += O.act_to_f64(y_sh[s], act)
        outs.append(O.f64_to_act(acc, act))
    inter = [dict(routes[r], **plans[r], counts_all=counts_all.astype(np.int32), xr=xr[r],
                  h=hs[r], y=ys[r], y_shared=y_sh[r], R_recv=Rr) for r in range(W)]
    return outs, inter
