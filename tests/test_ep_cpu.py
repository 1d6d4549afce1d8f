"""Host-side checks of the expert-parallel ABI (no GPU needed): sizes against
the oracle, validation, the ctypes mirrors of the header's structs, argument
errors caught before any launch, and the handle exchange of a process group
(gloo, two ranks)."""
import ctypes
import os
import time
import re

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import combine_moe_route_13_b200 as M
from combine_moe_route_13_b200 import ep as EP
from oracle import moe_oracle as O
from oracle import moe_oracle_ep as P
import workloads as W

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "moe_ep.h")


def cfg_of(name, **kw):
    w = W.WORKLOADS[name]
    d = dict(T=w.T, H=w.H, E=w.E, K=w.K, F=w.F, S=w.S,
             capacity=O.capacity(w.T, w.K, w.E, w.cf), row_align=w.row_align, act=w.act)
    d.update(kw)
    return M.make_config(**d)


@pytest.mark.parametrize("name,world", [("mixtral", 2), ("mixtral", 8), ("dsv3", 8), ("dsv3", 4),
                                        ("skewed", 8), ("kimi", 16), ("tiny", 2), ("mixtral", 1)])
def test_recv_rows_match_oracle(name, world):
    c = cfg_of(name)
    assert M.moe_ep_recv_rows(c, world) == P.recv_rows_max(c.T, c.K, c.E, c.capacity,
                                                            c.row_align, world)
    R = M.moe_ep_recv_rows(c, world)
    es = 4 if c.act_dtype == M.MOE_F32 else 2
    sym = M.moe_ep_symmetric_bytes(c, world)
    assert sym >= 2 * R * c.H * es + world * c.E * 4 + 3 * world * 4
    assert M.moe_ep_workspace_bytes(c, world) >= R * c.F * es


def test_one_rank_sizes_equal_the_one_rank_layer():
    c = cfg_of("mixtral")
    assert M.moe_ep_recv_rows(c, 1) == M.moe_max_rows(c)


@pytest.mark.parametrize("kw,world,rank,epoch,code", [
    (dict(), 3, 0, 1, M.MOE_ERR_INVALID_ARG),            # E % W
    (dict(S=2), 4, 0, 1, M.MOE_ERR_INVALID_ARG),         # S % W
    (dict(), 0, 0, 1, M.MOE_ERR_INVALID_ARG),
    (dict(), 2, 2, 1, M.MOE_ERR_INVALID_ARG),            # rank >= W
    (dict(), 2, -1, 1, M.MOE_ERR_INVALID_ARG),
    (dict(), 2, 0, 0, M.MOE_OK),                         # epoch 0: the device step counter
    (dict(n_shared=1), 2, 0, 1, M.MOE_OK),               # bf16 with a shared expert
    (dict(H=4100), 2, 0, 1, M.MOE_ERR_UNSUPPORTED),      # what the one-rank GEMM rejects
    (dict(), 2, 1, 7, M.MOE_OK),
])
def test_check(kw, world, rank, epoch, code):
    c = cfg_of("mixtral", **kw)
    assert M.moe_ep_check(c, M.make_ep(world, rank, epoch)) == code


@pytest.mark.parametrize("kw,flags,code", [
    (dict(), M.MOE_EP_TILE_SIGNAL, M.MOE_OK),
    (dict(), M.MOE_EP_TILE_SIGNAL | M.MOE_EP_REMOTE_FIRST, M.MOE_OK),
    (dict(n_shared=1), M.MOE_EP_TILE_SIGNAL, M.MOE_OK),
    (dict(), M.MOE_EP_REMOTE_FIRST, M.MOE_ERR_INVALID_ARG),    # the order knob alone
    (dict(), 4, M.MOE_ERR_INVALID_ARG),                        # an unknown flag
    (dict(row_align=64), M.MOE_EP_TILE_SIGNAL, M.MOE_ERR_UNSUPPORTED),   # 128-row blocks
])
def test_check_tile_signal_flags(kw, flags, code):
    # moe_ep.h: tile signalling needs bf16 and row_align % 128 == 0
    c = cfg_of("mixtral", **kw)
    assert M.moe_ep_check(c, M.make_ep(2, 0, 1, 0, flags)) == code


def test_tile_signal_needs_bf16_activations():
    c = cfg_of("tiny", S=2, row_align=128)   # fp32 activations
    assert M.moe_ep_check(c, M.make_ep(2, 0, 1, 0, M.MOE_EP_TILE_SIGNAL)) == M.MOE_ERR_UNSUPPORTED
    # the fp8 layer (bf16 activations, e4m3 payload) takes both tile flags: with
    # a valid configuration the missing workspace is the first error found
    c = cfg_of("mixtral")
    fake = 1 << 40
    for flags in (M.MOE_EP_TILE_SIGNAL, M.MOE_EP_TILE_SIGNAL | M.MOE_EP_REMOTE_FIRST):
        ep = M.make_ep(2, 0, 1, 0, flags)
        got = M.LIB.moe_ep_dispatch_fp8(ctypes.byref(c), ctypes.byref(ep), fake, fake, fake, None,
                                        1 << 40, None)
        assert got == M.MOE_ERR_WORKSPACE, flags


def test_fp8_remote_first_needs_its_tables_to_fit():
    # the remote-first order's two extra tables per local expert live in the
    # fp8 GEMM's shared memory: 512 local experts do not fit beside six stages
    c = M.make_config(T=16384, H=256, E=512, K=8, F=256, S=1, capacity=320, row_align=128)
    fake = 1 << 40
    for flags, code in ((M.MOE_EP_TILE_SIGNAL, M.MOE_ERR_WORKSPACE),
                        (M.MOE_EP_TILE_SIGNAL | M.MOE_EP_REMOTE_FIRST, M.MOE_ERR_UNSUPPORTED)):
        ep = M.make_ep(1, 0, 1, 0, flags)
        got = M.LIB.moe_ep_dispatch_fp8(ctypes.byref(c), ctypes.byref(ep), fake, fake, fake, None,
                                        1 << 40, None)
        assert got == code, (flags, got)


def test_shared_expert_with_fp32_activations():
    c = cfg_of("tiny", S=2, n_shared=1)   # fp32: the CUDA-core GEMM runs the shared expert
    assert M.moe_ep_check(c, M.make_ep(2, 0, 1)) == M.MOE_OK


@pytest.mark.parametrize("kw,code", [
    (dict(), M.MOE_OK),
    (dict(n_shared=1), M.MOE_OK),               # each rank's shared expert in fp8
    (dict(H=4160), M.MOE_ERR_UNSUPPORTED),      # H % 256 != 0
    (dict(F=14400), M.MOE_ERR_UNSUPPORTED),     # F % 128 != 0
])
def test_fp8_entry_points_check_the_fp8_limits(kw, code):
    c = cfg_of("mixtral", **kw)
    ep = M.make_ep(2, 0, 1)
    big, fake = 1 << 40, 1 << 40
    got = M.LIB.moe_ep_dispatch_fp8(ctypes.byref(c), ctypes.byref(ep), fake, fake, fake, None,
                                    big, None)
    # with a valid configuration the missing workspace is the first error found
    assert got == (M.MOE_ERR_WORKSPACE if code == M.MOE_OK else code)


def test_too_many_ranks_unsupported():
    c = M.make_config(T=64, H=256, E=128, K=2, F=256, S=128, capacity=8)
    assert M.moe_ep_check(c, M.make_ep(128, 0, 1)) == M.MOE_ERR_UNSUPPORTED
    assert M.moe_ep_check(c, M.make_ep(64, 63, 1)) == M.MOE_OK
    assert M.moe_ep_recv_rows(c, 128) == -1
    assert M.moe_ep_symmetric_bytes(c, 128) == 0


def _fields(struct):
    src = open(HEADER).read()
    body = re.search(r"typedef struct \{([^{}]*)\} " + struct + ";", src).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    return re.findall(r"\*?\b([A-Za-z_]+)\s*[,;]", body)


def test_structs_match_header():
    assert [n for n, _ in M.MoeEp._fields_] == _fields("moe_ep_t")
    assert ctypes.sizeof(M.MoeEp) == 20
    assert [n for n, _ in M.MoeEpAux._fields_] == _fields("moe_ep_aux_t")


def test_aux_layout_is_inside_the_buffers():
    c = cfg_of("mixtral")
    world = 4
    sym, ws = 1 << 40, 1 << 41   # host-only: nothing is dereferenced
    aux = M.MoeEpAux()
    ep = M.make_ep(world, 2, 1)
    assert M.LIB.moe_ep_aux(ctypes.byref(c), ctypes.byref(ep), sym, ws, ctypes.byref(aux)) == M.MOE_OK
    nsym = M.moe_ep_symmetric_bytes(c, world)
    nws = M.moe_ep_workspace_bytes(c, world)
    R = M.moe_ep_recv_rows(c, world)
    for f in ("counts_all", "flags", "y_ready", "xr", "y"):
        assert sym <= getattr(aux, f) < sym + nsym, f
    # the ready counters (2 banks of ceil(R/128)) lie before xr, inside the zeroed head
    assert aux.y_ready + 2 * ((R + 127) // 128) * 4 <= aux.xr
    assert aux.y + R * c.H * 2 <= sym + nsym
    for f in ("topk_idx", "expert_counts", "token_slot", "send_dst_row", "recv_offsets",
              "recv_counts", "recv_split", "h"):
        v = getattr(aux, f)
        assert ws + 256 <= v < ws + nws and v % 256 == 0, f
    assert aux.h + R * c.F * 2 <= ws + nws
    assert aux.h_shared is None and aux.y_shared is None
    cs = cfg_of("mixtral", n_shared=1)
    assert M.LIB.moe_ep_aux(ctypes.byref(cs), ctypes.byref(ep), sym, ws, ctypes.byref(aux)) == M.MOE_OK
    nws = M.moe_ep_workspace_bytes(cs, world)
    assert ws < aux.h_shared < aux.y_shared and aux.y_shared + cs.T * cs.H * 2 <= ws + nws


def test_entry_points_reject_bad_arguments_before_any_launch():
    lib = M.LIB
    c = cfg_of("tiny", S=2)
    ep = M.make_ep(2, 0, 1)
    big = 1 << 30
    fake = 1 << 40
    # no symmetric region / peers
    assert lib.moe_ep_route(ctypes.byref(c), ctypes.byref(ep), fake, None, fake, fake, big, None) \
        == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_dispatch(ctypes.byref(c), ctypes.byref(ep), fake, fake, None, fake, big,
                               None) == M.MOE_ERR_INVALID_ARG
    # workspace too small, or misaligned
    assert lib.moe_ep_combine(ctypes.byref(c), ctypes.byref(ep), fake, fake, fake, fake, 256,
                              None) == M.MOE_ERR_WORKSPACE
    assert lib.moe_ep_expert_mlp(ctypes.byref(c), ctypes.byref(ep), None, fake, fake, fake, fake,
                                 fake + 16, big, None) == M.MOE_ERR_WORKSPACE
    # weights missing
    assert lib.moe_ep_expert_mlp(ctypes.byref(c), ctypes.byref(ep), None, None, fake, fake, fake,
                                 fake, big, None) == M.MOE_ERR_INVALID_ARG
    # a shared expert needs x
    cs = cfg_of("mixtral", n_shared=1)
    assert lib.moe_ep_expert_mlp(ctypes.byref(cs), ctypes.byref(ep), None, fake, fake, fake, fake,
                                 fake, big, None) == M.MOE_ERR_INVALID_ARG
    # a bad config
    assert lib.moe_ep_layer_forward(None, ctypes.byref(ep), fake, fake, fake, fake, fake, fake,
                                    fake, None, fake, big, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_symmetric_init(ctypes.byref(c), 2, fake, 16, None) == M.MOE_ERR_WORKSPACE
    assert lib.moe_ep_workspace_init(ctypes.byref(c), 2, fake, 256, None) == M.MOE_ERR_WORKSPACE
    assert lib.moe_ipc_open(None, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_sym_alloc(0, None) == M.MOE_ERR_INVALID_ARG


# ---------------------------------------------------------------- handle exchange (gloo)

def _exchange_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        own = bytes([rank]) * 64
        opened = []

        def open_handle(h):
            opened.append(h[0])
            return 1000 + h[0]

        addrs = EP.exchange_addresses(own, 7 + rank, open_handle)
        q.put((rank, addrs, opened))
    finally:
        dist.destroy_process_group()


def test_handle_exchange_two_ranks():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_exchange_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(2):
        r, addrs, opened = q.get(timeout=120)
        got[r] = (addrs, opened)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # rank r keeps its own address and opens the other rank's handle, in rank order
    assert got[0] == ([7, 1001], [1])
    assert got[1] == ([1000, 8], [0])


# ---------------------------------------------------------------- EpGroup host logic (gloo)

def _group_worker(rank, world, port, q, device_epoch):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from combine_moe_route_13_b200 import _binding as B
        calls = []
        fake = {
            "moe_ep_check": lambda cfg, ep: B.MOE_OK,
            "moe_ep_symmetric_bytes": lambda cfg, w: 4096,
            "moe_ep_workspace_bytes": lambda cfg, w: 1024,
            "moe_ep_sym_alloc": lambda n: 1000 + rank,
            "moe_ipc_get_handle": lambda addr: bytes([addr % 256]) * 64,
            "moe_ipc_open": lambda h: calls.append(("open", h[0])) or 2000 + h[0],
            # rank 1 closes its import late: every rank's free must still wait for it
            "moe_ipc_close": lambda addr: (time.sleep(0.2 if rank == 1 else 0.0),
                                           calls.append(("close", addr, time.monotonic()))),
            "moe_ep_sym_free": lambda addr: calls.append(("free", addr, time.monotonic())),
            "moe_ep_workspace_init": lambda cfg, w, ws: calls.append(("ws_init", w)),
            "moe_ep_symmetric_init": lambda cfg, w, sym, n: calls.append(("sym_init", sym, n)),
            "moe_ep_layer_forward": lambda cfg, ep, *a: calls.append(
                ("forward", ep.world, ep.rank, ep.epoch)),
        }
        for k, v in fake.items():
            setattr(B, k, v)
        cfg = M.make_config(T=64, H=256, E=8, K=2, F=256, S=2, capacity=20)
        g = EP.EpGroup(cfg, device="cpu", device_epoch=device_epoch)
        peers = g.peers.tolist()
        for _ in range(3):
            g.forward(None, None, None, None, None)
        g.close()
        q.put((rank, g.addrs, peers, calls))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("device_epoch", [False, True])
def test_ep_group_setup_steps_and_close_two_ranks(device_epoch):
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_group_worker, args=(r, 2, port, q, device_epoch))
             for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        r, addrs, peers, calls = q.get(timeout=120)
        got[r] = (addrs, peers, calls)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        addrs, peers, calls = got[r]
        other = 1 - r
        # own region kept, the other rank's region opened from its handle, in rank order
        want = [1000 + r if i == r else 2000 + (1000 + other) % 256 for i in range(2)]
        assert addrs == [] and peers == want      # addrs cleared by close()
        names = [c[0] for c in calls]
        assert names == ["open", "ws_init", "sym_init", "forward", "forward", "forward",
                         "close", "free"]
        assert calls[2] == ("sym_init", 1000 + r, 4096)
        epochs = [c[3] for c in calls if c[0] == "forward"]
        assert epochs == ([0, 0, 0] if device_epoch else [1, 2, 3])
        assert all(c[1:3] == (2, r) for c in calls if c[0] == "forward")
        assert calls[-2][:2] == ("close", want[other]) and calls[-1][:2] == ("free", 1000 + r)
    # teardown order across the processes: every import is closed before any
    # exporter frees its region (CLOCK_MONOTONIC is shared by the processes)
    closes = [c[2] for r in range(2) for c in got[r][2] if c[0] == "close"]
    frees = [c[2] for r in range(2) for c in got[r][2] if c[0] == "free"]
    assert max(closes) < min(frees), (closes, frees)
