"""The expert-parallel group's CUDA IPC plumbing on a real GPU (EpGroup,
include/moe_ep.h: moe_ep_sym_alloc, moe_ipc_get_handle / moe_ipc_open /
moe_ipc_close, moe_ep_sym_free): two processes on the one GPU this test gets,
joined by a gloo process group, each allocate their symmetric region, swap
IPC handles, map the other's region, and write into it through the mapping;
after a barrier each finds the other's bytes in its own region, and both tear
the group down (every import closed before any region is freed).

No kernel that waits on another rank runs here: on one GPU nothing guarantees
that two processes' kernels run at the same time, so the layer's flag waits
are tested with the ranks emulated in one process (test_gpu_ep*.py). The
copies through the mapping are plain runtime copies.
"""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _ipc_worker(rank, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=2,
                            timeout=datetime.timedelta(seconds=120))
    try:
        import combine_moe_route_13_b200 as M
        from combine_moe_route_13_b200.ep import EpGroup
        from cuda.bindings import runtime as rt
        torch.cuda.set_device(0)
        cfg = M.make_config(T=256, H=256, E=8, K=2, F=256, S=2, capacity=80, row_align=128)
        g = EpGroup(cfg)
        other = 1 - rank
        n = 1 << 16
        assert g.sym_bytes >= 4 * n
        off = g.sym_bytes - 2 * n          # near the end of the region: rank r's bytes at + r * n
        (e0,) = rt.cudaMemset(g.sym + off, 0, 2 * n)   # this rank's test window, cleared
        torch.cuda.synchronize()
        dist.barrier()                      # both windows clear before anyone writes
        pat = torch.full((n,), 0x40 + rank, dtype=torch.uint8, device="cuda")
        d2d = rt.cudaMemcpyKind.cudaMemcpyDeviceToDevice
        (e1,) = rt.cudaMemcpy(g.addrs[other] + off + rank * n, pat.data_ptr(), n, d2d)
        torch.cuda.synchronize()
        dist.barrier()                      # both writes done
        got = torch.zeros(n, dtype=torch.uint8, device="cuda")
        (e2,) = rt.cudaMemcpy(got.data_ptr(), g.sym + off + other * n, n, d2d)
        torch.cuda.synchronize()
        mine = torch.zeros(n, dtype=torch.uint8, device="cuda")
        (e3,) = rt.cudaMemcpy(mine.data_ptr(), g.sym + off + rank * n, n, d2d)
        torch.cuda.synchronize()
        ok_other = bool((got == 0x40 + other).all())
        untouched = bool((mine == 0).all())   # cleared above; nobody wrote here
        addrs = list(g.addrs)
        g.close()
        q.put((rank, int(e0) + int(e1), int(e2), int(e3), ok_other, untouched, addrs, g.sym))
    finally:
        dist.destroy_process_group()


def test_ep_group_ipc_mapping_two_processes_one_gpu(cuda_ok):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ipc_worker, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        r, e1, e2, e3, ok_other, untouched, addrs, sym = q.get(timeout=300)
        got[r] = (e1, e2, e3, ok_other, untouched, addrs, sym)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(2):
        e1, e2, e3, ok_other, untouched, addrs, sym = got[r]
        assert (e1, e2, e3) == (0, 0, 0), got[r]
        assert ok_other, f"rank {r}: the other rank's bytes did not arrive through the mapping"
        assert untouched, f"rank {r}: bytes outside the written range changed"
        assert addrs[r] == sym and addrs[1 - r] != sym
