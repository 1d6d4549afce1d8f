"""Host-side setup of the expert-parallel layer (include/moe_ep.h).

EpGroup: one rank of a group of W processes, one GPU each. Its symmetric region
is its own cudaMalloc allocation (moe_ep_sym_alloc); the ranks swap CUDA IPC
handles through torch.distributed (all_gather_object: any backend) and map each
other's regions (moe_ipc_open), so that the kernels reach the peers' memory
with plain loads and stores over NVLink. No multicast object is created.

EpOnOneDevice: W ranks of the same layer on ONE device, for tests and
measurement where only one GPU is available. Each rank has its own symmetric
region and workspace; a step runs each of the four steps for every rank
before the next step, all in one stream, so every flag a kernel waits for was
set by a kernel that finished before it started.

Both are argument plumbing: every step of the layer runs in the library's
kernels.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch

from . import _binding as B


def exchange_addresses(own_handle: bytes, own_addr: int, open_handle: Callable[[bytes], int],
                       group=None) -> list:
    """Every rank's region as an address of this process: the ranks' handles are
    gathered in rank order, this rank keeps its own address and opens the
    others'. Returns [addr of rank 0, ..., addr of rank W-1]."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    handles = [None] * world
    dist.all_gather_object(handles, own_handle, group=group)
    if handles[rank] != own_handle:
        raise RuntimeError("handle exchange out of order")
    return [own_addr if r == rank else open_handle(h) for r, h in enumerate(handles)]


class EpGroup:
    """This process's rank of a W-GPU expert-parallel layer (W = the process
    group's size). `device` is this rank's GPU (default: torch.cuda's current
    device). device_epoch: number the steps with the device-resident step
    counter (epoch 0), so that a step can be captured in a CUDA graph.
    flags: MOE_EP_TILE_SIGNAL [| MOE_EP_REMOTE_FIRST] for the tile-signalled
    layer (the same on every rank)."""

    def __init__(self, cfg: B.MoeConfig, group=None, timeout_us: int = 0, device=None,
                 device_epoch: bool = False, flags: int = 0):
        import torch.distributed as dist
        self.cfg = cfg
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.timeout_us = int(timeout_us)
        self.device_epoch = bool(device_epoch)
        self.flags = int(flags)
        st = B.moe_ep_check(cfg, B.make_ep(self.world, self.rank, 1, self.timeout_us, self.flags))
        if st != B.MOE_OK:
            raise B.MoeError(st, "EpGroup")
        self.device = (torch.device("cuda", torch.cuda.current_device()) if device is None
                       else torch.device(device))
        self.sym_bytes = B.moe_ep_symmetric_bytes(cfg, self.world)
        self.sym = B.moe_ep_sym_alloc(self.sym_bytes)
        self.addrs = exchange_addresses(B.moe_ipc_get_handle(self.sym), self.sym, B.moe_ipc_open,
                                        group)
        self.peers = torch.tensor(self.addrs, dtype=torch.int64, device=self.device)
        self.ws = B.alloc_workspace(B.moe_ep_workspace_bytes(cfg, self.world), self.device)
        B.moe_ep_workspace_init(cfg, self.world, self.ws)
        B.moe_ep_symmetric_init(cfg, self.world, self.sym, self.sym_bytes)
        self._sync()
        dist.barrier(group=group)   # every region zeroed before any rank writes into one
        self.epoch = 0

    def _sync(self):
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)

    def _ep(self) -> B.MoeEp:
        return B.make_ep(self.world, self.rank, 0 if self.device_epoch else self.epoch,
                         self.timeout_us, self.flags)

    def forward(self, logits, x, w_gu_local, w_d_local, out, stream=None) -> B.MoeEpAux:
        """One step of this rank's layer (every rank calls it once per step)."""
        self.epoch += 1
        return B.moe_ep_layer_forward(self.cfg, self._ep(), logits, x, w_gu_local, w_d_local,
                                      self.sym, self.peers, out, self.ws, stream)

    def forward_fp8(self, logits, x, wq, out, stream=None) -> B.MoeEpAux:
        """One step with the fp8 payload; wq = (codes and scales of this rank's
        gate/up weights, codes and scales of its down weights)."""
        self.epoch += 1
        return B.moe_ep_layer_forward_fp8(self.cfg, self._ep(), logits, x, *wq, self.sym,
                                          self.peers, out, self.ws, stream)

    def close(self):
        import torch.distributed as dist
        self._sync()
        dist.barrier(group=self.group)   # nobody reads a region after it is unmapped
        for r, a in enumerate(self.addrs):
            if r != self.rank:
                B.moe_ipc_close(a)
        # an exported region is freed only after every importer has closed it
        # (freeing it while another process still has it open is undefined)
        dist.barrier(group=self.group)
        B.moe_ep_sym_free(self.sym)
        self.addrs = []


class EpOnOneDevice:
    """W ranks on one device (see the module doc). device_epoch: number the
    steps with the ranks' device-resident step counters (epoch 0) instead of
    host-side step numbers, so that a step can be captured in a CUDA graph and
    replayed. flags: MOE_EP_TILE_SIGNAL [| MOE_EP_REMOTE_FIRST]."""

    def __init__(self, cfg: B.MoeConfig, world: int, device="cuda", timeout_us: int = 0,
                 device_epoch: bool = False, flags: int = 0):
        self.cfg = cfg
        self.world = int(world)
        self.timeout_us = int(timeout_us)
        self.device_epoch = bool(device_epoch)
        self.flags = int(flags)
        st = B.moe_ep_check(cfg, B.make_ep(self.world, 0, 1, self.timeout_us, self.flags))
        if st != B.MOE_OK:
            raise B.MoeError(st, "EpOnOneDevice")
        nsym = B.moe_ep_symmetric_bytes(cfg, self.world)
        nws = B.moe_ep_workspace_bytes(cfg, self.world)
        self.sym = [torch.zeros(nsym, dtype=torch.uint8, device=device) for _ in range(self.world)]
        self.ws = [B.alloc_workspace(nws, device) for _ in range(self.world)]
        self.peers = torch.tensor([s.data_ptr() for s in self.sym], dtype=torch.int64,
                                  device=device)
        for s in self.sym:
            B.moe_ep_symmetric_init(cfg, self.world, s)
        for w in self.ws:
            B.moe_ep_workspace_init(cfg, self.world, w)
        self.epoch = 0

    def ep(self, rank: int) -> B.MoeEp:
        return B.make_ep(self.world, rank, 0 if self.device_epoch else self.epoch,
                         self.timeout_us, self.flags)

    def forward(self, logits: Sequence, x: Sequence, w_gu_local: Sequence, w_d_local: Sequence,
                out: Sequence, stream=None):
        """One step of every rank: route, dispatch, expert MLP, combine, each
        for ranks 0..W-1 in turn."""
        self.epoch += 1
        c, W = self.cfg, self.world
        for r in range(W):
            B.moe_ep_route(c, self.ep(r), logits[r], self.sym[r], self.peers, self.ws[r], stream)
        for r in range(W):
            B.moe_ep_dispatch(c, self.ep(r), x[r], self.sym[r], self.peers, self.ws[r], stream)
        for r in range(W):
            B.moe_ep_expert_mlp(c, self.ep(r), x[r] if c.n_shared else None, w_gu_local[r],
                                w_d_local[r], self.sym[r], self.peers, self.ws[r], stream)
        for r in range(W):
            B.moe_ep_combine(c, self.ep(r), self.sym[r], self.peers, out[r], self.ws[r], stream)

    def forward_fp8(self, logits: Sequence, x: Sequence, wq: Sequence, out: Sequence,
                    stream=None):
        """One step of every rank with the fp8 payload; wq[r] = (codes and scales
        of rank r's gate/up weights, codes and scales of its down weights)."""
        self.epoch += 1
        c, W = self.cfg, self.world
        for r in range(W):
            B.moe_ep_route(c, self.ep(r), logits[r], self.sym[r], self.peers, self.ws[r], stream)
        for r in range(W):
            B.moe_ep_dispatch_fp8(c, self.ep(r), x[r], self.sym[r], self.peers, self.ws[r], stream)
        for r in range(W):
            B.moe_ep_expert_mlp_fp8(c, self.ep(r), *wq[r], self.sym[r], self.peers, self.ws[r],
                                    stream)
        for r in range(W):
            B.moe_ep_combine(c, self.ep(r), self.sym[r], self.peers, out[r], self.ws[r], stream)

    def views(self, rank: int) -> dict:
        aux = B.moe_ep_aux(self.cfg, B.make_ep(self.world, rank, 1), self.sym[rank],
                           self.ws[rank])
        return B.ep_views(self.cfg, self.world, self.sym[rank], self.ws[rank], aux)

    def status(self, rank: int) -> int:
        return B.moe_get_device_status(self.ws[rank])
