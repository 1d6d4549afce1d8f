"""moe_route_topk_noalloc: the route entry point for callers that cannot
allocate device memory (code living inside another allocator, plug-ins handed
only their input and output buffers). It keeps its scratch in a fixed 1 MiB
device array inside the library instead of a caller workspace.

Checks, through the C ABI: two calls in a row (different inputs, so that the
shared scratch is reused) give exactly what moe_route_topk gives with its own
workspace and what the oracle's route gives (indices, counts, offsets and the
permutation bit for bit, weights within the router-weight tolerance), for each
of the three route block sizes (32, 64 and 128 tokens) and for a configuration
whose scratch fills the array exactly; a configuration needing more scratch
than the array holds is refused without launching anything. This file is
collected last on purpose.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_13_b200 as M
from oracle import moe_oracle as O
from _gpu_common import assert_route_equal

pytestmark = pytest.mark.gpu


def _route_both(cfg, logits):
    ref = M.alloc_route_outputs(cfg)
    ws = M.alloc_workspace(M.moe_route_workspace_bytes(cfg))
    M.moe_route_topk(cfg, logits, ref["topk_idx"], ref["topk_w"], ref["expert_counts"],
                     ref["overflow"], ref["expert_offsets"], ref["segment_offsets"],
                     ref["token_slot"], ref["row_src"], ref["totals"], ws)
    got = M.alloc_route_outputs(cfg)
    for t in got.values():   # garbage in the outputs: everything must be written
        t.fill_(-7)
    M.moe_route_topk_noalloc(cfg, logits, got["topk_idx"], got["topk_w"], got["expert_counts"],
                             got["overflow"], got["expert_offsets"], got["segment_offsets"],
                             got["token_slot"], got["row_src"], got["totals"])
    torch.cuda.synchronize()
    return ({k: v.cpu().numpy() for k, v in got.items()},
            {k: v.cpu().numpy() for k, v in ref.items()})


# route blocks of 32 tokens (T <= 9472), 64 (T <= 18944) and 128 (above); the
# last case needs ceil(32768/128) * 1024 * 4 B = 1 MiB: the array exactly
@pytest.mark.parametrize("T,E,K,S,cf,A", [(4096, 64, 6, 8, 1.0, 128),
                                          (16384, 64, 6, 8, 1.0, 128),
                                          (32768, 384, 8, 16, 1.25, 128),
                                          (32768, 1024, 8, 16, 1.25, 128)])
def test_noalloc_route_matches_workspace_route_and_oracle_twice(cuda_ok, T, E, K, S, cf, A):
    C = O.capacity(T, K, E, cf)
    cfg = M.make_config(T, 64, E, K, 64, S, C, A, "bf16")
    R = M.moe_max_rows(cfg)
    for call, seed in enumerate((1, 2)):
        g = torch.Generator().manual_seed(seed)
        lg = torch.randn(T, E, generator=g)
        lg[:, call] += 1.0            # a different hot expert on each call
        got, ref = _route_both(cfg, lg.cuda())
        assert_route_equal(got, ref, R)
        assert np.array_equal(got["topk_w"], ref["topk_w"])
        # and the oracle's route of the same logits (weights: fp32 exp vs float64)
        o = O.route(lg.numpy(), K, C, A, S)
        assert o["R_max"] == R
        assert_route_equal(got, o, R)


def test_noalloc_route_refuses_configs_beyond_its_scratch(cuda_ok):
    # ceil(T/128) * E int32 counters must fit in MOE_NOALLOC_SCRATCH_BYTES (1 MiB)
    T, E = 128 * 1024, 512            # 1024 blocks * 512 experts * 4 B = 2 MiB
    cfg = M.make_config(T, 64, E, 2, 64, 1, 1, 1, "bf16")
    dummy = torch.empty(1, dtype=torch.int32, device="cuda")
    f = torch.empty(1, dtype=torch.float32, device="cuda")
    code = M.LIB.moe_route_topk_noalloc(
        __import__("ctypes").byref(cfg), f.data_ptr(), dummy.data_ptr(), f.data_ptr(),
        dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
        dummy.data_ptr(), dummy.data_ptr(), None)
    assert code == M.MOE_ERR_WORKSPACE
