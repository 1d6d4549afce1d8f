"""The bounds-checked build of the library (libmoe_check.so: -DMOE_CHECK_BOUNDS,
see moe_debug_bounds_failures in include/moe.h). Every kernel there checks its
internal index invariants (decoded tiles, TMEM columns, shared-memory staging
offsets, table indices) and counts failures instead of stopping. These tests
run the small parity cases of the other GPU test files, and then three
full-size layers, against the oracle in a child process that loads the
checked build, and require them to pass with no failed check. (The driver's sanitizer is not available on this machine; this
is the library's own stand-in for it.)"""
import os
import subprocess
import sys
import tempfile

import pytest

import combine_moe_route_13_b200 as M

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECK_LIB = os.path.join(ROOT, "combine_moe_route_13_b200", "libmoe_check.so")

# small parity cases: one-rank layers (bf16 pair and single-CTA tiles, fp32,
# shared expert, overlap), fp8, router, and the expert-parallel layer with and
# without tile signalling
CASES = [
    "tests/test_gpu_parity.py::test_layer_forward_end_to_end",
    "tests/test_gpu_parity.py::test_expert_mlp_bf16",
    "tests/test_gpu_parity.py::test_dispatch_bit_exact",
    "tests/test_gpu_parity.py::test_combine_matches_explicit_weighted_sum",
    "tests/test_gpu_parity.py::test_route_bit_exact",
    "tests/test_gpu_shared.py",
    "tests/test_gpu_overlap.py::test_overlap_is_bit_identical",
    "tests/test_gpu_fp8.py",
    "tests/test_gpu_router.py",
    "tests/test_gpu_ep.py::test_ep_layer_matches_oracle",
    "tests/test_gpu_ep_tiles.py::test_tile_signalled_layer",
    "tests/test_gpu_ep_fp8.py::test_ep_fp8_layer",
    "tests/test_gpu_ep_fp8_tiles.py::test_tile_signalled_fp8_layer",
]

# full-size layers: the Kimi-K2-shaped layer in bf16 (with a shared expert)
# and fp8, and the tile-signalled expert-parallel Mixtral layer in remote-first
# order, so that every index the kernels compute at the largest shapes is checked
FULL_CASES = [
    "tests/test_gpu_workloads.py::test_workload_full_size[kimi-1]",
    "tests/test_gpu_fp8_workloads.py::test_workload_full_size_fp8[kimi-0]",
    "tests/test_gpu_ep_workloads.py::test_workload_full_size_ep[mixtral-2-3]",
]


def test_release_build_has_no_checks(cuda_ok):
    with pytest.raises(M.MoeError) as e:
        M.moe_debug_bounds_failures()
    assert e.value.code == M.MOE_ERR_UNSUPPORTED


def _run_checked(cases, select=None):
    assert os.path.exists(CHECK_LIB), "build it: python combine_moe_route_13_b200/build.py --check"
    with tempfile.TemporaryDirectory() as d:
        report = os.path.join(d, "bounds.txt")
        env = dict(os.environ, MOE_LIBRARY="libmoe_check.so", MOE_BOUNDS_REPORT=report)
        cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu"]
        if select:
            cmd += ["-k", select]
        r = subprocess.run(cmd + list(cases), cwd=ROOT, env=env, capture_output=True, text=True,
                           timeout=1500)
        assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
        with open(report) as f:
            n, line = (int(v) for v in f.read().split())
    assert n == 0, f"{n} failed bounds checks, the first at source line {line}"


def test_parity_cases_pass_with_no_failed_bounds_check(cuda_ok):
    _run_checked(CASES, "not mixtral and not full_size")


def test_full_size_layers_pass_with_no_failed_bounds_check(cuda_ok):
    _run_checked(FULL_CASES)
