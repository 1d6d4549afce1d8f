"""The synthetic input recipe (workloads.py) checked against its stated
distributions and shapes, on the CPU: router logits N(0,1) plus the
workload's per-expert bias (dsv3: N(0, 0.1^2); skewed: -2.4 ln(e+1)),
activations N(0,1), weights N(0, 0.02^2) in the activation dtype, a shared
expert as one more expert, and the same tensors for the same seed."""
import math

import numpy as np
import pytest
import torch

import workloads as W


def _std_ok(t, want, rel=0.05):
    s = float(t.double().std())
    return abs(s - want) <= rel * want, s


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_shapes_dtypes_and_unit_normals(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=0, device="cpu", weights=False)
    lg, x = inp["logits"], inp["x"]
    assert lg.shape == (wl.T, wl.E) and lg.dtype == torch.float32
    assert x.shape == (wl.T, wl.H) and x.dtype == wl.torch_act
    # bounds of five standard errors of the estimates (sample size n)
    n = x.numel()
    ok, s = _std_ok(x, 1.0, rel=5 / math.sqrt(2 * n) + 0.01)   # + bf16 rounding
    assert ok, f"x std {s}"
    assert abs(float(x.double().mean())) < 5 / math.sqrt(n)
    # the logits around each expert's column mean (its bias) are N(0,1)
    centred = lg.double() - lg.double().mean(dim=0, keepdim=True)
    ok, s = _std_ok(centred, 1.0, rel=5 / math.sqrt(2 * lg.numel()) + 1.0 / wl.T)
    assert ok, f"logit noise std {s}"


def test_skewed_bias_is_the_zipf_log_rank():
    wl = W.WORKLOADS["skewed"]
    lg = W.make_inputs(wl, seed=0, device="cpu", weights=False)["logits"].double()
    want = -2.4 * np.log(np.arange(1, wl.E + 1))
    got = lg.mean(dim=0).numpy()
    # column means of T = 16384 unit normals: standard error 1/128
    assert np.max(np.abs(got - want)) < 6 / math.sqrt(wl.T)


def test_dsv3_bias_has_std_0_1():
    wl = W.WORKLOADS["dsv3"]
    lg = W.make_inputs(wl, seed=0, device="cpu", weights=False)["logits"].double()
    col = lg.mean(dim=0)
    # Var(column mean) = 0.1^2 (the bias) + 1/T (the noise)
    s = float(col.std())
    assert abs(s - math.sqrt(0.01 + 1 / wl.T)) < 0.02, s
    # and no bias at all in mixtral
    m = W.make_inputs(W.WORKLOADS["mixtral"], seed=0, device="cpu", weights=False)["logits"]
    assert float(m.double().mean(dim=0).abs().max()) < 6 / math.sqrt(4096)


@pytest.mark.parametrize("n_shared", [0, 1])
def test_weights(n_shared):
    wl = W.small_case(64, 256, 8, 2, 384, 2, 1.25, "bf16", 128, n_shared=n_shared)
    inp = W.make_inputs(wl, seed=0, device="cpu")
    assert inp["w_gu"].shape == (wl.E + n_shared, 2 * wl.F, wl.H)
    assert inp["w_d"].shape == (wl.E + n_shared, wl.H, wl.F)
    for k in ("w_gu", "w_d"):
        assert inp[k].dtype == torch.bfloat16
        ok, s = _std_ok(inp[k], 0.02, rel=0.02)
        assert ok, f"{k} std {s}"
        assert abs(float(inp[k].double().mean())) < 1e-3


def test_same_seed_same_tensors_and_draw_order():
    wl = W.small_case(64, 256, 8, 2, 256, 2, 1.25, "bf16", 128)
    a = W.make_inputs(wl, seed=7, device="cpu")
    b = W.make_inputs(wl, seed=7, device="cpu")
    c = W.make_inputs(wl, seed=8, device="cpu")
    for k in a:
        assert torch.equal(a[k], b[k]), k
        assert not torch.equal(a[k], c[k]), k
    # the logits and x come first: drawing without weights gives the same ones
    d = W.make_inputs(wl, seed=7, device="cpu", weights=False)
    assert torch.equal(a["logits"], d["logits"]) and torch.equal(a["x"], d["x"])
