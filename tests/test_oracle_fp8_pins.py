"""Pins of the fp8 block-scaled oracle (CPU only).

Each function is checked against something it does not compute itself:
torch's float8_e4m3fn conversions (decode of all 256 codes, round-to-nearest-
even encode including every tie), brute force over exponents for the scale
rule, an independent inversion of the scale byte layout, and a torch
re-computation of the fp8 expert MLP whose every fp8 step goes through torch's
conversion.  Planted mistakes (a scale exponent off by one, a skipped
quantisation of h) must be caught."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from oracle import moe_oracle_fp8 as Q

F8 = torch.float8_e4m3fn


def torch_decode(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(F8).to(torch.float64).numpy()


def torch_encode(v32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(v32, np.float32)).to(F8).view(torch.uint8).numpy()


def test_decode_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours, ref = Q.e4m3_decode(codes), torch_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2
    assert np.array_equal(ours[~nan], ref[~nan])
    assert Q.e4m3_decode(np.array([0x7E], np.uint8))[0] == 448.0
    assert Q.e4m3_decode(np.array([0x01], np.uint8))[0] == 2.0 ** -9


def test_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    assert np.array_equal(Q.e4m3_encode(Q.e4m3_decode(codes)), codes)


def test_encode_ties_and_random_values_match_torch():
    pos = np.unique(Q.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = (pos[:-1] + pos[1:]) / 2          # every tie, exactly representable in fp32
    rng = np.random.default_rng(0)
    vals = np.concatenate([mids, -mids, rng.uniform(-448, 448, 20000),
                           rng.standard_normal(20000) * 0.01, [0.0, -0.0, 448.0, -448.0]])
    v32 = vals.astype(np.float32)
    assert np.array_equal(Q.e4m3_encode(v32.astype(np.float64)), torch_encode(v32))


def test_encode_rejects_out_of_range():
    with pytest.raises(ValueError):
        Q.e4m3_encode(np.array([449.0]))


def test_scale_exponent_is_the_smallest_fitting_power_of_two():
    rng = np.random.default_rng(1)
    amax = np.concatenate([
        np.exp2(rng.uniform(-140, 120, 3000)),
        448.0 * np.exp2(np.arange(-130, 110, dtype=np.float64)),            # exact boundaries
        np.nextafter(448.0 * np.exp2(np.arange(-120, 110, dtype=np.float64)), np.inf),
        [0.0, 1.0, 448.0, 449.0, 2.0 ** -150]])
    p = Q.scale_exponent(amax)
    for a, pe in zip(amax, p):
        best = -127
        while a > 448.0 * 2.0 ** best:
            best += 1
        assert pe == best, (a, pe, best)


def test_quantize_rows_bounds_and_minimality():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((37, 384)) * np.exp2(rng.integers(-20, 20, (37, 1)))
    v[3, :128] = 0.0                           # an all-zero block
    q, p = Q.quantize_rows(v)
    d = Q.dequantize_rows(q, p)
    scaled = np.abs(v.reshape(37, 3, 128)) / np.exp2(p)[:, :, None]
    assert scaled.max() <= 448.0
    amax = scaled.max(axis=2)
    # minimality: halving the scale would overflow, unless the block is all zero
    assert np.all((amax > 224.0) | (np.abs(v.reshape(37, 3, 128)).max(axis=2) == 0))
    assert p[3, 0] == -127 and np.all(q[3, :128] == 0)
    # error at most half a code step: 2^-4 relative for normals, 2^-10 * scale absolute below
    step = np.maximum(np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1e-300)))) / 8.0,
                      2.0 ** -9 * np.repeat(np.exp2(p), 128, axis=1))
    assert np.all(np.abs(d - v) <= step / 2 * (1 + 1e-12))


def test_quantize_matches_torch_conversion():
    rng = np.random.default_rng(3)
    v = (rng.standard_normal((9, 256)) * 3).astype(np.float32).astype(np.float64)
    q, p = Q.quantize_rows(v)
    for r in range(9):
        for b in range(2):
            blk = v[r, 128 * b:128 * (b + 1)]
            s = 2.0 ** p[r, b]
            assert np.array_equal(q[r, 128 * b:128 * (b + 1)], torch_encode((blk / s).astype(np.float32)))


def test_scale_layout_by_independent_inversion():
    rows, KB = 300, 6
    p = np.arange(rows * KB, dtype=np.int64).reshape(rows, KB) % 200 - 100
    buf = Q.scales_blocked(p, pad=127)
    assert buf.size == 3 * 2 * 512
    # walk the bytes and invert the position formula independently
    for off in range(buf.size):
        chunk, o = divmod(off, 512)
        rb, g = divmod(chunk, 2)
        row, kb = 128 * rb + 32 * ((o % 16) // 4) + o // 16, 4 * g + o % 4
        want = p[row, kb] + 127 if row < rows and kb < KB else 127
        assert buf[off] == want, (off, row, kb)
    assert np.array_equal(Q.scales_from_blocked(buf, rows, KB), p)


def _torch_mlp_fp8(xq, xe, wq_gu, wgu_e, wq_d, wd_e):
    """The fp8 MLP with every fp8 step through torch's float8 conversions."""
    def deq(c, pe):
        vals = torch_decode(c).reshape(c.shape[0], -1, 128)
        return (vals * np.exp2(pe)[:, :, None]).reshape(c.shape[0], -1)
    a, wgu, wd = deq(xq, xe), deq(wq_gu, wgu_e), deq(wq_d, wd_e)
    F = wgu.shape[0] // 2
    g, u = torch.from_numpy(a @ wgu[:F].T), torch.from_numpy(a @ wgu[F:].T)
    h32 = (torch.nn.functional.silu(g) * u).float().numpy()
    n = h32.shape[0]
    blocks = h32.reshape(n, F // 128, 128).astype(np.float64)
    amax = np.abs(blocks).max(axis=2)
    pe = np.array([[min(p for p in range(-127, 130) if a_ <= 448.0 * 2.0 ** p) for a_ in row]
                   for row in amax])
    hq = np.stack([torch_encode((blocks[i] / np.exp2(pe[i])[:, None]).astype(np.float32).reshape(-1))
                   for i in range(n)])
    y = deq(hq, pe) @ wd.T
    return hq, pe, torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _fp8_case(seed, n=40, H=256, F=256):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, H))
    wgu = rng.standard_normal((2 * F, H)) * 0.05
    wd = rng.standard_normal((H, F)) * 0.05
    xq, xe = Q.quantize_rows(x)
    gq, ge = Q.quantize_rows(wgu)
    dq, de = Q.quantize_rows(wd)
    return x, wgu, wd, xq, xe, gq, ge, dq, de


def test_expert_mlp_fp8_matches_torch_float8_pipeline():
    _, _, _, xq, xe, gq, ge, dq, de = _fp8_case(4)
    hq, he, y, _ = Q.expert_mlp_fp8_rows(xq, xe, gq, ge, dq, de)
    rq, re_, ry = _torch_mlp_fp8(xq, xe, gq, ge, dq, de)
    assert np.array_equal(hq, rq) and np.array_equal(he, re_)
    assert np.array_equal(y, ry)


def test_expert_mlp_fp8_is_close_to_the_bf16_definition():
    # the fp8 layer approximates the full-precision SwiGLU within a few percent
    x, wgu, wd, xq, xe, gq, ge, dq, de = _fp8_case(5)
    _, _, y, _ = Q.expert_mlp_fp8_rows(xq, xe, gq, ge, dq, de)
    g, u = x @ wgu[:256].T, x @ wgu[256:].T
    ref = (O.silu(g) * u) @ wd.T
    got = O.bf16_bits_to_f64(y)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 0.08, rel


def test_planted_scale_mistake_is_caught(monkeypatch):
    _, _, _, xq, xe, gq, ge, dq, de = _fp8_case(6)
    rq, re_, ry = _torch_mlp_fp8(xq, xe, gq, ge, dq, de)
    real = Q.scale_exponent
    monkeypatch.setattr(Q, "scale_exponent", lambda a: real(a) + 1)
    hq, he, y, _ = Q.expert_mlp_fp8_rows(xq, xe, gq, ge, dq, de)
    assert not np.array_equal(he, re_)
    assert not np.array_equal(hq, rq)


def test_skipping_h_quantisation_is_caught():
    _, _, _, xq, xe, gq, ge, dq, de = _fp8_case(7)
    _, _, ry = _torch_mlp_fp8(xq, xe, gq, ge, dq, de)
    _, _, y, h32 = Q.expert_mlp_fp8_rows(xq, xe, gq, ge, dq, de)
    assert np.array_equal(y, ry)
    # a version that multiplies the unquantised h differs from the pinned result
    y_skip = O.f64_to_bf16_bits(h32.astype(np.float64) @ Q.dequantize_rows(dq, de).T)
    assert not np.array_equal(y_skip, ry)


def test_dispatch_fp8_rows_are_the_token_quantisation():
    rng = np.random.default_rng(8)
    T, H, E, K = 50, 256, 4, 2
    x = O.f64_to_bf16_bits(rng.standard_normal((T, H)))
    r = O.route(rng.standard_normal((T, E)), K, O.capacity(T, K, E, 0.8), 4, 2)
    xq, xe = Q.dispatch_fp8(x, r["token_slot"], r["R_max"])
    for t in range(T):
        tq = torch_encode(O.bf16_bits_to_f64(x[t:t + 1]).reshape(2, 128).astype(np.float32)
                          / np.exp2(Q.scale_exponent(np.abs(O.bf16_bits_to_f64(x[t:t + 1]))
                                                      .reshape(2, 128).max(axis=1)))[:, None])
        for s in r["token_slot"][t]:
            if s >= 0:
                assert np.array_equal(xq[s], tq.reshape(-1))
    unused = r["row_src"] < 0
    assert np.all(xq[unused] == 0)


def test_layer_forward_fp8_combines_in_bf16():
    rng = np.random.default_rng(9)
    T, H, F, E, K = 64, 128, 128, 4, 2
    x = O.f64_to_bf16_bits(rng.standard_normal((T, H)))
    gq, ge = Q.quantize_rows(rng.standard_normal((E * 2 * F, H)) * 0.05)
    dq, de = Q.quantize_rows(rng.standard_normal((E * H, F)) * 0.05)
    gq, ge = gq.reshape(E, 2 * F, H), ge.reshape(E, 2 * F, 1)
    dq, de = dq.reshape(E, H, F), de.reshape(E, H, 1)
    lg = rng.standard_normal((T, E))
    out, r = Q.layer_forward_fp8(lg, x, gq, ge, dq, de, K, T, 1, 2)
    ref = O.combine(r["y"], r["token_slot"], r["topk_w"], O.ACT_BF16)
    assert np.array_equal(out, ref)


def test_fp8_shared_expert_is_the_dense_fp8_mlp_of_every_token():
    # every routed assignment dropped (C = 0): the layer is the shared expert
    # alone, i.e. the torch float8 pipeline applied to all tokens
    rng = np.random.default_rng(10)
    T, H, F, E, K = 48, 256, 256, 4, 2
    x = O.f64_to_bf16_bits(rng.standard_normal((T, H)))
    gq, ge = Q.quantize_rows(rng.standard_normal(((E + 1) * 2 * F, H)) * 0.05)
    dq, de = Q.quantize_rows(rng.standard_normal(((E + 1) * H, F)) * 0.05)
    gq, ge = gq.reshape(E + 1, 2 * F, H), ge.reshape(E + 1, 2 * F, 2)
    dq, de = dq.reshape(E + 1, H, F), de.reshape(E + 1, H, 2)
    lg = rng.standard_normal((T, E))
    out, r = Q.layer_forward_fp8(lg, x, gq, ge, dq, de, K, 0, 1, 2, n_shared=1)
    xq, xe = Q.quantize_rows(O.bf16_bits_to_f64(x))
    _, _, ry = _torch_mlp_fp8(xq, xe, gq[E], ge[E], dq[E], de[E])
    assert np.array_equal(out, ry)
    # with routing kept, out = routed combine + shared output
    out2, r2 = Q.layer_forward_fp8(lg, x, gq, ge, dq, de, K, T, 1, 2, n_shared=1)
    routed = O.combine(r2["y"], r2["token_slot"], r2["topk_w"], O.ACT_BF16,
                       y_shared=r2["y_shared"])
    assert np.array_equal(out2, routed)
    assert not np.array_equal(out2, O.combine(r2["y"], r2["token_slot"], r2["topk_w"], O.ACT_BF16))
