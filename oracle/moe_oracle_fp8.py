"""CPU oracle for the fp8 block-scaled variant of the expert layer.

TEST INFRASTRUCTURE ONLY, like ``moe_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` may import it, and it shares no
code with the CUDA library.

Sources.  "Enabling trillion-parameter models on AWS EFA", section "Оценка":
the dispatch payload is fp8 with block scaling and the combine stays bf16.
The pplx-kernels page, "Dispatch": the dispatch sends the token rows together
with their block scale factors.  The pages fix neither the fp8 format, nor the
block shape, nor the scale encoding.  The readings taken here (listed in the
design notes):

* values are e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
  infinities, largest finite 448), rounded to nearest-even;
* one scale per 128 consecutive elements of a row along the contraction
  dimension (1 x 128 blocks), for activations and weights alike;
* a scale is a power of two 2^p, stored as the byte p + 127 (UE8M0), and p is
  the smallest integer >= -127 with amax <= 448 * 2^p, so that every scaled
  value is finite and dividing by the scale is exact;
* the expert MLP consumes the dequantised values exactly (scale * value, real
  arithmetic): g, u from x and W_gu; h = silu(g) * u; h is quantised the same
  way (its 1 x 128 blocks along F) from its fp32 value, dequantised, and
  multiplied by W_d; y is rounded to bf16 once.  The quantisation decision for
  h is taken on fp32 values because that is the precision the kernel holds h
  in (a decided integer is compared in the kernel's precision).

Scales are returned as the integer exponents p; ``scales_blocked`` writes them
in the byte layout the library's kernels read (an interface layout, not an
arithmetic step: see its docstring).
"""
from __future__ import annotations

import numpy as np

from . import moe_oracle as O

E4M3_MAX = 448.0
BLOCK = 128          # elements per scale block along the contraction dimension
P_MIN = -127         # smallest scale exponent a UE8M0 byte can hold (byte 0)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each e4m3 code: exponent field 0 is subnormal, m * 2^-9;
    otherwise (1 + m/8) * 2^(e - 7); 0x7F / 0xFF are NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even e4m3 code of each value; |v| must not exceed 448.

    For |v| >= 2^-6 with binade e (2^e <= |v| < 2^(e+1)) the code is
    8 * (e + 6) + n, n = rne(|v| * 2^(3 - e)) in [8, 16]; below 2^-6 it is
    rne(|v| * 2^9) in [0, 8].  Both branches meet continuously (n = 16 is the
    next binade's n = 8, 8 in the subnormal branch is 2^-6), so a value that
    rounds up across a binade gets the right code.  The sign is the top bit
    (a negative zero keeps it)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    if np.any(~np.isfinite(a)) or np.any(a > E4M3_MAX):
        raise ValueError("e4m3_encode: value outside [-448, 448]")
    frac, ex = np.frexp(a)                  # a = frac * 2^ex, frac in [0.5, 1)
    e = ex.astype(np.int64) - 1             # binade of a
    normal = a >= 2.0 ** -6
    n_norm = np.rint(np.ldexp(a, (3 - np.where(normal, e, 0)).astype(np.int32)))
    n_sub = np.rint(np.ldexp(a, 9))
    code = np.where(normal, 8 * (e + 6) + n_norm, n_sub).astype(np.int64)
    code |= np.where(np.signbit(v), 0x80, 0)
    return code.astype(np.uint8)


def scale_exponent(amax: np.ndarray) -> np.ndarray:
    """Smallest p >= -127 with amax <= 448 * 2^p (amax = 0 gives -127).

    With amax = f * 2^x (f in [0.5, 1)) and 448 = 0.875 * 2^9, the condition
    is f * 2^x <= 0.875 * 2^(p + 9): p = x - 9 when f <= 0.875, else x - 8."""
    amax = np.asarray(amax, dtype=np.float64)
    f, x = np.frexp(amax)
    p = np.where(f <= 0.875, x - 9, x - 8).astype(np.int64)
    p = np.where(amax == 0, P_MIN, p)
    return np.maximum(p, P_MIN)


def quantize_rows(v: np.ndarray):
    """1 x 128 block quantisation of a [rows, K] matrix (K % 128 == 0).
    Returns (codes uint8 [rows, K], p int64 [rows, K/128])."""
    v = np.asarray(v, dtype=np.float64)
    rows, K = v.shape
    assert K % BLOCK == 0
    blocks = v.reshape(rows, K // BLOCK, BLOCK)
    p = scale_exponent(np.abs(blocks).max(axis=2)) if rows else np.zeros((0, K // BLOCK), np.int64)
    scaled = np.ldexp(blocks, (-p)[:, :, None].astype(np.int32))
    return e4m3_encode(scaled).reshape(rows, K), p


def dequantize_rows(codes: np.ndarray, p: np.ndarray) -> np.ndarray:
    """Exact values scale * e4m3(code) of a [rows, K] block-quantised matrix."""
    codes = np.asarray(codes, dtype=np.uint8)
    rows, K = codes.shape
    vals = e4m3_decode(codes).reshape(rows, K // BLOCK, BLOCK)
    return np.ldexp(vals, np.asarray(p)[:, :, None].astype(np.int32)).reshape(rows, K)


def _scale_positions(rows: int, KB: int) -> np.ndarray:
    """Byte offset of scale (r, kb): [rows, KB]."""
    KG = -(-KB // 4)
    r = np.arange(rows, dtype=np.int64)[:, None]
    kb = np.arange(KB, dtype=np.int64)[None, :]
    return ((r // 128) * KG + kb // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + kb % 4


def scales_blocked(p: np.ndarray, row_blocks: int | None = None, pad: int | None = None) -> np.ndarray:
    """The scale bytes (p + 127) in the byte layout the library's kernels read.

    With KG = ceil(KB / 4), for each block of 128 rows rb and each group of
    four 128-element k blocks g there is a 512-byte chunk at offset
    (rb * KG + g) * 512; the scale of row r = 128*rb + 32*j + i (i < 32,
    j < 4) for k block kb = 4*g + s is byte 16*i + 4*j + s of it (the position
    the tensor cores read it from after copying the chunk into tensor memory).
    Bytes of rows or k blocks past the matrix get `pad` (None leaves them 0).
    This is an interface layout of the library, written out here so that the
    kernels' scale output can be compared byte for byte."""
    p = np.asarray(p, dtype=np.int64)
    rows, KB = p.shape
    RB = -(-rows // 128) if row_blocks is None else row_blocks
    out = np.full(RB * (-(-KB // 4)) * 512, 0 if pad is None else pad, dtype=np.uint8)
    out[_scale_positions(rows, KB)] = (p + 127).astype(np.uint8)
    return out


def scales_from_blocked(buf: np.ndarray, rows: int, KB: int) -> np.ndarray:
    """Inverse of scales_blocked for the first `rows` rows: p [rows, KB]."""
    buf = np.asarray(buf, dtype=np.uint8)
    return buf[_scale_positions(rows, KB)].astype(np.int64) - 127


def dispatch_fp8(x_bf16: np.ndarray, token_slot: np.ndarray, R_max: int):
    """Dispatch with the fp8 payload: row token_slot[t,k] of the grouped buffer
    receives the 1 x 128 block quantisation of x[t] (codes and scales).  Rows no
    slot points at stay zero (codes) and p = P_MIN here; the library leaves them
    unwritten.  Returns (xq [R_max,H] uint8, xp_exp [R_max,H/128] int64)."""
    xv = O.bf16_bits_to_f64(x_bf16)
    T, H = xv.shape
    q, p = quantize_rows(xv)
    xq = np.zeros((R_max, H), np.uint8)
    xe = np.full((R_max, H // BLOCK), P_MIN, np.int64)
    slot = np.asarray(token_slot)
    for t in range(T):
        for s in slot[t]:
            if s >= 0:
                xq[s] = q[t]
                xe[s] = p[t]
    return xq, xe


def expert_mlp_fp8_rows(xq, x_exp, wq_gu_e, wgu_exp_e, wq_d_e, wd_exp_e):
    """One expert's SwiGLU on block-quantised rows.  Returns
    (hq uint8 [n,F], h_exp [n,F/128], y bf16 bits [n,H], h_f32 [n,F])."""
    a = dequantize_rows(xq, x_exp)
    wgu = dequantize_rows(wq_gu_e, wgu_exp_e)
    F = wgu.shape[0] // 2
    g = a @ wgu[:F].T
    u = a @ wgu[F:].T
    h32 = (O.silu(g) * u).astype(np.float32)
    hq, h_exp = quantize_rows(h32.astype(np.float64))
    y = dequantize_rows(hq, h_exp) @ dequantize_rows(wq_d_e, wd_exp_e).T
    return hq, h_exp, O.f64_to_bf16_bits(y), h32


def down_fp8_rows(hq, h_exp, wq_d_e, wd_exp_e):
    """y = dequant(h) W_d^T rounded to bf16 (the second GEMM alone)."""
    return O.f64_to_bf16_bits(dequantize_rows(hq, h_exp) @ dequantize_rows(wq_d_e, wd_exp_e).T)


def layer_forward_fp8(logits, x_bf16, wq_gu, wgu_exp, wq_d, wd_exp, K, C, A, S, n_shared=0):
    """route -> fp8 dispatch -> fp8 expert MLP -> bf16 combine.
    wq_gu [E',2F,H] codes with wgu_exp [E',2F,H/128]; wq_d [E',H,F] with
    wd_exp [E',H,F/128], E' = E + n_shared.  With n_shared = 1 the last expert is
    the shared expert: every token's quantised row goes through it and its bf16
    output is added with weight 1 (the combine of the bf16 layer).
    Returns (out bf16 bits [T,H], intermediates)."""
    r = O.route(logits, K, C, A, S)
    R = r["R_max"]
    xq, xe = dispatch_fp8(x_bf16, r["token_slot"], R)
    Ew, twoF, H = wq_gu.shape
    E = Ew - n_shared
    F = twoF // 2
    hq = np.zeros((R, F), np.uint8)
    he = np.full((R, F // BLOCK), P_MIN, np.int64)
    y = np.zeros((R, H), np.uint16)
    off, kept = r["expert_offsets"], r["kept"]
    for e in range(E):
        n = int(kept[e])
        if n == 0:
            continue
        sl = slice(int(off[e]), int(off[e]) + n)
        hq[sl], he[sl], y[sl], _ = expert_mlp_fp8_rows(xq[sl], xe[sl], wq_gu[e], wgu_exp[e],
                                                       wq_d[e], wd_exp[e])
    y_sh = hq_sh = he_sh = None
    if n_shared:
        tq, te = quantize_rows(O.bf16_bits_to_f64(x_bf16))
        hq_sh, he_sh, y_sh, _ = expert_mlp_fp8_rows(tq, te, wq_gu[E], wgu_exp[E], wq_d[E], wd_exp[E])
    out = O.combine(y, r["token_slot"], r["topk_w"], O.ACT_BF16, y_shared=y_sh)
    r.update(xq=xq, x_exp=xe, hq=hq, h_exp=he, y=y, y_shared=y_sh, hq_shared=hq_sh,
             h_exp_shared=he_sh)
    return out, r
