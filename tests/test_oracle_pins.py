"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each pin is one of: a value worked by hand from the pages (tests/golden/, with
the citation in the file), a library routine that computes the same thing by a
different route (numpy/torch IEEE casts, numpy integer and fp64 matmul), an
exact-rational model of binary32 arithmetic, a closed form (one-hot rows,
identity and permutation matrices), or an invariant the pages state (absmax
maps to +-127, dequant error <= scale/2, per-tensor equals per-channel when the
scales agree, pack/unpack round trip).  Each is chosen so that a plausible slip
in the oracle (a dropped term, a wrong sign or index, a transposed operand,
round-half-away instead of half-even, quantizing with the fp32 instead of the
stored fp16 scale) fails at least one of them.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# binary16 / bfloat16 codecs
# ----------------------------------------------------------------------------

def test_f16_decode_every_bit_pattern_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_decode(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def _f16_midpoints(rng, n):
    """binary32 values exactly halfway between adjacent binary16 values (ties)."""
    h = rng.integers(1, 0x7BFF, size=n).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2
    mid32 = mid.astype(np.float32)
    assert np.array_equal(mid32.astype(np.float64), mid)   # exact in binary32
    return mid32


def test_f32_to_f16_matches_numpy_including_ties_subnormals_overflow():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32),
        (rng.standard_normal(50_000) * 1e-5).astype(np.float32),      # fp16 subnormal range
        (rng.standard_normal(50_000) * 3e4).astype(np.float32),       # near overflow
        _f16_midpoints(rng, 50_000), -_f16_midpoints(rng, 50_000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, 2**-25, 2**-24, 1.5 * 2**-25, 5.9604645e-8],
                 dtype=np.float32),
    ])
    ours = oracle.f32_to_f16(vals)
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_f64_to_f16_matches_numpy():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.standard_normal(100_000) * s for s in (1e-6, 1e-2, 1.0, 300.0, 2e4)])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.round_f16(vals), ref)


def test_bf16_rounding_matches_torch_on_binary32_inputs():
    rng = np.random.default_rng(2)
    vals = np.concatenate([rng.standard_normal(200_000) * s for s in (1e-30, 1e-3, 1.0, 1e5, 1e30)]
                          ).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = oracle.round_bf16(vals.astype(np.float64))
    assert np.array_equal(ours, ref)
    assert np.array_equal(oracle.bf16_decode(ours),
                          torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_bf16_rounding_of_doubles_is_nearest_even():
    """Direct fp64 -> bf16: the result is the nearest neighbour, ties to the even code."""
    rng = np.random.default_rng(3)
    y = rng.standard_normal(20_000) * 10.0
    r = oracle.round_bf16(y).astype(np.int64)
    dec = lambda b: oracle.bf16_decode(np.asarray(b, dtype=np.uint16))
    mid, up, dn = dec(r), dec(r + 1), dec(r - 1)
    # for negative values the bit pattern grows with |y|, so neighbours are up/down in magnitude
    assert np.all(np.abs(y - mid) <= np.abs(y - up))
    assert np.all(np.abs(y - mid) <= np.abs(y - dn))
    # ties between two bf16 values go to the even code
    lo = np.array([0x3F80, 0x4000, 0x4101, 0xC0A3], dtype=np.int64)
    ties = (dec(lo) + dec(lo + 1)) / 2
    assert np.array_equal(oracle.round_bf16(ties) % 2, np.zeros(4, dtype=np.uint16))


# ----------------------------------------------------------------------------
# a1: symmetric per-row int8 quantization
# ----------------------------------------------------------------------------

def _read_rows(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append([p.strip() for p in line.split("|")])
    return rows


def test_quantize_rowwise_golden():
    rows = _read_rows("quantize_rowwise.txt")
    x = np.array([[float(v) for v in r[0].split()] for r in rows], dtype=np.float16)
    expect = np.array([[int(v) for v in r[1].split()] for r in rows], dtype=np.int8)
    q, s = oracle.quantize_rowwise_int8(x)
    assert np.array_equal(q, expect)
    amax = np.abs(x.astype(np.float32)).max(axis=1)
    amax = np.maximum(amax, np.float32(1e-10))
    assert np.array_equal(s, amax / np.float32(127.0))      # numpy binary32 division
    assert s[0] == 1.0


def _fl32(v: Fraction) -> Fraction:
    """Round an exact rational to the nearest binary32 (normal range), ties to even."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    quantum = Fraction(2) ** (e - 23)
    n = a / quantum
    r = round(n)                      # Fraction.__round__: half to even
    return sign * r * quantum


def test_quantize_rowwise_matches_exact_rational_binary32_model():
    """Every binary32 operation of the definition, modelled with exact rationals."""
    x = W.activations(24, 96, seed=11, outliers=True)
    q, s = oracle.quantize_rowwise_int8(x)
    for m in range(x.shape[0]):
        vals = [Fraction(float(v)) for v in x[m].astype(np.float64)]
        a = max(abs(v) for v in vals)
        inv = _fl32(Fraction(127) / a)
        for k, v in enumerate(vals):
            t = _fl32(v * inv)
            code = max(-127, min(127, round(t)))
            assert q[m, k] == code, (m, k)
        assert Fraction(float(s[m])) == _fl32(a / 127)


@pytest.mark.parametrize("seed,outliers", [(0, False), (1, True), (5, True)])
def test_quantize_rowwise_invariants(seed, outliers):
    x = W.activations(64, 512, seed=seed, outliers=outliers)
    q, s = oracle.quantize_rowwise_int8(x)
    xf = x.astype(np.float64)
    # the absmax element of every row maps to +-127, with its sign
    idx = np.abs(xf).argmax(axis=1)
    top = q[np.arange(64), idx].astype(int)
    assert np.array_equal(np.abs(top), np.full(64, 127))
    assert np.array_equal(np.sign(top), np.sign(xf[np.arange(64), idx]).astype(int))
    # range and dequant error <= scale/2, plus the binary32 roundings of 127/a, of x*inv and of
    # a/127: |x| <= 127*scale, three relative errors of 2^-24 each -> 127*3*2^-24*scale
    assert q.min() >= -127
    err = np.abs(xf - q.astype(np.float64) * s[:, None].astype(np.float64))
    assert np.all(err <= s[:, None] * (0.5 + 127 * 3 * 2.0 ** -24))
    # odd symmetry and monotonicity within a row
    qn, sn = oracle.quantize_rowwise_int8(-x)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    order = np.argsort(xf, axis=1, kind="stable")
    assert np.all(np.diff(np.take_along_axis(q.astype(int), order, axis=1), axis=1) >= 0)


def test_per_tensor_equals_per_channel_when_absmax_agrees():
    """Per-tensor quant is per-row quant with one shared scale: rows scaled to a common absmax."""
    x = W.activations(8, 256, seed=4).astype(np.float64)
    x = x / np.abs(x).max(axis=1, keepdims=True) * 3.0   # every row absmax 3 (exact in fp16)
    x16 = x.astype(np.float16)
    assert np.all(np.abs(x16.astype(np.float64)).max(axis=1) == 3.0)
    q_rows, s_rows = oracle.quantize_rowwise_int8(x16)
    q_flat, s_flat = oracle.quantize_rowwise_int8(x16.reshape(1, -1))
    assert np.all(s_rows == s_flat[0])
    assert np.array_equal(q_rows.reshape(1, -1), q_flat)


def test_quantize_rowwise_zero_row_and_tiny_rows():
    x = np.zeros((3, 32), np.float16)
    x[1, 5] = np.float16(6e-8)     # smallest fp16 subnormal region
    x[2, :] = np.float16(-1e-4)
    q, s = oracle.quantize_rowwise_int8(x)
    assert np.all(q[0] == 0) and s[0] == np.float32(1e-10) / np.float32(127)
    assert q[1, 5] == 127 and np.count_nonzero(q[1]) == 1
    assert np.all(q[2] == -127)


# ----------------------------------------------------------------------------
# a2: block-wise asymmetric 4-bit quantization and packing
# ----------------------------------------------------------------------------

def _unpack(qweight: np.ndarray) -> np.ndarray:
    """Unpack 8 nibbles per uint32 along K, nibble j at bits 4j (numpy bit ops)."""
    shifts = (4 * np.arange(8, dtype=np.uint32))
    return ((qweight[:, :, None] >> shifts) & 0xF).reshape(qweight.shape[0], -1).astype(np.uint8)


def test_block_asym4_golden():
    for name, expr, scale, zero, codes, words, _ in _read_rows("block_asym4.txt"):
        k = np.arange(64)
        w = np.asarray(eval(expr, {"k": k}), dtype=np.float64) * np.ones(64)
        w16 = w.astype(np.float16).reshape(1, 64)
        assert np.array_equal(w16.astype(np.float64).ravel(), w), name
        qw, sc, ze, q = oracle.quantize_block_asym4(w16, group=64)
        assert float(sc[0, 0]) == float(scale), name
        assert float(ze[0, 0]) == float(zero) and not np.signbit(ze[0, 0]), name
        expect = np.tile(np.array([int(c) for c in codes.split()]), 4)
        assert np.array_equal(q[0], expect), name
        assert [int(wd, 16) for wd in words.split()] == [int(qw[0, 0]), int(qw[0, 1])], name


@pytest.mark.parametrize("seed,factor", [(4, False), (9, True)])
def test_block_asym4_invariants(seed, factor):
    w = W.weights(48, 512, seed=seed, per_column_factor=factor)
    qw, sc, ze, q = oracle.quantize_block_asym4(w, group=64)
    assert np.array_equal(_unpack(qw), q)                      # pack/unpack round trip
    assert q.max() <= 15
    s = sc.astype(np.float64).T.repeat(64, axis=1)             # [N, K]
    z = ze.astype(np.float64).T.repeat(64, axis=1)
    assert np.all(ze.astype(np.float64) == np.round(ze.astype(np.float64)))
    wf = w.astype(np.float64)
    deq = (q.astype(np.float64) - z) * s
    # where no clamp was active the dequant error is at most half a step (+ binary32 rounding)
    free = (q > 0) & (q < 15)
    assert np.all(np.abs(wf - deq)[free] <= s[free] * (0.5 + 2.0 ** -18))
    # block minimum maps to code 0 or 1 (zero rounding), block maximum to 14 or 15
    blocks = wf.reshape(48, -1, 64)
    qb = q.reshape(48, -1, 64)
    qmin = np.take_along_axis(qb, blocks.argmin(axis=2)[..., None], axis=2)
    qmax = np.take_along_axis(qb, blocks.argmax(axis=2)[..., None], axis=2)
    assert qmin.max() <= 1 and qmax.min() >= 14
    # the scale is the fp16 rounding of (max-min)/15 in binary32
    rng = (blocks.max(axis=2) - blocks.min(axis=2)).astype(np.float32) / np.float32(15)
    assert np.array_equal(sc.T, np.maximum(rng, np.float32(1e-5)).astype(np.float16))


def test_block_asym4_quantizes_with_the_stored_fp16_scale():
    """A block whose binary32 scale and fp16 scale give different codes: the fp16 one wins."""
    rng = np.random.default_rng(7)
    hits = 0
    for _ in range(200):
        w = (rng.standard_normal((1, 64)) * 0.02).astype(np.float16)
        qw, sc, ze, q = oracle.quantize_block_asym4(w, group=64)
        wf = w.astype(np.float32).ravel()
        s32 = np.float32(wf.max() - wf.min()) / np.float32(15)
        s16 = np.float32(sc[0, 0])
        z = float(ze[0, 0])
        with_16 = np.clip(np.rint(wf / s16) + z, 0, 15)
        with_32 = np.clip(np.rint(wf / s32) + z, 0, 15)
        assert np.array_equal(q[0], with_16.astype(np.uint8))
        hits += int(not np.array_equal(with_16, with_32))
    assert hits > 0


# ----------------------------------------------------------------------------
# a3/a4: integer GEMM and the W8A8 epilogue
# ----------------------------------------------------------------------------

def _read_kv(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, rest = line.split(None, 1)
        rows = [[float(v) for v in r.split()] for r in rest.split(";")]
        out[key] = np.array(rows if len(rows) > 1 else rows[0])
    return out


def test_w8a8_golden():
    g = _read_kv("gemm_w8a8.txt")
    xq, wq = g["xq"].astype(np.int8), g["wq"].astype(np.int8)
    acc = oracle.gemm_i8_i64(xq, wq)
    assert np.array_equal(acc, g["acc"].astype(np.int64))
    y = oracle.w8a8_f64(xq, wq, g["x_scale"], g["w_scale"], g["bias"])
    assert np.array_equal(y, g["y"])
    assert np.array_equal(oracle.w8a8_epilogue_f64(acc, g["x_scale"], g["w_scale"], g["bias"]), g["y"])


# ----------------------------------------------------------------------------
# NEXT-2: asymmetric per-row int8 and the zero-point W8A8 product
# ----------------------------------------------------------------------------

def test_quantize_rowwise_asym_golden():
    rows = _read_rows("quantize_rowwise_asym.txt")
    x = np.array([[float(v) for v in r[0].split()] for r in rows], dtype=np.float16)
    expect = np.array([[int(v) for v in r[1].split()] for r in rows], dtype=np.int8)
    sz = np.array([[float(v) for v in r[2].split()] for r in rows])
    q, s, z, qs = oracle.quantize_rowwise_asym_int8(x)
    assert np.array_equal(q, expect)
    assert np.array_equal(s.astype(np.float64), sz[:, 0]) and np.array_equal(z.astype(np.float64), sz[:, 1])
    assert np.array_equal(qs, expect.astype(np.int64).sum(axis=1))


def test_quantize_rowwise_asym_invariants():
    """Invariants the pages' formulas fix: the row minimum maps to -128 and the
    maximum to 127 (min/s + z = -128 and max/s + z = 127 up to binary32
    rounding, far from a tie); every code dequantizes to within s/2 of its value
    (plus the binary32 rounding of x/s + z); qsum is the code row sum."""
    x = W.activations(64, 1000, seed=5, outliers=True)
    x[3] = np.abs(x[3])                  # all non-negative (post-ReLU-like) row
    q, s, z, qs = oracle.quantize_rowwise_asym_int8(x)
    xf = x.astype(np.float64)
    r = np.arange(x.shape[0])
    assert np.all(q[r, xf.argmin(axis=1)] == -128) and np.all(q[r, xf.argmax(axis=1)] == 127)
    deq = s.astype(np.float64)[:, None] * (q.astype(np.float64) - z.astype(np.float64)[:, None])
    slack = 2.0 ** -22 * (np.abs(xf) + 256 * s.astype(np.float64)[:, None])
    assert np.all(np.abs(deq - xf) <= s.astype(np.float64)[:, None] / 2 + slack)
    assert np.array_equal(qs, q.astype(np.int64).sum(axis=1))
    # the scale and zero are the page's binary32 expressions (numpy binary32 ops)
    mn, mx = x.astype(np.float32).min(axis=1), x.astype(np.float32).max(axis=1)
    s_ref = np.maximum((mx - mn) / np.float32(255.0), np.float32(1e-8))
    assert np.array_equal(s, s_ref)
    assert np.array_equal(z, -mn / s_ref - np.float32(128.0))


def test_quantize_rowwise_asym_constant_rows():
    """max == min: the scale is clamped to 1e-8 and the row lands on -128
    (x/s + z = x/s - x/s - 128)."""
    x = np.zeros((3, 40), np.float16)
    x[1] = 0.5
    x[2] = -3.0
    q, s, z, _ = oracle.quantize_rowwise_asym_int8(x)
    assert np.all(s == np.float32(1e-8)) and np.all(q == -128)


def test_w8a8_zp_matches_the_pages_integer_expansion():
    """Page "量化与多精度算子" §二: with x ~= s_x(q_x - z_x) and w ~= s_w(q_w - z_w)
    the product is the integer dot product plus correction terms,
      s_x s_w (sum q_x q_w - z_w sum q_x - z_x sum q_w + K z_x z_w),
    computed here from the exact int64 accumulator; the oracle sums the
    dequantized products directly.  Also: zero points of 0 give the symmetric
    W8A8 product exactly."""
    M, N, K = 6, 9, 300
    x = W.activations(M, K, seed=21, outliers=True)
    w = W.weights(N, K, seed=21, per_column_factor=True)
    xq, xs, xz, xsum = oracle.quantize_rowwise_asym_int8(x)
    wq, ws, wz, wsum = oracle.quantize_rowwise_asym_int8(w)
    b = W.bias(N, 21)
    y = oracle.w8a8_zp_f64(xq, xs, xz, wq, ws, wz, b)
    acc = xq.astype(np.int64) @ wq.astype(np.int64).T
    xz64, wz64 = xz.astype(np.float64)[:, None], wz.astype(np.float64)[None, :]
    corr = (acc - wz64 * xsum[:, None] - xz64 * wsum[None, :] + K * xz64 * wz64)
    y_exp = xs.astype(np.float64)[:, None] * ws.astype(np.float64)[None, :] * corr + b.astype(np.float64)[None, :]
    mag = (np.abs(xs.astype(np.float64))[:, None] * np.abs(ws.astype(np.float64))[None, :]
           * (np.abs(acc) + np.abs(wz64 * xsum[:, None]) + np.abs(xz64 * wsum[None, :]) + K * np.abs(xz64 * wz64)))
    assert np.all(np.abs(y - y_exp) <= 1e-12 * (mag + np.abs(b)[None, :]))
    # one asymmetric operand only (the other symmetric): same expansion with its z = 0
    wq_s, ws_s = oracle.quantize_rowwise_int8(w)
    y1 = oracle.w8a8_zp_f64(xq, xs, xz, wq_s, ws_s, None, None)
    acc1 = xq.astype(np.int64) @ wq_s.astype(np.int64).T
    wsum1 = wq_s.astype(np.int64).sum(axis=1)
    y1_exp = xs.astype(np.float64)[:, None] * ws_s.astype(np.float64)[None, :] * (acc1 - xz64 * wsum1[None, :])
    assert np.allclose(y1, y1_exp, rtol=1e-12, atol=0)
    # both symmetric: the a3+a4 oracle
    xq_s, xs_s = oracle.quantize_rowwise_int8(x)
    y0 = oracle.w8a8_zp_f64(xq_s, xs_s, None, wq_s, ws_s, None, b)
    assert np.allclose(y0, oracle.w8a8_f64(xq_s, wq_s, xs_s, ws_s, b), rtol=1e-13, atol=0)


# ----------------------------------------------------------------------------
# NEXT-3: symmetric int4, W4A8 through the int8 product, symmetric W4A16
# ----------------------------------------------------------------------------

def test_quantize_sym4_golden():
    r = _read_rows("quantize_sym4.txt")[0]
    w = np.zeros((1, 64), np.float16)
    w[0, :8] = [float(v) for v in r[0].split()]
    expect = np.array([int(v) for v in r[1].split()], np.int8)
    qw, sc, q = oracle.quantize_block_sym4(w, 64)
    assert np.array_equal(q[0, :8], expect) and not q[0, 8:].any()
    assert float(sc[0, 0]) == float(r[2]) and int(qw[0, 0]) == int(r[3], 16)
    qw_c, sc_c, q_c = oracle.quantize_channel_sym4(w)      # per-column: the same single block
    assert np.array_equal(q_c, q) and np.array_equal(qw_c, qw) and sc_c[0] == np.float32(1.0)


def test_quantize_sym4_floors_golden():
    """The two scale floors (block: 1e-5 on max|w|/7, then fp16; per-column:
    1e-10 on max|w|) and constant blocks at the code limit +-7, from the
    hand-worked rows of sym4_floor.txt."""
    for form, name, expr, sbits, codes, word, _ in _read_rows("sym4_floor.txt"):
        k = np.arange(64)
        w16 = (np.asarray(eval(expr, {"k": k}), dtype=np.float64) * np.ones(64)).astype(np.float16).reshape(1, 64)
        expect = np.array([int(c) for c in codes.split()], np.int8)
        if form == "block":
            qw, sc, q = oracle.quantize_block_sym4(w16, 64)
            assert int(sc.view(np.uint16)[0, 0]) == int(sbits, 16), name
        else:
            qw, sc, q = oracle.quantize_channel_sym4(w16)
            assert int(sc.view(np.uint32)[0]) == int(sbits, 16), name
        assert np.array_equal(q[0, :8], expect), name
        assert int(qw[0, 0]) == int(word, 16), name
        # the codes past k = 7 repeat the pattern of the expression (zero or the constant)
        assert np.all(q[0, 8:] == (expect[2] if name != "tiny" else 0)), name


def _unpack_signed(qw):
    nib = (qw[:, :, None] >> (4 * np.arange(8, dtype=np.uint32))[None, None, :]) & 0xF
    v = nib.astype(np.int16).reshape(qw.shape[0], -1)
    return np.where(v >= 8, v - 16, v).astype(np.int8)


@pytest.mark.parametrize("group", [64, 4096])
def test_quantize_sym4_invariants(group):
    """Unpacking the words (page "INT4/FP16混合精度GEMM" §4.2: (w >> 4i) & 0xF,
    sign-extended) gives back the codes; every weight is within s/2 of q s (no
    code reaches the clamp for these scales); each block's largest |w| maps to +-7."""
    w = W.weights(48, 4096, seed=8, per_column_factor=True)
    if group == 4096:
        qw, s, q = oracle.quantize_channel_sym4(w)
        s64 = np.repeat(s.astype(np.float64)[:, None], 4096, axis=1)
    else:
        qw, sc, q = oracle.quantize_block_sym4(w, group)
        s64 = np.repeat(sc.astype(np.float64).T, group, axis=1)
    assert np.array_equal(_unpack_signed(qw), q)
    wf = w.astype(np.float64)
    assert np.all(np.abs(q * s64 - wf) <= s64 / 2 * (1 + 2.0 ** -20))
    blocks = np.abs(wf).reshape(48, -1, group).argmax(axis=2)
    qb = q.reshape(48, -1, group)
    picked = np.take_along_axis(qb, blocks[:, :, None], axis=2)[:, :, 0]
    assert np.all(np.abs(picked) == 7)


def test_w4a8_equals_the_int8_product_of_the_unpacked_codes():
    """Page "Ascend C per-channel INT8 GEMM" §9.1: int4 unpacked to int8, then the
    int8 matmul -- so W4A8 is W8A8 on the unpacked codes (numpy int64 matmul
    and the W8A8 oracle give the same numbers)."""
    M, N, K = 7, 40, 512
    x = W.activations(M, K, seed=4, outliers=True)
    w = W.weights(N, K, seed=4, per_column_factor=True)
    xq, xs = oracle.quantize_rowwise_int8(x)
    qw, ws, q = oracle.quantize_channel_sym4(w)
    b = W.bias(N, 4)
    y = oracle.w4a8_f64(xq, qw, xs, ws, b)
    assert np.array_equal(y, oracle.w8a8_f64(xq, q, xs, ws, b))
    acc = xq.astype(np.int64) @ _unpack_signed(qw).astype(np.int64).T
    assert np.array_equal(y, oracle.w8a8_epilogue_f64(acc, xs, ws, b))


def test_w4a16_sym_equals_asymmetric_form_with_zero_eight():
    """A two's-complement code q is the offset code u = q + 8 = nibble ^ 8 with
    zero point 8: (u - 8) s = q s, so the symmetric product must equal the
    asymmetric W4A16 oracle fed those codes, bit for bit (same fp64 terms, same
    order).  One-hot rows give q s exactly."""
    M, N, K = 5, 24, 256
    x = W.activations(M, K, seed=6)
    w = W.weights(N, K, seed=6, per_column_factor=False)
    qw, sc, q = oracle.quantize_block_sym4(w, 64)
    y = oracle.w4a16_sym_f64(x, qw, sc, 64, None)
    z8 = np.full(sc.shape, 8, np.float16)
    assert np.array_equal(y, oracle.w4a16_f64(x, qw ^ np.uint32(0x88888888), sc, z8, 64, None))
    e = np.zeros((1, K), np.float16)
    e[0, 77] = 1.0
    col = oracle.w4a16_sym_f64(e, qw, sc, 64, None)[0]
    assert np.array_equal(col, q[:, 77].astype(np.float64) * sc[77 // 64].astype(np.float64))


# ----------------------------------------------------------------------------
# NEXT-4: GELU after the GEMM
# ----------------------------------------------------------------------------

def test_gelu_closed_forms():
    """gelu(y) = y Phi(y): Phi(0) = 1/2, Phi(1) and Phi(2) are textbook values of
    the standard normal CDF, gelu(y) - gelu(-y) = y for every y (Phi(-y) =
    1 - Phi(y)), and gelu(y) -> y, gelu(-y) -> 0 for large y."""
    phi1, phi2 = 0.8413447460685429, 0.9772498680518208
    g = oracle.gelu_f64(np.array([0.0, 1.0, 2.0, -1.0, 40.0, -40.0]))
    assert g[0] == 0.0
    assert abs(g[1] - phi1) <= 1e-15 and abs(g[2] - 2 * phi2) <= 2e-15
    assert abs(g[3] - (phi1 - 1.0)) <= 1e-15
    assert g[4] == 40.0 and abs(g[5]) < 1e-300
    y = np.random.default_rng(3).normal(size=1000) * 4
    assert np.allclose(oracle.gelu_f64(y) - oracle.gelu_f64(-y), y, rtol=0, atol=1e-14)


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 5, 7), (17, 9, 64), (5, 33, 300)])
def test_gemm_i8_matches_numpy_int64(M, N, K):
    rng = np.random.default_rng(M * 1000 + N * 10 + K)
    xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    wq = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
    ref = xq.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(oracle.gemm_i8_i64(xq, wq), ref)


def test_gemm_i8_identity_permutation_and_extremes():
    rng = np.random.default_rng(12)
    xq = rng.integers(-127, 128, size=(6, 32)).astype(np.int8)
    eye = np.eye(32, dtype=np.int8)
    assert np.array_equal(oracle.gemm_i8_i64(xq, eye), xq.astype(np.int64))
    perm = rng.permutation(32)
    assert np.array_equal(oracle.gemm_i8_i64(xq, eye[perm]), xq[:, perm].astype(np.int64))
    K = 4096
    lo = np.full((2, K), -127, np.int8)
    acc = oracle.gemm_i8_i64(lo, lo)
    assert np.all(acc == 127 * 127 * K) and acc.max() < 2 ** 31


def test_w8a8_equals_product_of_dequantized_operands():
    """(x_scale*Xq) @ (w_scale*Wq)^T + bias, computed by numpy fp64 matmul."""
    x = W.activations(12, 256, seed=0, outliers=True)
    w = W.weights(40, 256, seed=0)
    xq, xs = oracle.quantize_rowwise_int8(x)
    wq, ws = oracle.quantize_rowwise_int8(w)
    b = W.bias(40, seed=0)
    y = oracle.w8a8_f64(xq, wq, xs, ws, b)
    ref = (xs[:, None].astype(np.float64) * xq) @ (ws[:, None].astype(np.float64) * wq).T + b
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    # bias alone when X is zero; one-hot row picks a scaled column of Wq
    zero = np.zeros_like(xq)
    assert np.array_equal(oracle.w8a8_f64(zero, wq, xs, ws, b), np.tile(b.astype(np.float64), (12, 1)))
    onehot = np.zeros_like(xq)
    onehot[:, 17] = 1
    y1 = oracle.w8a8_f64(onehot, wq, xs, ws, None)
    assert np.array_equal(y1, xs[:, None].astype(np.float64) * ws[None, :] * wq[:, 17][None, :])


# ----------------------------------------------------------------------------
# a5/a6: weight-only products
# ----------------------------------------------------------------------------

def test_w8a16_matches_fp64_matmul_and_closed_forms():
    x = W.activations(5, 192, seed=3)
    w = W.weights(24, 192, seed=3)
    wq, ws = oracle.quantize_rowwise_int8(w)
    b = W.bias(24, seed=3)
    y = oracle.w8a16_f64(x, wq, ws, b)
    wdq = ws[:, None].astype(np.float64) * wq.astype(np.float64)     # [N,K]
    ref = x.astype(np.float64) @ wdq.T + b
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-13)
    onehot = np.zeros_like(x)
    onehot[:, 100] = 1.0
    assert np.array_equal(oracle.w8a16_f64(onehot, wq, ws, None), np.tile(wdq[:, 100], (5, 1)))


def test_w4a16_matches_fp64_matmul_and_closed_forms():
    x = W.activations(4, 256, seed=4)
    w = W.weights(20, 256, seed=4, per_column_factor=False)
    qw, sc, ze, q = oracle.quantize_block_asym4(w, group=64)
    # dequantize independently: numpy unpack, (q - z) * s with [K/64, N] scale/zero
    codes = _unpack(qw).astype(np.float64)                          # [N, K]
    s = sc.astype(np.float64).T.repeat(64, axis=1)
    z = ze.astype(np.float64).T.repeat(64, axis=1)
    wdq = (codes - z) * s
    y = oracle.w4a16_f64(x, qw, sc, ze, 64, None)
    assert np.allclose(y, x.astype(np.float64) @ wdq.T, rtol=1e-13, atol=1e-13)
    onehot = np.zeros_like(x)
    onehot[:, 130] = 1.0
    assert np.array_equal(oracle.w4a16_f64(onehot, qw, sc, ze, 64, None), np.tile(wdq[:, 130], (4, 1)))
    assert oracle.w4_dequant(qw, sc, ze, 64, 130, 7) == wdq[7, 130]
    b = W.bias(20, seed=4)
    zx = np.zeros_like(x)
    assert np.array_equal(oracle.w4a16_f64(zx, qw, sc, ze, 64, b), np.tile(b.astype(np.float64), (4, 1)))
    # the golden ramp block dequantizes exactly back to its weights
    kk = np.arange(64)
    ramp = (0.125 * ((kk % 16) - 3)).astype(np.float16).reshape(1, 64)
    qw1, sc1, ze1, _ = oracle.quantize_block_asym4(ramp, 64)
    eye = np.eye(64, dtype=np.float16)
    assert np.array_equal(oracle.w4a16_f64(eye, qw1, sc1, ze1, 64, None)[:, 0], ramp[0].astype(np.float64))


def test_quantization_error_per_channel_below_per_tensor():
    """Direction of the per-tensor vs per-channel comparison (values unpinned: no real weights)."""
    w = W.weights(256, 512, seed=6)
    q_ch, s_ch = oracle.quantize_rowwise_int8(w)
    q_t, s_t = oracle.quantize_rowwise_int8(w.reshape(1, -1))
    wf = w.astype(np.float64)
    err_ch = np.mean((wf - q_ch * s_ch[:, None].astype(np.float64)) ** 2)
    err_t = np.mean((wf - q_t.reshape(w.shape) * float(s_t[0])) ** 2)
    assert err_ch < err_t / 4
