"""Helpers for the GPU parity tests: move seeded inputs to the device, compare
kernel outputs with the oracle at the tolerances the hot path states."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle

requires_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def dev(a: np.ndarray, dtype=None, ld: int | None = None) -> torch.Tensor:
    """numpy -> CUDA tensor; with ld, a [rows, ld] buffer whose first cols hold `a`."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    if ld is not None and ld != t.shape[1]:
        buf = torch.zeros((t.shape[0], ld), dtype=t.dtype)
        buf[:, : t.shape[1]] = t
        return buf.cuda()[:, : t.shape[1]]
    return t.cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy()


def bits16(t: torch.Tensor) -> np.ndarray:
    """fp16/bf16 CUDA tensor -> uint16 bit patterns."""
    return host(t.contiguous().view(torch.int16)).view(np.uint16)


def ordered16(bits: np.ndarray) -> np.ndarray:
    """Sign-magnitude 16-bit float patterns -> integers ordered like the values
    (adjacent representable values differ by 1)."""
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def assert_within_one_ulp16(got_bits: np.ndarray, ref_bits: np.ndarray, what: str) -> None:
    d = np.abs(ordered16(got_bits) - ordered16(ref_bits))
    bad = np.argwhere(d > 1)
    assert bad.size == 0, f"{what}: {bad.shape[0]} outputs differ by more than 1 ulp, first at {bad[0]}"


def decode16(bits: np.ndarray, kind: str) -> np.ndarray:
    return oracle.f16_decode(bits) if kind == "f16" else oracle.bf16_decode(bits)


def assert_w8a8_half(got_bits: np.ndarray, y64: np.ndarray, mag: np.ndarray, kind: str, what: str) -> None:
    """fp16/bf16 W8A8 output.  The kernel rounds an fp32 value y32 with
    |y32 - y64| <= 1e-6 * mag (mag = |acc*xs*ws| + |bias|, the fp32 epilogue
    bar) to the output type, so |out - y64| <= ulp(out)/2 + 1e-6 * mag.  That
    is within 1 ulp of round(y64) except where acc*xs*ws and bias nearly
    cancel; both forms are accepted, nothing looser."""
    ref_bits = round16(y64, kind)
    one_ulp = np.abs(ordered16(got_bits) - ordered16(ref_bits)) <= 1
    got = decode16(got_bits, kind)
    nxt = decode16((got_bits.astype(np.int64) + 1).astype(np.uint16), kind)
    ulp = np.abs(nxt - got)
    bound = np.abs(got - y64) <= 0.5 * ulp + 1e-6 * mag
    bad = np.argwhere(~(one_ulp | bound))
    assert bad.size == 0, f"{what}: {bad.shape[0]} outputs outside the bound, first at {bad[0]}"


def w8a8_magnitude(acc: np.ndarray, xs, ws, bias) -> np.ndarray:
    mag = np.abs(acc.astype(np.float64) * xs[:, None].astype(np.float64) * ws[None, :].astype(np.float64))
    if bias is not None:
        mag = mag + np.abs(bias.astype(np.float64))[None, :]
    return mag


def assert_w8a8_f32(y: np.ndarray, acc: np.ndarray, xs, ws, bias, y64: np.ndarray) -> None:
    """fp32 epilogue: |y - y64| <= 1e-6 * (|acc * xs * ws| + |bias|)."""
    mag = np.abs(acc.astype(np.float64) * xs[:, None].astype(np.float64) * ws[None, :].astype(np.float64))
    if bias is not None:
        mag = mag + np.abs(bias.astype(np.float64))[None, :]
    err = np.abs(y.astype(np.float64) - y64)
    bad = err > 1e-6 * mag + 1e-30
    assert not bad.any(), f"{bad.sum()} fp32 outputs outside 1e-6 relative; worst {np.max(err / (mag + 1e-30))}"


def rel_frobenius(y: np.ndarray, y64: np.ndarray) -> float:
    return float(np.linalg.norm(y.astype(np.float64) - y64) / max(np.linalg.norm(y64), 1e-300))


def round16(y64: np.ndarray, kind: str) -> np.ndarray:
    return oracle.round_f16(y64) if kind == "f16" else oracle.round_bf16(y64)


# ----------------------------------------------------------------------------
# Weight-only GEMMs: an element-wise bound from the arithmetic
# ----------------------------------------------------------------------------
# The kernels form each weight's fp16 A operand (int8 codes exactly; int4
# (q - z) * s rounded once to fp16: relative error <= 2^-11, or at most 2^-25
# absolute where the product is an fp16 subnormal), multiply it by the fp16 X
# element exactly (an fp16 x fp16 product fits in binary32), sum the K products
# in fp32 on the tensor cores and across the K-split CTAs (at most K + 8
# additions; each, whatever the tensor core's internal order and rounding, is
# taken to lose at most 2^-23 of the running magnitude sum_k |x_k w_k| -- a
# truncating binary32 addition), then scale (W8A16), add the bias (one binary32
# rounding each, 2^-23 of |y| + |bias| for both) and round to fp16 (half an ulp).
# The oracle is the fp64 product of the exactly dequantized weights.  Hence
#   |y - y64| <= ulp16(y)/2 + (c_deq + (K + 8) 2^-23) sum_k |x_k| |w_kn|
#                + a_deq sum_k |x_k| + 2^-23 (|y64| + |bias_n|)
# with c_deq = 2^-11, a_deq = 2^-25 for the int4 forms and 0, 0 for W8A16.
# With a GELU epilogue the bound above applies to the pre-activation value v,
# gelu' <= 1.13 carries it through, and the binary32 evaluation of
# 0.5 v (1 + erf(v / sqrt 2)) adds at most 2^-20 |v|.

def unpack_u4(qweight: np.ndarray) -> np.ndarray:
    """[N, K/8] uint32 -> [N, K] nibble values 0..15 (nibble j of word p is k = 8p + j)."""
    q = np.asarray(qweight).view(np.uint32)
    shifts = 4 * np.arange(8, dtype=np.uint32)
    return ((q[:, :, None] >> shifts) & 0xF).reshape(q.shape[0], -1).astype(np.int64)


def w8_dequant(wq: np.ndarray, ws: np.ndarray) -> np.ndarray:
    """Exact fp64 dequantized W8A16 weights [N, K] = w_scale[n] * q[n, k]."""
    return wq.astype(np.float64) * ws.astype(np.float64)[:, None]


def w4_dequant(qweight, scale, zero, group=64) -> np.ndarray:
    """Exact fp64 dequantized W4A16 weights [N, K] = (q - z) * s (scale/zero [K/group, N])."""
    q = unpack_u4(qweight).astype(np.float64)
    s = np.repeat(scale.astype(np.float64).T, group, axis=1)
    z = np.repeat(zero.astype(np.float64).T, group, axis=1)
    return (q - z) * s


def w4sym_dequant(qweight, scale, group=64) -> np.ndarray:
    """Exact fp64 dequantized symmetric int4 weights [N, K] = q * s (two's-complement codes)."""
    u = unpack_u4(qweight)
    q = np.where(u >= 8, u - 16, u).astype(np.float64)
    return q * np.repeat(scale.astype(np.float64).T, group, axis=1)


def wonly_bound(x: np.ndarray, wdeq: np.ndarray, y64_pre: np.ndarray, bias, int4: bool) -> np.ndarray:
    """The arithmetic part of the bound above (without the output half-ulp), for the
    pre-activation value: [M, N]."""
    K = x.shape[1]
    xa = np.abs(x.astype(np.float64))
    mag = xa @ np.abs(wdeq).T
    c_deq, a_deq = (2.0 ** -11, 2.0 ** -25) if int4 else (0.0, 0.0)
    b = 0.0 if bias is None else np.abs(bias.astype(np.float64))[None, :]
    return ((c_deq + (K + 8) * 2.0 ** -23) * mag + a_deq * xa.sum(axis=1, keepdims=True)
            + 2.0 ** -23 * (np.abs(y64_pre) + b))


def assert_wonly_elementwise(y: torch.Tensor, x: np.ndarray, wdeq: np.ndarray, y64_pre: np.ndarray, bias,
                             int4: bool, what: str, gelu: bool = False) -> None:
    """fp16 output y [M, N] of a weight-only GEMM against the fp64 oracle value,
    element by element, within the bound derived above."""
    got_bits = bits16(y)
    got = oracle.f16_decode(got_bits)
    nxt = oracle.f16_decode((got_bits.astype(np.int64) + 1).astype(np.uint16))
    half_ulp = 0.5 * np.abs(nxt - got)
    pre = wonly_bound(x, wdeq, y64_pre, bias, int4)
    if gelu:
        ref = oracle.gelu_f64(y64_pre)
        bound = half_ulp + 1.13 * pre + 2.0 ** -20 * np.abs(y64_pre)
    else:
        ref = y64_pre
        bound = half_ulp + pre
    err = np.abs(got - ref)
    bad = np.argwhere(~(err <= bound))
    assert bad.size == 0, (f"{what}: {bad.shape[0]} outputs outside the element-wise bound, first at "
                           f"{tuple(bad[0])}: |err| {err[tuple(bad[0])]:.3e} > {bound[tuple(bad[0])]:.3e}")
    # the margin actually used, for the record
    return float(np.max(err / np.maximum(bound, 1e-300)))
