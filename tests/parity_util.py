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
