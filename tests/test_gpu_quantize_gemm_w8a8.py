"""GPU parity for the fused per-row quantize + W8A8 decode GEMM
(qg_quantize_gemm_w8a8), called through the C ABI.

The fused kernel takes the same binary32 decisions as the two separate calls,
so its codes, scales and outputs must match qg_quantize_rowwise_int8 followed
by qg_gemm_w8a8 bit for bit, and the oracle at the W8A8 bars: codes, scales and
int32 accumulators bit-exact, fp16/bf16 within the W8A8 half-precision bound.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import (assert_w8a8_f32, assert_w8a8_half, bits16, dev, host, requires_cuda,
                         w8a8_magnitude)

pytestmark = [pytest.mark.gpu, requires_cuda]


def qg():
    import int4_quantized_gemm_b200 as q
    return q


def _inputs(M, N, K, seed, outliers=True):
    x = W.activations(M, K, seed=seed, outliers=outliers)
    w = W.weights(N, K, seed=seed, per_column_factor=True)
    wq, ws = oracle.quantize_rowwise_int8(w)
    return x, wq, ws, W.bias(N, seed)


def _ld(K, elem):
    per16 = 16 // elem
    return (K + per16 - 1) // per16 * per16


# decode batches on both sides of the 16/32/64 tile widths, K with ragged 128-byte
# blocks and ragged 16-element chunks, N with a ragged 128-row tile
SHAPES = [(1, 4096, 4096), (16, 4096, 4096), (16, 11008, 4096), (5, 520, 1000), (17, 300, 264),
          (33, 264, 520), (64, 256, 4096), (3, 128, 8), (16, 136, 1104)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("dtype", [torch.float16, torch.int32])
def test_fused_equals_quantize_then_gemm_bit_for_bit(M, N, K, dtype):
    q = qg()
    x, wq, ws, b = _inputs(M, N, K, seed=M * 7 + N)
    dx = dev(x, ld=_ld(K, 2))
    dwq = dev(wq, ld=_ld(K, 1))
    dws, db = dev(ws), dev(b)
    raw = dtype == torch.int32
    xq2 = torch.zeros((M, _ld(K, 1)), dtype=torch.int8, device="cuda")[:, :K]
    xs2 = torch.zeros(M, dtype=torch.float32, device="cuda")
    y2 = q.quantize_gemm_w8a8(dx, dwq, None if raw else dws, None if raw else db, out_dtype=dtype,
                              xq_out=xq2, x_scale_out=xs2)
    xq1, xs1 = q.quantize_rowwise_int8(dx)
    y1 = q.gemm_w8a8(xq1, dwq, None if raw else xs1, None if raw else dws, None if raw else db,
                     out_dtype=dtype)
    torch.cuda.synchronize()
    assert torch.equal(xq2, xq1) and torch.equal(xs2, xs1)
    if dtype == torch.float16:
        assert np.array_equal(bits16(y2), bits16(y1))
    else:
        assert torch.equal(y2, y1)
    q.check_device_errors()


@pytest.mark.parametrize("M,N,K,kind", [(16, 4096, 4096, "f16"), (1, 11008, 4096, "bf16"),
                                        (40, 520, 1000, "f16")])
def test_fused_against_the_oracle(M, N, K, kind):
    q = qg()
    x, wq, ws, b = _inputs(M, N, K, seed=11)
    xq_ref, xs_ref = oracle.quantize_rowwise_int8(x)
    acc = oracle.gemm_i8_i64(xq_ref, wq)
    y64 = oracle.w8a8_epilogue_f64(acc, xs_ref, ws, b)
    dt = torch.float16 if kind == "f16" else torch.bfloat16
    xq = torch.zeros((M, _ld(K, 1)), dtype=torch.int8, device="cuda")[:, :K]
    xs = torch.zeros(M, dtype=torch.float32, device="cuda")
    y = q.quantize_gemm_w8a8(dev(x, ld=_ld(K, 2)), dev(wq, ld=_ld(K, 1)), dev(ws), dev(b), out_dtype=dt,
                             xq_out=xq, x_scale_out=xs)
    yf = q.quantize_gemm_w8a8(dev(x, ld=_ld(K, 2)), dev(wq, ld=_ld(K, 1)), dev(ws), dev(b),
                              out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(xs).view(np.uint32), xs_ref.view(np.uint32))
    assert_w8a8_half(bits16(y), y64, w8a8_magnitude(acc, xs_ref, ws, b), kind, f"fused {M}x{N}x{K}")
    assert_w8a8_f32(host(yf), acc, xs_ref, ws, b, y64)


def test_fused_zero_rows_ties_and_no_optional_outputs():
    q = qg()
    M, N, K = 8, 384, 512
    x, wq, ws, b = _inputs(M, N, K, seed=3)
    x[0] = 0                                      # all-zero row: scale 1e-10/127, codes 0
    x[1, :8] = np.array([127, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -127], np.float16)
    x[1, 8:] = 0                                  # exact .5 ties, half to even
    xq_ref, xs_ref = oracle.quantize_rowwise_int8(x)
    acc = oracle.gemm_i8_i64(xq_ref, wq)
    y = torch.full((M, N), -1, dtype=torch.int32, device="cuda")
    q.quantize_gemm_w8a8(dev(x), dev(wq), None, None, out_dtype=torch.int32, out=y)
    torch.cuda.synchronize()
    assert np.array_equal(host(y).astype(np.int64), acc)
    assert xs_ref[0] == np.float32(1e-10) / np.float32(127)


def test_fused_degenerate_sizes_and_limits():
    q = qg()
    b = torch.arange(24, dtype=torch.float32, device="cuda")
    ws = torch.ones(24, device="cuda")
    # K == 0: Y = bias; the row scales are those of an all-zero row
    xs = torch.full((3,), -1.0, device="cuda")
    xq = torch.zeros((3, 16), dtype=torch.int8, device="cuda")[:, :0]
    y = q.quantize_gemm_w8a8(torch.zeros((3, 0), dtype=torch.float16, device="cuda"),
                             torch.zeros((24, 0), dtype=torch.int8, device="cuda"), ws, b,
                             xq_out=xq, x_scale_out=xs)
    torch.cuda.synchronize()
    assert torch.equal(y.float(), b.expand(3, 24))
    assert np.array_equal(host(xs), np.full(3, np.float32(1e-10) / np.float32(127), np.float32))
    # M == 0 is a no-op; M > 64 is not a decode batch
    y0 = q.quantize_gemm_w8a8(torch.zeros((0, 64), dtype=torch.float16, device="cuda"),
                              torch.zeros((24, 64), dtype=torch.int8, device="cuda"), ws, b)
    assert y0.shape == (0, 24)
    with pytest.raises(q.QGError):
        q.quantize_gemm_w8a8(torch.zeros((65, 64), dtype=torch.float16, device="cuda"),
                             torch.zeros((24, 64), dtype=torch.int8, device="cuda"), ws, b)
    q.check_device_errors()
