"""GPU parity for the asymmetric per-row int8 quantizer and the zero-point W8A8
GEMM, called through the C ABI and compared with the oracle.

Bars: codes, scales, zero points and code sums bit-exact; fp32 outputs within
1e-6 of the magnitude |s_x s_w| (|acc| + |z_w sum q_x| + |z_x sum q_w| +
K |z_x z_w|) + |bias| (the kernel forms the bracket in fp64 and rounds it to
fp32 once, then scales like the symmetric W8A8); fp16/bf16 outputs within the
W8A8 half-precision bound with that magnitude.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import assert_w8a8_half, bits16, dev, host, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]


def qg():
    import int4_quantized_gemm_b200 as q
    return q


def _ld(K, elem):
    per16 = 16 // elem
    return (K + per16 - 1) // per16 * per16


@pytest.mark.parametrize("M,K,relu", [(16, 4096, False), (1, 4096, True), (300, 1000, True), (5, 7, False),
                                      (64, 8192, False), (2048, 4096, True)])
def test_quantize_rowwise_asym_bit_exact(M, K, relu):
    x = W.activations(M, K, seed=M + K, outliers=True)
    if relu:
        x = np.maximum(x, np.float16(0))          # all non-negative rows: z near -128
    q_ref, s_ref, z_ref, qs_ref = oracle.quantize_rowwise_asym_int8(x)
    q, s, z, qs = qg().quantize_rowwise_asym_int8(dev(x, ld=_ld(K, 2)))
    torch.cuda.synchronize()
    assert np.array_equal(host(q), q_ref)
    assert np.array_equal(host(s).view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(host(z).view(np.uint32), z_ref.view(np.uint32))
    assert np.array_equal(host(qs), qs_ref)


def test_quantize_rowwise_asym_constant_and_golden_rows():
    x = np.zeros((4, 64), np.float16)
    x[1] = 0.5
    x[2, :6] = [-16, -1, 0, 0.0625, 0.1875, 15.875]   # the worked example: s = 0.125, z = 0
    x[2, 6:] = 0
    x[3, :6] = [-8, 0, 0.0625, 0.1875, 23.875, -8]    # s = 0.125, z = -64
    x[3, 6:] = 0
    q_ref, s_ref, z_ref, qs_ref = oracle.quantize_rowwise_asym_int8(x)
    q, s, z, qs = qg().quantize_rowwise_asym_int8(dev(x))
    torch.cuda.synchronize()
    assert np.array_equal(host(q), q_ref) and np.array_equal(host(qs), qs_ref)
    assert np.array_equal(host(s), s_ref) and np.array_equal(host(z), z_ref)
    assert list(host(q)[2, :6]) == [-128, -8, 0, 0, 2, 127]
    assert list(host(q)[3, :6]) == [-128, -64, -64, -62, 127, -128]


def _zp_case(M, N, K, seed, x_asym=True, w_asym=True, relu=True):
    x = W.activations(M, K, seed=seed, outliers=True)
    if relu:
        x = np.maximum(x, np.float16(0))
    w = W.weights(N, K, seed=seed, per_column_factor=True)
    if x_asym:
        xq, xs, xz, xsum = oracle.quantize_rowwise_asym_int8(x)
    else:
        xq, xs = oracle.quantize_rowwise_int8(x)
        xz, xsum = None, xq.astype(np.int64).sum(axis=1).astype(np.int32)
    if w_asym:
        wq, ws, wz, wsum = oracle.quantize_rowwise_asym_int8(w)
    else:
        wq, ws = oracle.quantize_rowwise_int8(w)
        wz, wsum = None, wq.astype(np.int64).sum(axis=1).astype(np.int32)
    b = W.bias(N, seed)
    return xq, xs, xz, xsum, wq, ws, wz, wsum, b


def _magnitude(xq, xs, xz, xsum, wq, ws, wz, wsum, b):
    K = xq.shape[1]
    acc = oracle.gemm_i8_i64(xq, wq).astype(np.float64)
    xz64 = (np.zeros(len(xs)) if xz is None else xz.astype(np.float64))[:, None]
    wz64 = (np.zeros(len(ws)) if wz is None else wz.astype(np.float64))[None, :]
    inner = (np.abs(acc) + np.abs(wz64 * xsum.astype(np.float64)[:, None])
             + np.abs(xz64 * wsum.astype(np.float64)[None, :]) + K * np.abs(xz64 * wz64))
    return np.abs(xs.astype(np.float64))[:, None] * np.abs(ws.astype(np.float64))[None, :] * inner \
        + np.abs(b.astype(np.float64))[None, :]


def _run(case, dtype, zp_x=True, zp_w=True):
    xq, xs, xz, xsum, wq, ws, wz, wsum, b = case
    K = xq.shape[1]
    d = lambda a: None if a is None else dev(a)
    return qg().gemm_w8a8_zp(dev(xq, ld=_ld(K, 1)), dev(xs), d(xz), dev(xsum), dev(wq, ld=_ld(K, 1)), dev(ws),
                             d(wz), dev(wsum), dev(b), out_dtype=dtype)


# decode (swap-AB, single CTA and K-split clusters) and prefill tiles, ragged M/N/K
ZP_SHAPES = [(1, 4096, 4096), (16, 4096, 4096), (16, 11008, 4096), (5, 520, 1000), (33, 300, 264),
             (64, 264, 520), (129, 520, 1000), (300, 777, 1104), (1024, 1024, 4096)]


@pytest.mark.parametrize("M,N,K", ZP_SHAPES)
def test_w8a8_zp_f32_against_the_oracle(M, N, K):
    case = _zp_case(M, N, K, seed=M + 3 * N)
    xq, xs, xz, xsum, wq, ws, wz, wsum, b = case
    y64 = oracle.w8a8_zp_f64(xq, xs, xz, wq, ws, wz, b)
    y = _run(case, torch.float32)
    torch.cuda.synchronize()
    mag = _magnitude(*case)
    err = np.abs(host(y).astype(np.float64) - y64)
    assert np.all(err <= 1e-6 * mag + 1e-30), f"worst {np.max(err / (mag + 1e-30)):.3e}"


@pytest.mark.parametrize("M,N,K,kind,x_asym,w_asym", [
    (16, 4096, 4096, "f16", True, True), (16, 4096, 4096, "f16", True, False),
    (16, 4096, 4096, "bf16", False, True), (256, 1000, 4096, "bf16", True, True),
    (3, 520, 1000, "f16", False, False)])
def test_w8a8_zp_half_outputs(M, N, K, kind, x_asym, w_asym):
    case = _zp_case(M, N, K, seed=7, x_asym=x_asym, w_asym=w_asym)
    xq, xs, xz, xsum, wq, ws, wz, wsum, b = case
    y64 = oracle.w8a8_zp_f64(xq, xs, xz, wq, ws, wz, b)
    dt = torch.float16 if kind == "f16" else torch.bfloat16
    y = _run(case, dt)
    torch.cuda.synchronize()
    assert_w8a8_half(bits16(y), y64, _magnitude(*case), kind, f"zp {kind} {M}x{N}x{K}")


def test_w8a8_zp_raw_accumulator_and_pipeline_from_gpu_quantizers():
    q = qg()
    M, N, K = 16, 1024, 4096
    x = np.maximum(W.activations(M, K, seed=31, outliers=True), np.float16(0))
    w = W.weights(N, K, seed=31, per_column_factor=True)
    xq, xs, xz, xsum = q.quantize_rowwise_asym_int8(dev(x))
    wq, ws, wz, wsum = q.quantize_rowwise_asym_int8(dev(w))
    acc = q.gemm_w8a8_zp(xq, None, None, None, wq, None, None, None, out_dtype=torch.int32)
    y = q.gemm_w8a8_zp(xq, xs, xz, xsum, wq, ws, wz, wsum, out_dtype=torch.float32)
    torch.cuda.synchronize()
    xq_r, xs_r, xz_r, xsum_r = oracle.quantize_rowwise_asym_int8(x)
    wq_r, ws_r, wz_r, wsum_r = oracle.quantize_rowwise_asym_int8(w)
    assert np.array_equal(host(acc).astype(np.int64), oracle.gemm_i8_i64(xq_r, wq_r))
    y64 = oracle.w8a8_zp_f64(xq_r, xs_r, xz_r, wq_r, ws_r, wz_r, None)
    mag = _magnitude(xq_r, xs_r, xz_r, xsum_r, wq_r, ws_r, wz_r, wsum_r, np.zeros(N, np.float32))
    err = np.abs(host(y).astype(np.float64) - y64)
    assert np.all(err <= 1e-6 * mag + 1e-30), f"worst {np.max(err / (mag + 1e-30)):.3e}"


def test_w8a8_zp_argument_checks_and_empty_sums():
    q = qg()
    xq = torch.zeros((4, 64), dtype=torch.int8, device="cuda")
    wq = torch.zeros((8, 64), dtype=torch.int8, device="cuda")
    f4, f8 = torch.ones(4, device="cuda"), torch.ones(8, device="cuda")
    with pytest.raises(q.QGError):      # w_zero without the Xq row sums
        q.gemm_w8a8_zp(xq, f4, None, None, wq, f8, f8, torch.zeros(8, dtype=torch.int32, device="cuda"))
    b = torch.arange(8, dtype=torch.float32, device="cuda")
    y = q.gemm_w8a8_zp(torch.zeros((4, 0), dtype=torch.int8, device="cuda"), f4, f4,
                       torch.zeros(4, dtype=torch.int32, device="cuda"),
                       torch.zeros((8, 0), dtype=torch.int8, device="cuda"), f8, f8,
                       torch.zeros(8, dtype=torch.int32, device="cuda"), b, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y, b.expand(4, 8))   # K == 0: the empty sum, K z_x z_w = 0
    q.check_device_errors()
