"""GPU parity: rowwise int8 quantize, block 4-bit quantize and the W8A8 GEMM,
called through the C ABI (the Python binding) and compared element by element
with the oracle on the same seeded inputs.

Bars: int8 codes, scales, packed words and raw int32 accumulators bit-exact;
fp32 epilogue within 1e-6 relative to |acc*xs*ws| + |bias|; fp16/bf16 outputs
within 1 ulp of the nearest-even rounding of the fp64 oracle value.
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


# ----------------------------------------------------------------------------
# a1: rowwise quantize
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("M,K,ld,outliers", [
    (1, 4096, 4096, True), (16, 4096, 4096, True), (3, 256, 256, False), (37, 1000, 1000, True),
    (300, 1001, 1008, True), (5, 7, 8, False), (64, 8192, 8192, True), (2048, 4096, 4096, True),
])
def test_quantize_rowwise_bit_exact(M, K, ld, outliers):
    x = W.activations(M, K, seed=M + K, outliers=outliers)
    q_ref, s_ref = oracle.quantize_rowwise_int8(x)
    xt = dev(x, ld=ld)
    xq, xs = qg().quantize_rowwise_int8(xt)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), q_ref)
    assert np.array_equal(host(xs).view(np.uint32), s_ref.view(np.uint32))


def test_quantize_rowwise_zero_rows_ties_and_full_size():
    x = W.activations(8192, 4096, seed=1, outliers=True)
    x[0] = 0                                              # all-zero row: scale 1e-10/127
    x[1, :8] = np.array([127, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -127], np.float16)
    x[1, 8:] = 0
    q_ref, s_ref = oracle.quantize_rowwise_int8(x)
    xq, xs = qg().quantize_rowwise_int8(dev(x))
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), q_ref)
    assert np.array_equal(host(xs), s_ref)
    assert list(host(xq)[1, :8]) == [127, 2, 4, -2, -4, 0, 2, -127]


# ----------------------------------------------------------------------------
# a2: block-asymmetric 4-bit quantize + pack
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(1, 64), (24, 192), (11008, 4096)])
def test_quantize_block_asym4_bit_exact(N, K):
    w = W.weights(N, K, seed=4, per_column_factor=False)
    qw_ref, sc_ref, ze_ref, _ = oracle.quantize_block_asym4(w, 64)
    qw, sc, ze = qg().quantize_block_asym4(dev(w))
    torch.cuda.synchronize()
    assert np.array_equal(host(qw).view(np.uint32), qw_ref)
    assert np.array_equal(bits16(sc), sc_ref.view(np.uint16))
    assert np.array_equal(bits16(ze), ze_ref.view(np.uint16))


# ----------------------------------------------------------------------------
# a3/a4: W8A8
# ----------------------------------------------------------------------------

def _w8a8_inputs(M, N, K, seed, outliers=True, factor=True, with_bias=True):
    x = W.activations(M, K, seed=seed, outliers=outliers)
    w = W.weights(N, K, seed=seed, per_column_factor=factor)
    xq, xs = oracle.quantize_rowwise_int8(x)
    wq, ws = oracle.quantize_rowwise_int8(w)
    b = W.bias(N, seed) if with_bias else None
    return xq, xs, wq, ws, b


# shapes: decode (swap-AB, split-K clusters), mid, prefill tiles with ragged M/N/K tails
W8A8_SHAPES = [
    (129, 520, 1000), (300, 777, 1104), (65, 300, 256), (1024, 1024, 4096), (64, 11008, 4096),
    (16, 256, 256), (3, 520, 1000), (17, 200, 4096), (33, 384, 512),
    (1, 4096, 4096), (8, 4096, 4096), (16, 4096, 4096),
]


@pytest.mark.parametrize("M,N,K", W8A8_SHAPES)
def test_w8a8_int32_accumulator_bit_exact(M, N, K):
    xq, xs, wq, ws, _ = _w8a8_inputs(M, N, K, seed=M + N)
    acc_ref = oracle.gemm_i8_i64(xq, wq)
    assert np.abs(acc_ref).max() < 2 ** 31
    ldx = (K + 15) // 16 * 16
    y = torch.full((M, N), -1, dtype=torch.int32, device="cuda")
    qg().gemm_w8a8(dev(xq, ld=ldx), dev(wq, ld=ldx), None, None, None, out_dtype=torch.int32, out=y)
    torch.cuda.synchronize()
    assert np.array_equal(host(y).astype(np.int64), acc_ref)


@pytest.mark.parametrize("M,N,K", [(16, 256, 256), (1, 4096, 4096), (300, 777, 1104), (129, 520, 1000)])
def test_w8a8_f32_epilogue(M, N, K):
    xq, xs, wq, ws, b = _w8a8_inputs(M, N, K, seed=0, outliers=(M != 16))
    acc = oracle.gemm_i8_i64(xq, wq)
    y64 = oracle.w8a8_epilogue_f64(acc, xs, ws, b)
    ldx = (K + 15) // 16 * 16
    y = qg().gemm_w8a8(dev(xq, ld=ldx), dev(wq, ld=ldx), dev(xs), dev(ws), dev(b), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_w8a8_f32(host(y), acc, xs, ws, b, y64)


@pytest.mark.parametrize("M,N,K,kind", [(1, 4096, 4096, "f16"), (8, 4096, 4096, "f16"), (16, 4096, 4096, "f16"),
                                        (33, 4096, 4096, "f16"), (256, 1000, 4096, "bf16"),
                                        (2048, 4096, 4096, "bf16")])
def test_w8a8_half_outputs_within_one_ulp(M, N, K, kind):
    xq, xs, wq, ws, b = _w8a8_inputs(M, N, K, seed=1 if kind == "f16" else 2)
    acc = oracle.gemm_i8_i64(xq, wq)
    y64 = oracle.w8a8_epilogue_f64(acc, xs, ws, b)
    dt = torch.float16 if kind == "f16" else torch.bfloat16
    y = qg().gemm_w8a8(dev(xq), dev(wq), dev(xs), dev(ws), dev(b), out_dtype=dt)
    torch.cuda.synchronize()
    assert_w8a8_half(bits16(y), y64, w8a8_magnitude(acc, xs, ws, b), kind, f"w8a8 {kind} {M}x{N}x{K}")


@pytest.mark.parametrize("M,N", [(8192, 11008), (2048, 11008), (8192, 4096)])
def test_w8a8_prefill_full_size_sampled_rows(M, N):
    """Full-size prefill launch; 48 seeded rows checked against the oracle."""
    K = 4096
    xq, xs, wq, ws, b = _w8a8_inputs(M, N, K, seed=2)
    y = qg().gemm_w8a8(dev(xq), dev(wq), dev(xs), dev(ws), dev(b), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows = W.sample_rows(M, 48, seed=M + N)
    acc = oracle.gemm_i8_i64(xq[rows], wq)
    y64 = oracle.w8a8_epilogue_f64(acc, xs[rows], ws, b)
    assert_w8a8_half(bits16(y)[rows], y64, w8a8_magnitude(acc, xs[rows], ws, b), "bf16", f"w8a8 prefill {M}x{N}")


def test_w8a8_no_bias_and_strided_output():
    M, N, K = 40, 300, 512
    xq, xs, wq, ws, _ = _w8a8_inputs(M, N, K, seed=7, with_bias=False)
    acc = oracle.gemm_i8_i64(xq, wq)
    y64 = oracle.w8a8_epilogue_f64(acc, xs, ws, None)
    buf = torch.zeros((M, 320), dtype=torch.float16, device="cuda")
    y = buf[:, :N]
    qg().gemm_w8a8(dev(xq), dev(wq), dev(xs), dev(ws), None, out_dtype=torch.float16, out=y)
    torch.cuda.synchronize()
    assert_w8a8_half(bits16(y), y64, w8a8_magnitude(acc, xs, ws, None), "f16", "w8a8 strided")
    assert torch.all(buf[:, N:] == 0)


def test_w8a8_degenerate_sizes():
    q = qg()
    xq = torch.zeros((4, 0), dtype=torch.int8, device="cuda")
    wq = torch.zeros((8, 0), dtype=torch.int8, device="cuda")
    b = torch.arange(8, dtype=torch.float32, device="cuda")
    xs = torch.ones(4, device="cuda")
    ws = torch.ones(8, device="cuda")
    y = q.gemm_w8a8(xq, wq, xs, ws, b, out_dtype=torch.float32)       # K = 0: Y = bias
    torch.cuda.synchronize()
    assert torch.equal(y, b.expand(4, 8))
    y0 = q.gemm_w8a8(torch.zeros((0, 64), dtype=torch.int8, device="cuda"),
                     torch.zeros((8, 64), dtype=torch.int8, device="cuda"),
                     torch.ones(0, device="cuda"), ws, None, out_dtype=torch.float32)
    assert y0.shape == (0, 8)
    q.check_device_errors()


def test_device_status_clean_after_all_launches():
    qg().check_device_errors()


# ----------------------------------------------------------------------------
# decode paths: stream-K (workspace) and cluster split-K (no workspace)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 4096, 4096), (16, 256, 256), (3, 520, 1000),
                                   (33, 384, 512), (64, 11008, 4096), (16, 11008, 4096), (8, 128, 128)])
def test_w8a8_decode_stream_k_and_cluster_paths_bit_exact(M, N, K):
    xq, xs, wq, ws, b = _w8a8_inputs(M, N, K, seed=N + K)
    acc_ref = oracle.gemm_i8_i64(xq, wq)
    ldx = (K + 15) // 16 * 16
    dx, dw = dev(xq, ld=ldx), dev(wq, ld=ldx)
    q = qg()
    for ws_mode in ("auto", None, "auto"):      # the second stream-K call checks the tickets were reset
        y = torch.full((M, N), -7, dtype=torch.int32, device="cuda")
        q.gemm_w8a8(dx, dw, None, None, None, out_dtype=torch.int32, out=y, workspace=ws_mode)
        torch.cuda.synchronize()
        assert np.array_equal(host(y).astype(np.int64), acc_ref), ws_mode
    y64 = oracle.w8a8_epilogue_f64(acc_ref, xs, ws, b)
    yh = q.gemm_w8a8(dx, dw, dev(xs), dev(ws), dev(b), out_dtype=torch.float16)
    torch.cuda.synchronize()
    assert_w8a8_half(bits16(yh), y64, w8a8_magnitude(acc_ref, xs, ws, b), "f16", f"w8a8 stream-K {M}x{N}x{K}")
    q.check_device_errors()
