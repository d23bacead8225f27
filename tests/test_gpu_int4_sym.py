"""GPU parity for symmetric int4 weights: the two quantizers (bit-exact codes,
packed words and scales), W4A8 on the int8 tensor cores (int32 accumulator
bit-exact; fp32 and fp16/bf16 outputs at the W8A8 bars, since its epilogue is
the W8A8 one), and the symmetric group-int4 W4A16 (relative Frobenius <= 2e-3,
one-hot rows bit-exact fp16(q * s)), all against the oracle through the C ABI.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import (assert_w8a8_f32, assert_w8a8_half, assert_wonly_elementwise, bits16, dev, host,
                         rel_frobenius, requires_cuda, w4sym_dequant, w8a8_magnitude)

pytestmark = [pytest.mark.gpu, requires_cuda]


def qg():
    import int4_quantized_gemm_b200 as q
    return q


def _unpack(qw):
    nib = (qw[:, :, None] >> (4 * np.arange(8, dtype=np.uint32))[None, None, :]) & 0xF
    v = nib.astype(np.int16).reshape(qw.shape[0], -1)
    return np.where(v >= 8, v - 16, v).astype(np.int8)


@pytest.mark.parametrize("N,K", [(1, 64), (24, 192), (11008, 4096)])
def test_quantize_sym4_bit_exact(N, K):
    w = W.weights(N, K, seed=12, per_column_factor=True)
    qw_r, sc_r, _ = oracle.quantize_block_sym4(w, 64)
    qw, sc = qg().quantize_block_sym4(dev(w))
    qc_r, sc2_r, _ = oracle.quantize_channel_sym4(w)
    qc, sc2 = qg().quantize_channel_sym4(dev(w))
    torch.cuda.synchronize()
    assert np.array_equal(host(qw).view(np.uint32), qw_r)
    assert np.array_equal(bits16(sc), sc_r.view(np.uint16))
    assert np.array_equal(host(qc).view(np.uint32), qc_r)
    assert np.array_equal(host(sc2).view(np.uint32), sc2_r.view(np.uint32))


def _w4a8_case(M, N, K, seed):
    x = W.activations(M, K, seed=seed, outliers=True)
    w = W.weights(N, K, seed=seed, per_column_factor=True)
    xq, xs = oracle.quantize_rowwise_int8(x)
    qw, ws, q = oracle.quantize_channel_sym4(w)
    return xq, xs, qw, ws, q, W.bias(N, seed)


# decode (swap-AB, K-split clusters), ragged N and K blocks, and M > 64 on 64-row tiles
W4A8_SHAPES = [(1, 4096, 4096), (16, 4096, 4096), (16, 11008, 4096), (5, 520, 1056), (33, 300, 288),
               (64, 264, 512), (100, 777, 1024), (300, 520, 2048)]


@pytest.mark.parametrize("M,N,K", W4A8_SHAPES)
def test_w4a8_int32_accumulator_bit_exact(M, N, K):
    xq, xs, qw, ws, q, b = _w4a8_case(M, N, K, seed=M + N)
    acc_ref = oracle.gemm_i8_i64(xq, q)
    ld = (K + 15) // 16 * 16
    y = torch.full((M, N), -1, dtype=torch.int32, device="cuda")
    qg().gemm_w4a8(dev(xq, ld=ld), dev(qw.view(np.int32)), None, None, None, out_dtype=torch.int32, out=y)
    torch.cuda.synchronize()
    assert np.array_equal(host(y).astype(np.int64), acc_ref)


@pytest.mark.parametrize("M,N,K,kind", [(16, 4096, 4096, "f32"), (16, 11008, 4096, "f16"),
                                        (3, 520, 1056, "bf16"), (200, 1024, 4096, "f16")])
def test_w4a8_epilogue_against_the_oracle(M, N, K, kind):
    xq, xs, qw, ws, q, b = _w4a8_case(M, N, K, seed=3)
    acc = oracle.gemm_i8_i64(xq, q)
    y64 = oracle.w4a8_f64(xq, qw, xs, ws, b)
    dt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[kind]
    ld = (K + 15) // 16 * 16
    y = qg().gemm_w4a8(dev(xq, ld=ld), dev(qw.view(np.int32)), dev(xs), dev(ws), dev(b), out_dtype=dt)
    torch.cuda.synchronize()
    if kind == "f32":
        assert_w8a8_f32(host(y), acc, xs, ws, b, y64)
    else:
        assert_w8a8_half(bits16(y), y64, w8a8_magnitude(acc, xs, ws, b), kind, f"w4a8 {kind} {M}x{N}x{K}")


def test_w4a8_pipeline_from_gpu_quantizers_and_extreme_codes():
    q = qg()
    M, N, K = 16, 1024, 4096
    x = W.activations(M, K, seed=14, outliers=True)
    w = W.weights(N, K, seed=14, per_column_factor=True)
    xq, xs = q.quantize_rowwise_int8(dev(x))
    qw, ws = q.quantize_channel_sym4(dev(w))
    y = q.gemm_w4a8(xq, qw, None, None, None, out_dtype=torch.int32)
    torch.cuda.synchronize()
    assert np.array_equal(host(y).astype(np.int64), oracle.gemm_i8_i64(host(xq), _unpack(host(qw).view(np.uint32))))
    # every nibble value, including -8, through the unpacker: codes -8..7 repeated
    codes = np.tile(np.arange(-8, 8, dtype=np.int8), (64, 256))[:, :4096]
    words = np.zeros((64, 512), np.uint32)
    for j in range(8):
        words |= (codes[:, j::8].astype(np.uint32) & 0xF) << np.uint32(4 * j)
    ones = np.ones((3, 4096), np.int8)
    ones[1] = -1
    ones[2, ::2] = 127
    yy = q.gemm_w4a8(dev(ones), dev(words.view(np.int32)), None, None, None, out_dtype=torch.int32)
    torch.cuda.synchronize()
    assert np.array_equal(host(yy).astype(np.int64), ones.astype(np.int64) @ codes.astype(np.int64).T)


@pytest.mark.parametrize("M,N,K", [(16, 11008, 4096), (1, 4096, 4096), (40, 520, 1024), (256, 1024, 4096),
                                   (3, 136, 192)])
def test_w4a16_sym_frobenius(M, N, K):
    x = W.activations(M, K, seed=5)
    w = W.weights(N, K, seed=5, per_column_factor=False)
    qw, sc, _ = oracle.quantize_block_sym4(w, 64)
    b = W.bias(N, 5)
    y64 = oracle.w4a16_sym_f64(x, qw, sc, 64, b)
    y = qg().gemm_w4a16_sym(dev(x), dev(qw.view(np.int32)), dev(sc), 64, dev(b))
    torch.cuda.synchronize()
    assert rel_frobenius(host(y).astype(np.float64), y64) <= 2e-3
    assert_wonly_elementwise(y, x, w4sym_dequant(qw, sc), y64, b, int4=True, what=f"w4a16 sym {M}x{N}x{K}")


def test_w4a16_sym_one_hot_rows_are_bit_exact():
    M, N, K = 16, 4096, 4096
    w = W.weights(N, K, seed=7, per_column_factor=False)
    qw, sc, q = oracle.quantize_block_sym4(w, 64)
    x = np.zeros((M, K), np.float16)
    cols = W.sample_rows(K, M, seed=7)
    x[np.arange(M), cols] = 1.0
    y = qg().gemm_w4a16_sym(dev(x), dev(qw.view(np.int32)), dev(sc), 64)
    torch.cuda.synchronize()
    ref = oracle.round_f16(q[:, cols].T.astype(np.float64) * sc.astype(np.float64)[cols // 64, :])
    assert np.array_equal(bits16(y), ref)
    qg().check_device_errors()
