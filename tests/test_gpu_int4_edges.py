"""GPU parity on the cases where the 4-bit weight quantizers' floors and clamps
act, through the C ABI, against the oracle.

The weights come from workloads.edge_weights: 64-element blocks of hand-chosen
patterns (ramps whose asymmetric zero point is each of 0..15, all-zero and
constant blocks, all-positive and all-negative blocks, a tiny block, whole
zero and constant rows) mixed with N(0, 0.02) blocks.  Quantizer outputs
(packed words, fp16 scales and zero points, fp32 per-column scales) must be
bit-exact; the GEMMs on these weights (zero points spanning 0..15, so q - z
spans -15..15; subnormal fp16 scales) must meet the element-wise weight-only
bound of parity_util and the relative Frobenius bound 2e-3, and W4A8's int32
accumulator must be exact.  Pages: "从零实现大语言模型 INT8 量化" 第一步/第二步
(block scale and zero point), "量化算法的本质" (the 1e-5 and 1e-10 floors, code
clamp), "INT4/FP16混合精度GEMM" §5.1 (symmetric int4).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import (assert_w8a8_f32, assert_wonly_elementwise, bits16, dev, host, rel_frobenius,
                         requires_cuda, w4_dequant, w4sym_dequant)

pytestmark = [pytest.mark.gpu, requires_cuda]
SHAPES = [(11008, 4096), (520, 1024), (24, 64)]


def qg():
    import int4_quantized_gemm_b200 as q
    return q


@pytest.mark.parametrize("N,K", SHAPES)
def test_block_asym4_quantizer_on_edge_blocks_bit_exact(N, K):
    w = W.edge_weights(N, K, seed=N)
    qw_r, sc_r, ze_r, _ = oracle.quantize_block_asym4(w, 64)
    qw, sc, ze = qg().quantize_block_asym4(dev(w))
    torch.cuda.synchronize()
    if N >= 24 * 11:
        assert sorted(set(ze_r.astype(np.float64).ravel().tolist())) == [float(z) for z in range(16)]
    assert np.array_equal(host(qw).view(np.uint32), qw_r)
    assert np.array_equal(bits16(sc), sc_r.view(np.uint16))
    assert np.array_equal(bits16(ze), ze_r.view(np.uint16))


@pytest.mark.parametrize("N,K", SHAPES)
def test_sym4_quantizers_on_edge_blocks_bit_exact(N, K):
    w = W.edge_weights(N, K, seed=N + 1)
    qw_r, sc_r, _ = oracle.quantize_block_sym4(w, 64)
    qc_r, sc2_r, _ = oracle.quantize_channel_sym4(w)
    qw, sc = qg().quantize_block_sym4(dev(w))
    qc, sc2 = qg().quantize_channel_sym4(dev(w))
    torch.cuda.synchronize()
    # the floors are taken: the 1e-5 block floor (fp16 bits 0x00A8) and 1e-10/7 per column
    assert (sc_r.view(np.uint16) == 0x00A8).any()
    assert (sc2_r.view(np.uint32) == 0x2D7B5123).any()
    assert np.array_equal(host(qw).view(np.uint32), qw_r)
    assert np.array_equal(bits16(sc), sc_r.view(np.uint16))
    assert np.array_equal(host(qc).view(np.uint32), qc_r)
    assert np.array_equal(host(sc2).view(np.uint32), sc2_r.view(np.uint32))


@pytest.mark.parametrize("M,N,K", [(16, 11008, 4096), (1, 11008, 4096), (5, 520, 1024), (200, 520, 1024)])
def test_w4a16_with_zero_points_spanning_0_to_15(M, N, K):
    w = W.edge_weights(N, K, seed=N)
    qw, sc, ze, _ = oracle.quantize_block_asym4(w, 64)
    x = W.activations(M, K, seed=M + 40)
    b = W.bias(N, M)
    y64 = oracle.w4a16_f64(x, qw, sc, ze, 64, b)
    y = qg().gemm_w4a16(dev(x), dev(qw.view(np.int32)), dev(sc), dev(ze), 64, dev(b))
    torch.cuda.synchronize()
    assert rel_frobenius(host(y).astype(np.float64), y64) <= 2e-3
    assert_wonly_elementwise(y, x, w4_dequant(qw, sc, ze), y64, b, int4=True, what=f"w4a16 edges {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(16, 11008, 4096), (3, 520, 1024)])
def test_w4a16_sym_on_edge_blocks(M, N, K):
    w = W.edge_weights(N, K, seed=N + 1)
    qw, sc, _ = oracle.quantize_block_sym4(w, 64)
    x = W.activations(M, K, seed=M + 41)
    y64 = oracle.w4a16_sym_f64(x, qw, sc, 64, None)
    y = qg().gemm_w4a16_sym(dev(x), dev(qw.view(np.int32)), dev(sc), 64)
    torch.cuda.synchronize()
    assert rel_frobenius(host(y).astype(np.float64), y64) <= 2e-3
    assert_wonly_elementwise(y, x, w4sym_dequant(qw, sc), y64, None, int4=True,
                             what=f"w4a16 sym edges {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(16, 11008, 4096), (7, 520, 1024)])
def test_w4a8_on_edge_columns(M, N, K):
    """Per-column symmetric int4 codes of the edge weights (zero columns with
    the 1e-10 floor, constant columns at -7) through W4A8: the int32
    accumulator is exact and the fp32 epilogue meets the W8A8 bar."""
    w = W.edge_weights(N, K, seed=N + 2)
    x = W.activations(M, K, seed=M + 42, outliers=True)
    xq, xs = oracle.quantize_rowwise_int8(x)
    qw, ws, q = oracle.quantize_channel_sym4(w)
    b = W.bias(N, M)
    acc = oracle.gemm_i8_i64(xq, q)
    ld = (K + 15) // 16 * 16
    yi = qg().gemm_w4a8(dev(xq, ld=ld), dev(qw.view(np.int32)), None, None, None, out_dtype=torch.int32)
    y = qg().gemm_w4a8(dev(xq, ld=ld), dev(qw.view(np.int32)), dev(xs), dev(ws), dev(b), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(host(yi).astype(np.int64), acc)
    assert_w8a8_f32(host(y), acc, xs, ws, b, oracle.w4a8_f64(xq, qw, xs, ws, b))
    qg().check_device_errors()
