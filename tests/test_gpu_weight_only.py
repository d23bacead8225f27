"""GPU parity for the weight-only GEMMs (W8A16, W4A16) through the C ABI.

Bars: relative Frobenius error <= 2e-3 against the fp64 product of the
dequantized weights (the oracle), on the same seeded inputs, and every output
element within the element-wise bound derived from the kernels' arithmetic
(parity_util.assert_wonly_elementwise).  One-hot rows of X
reduce the product to a dequantized weight column, which gives a per-element
closed form: bit-exact for W4A16 (the kernel forms fp16((q - z) * s) once and
multiplies it by 1.0 exactly) and within 1 ulp for W8A16 (w_scale * q rounded
in fp32, then to fp16).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import (assert_within_one_ulp16, assert_wonly_elementwise, bits16, dev, host, rel_frobenius,
                         requires_cuda, w4_dequant, w8_dequant)

pytestmark = [pytest.mark.gpu, requires_cuda]
TOL = 2e-3


def qg():
    import int4_quantized_gemm_b200 as q
    return q


def _w8_inputs(M, N, K, seed, factor=True, with_bias=False):
    x = W.activations(M, K, seed=seed)
    w = W.weights(N, K, seed=seed, per_column_factor=factor)
    wq, ws = oracle.quantize_rowwise_int8(w)
    b = W.bias(N, seed) if with_bias else None
    return x, wq, ws, b


def _w4_inputs(M, N, K, seed, with_bias=False):
    x = W.activations(M, K, seed=seed)
    w = W.weights(N, K, seed=seed, per_column_factor=False)
    qw, sc, ze, _ = oracle.quantize_block_asym4(w, 64)
    b = W.bias(N, seed) if with_bias else None
    return x, qw, sc, ze, b


W8A16_SHAPES = [
    (1, 4096, 4096), (16, 4096, 4096), (16, 11008, 4096), (3, 520, 1000), (33, 300, 256),
    (64, 264, 512), (100, 777, 520), (129, 200, 256), (300, 520, 384), (256, 1024, 4096),
]


@pytest.mark.parametrize("M,N,K", W8A16_SHAPES)
def test_w8a16_frobenius(M, N, K):
    x, wq, ws, b = _w8_inputs(M, N, K, seed=3, with_bias=(M % 2 == 1))
    y64 = oracle.w8a16_f64(x, wq, ws, b)
    ldx = (K + 7) // 8 * 8
    ldw = (K + 15) // 16 * 16
    y = qg().gemm_w8a16(dev(x, ld=ldx), dev(wq, ld=ldw), dev(ws), None if b is None else dev(b))
    torch.cuda.synchronize()
    err = rel_frobenius(host(y).astype(np.float64), y64)
    assert err <= TOL, f"W8A16 {M}x{N}x{K}: relative Frobenius error {err:.3e}"
    assert_wonly_elementwise(y, x, w8_dequant(wq, ws), y64, b, int4=False, what=f"W8A16 {M}x{N}x{K}")


@pytest.mark.parametrize("M,N", [(256, 11008), (256, 4096)])
def test_w8a16_full_size_sampled_rows(M, N):
    K = 4096
    x, wq, ws, _ = _w8_inputs(M, N, K, seed=3)
    y = qg().gemm_w8a16(dev(x), dev(wq), dev(ws))
    torch.cuda.synchronize()
    rows = W.sample_rows(M, 24, seed=N)
    y64 = oracle.w8a16_f64(x[rows], wq, ws, None)
    err = rel_frobenius(host(y)[rows].astype(np.float64), y64)
    assert err <= TOL, err
    assert_wonly_elementwise(y[torch.from_numpy(rows).cuda()], x[rows], w8_dequant(wq, ws), y64, None, int4=False,
                             what=f"W8A16 {M}x{N}x{K} sampled rows")


def test_w8a16_one_hot_rows_give_scaled_columns():
    M, N, K = 16, 4096, 4096
    _, wq, ws, _ = _w8_inputs(M, N, K, seed=5)
    x = np.zeros((M, K), np.float16)
    cols = W.sample_rows(K, M, seed=5)
    x[np.arange(M), cols] = 1.0
    y = qg().gemm_w8a16(dev(x), dev(wq), dev(ws))
    torch.cuda.synchronize()
    ref = oracle.round_f16(ws[None, :].astype(np.float64) * wq[:, cols].T.astype(np.float64))
    assert_within_one_ulp16(bits16(y), ref, "w8a16 one-hot")


W4A16_SHAPES = [
    (1, 11008, 4096), (16, 11008, 4096), (16, 4096, 4096), (3, 520, 1024), (40, 264, 512),
    (129, 256, 320), (300, 136, 192), (64, 1024, 4096),
]


@pytest.mark.parametrize("M,N,K", W4A16_SHAPES)
def test_w4a16_frobenius(M, N, K):
    x, qw, sc, ze, b = _w4_inputs(M, N, K, seed=4, with_bias=(M % 2 == 1))
    y64 = oracle.w4a16_f64(x, qw, sc, ze, 64, b)
    y = qg().gemm_w4a16(dev(x), dev(qw.view(np.int32)), dev(sc), dev(ze), 64,
                        None if b is None else dev(b))
    torch.cuda.synchronize()
    err = rel_frobenius(host(y).astype(np.float64), y64)
    assert err <= TOL, f"W4A16 {M}x{N}x{K}: relative Frobenius error {err:.3e}"
    assert_wonly_elementwise(y, x, w4_dequant(qw, sc, ze), y64, b, int4=True, what=f"W4A16 {M}x{N}x{K}")


@pytest.mark.parametrize("M,N", [(256, 11008), (512, 4096)])
def test_w4a16_full_size_sampled_rows(M, N):
    """Larger M: several 128-wide X tiles per weight tile (one or two waves)."""
    K = 4096
    x, qw, sc, ze, _ = _w4_inputs(M, N, K, seed=8)
    y = qg().gemm_w4a16(dev(x), dev(qw.view(np.int32)), dev(sc), dev(ze))
    torch.cuda.synchronize()
    rows = W.sample_rows(M, 24, seed=N + 1)
    y64 = oracle.w4a16_f64(x[rows], qw, sc, ze, 64, None)
    err = rel_frobenius(host(y)[rows].astype(np.float64), y64)
    assert err <= TOL, err
    assert_wonly_elementwise(y[torch.from_numpy(rows).cuda()], x[rows], w4_dequant(qw, sc, ze), y64, None,
                             int4=True, what=f"W4A16 {M}x{N}x{K} sampled rows")


def test_weight_only_outputs_into_column_slices():
    """Outputs written through a leading dimension larger than N (column slices
    of one wider buffer) equal the contiguous outputs bit for bit and leave the
    rest of the buffer untouched."""
    q = qg()
    M, N, K = 16, 1000, 1024
    x, wq, ws, b = _w8_inputs(M, N, K, seed=12, with_bias=True)
    _, qw, sc, ze, _ = _w4_inputs(M, N, K, seed=12)
    dx = dev(x)
    buf = torch.zeros((M, 2 * N + 24), dtype=torch.float16, device="cuda")
    y8, y4 = buf[:, 8:8 + N], buf[:, 16 + N:16 + 2 * N]
    q.gemm_w8a16(dx, dev(wq), dev(ws), dev(b), out=y8)
    q.gemm_w4a16(dx, dev(qw.view(np.int32)), dev(sc), dev(ze), out=y4)
    r8 = q.gemm_w8a16(dx, dev(wq), dev(ws), dev(b))
    r4 = q.gemm_w4a16(dx, dev(qw.view(np.int32)), dev(sc), dev(ze))
    torch.cuda.synchronize()
    assert torch.equal(y8.view(torch.int16), r8.view(torch.int16))
    assert torch.equal(y4.view(torch.int16), r4.view(torch.int16))
    assert torch.all(buf[:, :8] == 0) and torch.all(buf[:, 8 + N:16 + N] == 0) and torch.all(buf[:, 16 + 2 * N:] == 0)


def test_w4a16_one_hot_rows_are_bit_exact_dequantized_columns():
    M, N, K = 16, 11008, 4096
    _, qw, sc, ze, _ = _w4_inputs(M, N, K, seed=6)
    x = np.zeros((M, K), np.float16)
    cols = W.sample_rows(K, M, seed=6)
    x[np.arange(M), cols] = 1.0
    y = qg().gemm_w4a16(dev(x), dev(qw.view(np.int32)), dev(sc), dev(ze))
    torch.cuda.synchronize()
    # (q - z) * s rounded once to fp16, per the kernel's dequant
    codes = ((qw[:, cols // 8] >> (4 * (cols % 8)).astype(np.uint32)) & 0xF).astype(np.float64)  # [N, M]
    s = sc.astype(np.float64)[cols // 64, :].T
    z = ze.astype(np.float64)[cols // 64, :].T
    ref = oracle.round_f16(((codes - z) * s).T)
    assert np.array_equal(bits16(y), ref)


def test_w4a16_pipeline_from_gpu_quantizer():
    """GPU block quantizer -> GPU W4A16, against the oracle on the oracle's own codes."""
    M, N, K = 16, 11008, 4096
    x = W.activations(M, K, seed=8)
    w = W.weights(N, K, seed=8, per_column_factor=False)
    qw, sc, ze = qg().quantize_block_asym4(dev(w))
    y = qg().gemm_w4a16(dev(x), qw, sc, ze)
    torch.cuda.synchronize()
    qw_r, sc_r, ze_r, _ = oracle.quantize_block_asym4(w, 64)
    y64 = oracle.w4a16_f64(x, qw_r, sc_r, ze_r, 64, None)
    assert rel_frobenius(host(y).astype(np.float64), y64) <= TOL
    assert_wonly_elementwise(y, x, w4_dequant(qw_r, sc_r, ze_r), y64, None, int4=True, what="W4A16 pipeline")


def test_weight_only_degenerate_sizes_and_status():
    q = qg()
    b = torch.arange(24, dtype=torch.float32, device="cuda")
    y = q.gemm_w8a16(torch.zeros((3, 0), dtype=torch.float16, device="cuda"),
                     torch.zeros((24, 0), dtype=torch.int8, device="cuda"),
                     torch.ones(24, device="cuda"), b)
    torch.cuda.synchronize()
    assert torch.equal(y.float(), b.expand(3, 24))
    y0 = q.gemm_w4a16(torch.zeros((0, 64), dtype=torch.float16, device="cuda"),
                      torch.zeros((24, 8), dtype=torch.int32, device="cuda"),
                      torch.ones((1, 24), dtype=torch.float16, device="cuda"),
                      torch.zeros((1, 24), dtype=torch.float16, device="cuda"))
    assert y0.shape == (0, 24)
    q.check_device_errors()


@pytest.mark.parametrize("M,N,K", [(1, 11008, 4096), (16, 4096, 4096), (16, 264, 512), (3, 520, 1024),
                                   (40, 520, 1024), (64, 1024, 4096), (16, 128, 128)])
def test_weight_only_decode_stream_k_and_cluster_paths(M, N, K):
    q = qg()
    x, wq, ws, b = _w8_inputs(M, N, K, seed=9, with_bias=True)
    y8_ref = oracle.w8a16_f64(x, wq, ws, b)
    _, qw, sc, ze, _ = _w4_inputs(M, N, K, seed=10)
    y4_ref = oracle.w4a16_f64(x, qw, sc, ze, 64, b)
    dx, dwq, dws, db = dev(x), dev(wq), dev(ws), dev(b)
    dqw, dsc, dze = dev(qw.view(np.int32)), dev(sc), dev(ze)
    outs8, outs4 = [], []
    for ws_mode in ("auto", None, "auto"):
        y8 = q.gemm_w8a16(dx, dwq, dws, db, workspace=ws_mode)
        y4 = q.gemm_w4a16(dx, dqw, dsc, dze, 64, db, workspace=ws_mode)
        torch.cuda.synchronize()
        assert rel_frobenius(host(y8).astype(np.float64), y8_ref) <= TOL, ("w8a16", ws_mode)
        assert rel_frobenius(host(y4).astype(np.float64), y4_ref) <= TOL, ("w4a16", ws_mode)
        assert_wonly_elementwise(y8, x, w8_dequant(wq, ws), y8_ref, b, int4=False, what=f"w8a16 {ws_mode}")
        assert_wonly_elementwise(y4, x, w4_dequant(qw, sc, ze), y4_ref, b, int4=True, what=f"w4a16 {ws_mode}")
        outs8.append(host(y8))
        outs4.append(host(y4))
    # stream-K sums partials in a fixed order: repeated calls are bitwise identical
    assert np.array_equal(outs8[0], outs8[2]) and np.array_equal(outs4[0], outs4[2])
    q.check_device_errors()


@pytest.mark.parametrize("M,N,K", [(130, 3000, 1024), (200, 2048, 2048), (256, 1024, 4096), (96, 520, 4096),
                                   (640, 264, 1024), (100, 1000, 8192), (200, 1024, 512)])
def test_wide_token_tiles_with_k_split_clusters(M, N, K):
    """M > 64 runs the wide-tile kernel: one dequantization per weight block for
    128/256 tokens, K split over clusters of 1 (200x1024x512), 2 (130x3000,
    640x264), 4 (200x2048, 256x1024) and 8 CTAs (96x520, 100x1000x8192) with
    the partial rows summed through distributed shared memory, ragged N and M,
    several token tiles (M = 640)."""
    q = qg()
    x, wq, ws, b = _w8_inputs(M, N, K, seed=31, with_bias=True)
    _, qw, sc, ze, _ = _w4_inputs(M, N, K, seed=32)
    y8_64 = oracle.w8a16_f64(x, wq, ws, b)
    y4_64 = oracle.w4a16_f64(x, qw, sc, ze, 64, b)
    dx = dev(x)
    y8 = q.gemm_w8a16(dx, dev(wq), dev(ws), dev(b))
    y4 = q.gemm_w4a16(dx, dev(qw.view(np.int32)), dev(sc), dev(ze), 64, dev(b))
    torch.cuda.synchronize()
    assert rel_frobenius(host(y8).astype(np.float64), y8_64) <= TOL
    assert rel_frobenius(host(y4).astype(np.float64), y4_64) <= TOL
    assert_wonly_elementwise(y8, x, w8_dequant(wq, ws), y8_64, b, int4=False, what=f"wide W8A16 {M}x{N}x{K}")
    assert_wonly_elementwise(y4, x, w4_dequant(qw, sc, ze), y4_64, b, int4=True, what=f"wide W4A16 {M}x{N}x{K}")
    # an output whose row pitch (N + 3 elements) rules out the tile store: element stores, same bits
    buf8 = torch.zeros((M, N + 3), dtype=torch.float16, device="cuda")
    buf4 = torch.zeros((M, N + 3), dtype=torch.float16, device="cuda")
    q.gemm_w8a16(dx, dev(wq), dev(ws), dev(b), out=buf8[:, :N])
    q.gemm_w4a16(dx, dev(qw.view(np.int32)), dev(sc), dev(ze), 64, dev(b), out=buf4[:, :N])
    torch.cuda.synchronize()
    assert torch.equal(buf8[:, :N].view(torch.int16), y8.view(torch.int16))
    assert torch.equal(buf4[:, :N].view(torch.int16), y4.view(torch.int16))
    assert not buf8[:, N:].any() and not buf4[:, N:].any()
    q.check_device_errors()


@pytest.mark.parametrize("M,K", [(100, 8192), (256, 4096), (200, 2048)])
def test_wide_split_tail_ragged_columns(M, K):
    """The split-K tail writes 8 output columns per 16-byte store where the
    output allows it.  N = 1001 (W8A16 only: no quantization groups along N)
    leaves a last group of one column, written element by element; with a row
    pitch of 1008 the other groups take the 16-byte stores, with a pitch of 1001
    every group is written element by element.  Both equal the contiguous
    result bit for bit and meet the element-wise bound."""
    q = qg()
    N = 1001
    x, wq, ws, b = _w8_inputs(M, N, K, seed=35, with_bias=True)
    y64 = oracle.w8a16_f64(x, wq, ws, b)
    dx, dwq, dws, db = dev(x), dev(wq), dev(ws), dev(b)
    y = q.gemm_w8a16(dx, dwq, dws, db)
    buf = torch.zeros((M, 1008), dtype=torch.float16, device="cuda")
    q.gemm_w8a16(dx, dwq, dws, db, out=buf[:, :N])
    torch.cuda.synchronize()
    assert torch.equal(buf[:, :N].view(torch.int16), y.view(torch.int16))
    assert not buf[:, N:].any()
    assert_wonly_elementwise(y, x, w8_dequant(wq, ws), y64, b, int4=False, what=f"ragged W8A16 {M}x{N}x{K}")
    q.check_device_errors()


def test_token_tile_widths_agree():
    """The same product on decode tiles (64 tokens) and on wide tiles of 128 and
    256 tokens (forced with the QG_WONLY_BN switch): every width meets the bound."""
    q = qg()
    M, N, K = 256, 1024, 2048
    x, wq, ws, b = _w8_inputs(M, N, K, seed=33, with_bias=True)
    _, qw, sc, ze, _ = _w4_inputs(M, N, K, seed=34)
    y8_64 = oracle.w8a16_f64(x, wq, ws, b)
    y4_64 = oracle.w4a16_f64(x, qw, sc, ze, 64, b)
    try:
        for bn in (64, 128, 256):
            q.set_tuning("QG_WONLY_BN", bn)
            y8 = q.gemm_w8a16(dev(x), dev(wq), dev(ws), dev(b))
            y4 = q.gemm_w4a16(dev(x), dev(qw.view(np.int32)), dev(sc), dev(ze), 64, dev(b))
            torch.cuda.synchronize()
            assert_wonly_elementwise(y8, x, w8_dequant(wq, ws), y8_64, b, int4=False, what=f"W8A16 bn={bn}")
            assert_wonly_elementwise(y4, x, w4_dequant(qw, sc, ze), y4_64, b, int4=True, what=f"W4A16 bn={bn}")
    finally:
        q.set_tuning("QG_WONLY_BN", 0)
    q.check_device_errors()
