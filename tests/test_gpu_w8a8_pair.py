"""GPU parity for the CTA-pair prefill W8A8 tiles (256-row output tiles of 224
to 256 columns on two-CTA clusters, tcgen05 cta_group::2), through the C ABI.

The pair tiles take every floating-point decision the one-SM tiles take (same
int32 accumulator, same fp32 epilogue per element), so for M > 128 the output of
a launch on pair tiles must equal, bit for bit, the output of the same launch on
one-SM tiles (the QG_W8A8_PAIR switch set to 0), and the int32 accumulator
must equal the oracle's exact sum.  Shapes cover ragged M, N and K tails (a pair
whose odd CTA holds no valid row, N and K not multiples of the tile), one tile
per pair and several tiles per pair (both accumulator buffers in use).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import assert_w8a8_half, bits16, dev, host, requires_cuda, w8a8_magnitude

pytestmark = [pytest.mark.gpu, requires_cuda]


def qg():
    import int4_quantized_gemm_b200 as q
    return q


def _inputs(M, N, K, seed):
    x = W.activations(M, K, seed=seed, outliers=True)
    w = W.weights(N, K, seed=seed, per_column_factor=True)
    xq, xs = oracle.quantize_rowwise_int8(x)
    wq, ws = oracle.quantize_rowwise_int8(w)
    return xq, xs, wq, ws, W.bias(N, seed)


def _ld(K):
    return (K + 15) // 16 * 16


def _both(call):
    """call() on one-SM tiles, then on pair tiles (the default)."""
    q = qg()
    try:
        q.set_tuning("QG_W8A8_PAIR", 0)
        one = call()
        torch.cuda.synchronize()
        q.set_tuning("QG_W8A8_PAIR", 1)
        pair = call()
        torch.cuda.synchronize()
    finally:
        q.set_tuning("QG_W8A8_PAIR", 1)
    return one, pair


PAIR_SHAPES = [(129, 520, 1000), (257, 300, 160), (300, 777, 1104), (512, 512, 512), (1024, 1024, 4096),
               (2048, 11008, 4096)]


@pytest.mark.parametrize("M,N,K", PAIR_SHAPES)
def test_pair_int32_accumulator_equals_the_oracle_and_one_sm_tiles(M, N, K):
    xq, xs, wq, ws, _ = _inputs(M, N, K, seed=M + N + K)
    q = qg()
    dx, dw = dev(xq, ld=_ld(K)), dev(wq, ld=_ld(K))
    one, pair = _both(lambda: q.gemm_w8a8(dx, dw, None, None, None, out_dtype=torch.int32))
    assert torch.equal(one, pair)
    if M * N * K <= 2 ** 31:
        assert np.array_equal(host(pair).astype(np.int64), oracle.gemm_i8_i64(xq, wq))
    else:  # full size: 40 seeded rows against the oracle
        rows = W.sample_rows(M, 40, seed=M)
        assert np.array_equal(host(pair)[rows].astype(np.int64), oracle.gemm_i8_i64(xq[rows], wq))
    q.check_device_errors()


@pytest.mark.parametrize("M,N,K,kind", [(300, 777, 1104, "f16"), (1024, 1024, 4096, "bf16"),
                                        (2048, 4096, 4096, "f32")])
def test_pair_epilogue_bit_identical_to_one_sm_tiles(M, N, K, kind):
    xq, xs, wq, ws, b = _inputs(M, N, K, seed=5)
    q = qg()
    dt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[kind]
    args = (dev(xq, ld=_ld(K)), dev(wq, ld=_ld(K)), dev(xs), dev(ws), dev(b))
    one, pair = _both(lambda: q.gemm_w8a8(*args, out_dtype=dt))
    assert torch.equal(one.view(torch.int16) if kind != "f32" else one.view(torch.int32),
                       pair.view(torch.int16) if kind != "f32" else pair.view(torch.int32))
    if kind != "f32":
        acc = oracle.gemm_i8_i64(xq, wq)
        y64 = oracle.w8a8_epilogue_f64(acc, xs, ws, b)
        assert_w8a8_half(bits16(pair), y64, w8a8_magnitude(acc, xs, ws, b), kind, f"pair {kind} {M}x{N}x{K}")


def test_pair_zero_point_and_gelu_epilogues_bit_identical():
    q = qg()
    M, N, K = 384, 640, 1024
    x = np.maximum(W.activations(M, K, seed=9, outliers=True), np.float16(0))
    w = W.weights(N, K, seed=9, per_column_factor=True)
    xq, xs, xz, xsum = oracle.quantize_rowwise_asym_int8(x)
    wq, ws, wz, wsum = oracle.quantize_rowwise_asym_int8(w)
    b = W.bias(N, 9)
    zargs = (dev(xq), dev(xs), dev(xz), dev(xsum), dev(wq), dev(ws), dev(wz), dev(wsum), dev(b))
    one, pair = _both(lambda: q.gemm_w8a8_zp(*zargs, out_dtype=torch.float32))
    assert torch.equal(one.view(torch.int32), pair.view(torch.int32))
    y64 = oracle.w8a8_zp_f64(xq, xs, xz, wq, ws, wz, b)
    assert np.max(np.abs(host(pair).astype(np.float64) - y64)) <= 1e-5 * np.abs(y64).max()
    sq, ss = oracle.quantize_rowwise_int8(x)
    gargs = (dev(sq), dev(wq), dev(ss), dev(ws), dev(b), "gelu")
    one, pair = _both(lambda: q.gemm_w8a8_act(*gargs, out_dtype=torch.float16))
    assert torch.equal(one.view(torch.int16), pair.view(torch.int16))
    q.check_device_errors()


@pytest.mark.parametrize("M,N,K", [(300, 777, 1104), (1024, 1000, 2048)])
def test_pair_tile_widths_agree(M, N, K):
    """The pair tile width (output columns per tile, chosen by waves; the
    QG_PAIR_N switch forces it) changes only which CTA pair computes which
    columns: at 256, 240, 224 and 128 columns the int32 accumulator equals the
    oracle's exact sum and the bf16 outputs are the same bits."""
    xq, xs, wq, ws, b = _inputs(M, N, K, seed=9)
    q = qg()
    dx, dw = dev(xq, ld=_ld(K)), dev(wq, ld=_ld(K))
    dxs, dws, db = dev(xs), dev(ws), dev(b)
    acc = oracle.gemm_i8_i64(xq, wq)
    outs = []
    try:
        for pn in (256, 240, 224, 128):
            q.set_tuning("QG_PAIR_N", pn)
            raw = q.gemm_w8a8(dx, dw, None, None, None, out_dtype=torch.int32)
            y = q.gemm_w8a8(dx, dw, dxs, dws, db, out_dtype=torch.bfloat16)
            torch.cuda.synchronize()
            assert np.array_equal(host(raw).astype(np.int64), acc), pn
            outs.append(bits16(y))
    finally:
        q.set_tuning("QG_PAIR_N", 0)
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    q.check_device_errors()
