"""GPU parity for the GEMMs with a fused GELU epilogue (qg_gemm_*_act), through
the C ABI, against the oracle's GEMM followed by the oracle's GELU.

Bars.  W8A8: the kernel applies gelu to the fp32 epilogue value v, which is
within 1e-6 * mag of the fp64 result (the W8A8 bar).  gelu' is at most 1.13,
and the fp32 evaluation of 0.5 v (1 + erf(v / sqrt 2)) adds a few ulp of |v|
<= mag, so |out - gelu(y64)| <= 2.5e-6 * mag for fp32 outputs, plus half an
output ulp for fp16/bf16 (or 1 ulp of the rounded fp64 value).  Weight-only:
relative Frobenius error <= 2e-3 and the element-wise bound of the plain
weight-only GEMMs carried through gelu (parity_util.assert_wonly_elementwise).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import (assert_w8a8_half, assert_wonly_elementwise, bits16, dev, host, rel_frobenius, requires_cuda,
                         w4_dequant, w8_dequant, w8a8_magnitude)

pytestmark = [pytest.mark.gpu, requires_cuda]
GELU_MAG = 2.5


def qg():
    import int4_quantized_gemm_b200 as q
    return q


def _w8a8(M, N, K, seed):
    x = W.activations(M, K, seed=seed, outliers=True)
    w = W.weights(N, K, seed=seed, per_column_factor=True)
    xq, xs = oracle.quantize_rowwise_int8(x)
    wq, ws = oracle.quantize_rowwise_int8(w)
    return xq, xs, wq, ws, W.bias(N, seed)


@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (1, 11008, 4096), (3, 520, 1000), (300, 777, 1104),
                                   (1024, 1024, 4096)])
def test_w8a8_gelu_f32(M, N, K):
    xq, xs, wq, ws, b = _w8a8(M, N, K, seed=M + N)
    acc = oracle.gemm_i8_i64(xq, wq)
    g64 = oracle.gelu_f64(oracle.w8a8_epilogue_f64(acc, xs, ws, b))
    ld = (K + 15) // 16 * 16
    y = qg().gemm_w8a8_act(dev(xq, ld=ld), dev(wq, ld=ld), dev(xs), dev(ws), dev(b), "gelu",
                           out_dtype=torch.float32)
    torch.cuda.synchronize()
    mag = w8a8_magnitude(acc, xs, ws, b)
    err = np.abs(host(y).astype(np.float64) - g64)
    assert np.all(err <= GELU_MAG * 1e-6 * mag + 1e-30), f"worst {np.max(err / (mag + 1e-30)):.3e}"


@pytest.mark.parametrize("M,N,K,kind", [(16, 4096, 4096, "f16"), (256, 1000, 4096, "bf16")])
def test_w8a8_gelu_half(M, N, K, kind):
    xq, xs, wq, ws, b = _w8a8(M, N, K, seed=5)
    acc = oracle.gemm_i8_i64(xq, wq)
    g64 = oracle.gelu_f64(oracle.w8a8_epilogue_f64(acc, xs, ws, b))
    dt = torch.float16 if kind == "f16" else torch.bfloat16
    y = qg().gemm_w8a8_act(dev(xq), dev(wq), dev(xs), dev(ws), dev(b), "gelu", out_dtype=dt)
    torch.cuda.synchronize()
    assert_w8a8_half(bits16(y), g64, GELU_MAG * w8a8_magnitude(acc, xs, ws, b), kind, f"gelu {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(16, 11008, 4096), (1, 4096, 4096), (40, 520, 1024), (256, 1024, 4096)])
def test_weight_only_gelu(M, N, K):
    q = qg()
    x = W.activations(M, K, seed=9)
    w = W.weights(N, K, seed=9, per_column_factor=False)
    b = W.bias(N, 9)
    wq, ws = oracle.quantize_rowwise_int8(w)
    qw, sc, ze, _ = oracle.quantize_block_asym4(w, 64)
    v8 = oracle.w8a16_f64(x, wq, ws, b)
    v4 = oracle.w4a16_f64(x, qw, sc, ze, 64, b)
    g8, g4 = oracle.gelu_f64(v8), oracle.gelu_f64(v4)
    y8 = q.gemm_w8a16_act(dev(x), dev(wq), dev(ws), dev(b), "gelu")
    y4 = q.gemm_w4a16_act(dev(x), dev(qw.view(np.int32)), dev(sc), dev(ze), 64, dev(b), "gelu")
    torch.cuda.synchronize()
    assert rel_frobenius(host(y8).astype(np.float64), g8) <= 2e-3
    assert rel_frobenius(host(y4).astype(np.float64), g4) <= 2e-3
    assert_wonly_elementwise(y8, x, w8_dequant(wq, ws), v8, b, int4=False, what="w8a16 gelu", gelu=True)
    assert_wonly_elementwise(y4, x, w4_dequant(qw, sc, ze), v4, b, int4=True, what="w4a16 gelu", gelu=True)


def test_activation_none_matches_the_plain_gemm_and_edge_cases():
    q = qg()
    xq, xs, wq, ws, b = _w8a8(16, 4096, 4096, seed=2)
    y0 = q.gemm_w8a8(dev(xq), dev(wq), dev(xs), dev(ws), dev(b), out_dtype=torch.float32)
    y1 = q.gemm_w8a8_act(dev(xq), dev(wq), dev(xs), dev(ws), dev(b), "none", out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    # K == 0: gelu of the bias
    bb = torch.linspace(-3, 3, 24, device="cuda")
    y = q.gemm_w8a8_act(torch.zeros((2, 0), dtype=torch.int8, device="cuda"),
                        torch.zeros((24, 0), dtype=torch.int8, device="cuda"),
                        torch.ones(2, device="cuda"), torch.ones(24, device="cuda"), bb, "gelu",
                        out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.gelu_f64(host(bb).astype(np.float64))
    assert np.allclose(host(y)[0].astype(np.float64), ref, rtol=0, atol=1e-6)
    with pytest.raises(q.QGError):          # an activation on the raw int32 accumulator
        q.gemm_w8a8_act(dev(xq), dev(wq), dev(xs), dev(ws), None, "gelu", out_dtype=torch.int32)
    q.check_device_errors()
