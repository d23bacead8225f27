"""The debug library (libqg_debug.so: the same sources built with QG_DEBUG)
checks on the device every TMA coordinate against the 16-byte rule for its
innermost coordinate and the hand-computed offsets of the split-K exchanges
against their shared-memory areas.  A failed check records QG_ERR_DEBUG_CHECK
and skips the access, so a clean run proves those accesses in range for the
shapes below; the results must equal the release library's bit for bit (the
checks change no arithmetic).  Every kernel family runs: the quantizers, W8A8
decode (cluster split-K) and prefill (one-SM tiles, CTA pairs), the fused
quantize + W8A8, W4A8, W8A16 / W4A16 decode (cluster split-K, stream-K with a
workspace, the allocation-free entry) and the wide-tile kernel with and
without a K split.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import dev, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]


def qg():
    import int4_quantized_gemm_b200 as q
    return q


@pytest.fixture(scope="module")
def libs():
    q = qg()
    if not os.path.exists(q.DEBUG_LIB_PATH):
        pytest.fail("libqg_debug.so is missing: build it with int4_quantized_gemm_b200/build.py --debug")
    dbg = ctypes.CDLL(q.DEBUG_LIB_PATH)
    for name, (args, res) in q.SIGNATURES.items():
        f = getattr(dbg, name)
        f.argtypes = args
        f.restype = res
    assert dbg.qg_debug_checks() == 1 and q.raw.qg_debug_checks() == 0
    return q.raw, dbg


def _both(libs, call):
    """call() through the release library, then through the debug library; the
    debug run must report no failed check."""
    q = qg()
    rel, dbg = libs
    outs = []
    try:
        for lib in (rel, dbg):
            q.raw = lib
            outs.append(call())
            torch.cuda.synchronize()
            q.check_device_errors()
    finally:
        q.raw = rel
    return outs


def _same(a, b):
    if isinstance(a, (tuple, list)):
        for x, y in zip(a, b):
            _same(x, y)
        return
    assert a.dtype == b.dtype and a.shape == b.shape
    if a.dtype in (torch.float16, torch.bfloat16):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    elif a.dtype == torch.float32:
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    else:
        assert torch.equal(a, b)


def _w8(M, N, K, seed):
    x = W.activations(M, K, seed=seed, outliers=True)
    w = W.weights(N, K, seed=seed)
    xq, xs = oracle.quantize_rowwise_int8(x)
    wq, ws = oracle.quantize_rowwise_int8(w)
    ld8, ld16 = (K + 15) // 16 * 16, (K + 7) // 8 * 8  # rows on 16-byte boundaries
    return dev(x, ld=ld16), dev(xq, ld=ld8), dev(xs), dev(wq, ld=ld8), dev(ws), dev(W.bias(N, seed))


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 4096, 4096), (16, 520, 1000), (64, 1024, 2048),
                                   (100, 777, 1104), (300, 777, 1104), (1024, 1000, 2048)])
def test_w8a8_paths_pass_the_checks(libs, M, N, K):
    q = qg()
    x, xq, xs, wq, ws, b = _w8(M, N, K, seed=M + N)
    a, d = _both(libs, lambda: (q.gemm_w8a8(xq, wq, xs, ws, b, out_dtype=torch.float16),
                                q.gemm_w8a8(xq, wq, None, None, None, out_dtype=torch.int32)))
    _same(a, d)


@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (5, 520, 1024)])
def test_fused_quantize_and_w4a8_pass_the_checks(libs, M, N, K):
    q = qg()
    x, _, _, wq, ws, b = _w8(M, N, K, seed=3)
    w = W.weights(N, K, seed=4)
    qw, sc = q.quantize_channel_sym4(torch.from_numpy(w).cuda())
    a, d = _both(libs, lambda: (q.quantize_gemm_w8a8(x, wq, ws, b, out_dtype=torch.float16),
                                q.gemm_w4a8(q.quantize_rowwise_int8(x)[0], qw, q.quantize_rowwise_int8(x)[1], sc, b,
                                            out_dtype=torch.float16)))
    _same(a, d)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 11008, 4096), (16, 520, 1024), (64, 264, 512),
                                   (100, 520, 4096), (256, 1024, 4096), (200, 1024, 512), (96, 520, 4096)])
def test_weight_only_paths_pass_the_checks(libs, M, N, K):
    q = qg()
    x = W.activations(M, K, seed=M)
    w = W.weights(N, K, seed=N, per_column_factor=False)
    wq, ws = oracle.quantize_rowwise_int8(w)
    qw, sc, ze, _ = oracle.quantize_block_asym4(w, 64)
    dx, dwq, dws, dqw, dsc, dze = dev(x), dev(wq), dev(ws), dev(qw.view(np.int32)), dev(sc), dev(ze)
    work = None
    n = int(q.raw.qg_gemm_workspace_size(M, N, K))
    if n:
        work = torch.zeros(n, dtype=torch.uint8, device="cuda")

    def call():
        outs = [q.gemm_w8a16(dx, dwq, dws), q.gemm_w4a16(dx, dqw, dsc, dze),
                q.gemm_w4a16(dx, dqw, dsc, dze, static_weights=True)]
        if work is not None:  # the stream-K decode kernel
            outs += [q.gemm_w8a16(dx, dwq, dws, workspace=work), q.gemm_w4a16(dx, dqw, dsc, dze, workspace=work)]
        return outs

    a, d = _both(libs, call)
    _same(a, d)


def test_quantizers_and_no_alloc_pass_the_checks(libs):
    q = qg()
    M, N, K = 16, 4096, 4096
    x = torch.from_numpy(W.activations(M, K, seed=9)).cuda()
    w = torch.from_numpy(W.edge_weights(512, 1024, seed=9)).cuda()
    qw, sc, ze, _ = oracle.quantize_block_asym4(W.weights(N, K, seed=9, per_column_factor=False), 64)
    dqw, dsc, dze = dev(qw.view(np.int32)), dev(sc), dev(ze)

    def call():
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        q.gemm_w4a16_noalloc(x, dqw, dsc, dze, out=y)
        return [*q.quantize_rowwise_int8(x), *q.quantize_block_asym4(w), *q.quantize_rowwise_asym_int8(x), y]

    a, d = _both(libs, call)
    _same(a, d)
