"""QG_FLAG_STATIC_WEIGHTS (the *_ex GEMM entry points): the decode kernels load
and dequantize their first weight tiles before waiting on the preceding kernel.
The arithmetic is unchanged, so every output must equal the plain call's bit
for bit, on the decode shapes (single CTA, K-split clusters, ragged N and K,
fewer K blocks than ring stages) and, for the paths that ignore the flag
(larger M, a workspace), as well.  A chain of flagged calls on one stream (each
kernel's weight loads overlapping the previous kernel) is checked against the
oracle.  The weights here are written, and synchronized, before any flagged
call, which is the flag's contract.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import assert_w8a8_f32, assert_wonly_elementwise, dev, host, requires_cuda, w4_dequant, w8_dequant

pytestmark = [pytest.mark.gpu, requires_cuda]
SHAPES = [(1, 4096, 4096), (16, 11008, 4096), (16, 4096, 4096), (5, 520, 1024), (33, 304, 256), (64, 264, 512),
          (16, 128, 128), (100, 776, 1024)]


def qg():
    import int4_quantized_gemm_b200 as q
    return q


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_static_weight_calls_equal_the_plain_calls(M, N, K):
    q = qg()
    x = W.activations(M, K, seed=61, outliers=True)
    w = W.weights(N, K, seed=61, per_column_factor=True)
    b = W.bias(N, 61)
    xq, xs = oracle.quantize_rowwise_int8(x)
    wq, ws = oracle.quantize_rowwise_int8(w)
    qw, sc, ze, _ = oracle.quantize_block_asym4(w, 64)
    dx, dxq, dxs, dwq, dws, db = dev(x), dev(xq), dev(xs), dev(wq), dev(ws), dev(b)
    dqw, dsc, dze = dev(qw.view(np.int32)), dev(sc), dev(ze)
    torch.cuda.synchronize()
    a0 = q.gemm_w8a8(dxq, dwq, dxs, dws, db, out_dtype=torch.float16)
    a1 = q.gemm_w8a8(dxq, dwq, dxs, dws, db, out_dtype=torch.float16, static_weights=True)
    i1 = q.gemm_w8a8(dxq, dwq, None, None, None, out_dtype=torch.int32, static_weights=True)
    b0 = q.gemm_w8a16(dx, dwq, dws, db)
    b1 = q.gemm_w8a16(dx, dwq, dws, db, static_weights=True)
    c0 = q.gemm_w4a16(dx, dqw, dsc, dze, 64, db)
    c1 = q.gemm_w4a16(dx, dqw, dsc, dze, 64, db, static_weights=True)
    torch.cuda.synchronize()
    q.check_device_errors()
    assert torch.equal(a0.view(torch.int16), a1.view(torch.int16))
    assert torch.equal(b0.view(torch.int16), b1.view(torch.int16))
    assert torch.equal(c0.view(torch.int16), c1.view(torch.int16))
    assert np.array_equal(host(i1).astype(np.int64), oracle.gemm_i8_i64(xq, wq))


def test_a_chain_of_static_weight_calls_matches_the_oracle():
    """quantize -> W8A8 -> W8A16 -> W4A16, repeated over four weight sets on one
    stream with the flag: the decode step of the benchmark."""
    q = qg()
    M, K = 16, 4096
    sets = []
    for r in range(4):
        x = W.activations(M, K, seed=70 + r, outliers=True)
        w1 = W.weights(4096, K, seed=70 + r)
        w2 = W.weights(11008, K, seed=80 + r)
        w3 = W.weights(11008, K, seed=90 + r, per_column_factor=False)
        wq1, ws1 = oracle.quantize_rowwise_int8(w1)
        wq2, ws2 = oracle.quantize_rowwise_int8(w2)
        qw, sc, ze, _ = oracle.quantize_block_asym4(w3, 64)
        b1 = W.bias(4096, 70 + r)
        sets.append(dict(x=x, wq1=wq1, ws1=ws1, b1=b1, wq2=wq2, ws2=ws2, qw=qw, sc=sc, ze=ze,
                         d=dict(x=dev(x), wq1=dev(wq1), ws1=dev(ws1), b1=dev(b1), wq2=dev(wq2), ws2=dev(ws2),
                                qw=dev(qw.view(np.int32)), sc=dev(sc), ze=dev(ze))))
    torch.cuda.synchronize()   # every weight is written before the first flagged call
    outs = []
    for rep in range(2):
        for t in sets:
            d = t["d"]
            xq, xs = q.quantize_rowwise_int8(d["x"])
            y1 = q.gemm_w8a8(xq, d["wq1"], xs, d["ws1"], d["b1"], out_dtype=torch.float32, static_weights=True)
            y2 = q.gemm_w8a16(d["x"], d["wq2"], d["ws2"], static_weights=True)
            y3 = q.gemm_w4a16(d["x"], d["qw"], d["sc"], d["ze"], static_weights=True)
            outs.append((t, y1, y2, y3))
    torch.cuda.synchronize()
    q.check_device_errors()
    for t, y1, y2, y3 in outs[len(sets):]:   # the second pass: every kernel preceded by another
        xq_r, xs_r = oracle.quantize_rowwise_int8(t["x"])
        acc = oracle.gemm_i8_i64(xq_r, t["wq1"])
        assert_w8a8_f32(host(y1), acc, xs_r, t["ws1"], t["b1"], oracle.w8a8_f64(xq_r, t["wq1"], xs_r, t["ws1"], t["b1"]))
        assert_wonly_elementwise(y2, t["x"], w8_dequant(t["wq2"], t["ws2"]),
                                 oracle.w8a16_f64(t["x"], t["wq2"], t["ws2"], None), None, int4=False,
                                 what="chained w8a16")
        assert_wonly_elementwise(y3, t["x"], w4_dequant(t["qw"], t["sc"], t["ze"]),
                                 oracle.w4a16_f64(t["x"], t["qw"], t["sc"], t["ze"], 64, None), None, int4=True,
                                 what="chained w4a16")


def test_unknown_flag_bits_are_rejected():
    q = qg()
    x = torch.zeros((2, 64), dtype=torch.float16, device="cuda")
    wq = torch.zeros((8, 64), dtype=torch.int8, device="cuda")
    y = torch.zeros((2, 8), dtype=torch.float16, device="cuda")
    st = q.raw.qg_gemm_w8a16_ex(x.data_ptr(), 64, wq.data_ptr(), 64, torch.ones(8, device="cuda").data_ptr(), None,
                                y.data_ptr(), 8, 2, 8, 64, None, 0, 6, torch.cuda.current_stream().cuda_stream)
    assert st == q.QG_ERR_INVALID_ARG


def test_two_stream_step_in_a_graph_equals_the_one_stream_step():
    """The decode step as the benchmark schedules it: quantize -> W8A8 on the
    step's stream, W4A16 -> W8A16 (flagged calls) on a second stream forked
    from it and joined at the end of the step, eight steps over two weight
    sets captured in one CUDA graph.  Every output equals the one-stream
    step's bit for bit, also when kernels of the two streams overlap."""
    q = qg()
    M, K = 16, 4096
    dev_ = torch.device("cuda")
    sets = []
    for r in range(2):
        x = W.activations(M, K, seed=200 + r, outliers=True)
        wq1, ws1 = oracle.quantize_rowwise_int8(W.weights(4096, K, seed=210 + r))
        wq2, ws2 = oracle.quantize_rowwise_int8(W.weights(11008, K, seed=220 + r))
        qw, sc, ze, _ = oracle.quantize_block_asym4(W.weights(11008, K, seed=230 + r, per_column_factor=False), 64)
        sets.append(dict(x=dev(x), wq1=dev(wq1), ws1=dev(ws1), b1=dev(W.bias(4096, 200 + r)), wq2=dev(wq2),
                         ws2=dev(ws2), qw=dev(qw.view(np.int32)), sc=dev(sc), ze=dev(ze),
                         xq=torch.empty((M, K), dtype=torch.int8, device=dev_),
                         xs=torch.empty(M, dtype=torch.float32, device=dev_),
                         y=[torch.empty((M, n), dtype=torch.float16, device=dev_) for n in (4096, 11008, 11008)]))
    torch.cuda.synchronize()
    side = torch.cuda.Stream()

    def chain_a(d, y):
        q.quantize_rowwise_int8(d["x"], out=d["xq"], scale_out=d["xs"])
        q.gemm_w8a8(d["xq"], d["wq1"], d["xs"], d["ws1"], d["b1"], out_dtype=torch.float16, out=y[0],
                    static_weights=True)

    def chain_b(d, y):
        q.gemm_w4a16(d["x"], d["qw"], d["sc"], d["ze"], out=y[2], static_weights=True)
        q.gemm_w8a16(d["x"], d["wq2"], d["ws2"], out=y[1], static_weights=True)

    def two_stream_step(d, y):
        cur = torch.cuda.current_stream()
        side.wait_stream(cur)
        with torch.cuda.stream(side):
            chain_b(d, y)
        chain_a(d, y)
        cur.wait_stream(side)

    ref = []
    for d in sets:
        y = [torch.empty_like(t) for t in d["y"]]
        chain_a(d, y)
        chain_b(d, y)
        ref.append(y)
    torch.cuda.synchronize()
    q.check_device_errors()
    eager = []
    for d in sets:
        two_stream_step(d, d["y"])
        eager.append([t.clone() for t in d["y"]])
    torch.cuda.synchronize()
    for d in sets:
        for t in d["y"]:
            t.zero_()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(8):
                two_stream_step(sets[i % 2], sets[i % 2]["y"])
    with torch.cuda.stream(stream):
        g.replay()
        g.replay()
    stream.synchronize()
    q.check_device_errors()
    for r, d in enumerate(sets):
        for a, b, c in zip(ref[r], eager[r], d["y"]):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
            assert torch.equal(a.view(torch.int16), c.view(torch.int16))
    del g
