"""Launch plans (qg_plan_*): a plan binds one call's arguments once and each
launch makes that call, so every output must equal the direct call's bit for
bit -- on the decode shapes of the hot path, ragged and padded shapes, the
larger-M tilings, with and without QG_FLAG_STATIC_WEIGHTS and with a stream-K
workspace.  A plan binds buffers, not values: inputs rewritten in place between
launches give the new results.  Plans launched inside a CUDA graph capture and
on an explicit stream behave the same.
"""
from __future__ import annotations

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


def _same(a, b, what):
    assert a.dtype == b.dtype and a.shape == b.shape, what
    if a.dtype in (torch.float16, torch.bfloat16):
        a, b = a.view(torch.int16), b.view(torch.int16)
    elif a.dtype == torch.float32:
        a, b = a.view(torch.int32), b.view(torch.int32)
    assert torch.equal(a, b), what


def _operands(M, N, K, seed):
    x = W.activations(M, K, seed=seed, outliers=True)
    w = W.weights(N, K, seed=seed + 1)
    xq, xs = oracle.quantize_rowwise_int8(x)
    wq, ws = oracle.quantize_rowwise_int8(w)
    ld8, ld16 = (K + 15) // 16 * 16, (K + 7) // 8 * 8  # rows on 16-byte boundaries
    d = dict(x=dev(x, ld=ld16), xq=dev(xq, ld=ld8), xs=dev(xs), wq=dev(wq, ld=ld8), ws=dev(ws),
             b=dev(W.bias(N, seed)))
    if K % 64 == 0:  # 4-bit weights: whole groups of 64
        qw, sc, ze, _ = oracle.quantize_block_asym4(W.weights(N, K, seed=seed + 2, per_column_factor=False), 64)
        d.update(qw=dev(qw.view(np.int32)), sc=dev(sc), ze=dev(ze))
    return d


SHAPES = [(16, 4096, 4096), (16, 11008, 4096), (1, 4096, 4096), (5, 520, 1000), (64, 264, 512),
          (100, 776, 1024), (300, 1000, 2048)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("static", [False, True])
def test_plans_equal_the_direct_calls(M, N, K, static):
    q = qg()
    d = _operands(M, N, K, seed=M + N)
    torch.cuda.synchronize()  # the weights are written before any flagged call
    ref = [q.quantize_rowwise_int8(d["x"]),
           q.gemm_w8a8(d["xq"], d["wq"], d["xs"], d["ws"], d["b"], out_dtype=torch.float16, static_weights=static),
           q.gemm_w8a8(d["xq"], d["wq"], None, None, None, out_dtype=torch.int32, static_weights=static),
           q.gemm_w8a16(d["x"], d["wq"], d["ws"], d["b"], static_weights=static)]
    plans = [q.plan_quantize_rowwise_int8(d["x"]),
             q.plan_gemm_w8a8(d["xq"], d["wq"], d["xs"], d["ws"], d["b"], out_dtype=torch.float16,
                              static_weights=static),
             q.plan_gemm_w8a8(d["xq"], d["wq"], None, None, None, out_dtype=torch.int32, static_weights=static),
             q.plan_gemm_w8a16(d["x"], d["wq"], d["ws"], d["b"], static_weights=static)]
    if "qw" in d:
        ref.append(q.gemm_w4a16(d["x"], d["qw"], d["sc"], d["ze"], 64, d["b"], static_weights=static))
        plans.append(q.plan_gemm_w4a16(d["x"], d["qw"], d["sc"], d["ze"], 64, d["b"], static_weights=static))
    for p in plans:
        p.launch()
        p()  # twice: a launch leaves the plan unchanged
    torch.cuda.synchronize()
    q.check_device_errors()
    _same(ref[0][0], plans[0].out[0], "xq")
    _same(ref[0][1], plans[0].out[1], "x_scale")
    for r, p, what in zip(ref[1:], plans[1:], ("w8a8 f16", "w8a8 i32", "w8a16", "w4a16")):
        _same(r, p.out, what)
    for p in plans:
        p.close()
        p.close()  # idempotent


def test_a_plan_reads_its_buffers_at_each_launch():
    """Bound to the activation buffer: new values written in place between
    launches (the decode loop) give the new step's results."""
    q = qg()
    M, N, K = 16, 4096, 4096
    d = _operands(M, N, K, seed=7)
    x = d["x"]
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    pq = q.plan_quantize_rowwise_int8(x, out=xq, scale_out=xs)
    pa = q.plan_gemm_w8a8(xq, d["wq"], xs, d["ws"], d["b"], out_dtype=torch.float32, static_weights=True)
    pb = q.plan_gemm_w8a16(x, d["wq"], d["ws"], static_weights=True)
    pc = q.plan_gemm_w4a16(x, d["qw"], d["sc"], d["ze"], static_weights=True)
    for step in range(3):
        x.copy_(dev(W.activations(M, K, seed=100 + step, outliers=True)))
        for p in (pq, pa, pb, pc):
            p.launch()
        got = [pa.out.clone(), pb.out.clone(), pc.out.clone(), xq.clone(), xs.clone()]
        rq, rs = q.quantize_rowwise_int8(x)
        ref = [q.gemm_w8a8(rq, d["wq"], rs, d["ws"], d["b"], out_dtype=torch.float32),
               q.gemm_w8a16(x, d["wq"], d["ws"]), q.gemm_w4a16(x, d["qw"], d["sc"], d["ze"]), rq, rs]
        torch.cuda.synchronize()
        for g, r in zip(got, ref):
            _same(r.contiguous(), g.contiguous(), f"step {step}")
    q.check_device_errors()


def test_plans_in_a_graph_and_on_a_given_stream():
    q = qg()
    M, N, K = 16, 11008, 4096
    d = _operands(M, N, K, seed=11)
    torch.cuda.synchronize()
    ref = [q.gemm_w8a16(d["x"], d["wq"], d["ws"], d["b"]), q.gemm_w4a16(d["x"], d["qw"], d["sc"], d["ze"])]
    pb = q.plan_gemm_w8a16(d["x"], d["wq"], d["ws"], d["b"], static_weights=True)
    pc = q.plan_gemm_w4a16(d["x"], d["qw"], d["sc"], d["ze"], static_weights=True)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    pb.launch(s)
    pc.launch(s.cuda_stream)
    s.synchronize()
    _same(ref[0], pb.out, "w8a16 on a stream")
    _same(ref[1], pc.out, "w4a16 on a stream")
    pb.out.zero_()
    pc.out.zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(4):
                pc.launch()
                pb.launch()
    with torch.cuda.stream(s):
        g.replay()
    s.synchronize()
    q.check_device_errors()
    _same(ref[0], pb.out, "w8a16 in a graph")
    _same(ref[1], pc.out, "w4a16 in a graph")
    del g


def test_a_plan_with_a_workspace_runs_the_stream_k_kernels():
    q = qg()
    M, N, K = 16, 4096, 4096
    d = _operands(M, N, K, seed=13)
    n = int(q.raw.qg_gemm_workspace_size(M, N, K))
    assert n > 0
    w1 = torch.zeros(n, dtype=torch.uint8, device="cuda")
    w2 = torch.zeros(n, dtype=torch.uint8, device="cuda")
    ref = [q.gemm_w8a16(d["x"], d["wq"], d["ws"], workspace=w1), q.gemm_w4a16(d["x"], d["qw"], d["sc"], d["ze"],
                                                                             workspace=w1)]
    plans = [q.plan_gemm_w8a16(d["x"], d["wq"], d["ws"], workspace=w2),
             q.plan_gemm_w4a16(d["x"], d["qw"], d["sc"], d["ze"], workspace=w2)]
    for p in plans:
        p.launch()
    torch.cuda.synchronize()
    q.check_device_errors()
    for r, p in zip(ref, plans):
        _same(r, p.out, "stream-K plan")
    with pytest.raises(ValueError):
        q.plan_gemm_w8a16(d["x"], d["wq"], d["ws"], workspace="auto")
