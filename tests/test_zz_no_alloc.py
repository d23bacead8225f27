"""qg_gemm_w4a16_noalloc: the W4A16 decode GEMM that allocates no device memory.

Some callers may not allocate: code running inside a runtime that owns all
device memory through its own pool and forbids allocation while it executes,
or latency-bound decode loops that cannot pay for cudaMalloc/cudaFree (which
may synchronize the device).  For them the library keeps the stream-K kernel's
scratch in a static device array.  These tests call that entry point through
the C ABI and check it against the regular qg_gemm_w4a16 on the same inputs.

The file is named so that pytest collects it last.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import host, rel_frobenius, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]
TOL = 2e-3   # the weight-only relative Frobenius bound used by the other parity tests


def _inputs(M, N, K, seed):
    x = W.activations(M, K, seed=seed)
    w = W.weights(N, K, seed=seed, per_column_factor=False)
    qw, sc, ze, _ = oracle.quantize_block_asym4(w, 64)
    b = W.bias(N, seed)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return dict(x=d(x), qw=d(qw.view(np.int32)), sc=d(sc), ze=d(ze), b=d(b), M=M, N=N, K=K)


def _noalloc_raw(q, t, y):
    """One call of qg_gemm_w4a16_noalloc through the C ABI; returns its status."""
    vp = lambda a: ctypes.c_void_p(a.data_ptr())
    return q.raw.qg_gemm_w4a16_noalloc(vp(t["x"]), t["K"], vp(t["qw"]), vp(t["sc"]), vp(t["ze"]), 64,
                                       vp(t["b"]), vp(y), t["N"], t["M"], t["N"], t["K"],
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_the_allocating_entry_point_on_two_calls_in_a_row():
    import int4_quantized_gemm_b200 as q
    a = _inputs(16, 11008, 4096, seed=21)
    b = _inputs(5, 4096, 2048, seed=22)
    ya = torch.full((a["M"], a["N"]), float("nan"), dtype=torch.float16, device="cuda")
    yb = torch.full((b["M"], b["N"]), float("nan"), dtype=torch.float16, device="cuda")
    # two calls back to back on one stream: the second finds the first's scratch contents
    assert _noalloc_raw(q, a, ya) == q.QG_OK, q.raw.qg_last_error_message()
    assert _noalloc_raw(q, b, yb) == q.QG_OK, q.raw.qg_last_error_message()
    torch.cuda.synchronize()
    q.check_device_errors()
    for t, y in ((a, ya), (b, yb)):
        ref = q.gemm_w4a16(t["x"], t["qw"], t["sc"], t["ze"], 64, t["b"])              # cluster path
        ref_ws = q.gemm_w4a16(t["x"], t["qw"], t["sc"], t["ze"], 64, t["b"], workspace="auto")
        torch.cuda.synchronize()
        got = host(y).astype(np.float64)
        assert np.isfinite(got).all()
        assert rel_frobenius(got, host(ref).astype(np.float64)) <= TOL, (t["M"], t["N"], t["K"])
        # same stream-K kernel and combine order as a caller-provided workspace: identical bits
        assert torch.equal(y, ref_ws), (t["M"], t["N"], t["K"])


def test_noalloc_calls_allocate_no_device_memory():
    """After a warm-up call (which loads the kernel and looks up the array's
    address), repeated calls with caller-given outputs change neither what the
    torch allocator holds nor the device's free memory."""
    import int4_quantized_gemm_b200 as q
    t = _inputs(16, 4096, 4096, seed=24)
    y = torch.empty((16, 4096), dtype=torch.float16, device="cuda")
    ref = torch.empty_like(y)
    assert _noalloc_raw(q, t, y) == q.QG_OK, q.raw.qg_last_error_message()
    q.gemm_w4a16_noalloc(t["x"], t["qw"], t["sc"], t["ze"], 64, t["b"], out=ref)   # the Python wrapper
    torch.cuda.synchronize()
    held = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        assert _noalloc_raw(q, t, y) == q.QG_OK, q.raw.qg_last_error_message()
        q.gemm_w4a16_noalloc(t["x"], t["qw"], t["sc"], t["ze"], 64, t["b"], out=y)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == held
    assert free1 == free0
    q.check_device_errors()
    assert torch.equal(y, ref)


def test_noalloc_rejects_sizes_beyond_its_static_scratch():
    import int4_quantized_gemm_b200 as q
    t = _inputs(17, 256, 512, seed=23)
    y = torch.zeros((17, 256), dtype=torch.float16, device="cuda")
    assert _noalloc_raw(q, t, y) == q.QG_ERR_UNSUPPORTED
    assert "M=17" in q.raw.qg_last_error_message().decode()
    torch.cuda.synchronize()
    assert not y.any()   # nothing was launched
    # a rejected argument is reported before anything is enqueued or the shared array is touched
    t = _inputs(4, 256, 512, seed=25)
    y4 = torch.zeros((4, 256), dtype=torch.float16, device="cuda")
    vp = lambda a: ctypes.c_void_p(a.data_ptr())
    st = q.raw.qg_gemm_w4a16_noalloc(vp(t["x"]), t["K"], vp(t["qw"]), vp(t["sc"]), vp(t["ze"]), 63,
                                     vp(t["b"]), vp(y4), 256, 4, 256, 512,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == q.QG_ERR_UNSUPPORTED and "group 63" in q.raw.qg_last_error_message().decode()
    torch.cuda.synchronize()
    assert not y4.any()
