"""The device-side timeout path, exercised on purpose and without a fault.

Every mbarrier wait in the kernels is bounded; when one expires the kernel
records QG_ERR_TIMEOUT in its status word, waits (bounded) for the copies it
issued, frees its tensor memory and returns.  qg_debug_inject_timeout arms one
launch to withhold the copy of its first CTA's first K block (so the waits on it
can never complete) and to give up after a few milliseconds.  These tests check
that the host then sees QG_ERR_TIMEOUT, and that the same stream and context
keep working: the next launch is correct.  ("INT4/FP16混合精度GEMM" §7.1: the
checks to make when a kernel misbehaves; nothing here traps or faults.)
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import assert_wonly_elementwise, dev, host, rel_frobenius, requires_cuda, w4_dequant, w8_dequant

pytestmark = [pytest.mark.gpu, requires_cuda]
LIMIT_US = 3000


def qg():
    import int4_quantized_gemm_b200 as q
    return q


def _expect_timeout(q):
    with pytest.raises(q.QGError) as e:
        q.check_device_errors()
    assert e.value.status == q.QG_ERR_TIMEOUT, str(e.value)


@pytest.mark.parametrize("form", ["w8a16", "w4a16"])
def test_weight_only_kernel_times_out_cleanly_and_the_next_launch_is_correct(form):
    q = qg()
    M, N, K = 16, 128, 128      # one CTA: one weight tile, one K block
    x = W.activations(M, K, seed=51)
    w = W.weights(N, K, seed=51, per_column_factor=False)
    if form == "w8a16":
        wq, ws = oracle.quantize_rowwise_int8(w)
        args = (dev(x), dev(wq), dev(ws))
        call, y64, wdeq = q.gemm_w8a16, oracle.w8a16_f64(x, wq, ws, None), w8_dequant(wq, ws)
    else:
        qw, sc, ze, _ = oracle.quantize_block_asym4(w, 64)
        args = (dev(x), dev(qw.view(np.int32)), dev(sc), dev(ze))
        call, y64, wdeq = q.gemm_w4a16, oracle.w4a16_f64(x, qw, sc, ze, 64, None), w4_dequant(qw, sc, ze)
    q.check_device_errors()                                  # nothing pending
    q.debug_inject_timeout(q.QG_DEBUG_WEIGHT_ONLY, LIMIT_US)
    call(*args)
    _expect_timeout(q)
    q.check_device_errors()                                  # read and cleared
    y = call(*args)                                          # same stream, same context
    q.check_device_errors()
    assert rel_frobenius(host(y).astype(np.float64), y64) <= 2e-3
    assert_wonly_elementwise(y, x, wdeq, y64, None, int4=(form == "w4a16"), what=f"{form} after a timeout")


def test_stream_k_timeout_through_the_allocation_free_entry_point():
    """The stream-K kernel behind qg_gemm_w4a16_noalloc: a launch that times
    out leaves tile counters set in the static scratch; the next call clears
    them first, so it matches, bit for bit, the same kernel run on a fresh
    caller workspace."""
    q = qg()
    M, N, K = 16, 4096, 4096
    x = W.activations(M, K, seed=52)
    w = W.weights(N, K, seed=52, per_column_factor=False)
    qw, sc, ze, _ = oracle.quantize_block_asym4(w, 64)
    t = dict(x=dev(x), qw=dev(qw.view(np.int32)), sc=dev(sc), ze=dev(ze))
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    vp = lambda a: ctypes.c_void_p(a.data_ptr())

    def noalloc():
        return q.raw.qg_gemm_w4a16_noalloc(vp(t["x"]), K, vp(t["qw"]), vp(t["sc"]), vp(t["ze"]), 64, None,
                                           vp(y), N, M, N, K,
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))

    q.check_device_errors()
    q.debug_inject_timeout(q.QG_DEBUG_STREAM_K, LIMIT_US)
    assert noalloc() == q.QG_OK, q.raw.qg_last_error_message()
    _expect_timeout(q)
    assert noalloc() == q.QG_OK, q.raw.qg_last_error_message()
    ref = q.gemm_w4a16(t["x"], t["qw"], t["sc"], t["ze"], 64, None,
                       workspace=torch.zeros(q.raw.qg_gemm_workspace_size(M, N, K), dtype=torch.uint8,
                                             device="cuda"))
    torch.cuda.synchronize()
    q.check_device_errors()
    assert torch.equal(y, ref)
    y64 = oracle.w4a16_f64(x, qw, sc, ze, 64, None)
    assert_wonly_elementwise(y, x, w4_dequant(qw, sc, ze), y64, None, int4=True, what="stream-K after a timeout")
