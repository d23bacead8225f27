"""int4_quantized_gemm_b200 -- Python binding of libqg.so (the C ABI in include/qg.h).

Argument marshalling only: every step of the computation runs in the library's
sm_100a CUDA kernels.  PyTorch supplies device memory (tensor ``data_ptr()``),
the current CUDA stream, and allocates outputs.  There is no CPU fallback: if
``libqg.so`` is missing or no sm_100 device is present, calls raise.

Functions (same names as the C entry points, minus the ``qg_`` prefix):
    quantize_rowwise_int8(x)                    -> (xq int8 [M,K], x_scale f32 [M])
    quantize_block_asym4(w, group=64)           -> (qweight int32 [N,K/8], scale f16 [K/64,N], zero f16 [K/64,N])
    gemm_w8a8(xq, wq, x_scale, w_scale, bias=None, out_dtype=torch.float16) -> y [M,N]
    gemm_w8a16(x, wq, w_scale, bias=None)       -> y fp16 [M,N]
    gemm_w4a16(x, qweight, scale, zero, group=64, bias=None) -> y fp16 [M,N]
Launch plans bind one call's arguments once for loops over preallocated buffers:
    plan_quantize_rowwise_int8 / plan_gemm_w8a8 / plan_gemm_w8a16 / plan_gemm_w4a16
    (same arguments as the calls)           -> Plan; plan.launch(stream=None), plan.out
The GEMMs take workspace=None (the default: decode shapes run the cluster
split-K kernels, no scratch memory), "auto" (a per-stream workspace kept by this
module; decode shapes then run the stream-K kernels) or a caller's zero-filled
CUDA uint8 tensor.
Weights are passed as their [N, K] storage (row n = output column n of the
column-major [K, N] weight).  ``raw`` exposes the ctypes library itself.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqg.so")

QG_OK, QG_ERR_INVALID_ARG, QG_ERR_ALIGNMENT, QG_ERR_UNSUPPORTED, QG_ERR_CUDA, QG_ERR_TIMEOUT, \
    QG_ERR_NO_DEVICE, QG_ERR_DEBUG_CHECK = range(8)
DEBUG_LIB_PATH = os.path.join(_PKG, "libqg_debug.so")
QG_F32, QG_F16, QG_BF16, QG_I32 = range(4)
QG_DEBUG_WEIGHT_ONLY, QG_DEBUG_STREAM_K = 1, 2
QG_FLAG_STATIC_WEIGHTS = 1

_DTYPE_CODE = {torch.float32: QG_F32, torch.float16: QG_F16, torch.bfloat16: QG_BF16, torch.int32: QG_I32}

# C signatures of every exported symbol of include/qg.h.
_i64, _vp, _int, _sz = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_pp = ctypes.POINTER(ctypes.c_void_p)
SIGNATURES = {
    "qg_status_string": ([_int], ctypes.c_char_p),
    "qg_last_error_message": ([], ctypes.c_char_p),
    "qg_version": ([], _int),
    "qg_gemm_workspace_size": ([_i64, _i64, _i64], _sz),
    "qg_check_device_errors": ([_vp], _int),
    "qg_quantize_rowwise_int8": ([_vp, _i64, _vp, _i64, _vp, _i64, _i64, _vp], _int),
    "qg_quantize_block_asym4": ([_vp, _i64, _vp, _vp, _vp, _i64, _i64, _i64, _vp], _int),
    "qg_gemm_w8a8": ([_vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64, _i64, _vp, _sz, _vp], _int),
    "qg_gemm_w8a16": ([_vp, _i64, _vp, _i64, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _sz, _vp], _int),
    "qg_gemm_w4a16": ([_vp, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _sz, _vp], _int),
    "qg_quantize_block_sym4": ([_vp, _i64, _vp, _vp, _i64, _i64, _i64, _vp], _int),
    "qg_quantize_channel_sym4": ([_vp, _i64, _vp, _vp, _i64, _i64, _vp], _int),
    "qg_gemm_w4a8": ([_vp, _i64, _vp, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64, _i64, _vp], _int),
    "qg_gemm_w4a16_sym": ([_vp, _i64, _vp, _vp, _i64, _vp, _vp, _i64, _i64, _i64, _i64, _vp], _int),
    "qg_gemm_w8a8_act": ([_vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64, _i64, _int, _vp], _int),
    "qg_gemm_w8a16_act": ([_vp, _i64, _vp, _i64, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _int, _vp], _int),
    "qg_gemm_w4a16_act": ([_vp, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _i64, _i64, _i64, _i64, _int, _vp], _int),
    "qg_quantize_rowwise_asym_int8": ([_vp, _i64, _vp, _i64, _vp, _vp, _vp, _i64, _i64, _vp], _int),
    "qg_gemm_w8a8_zp": ([_vp, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64,
                         _i64, _vp], _int),
    "qg_quantize_gemm_w8a8": ([_vp, _i64, _vp, _i64, _vp, _vp, _vp, _int, _i64, _vp, _i64, _vp, _i64, _i64, _i64, _vp], _int),
    "qg_gemm_w4a16_noalloc": ([_vp, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _i64, _i64, _i64, _i64, _vp], _int),
    "qg_set_tuning": ([ctypes.c_char_p, _int], _int),
    "qg_debug_checks": ([], _int),
    "qg_debug_inject_timeout": ([_int, _int], _int),
    "qg_gemm_w8a8_ex": ([_vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64, _i64, _vp, _sz,
                         ctypes.c_uint, _vp], _int),
    "qg_gemm_w8a16_ex": ([_vp, _i64, _vp, _i64, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _sz, ctypes.c_uint,
                          _vp], _int),
    "qg_gemm_w4a16_ex": ([_vp, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _sz,
                          ctypes.c_uint, _vp], _int),
    "qg_plan_quantize_rowwise_int8": ([_pp, _vp, _i64, _vp, _i64, _vp, _i64, _i64], _int),
    "qg_plan_gemm_w8a8": ([_pp, _vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64, _i64, _vp, _sz,
                           ctypes.c_uint], _int),
    "qg_plan_gemm_w8a16": ([_pp, _vp, _i64, _vp, _i64, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _sz,
                            ctypes.c_uint], _int),
    "qg_plan_gemm_w4a16": ([_pp, _vp, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _sz,
                            ctypes.c_uint], _int),
    "qg_plan_launch": ([_vp, _vp], _int),
    "qg_plan_destroy": ([_vp], None),
}


class QGError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = raw.qg_last_error_message().decode(errors="replace") if raw is not None else ""
        name = raw.qg_status_string(status).decode() if raw is not None else str(status)
        super().__init__(f"{where}: {name}: {msg}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python int4_quantized_gemm_b200/build.py` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


raw = _load()


def _check(status: int, where: str) -> None:
    if status != QG_OK:
        raise QGError(status, where)


_current_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream() -> int:
    """The current CUDA stream of the current device as a raw handle.  Building a
    torch.cuda.Stream object costs ~3 us per call; the raw lookup is used when
    this torch provides it."""
    if _current_raw_stream is not None:
        return _current_raw_stream(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: torch.Tensor | None):
    # a plain int: ctypes turns it into the c_void_p argument itself
    return None if t is None else t.data_ptr()


def _rowmajor(t: torch.Tensor, name: str, dtype: torch.dtype) -> int:
    """Check a 2-D CUDA tensor with unit inner stride; return its leading dimension.
    (Shape and strides are read once each: this runs several times per call.)"""
    if t.dtype is not dtype or not t.is_cuda:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    shape = t.shape
    st = t.stride()
    if len(shape) != 2 or (shape[1] > 1 and st[1] != 1):
        raise ValueError(f"{name} must be 2-D with unit stride along its last dimension")
    return st[0] if shape[0] > 1 else max(st[0], shape[1])


def _vec(t: torch.Tensor | None, name: str, dtype: torch.dtype, n: int):
    if t is None:
        return None
    if t.dtype is not dtype or not t.is_cuda or t.numel() != n or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} vector of {n} elements")
    return t


_WORKSPACES: dict = {}


def workspace_for(M: int, N: int, K: int, device) -> torch.Tensor | None:
    """The GEMM workspace of the current stream on `device` (zero-filled once and
    reused; the kernels leave it zeroed), grown when a larger problem needs
    more.  None when the shape needs none.  Create it outside CUDA-graph
    capture (an eager call of the same shape does) so captured calls keep a
    fixed address."""
    need = int(raw.qg_gemm_workspace_size(M, N, K))
    if need == 0:
        return None
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    t = _WORKSPACES.get(key)
    if t is None or t.numel() < need:
        t = torch.zeros(need, dtype=torch.uint8, device=device)
        _WORKSPACES[key] = t
    return t


def _ws_args(workspace, M, N, K, device):
    """(workspace tensor or None, c_void_p, bytes) for the C call."""
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a CUDA uint8 tensor")
        workspace = workspace_for(M, N, K, device)
    if workspace is None:
        return None, None, 0
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA uint8 tensor")
    return workspace, ctypes.c_void_p(workspace.data_ptr()), workspace.numel()


def debug_inject_timeout(family: int, wait_limit_us: int) -> None:
    """Arm the next launch of a kernel family to time out on purpose
    (qg_debug_inject_timeout; tests of the timeout path only)."""
    _check(raw.qg_debug_inject_timeout(int(family), int(wait_limit_us)), "qg_debug_inject_timeout")


def set_tuning(name: str, value: int) -> None:
    """Set a kernel-choice switch of the library (qg_set_tuning; e.g.
    "QG_W8A8_PAIR" = 0 runs prefill W8A8 on one-SM tiles).  Results do not
    depend on any switch."""
    _check(raw.qg_set_tuning(name.encode(), int(value)), "qg_set_tuning")


def check_device_errors() -> None:
    """Synchronize the current stream and raise if a kernel recorded a timeout."""
    _check(raw.qg_check_device_errors(_stream()), "qg_check_device_errors")


def _quantize_rowwise_args(x, out, scale_out):
    """(xq, x_scale, the C arguments but the stream) of qg_quantize_rowwise_int8."""
    ldx = _rowmajor(x, "x", torch.float16)
    M, K = x.shape
    if out is None:
        # rows padded to a multiple of 16 bytes (ABI alignment); a [M, K] view is returned
        out = torch.empty((M, (K + 15) // 16 * 16), dtype=torch.int8, device=x.device)[:, :K]
    xq = out
    xs = scale_out if scale_out is not None else torch.empty(M, dtype=torch.float32, device=x.device)
    ldq = _rowmajor(xq, "out", torch.int8)
    _vec(xs, "scale_out", torch.float32, M)
    return xq, xs, (_ptr(x), ldx, _ptr(xq), ldq, _ptr(xs), M, K)


def quantize_rowwise_int8(x: torch.Tensor, out: torch.Tensor | None = None,
                          scale_out: torch.Tensor | None = None):
    xq, xs, a = _quantize_rowwise_args(x, out, scale_out)
    _check(raw.qg_quantize_rowwise_int8(*a, _stream()), "qg_quantize_rowwise_int8")
    return xq, xs


def quantize_block_asym4(w: torch.Tensor, group: int = 64):
    ldw = _rowmajor(w, "w", torch.float16)
    N, K = w.shape
    qweight = torch.empty((N, K // 8), dtype=torch.int32, device=w.device)
    scale = torch.empty((K // group, N), dtype=torch.float16, device=w.device)
    zero = torch.empty((K // group, N), dtype=torch.float16, device=w.device)
    _check(raw.qg_quantize_block_asym4(_ptr(w), ldw, _ptr(qweight), _ptr(scale), _ptr(zero), N, K,
                                       group, _stream()), "qg_quantize_block_asym4")
    return qweight, scale, zero


def _w8a8_args(xq, wq, x_scale, w_scale, bias, out_dtype, out, workspace):
    """(y, workspace tensor or None, the C arguments but flags and stream) of qg_gemm_w8a8_ex."""
    ldx = _rowmajor(xq, "xq", torch.int8)
    ldw = _rowmajor(wq, "wq", torch.int8)
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"wq must be [N, K] = [*, {K}], got {tuple(wq.shape)}")
    y = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=xq.device)
    ldy = _rowmajor(y, "out", out_dtype)
    _vec(x_scale, "x_scale", torch.float32, M)
    _vec(w_scale, "w_scale", torch.float32, N)
    _vec(bias, "bias", torch.float32, N)
    wst, wsp, wsn = _ws_args(workspace, M, N, K, xq.device)
    return y, wst, (_ptr(xq), ldx, _ptr(wq), ldw, _ptr(x_scale), _ptr(w_scale), _ptr(bias), _ptr(y),
                    _DTYPE_CODE[out_dtype], ldy, M, N, K, wsp, wsn)


def gemm_w8a8(xq: torch.Tensor, wq: torch.Tensor, x_scale: torch.Tensor | None,
              w_scale: torch.Tensor | None, bias: torch.Tensor | None = None,
              out_dtype: torch.dtype = torch.float16, out: torch.Tensor | None = None,
              workspace=None, static_weights: bool = False) -> torch.Tensor:
    """static_weights=True calls qg_gemm_w8a8_ex with QG_FLAG_STATIC_WEIGHTS (the
    caller guarantees no kernel still in flight writes wq)."""
    y, _, a = _w8a8_args(xq, wq, x_scale, w_scale, bias, out_dtype, out, workspace)
    if static_weights:
        _check(raw.qg_gemm_w8a8_ex(*a, QG_FLAG_STATIC_WEIGHTS, _stream()), "qg_gemm_w8a8_ex")
    else:
        _check(raw.qg_gemm_w8a8(*a, _stream()), "qg_gemm_w8a8")
    return y


def quantize_block_sym4(w: torch.Tensor, group: int = 64):
    """Block-wise symmetric int4 of fp16 W [N, K] -> (qweight int32 [N, K/8], scale fp16 [K/group, N])."""
    ldw = _rowmajor(w, "w", torch.float16)
    N, K = w.shape
    qweight = torch.empty((N, K // 8), dtype=torch.int32, device=w.device)
    scale = torch.empty((K // group, N), dtype=torch.float16, device=w.device)
    _check(raw.qg_quantize_block_sym4(_ptr(w), ldw, _ptr(qweight), _ptr(scale), N, K, group, _stream()),
           "qg_quantize_block_sym4")
    return qweight, scale


def quantize_channel_sym4(w: torch.Tensor):
    """Per-column symmetric int4 of fp16 W [N, K] -> (qweight int32 [N, K/8], scale f32 [N])."""
    ldw = _rowmajor(w, "w", torch.float16)
    N, K = w.shape
    qweight = torch.empty((N, K // 8), dtype=torch.int32, device=w.device)
    scale = torch.empty(N, dtype=torch.float32, device=w.device)
    _check(raw.qg_quantize_channel_sym4(_ptr(w), ldw, _ptr(qweight), _ptr(scale), N, K, _stream()),
           "qg_quantize_channel_sym4")
    return qweight, scale


def gemm_w4a8(xq: torch.Tensor, qweight: torch.Tensor, x_scale: torch.Tensor | None,
              w_scale: torch.Tensor | None, bias: torch.Tensor | None = None,
              out_dtype: torch.dtype = torch.float16, out: torch.Tensor | None = None) -> torch.Tensor:
    """int8 X x per-column symmetric int4 W on the int8 tensor cores (qg_gemm_w4a8)."""
    ldx = _rowmajor(xq, "xq", torch.int8)
    M, K = xq.shape
    N = qweight.shape[0]
    if qweight.dtype != torch.int32 or tuple(qweight.shape) != (N, K // 8) or not qweight.is_contiguous():
        raise ValueError(f"qweight must be contiguous int32 [N, K/8] = [{N}, {K // 8}]")
    y = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=xq.device)
    ldy = _rowmajor(y, "out", out_dtype)
    _vec(x_scale, "x_scale", torch.float32, M)
    _vec(w_scale, "w_scale", torch.float32, N)
    _vec(bias, "bias", torch.float32, N)
    _check(raw.qg_gemm_w4a8(_ptr(xq), ldx, _ptr(qweight), _ptr(x_scale), _ptr(w_scale), _ptr(bias), _ptr(y),
                            _DTYPE_CODE[out_dtype], ldy, M, N, K, _stream()), "qg_gemm_w4a8")
    return y


def gemm_w4a16_sym(x: torch.Tensor, qweight: torch.Tensor, scale: torch.Tensor, group: int = 64,
                   bias: torch.Tensor | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """W4A16 with symmetric group-int4 weights, no zero points (qg_gemm_w4a16_sym)."""
    ldx = _rowmajor(x, "x", torch.float16)
    M, K = x.shape
    N = qweight.shape[0]
    if qweight.dtype != torch.int32 or tuple(qweight.shape) != (N, K // 8) or not qweight.is_contiguous():
        raise ValueError(f"qweight must be contiguous int32 [N, K/8] = [{N}, {K // 8}]")
    if scale.dtype != torch.float16 or tuple(scale.shape) != (K // group, N) or not scale.is_contiguous():
        raise ValueError(f"scale must be contiguous fp16 [K/group, N] = [{K // group}, {N}]")
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    ldy = _rowmajor(y, "out", torch.float16)
    _vec(bias, "bias", torch.float32, N)
    _check(raw.qg_gemm_w4a16_sym(_ptr(x), ldx, _ptr(qweight), _ptr(scale), group, _ptr(bias), _ptr(y), ldy,
                                 M, N, K, _stream()), "qg_gemm_w4a16_sym")
    return y


_ACTIVATIONS = {"none": 0, "gelu": 1}


def _act_code(activation: str) -> int:
    if activation not in _ACTIVATIONS:
        raise ValueError(f"activation must be one of {sorted(_ACTIVATIONS)}, got {activation!r}")
    return _ACTIVATIONS[activation]


def gemm_w8a8_act(xq: torch.Tensor, wq: torch.Tensor, x_scale: torch.Tensor, w_scale: torch.Tensor,
                  bias: torch.Tensor | None = None, activation: str = "gelu",
                  out_dtype: torch.dtype = torch.float16, out: torch.Tensor | None = None) -> torch.Tensor:
    """act(W8A8) with the activation fused into the epilogue (qg_gemm_w8a8_act)."""
    ldx = _rowmajor(xq, "xq", torch.int8)
    ldw = _rowmajor(wq, "wq", torch.int8)
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"wq must be [N, K] = [*, {K}], got {tuple(wq.shape)}")
    y = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=xq.device)
    ldy = _rowmajor(y, "out", out_dtype)
    _vec(x_scale, "x_scale", torch.float32, M)
    _vec(w_scale, "w_scale", torch.float32, N)
    _vec(bias, "bias", torch.float32, N)
    _check(raw.qg_gemm_w8a8_act(_ptr(xq), ldx, _ptr(wq), ldw, _ptr(x_scale), _ptr(w_scale), _ptr(bias),
                                _ptr(y), _DTYPE_CODE[out_dtype], ldy, M, N, K, _act_code(activation),
                                _stream()), "qg_gemm_w8a8_act")
    return y


def gemm_w8a16_act(x: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                   bias: torch.Tensor | None = None, activation: str = "gelu",
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """act(W8A16) with the activation fused into the epilogue (qg_gemm_w8a16_act)."""
    ldx = _rowmajor(x, "x", torch.float16)
    ldw = _rowmajor(wq, "wq", torch.int8)
    M, K = x.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"wq must be [N, K] = [*, {K}], got {tuple(wq.shape)}")
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    ldy = _rowmajor(y, "out", torch.float16)
    _vec(w_scale, "w_scale", torch.float32, N)
    _vec(bias, "bias", torch.float32, N)
    _check(raw.qg_gemm_w8a16_act(_ptr(x), ldx, _ptr(wq), ldw, _ptr(w_scale), _ptr(bias), _ptr(y), ldy,
                                 M, N, K, _act_code(activation), _stream()), "qg_gemm_w8a16_act")
    return y


def gemm_w4a16_act(x: torch.Tensor, qweight: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
                   group: int = 64, bias: torch.Tensor | None = None, activation: str = "gelu",
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """act(W4A16) with the activation fused into the epilogue (qg_gemm_w4a16_act)."""
    ldx = _rowmajor(x, "x", torch.float16)
    M, K = x.shape
    N = qweight.shape[0]
    if qweight.dtype != torch.int32 or tuple(qweight.shape) != (N, K // 8) or not qweight.is_contiguous():
        raise ValueError(f"qweight must be contiguous int32 [N, K/8] = [{N}, {K // 8}]")
    for name, t in (("scale", scale), ("zero", zero)):
        if t.dtype != torch.float16 or tuple(t.shape) != (K // group, N) or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous fp16 [K/group, N] = [{K // group}, {N}]")
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    ldy = _rowmajor(y, "out", torch.float16)
    _vec(bias, "bias", torch.float32, N)
    _check(raw.qg_gemm_w4a16_act(_ptr(x), ldx, _ptr(qweight), _ptr(scale), _ptr(zero), group, _ptr(bias),
                                 _ptr(y), ldy, M, N, K, _act_code(activation), _stream()), "qg_gemm_w4a16_act")
    return y


def quantize_rowwise_asym_int8(x: torch.Tensor, out: torch.Tensor | None = None):
    """Asymmetric per-row int8 quantization of fp16 X [M, K] -> (q, scale, zero, qsum)."""
    ldx = _rowmajor(x, "x", torch.float16)
    M, K = x.shape
    if out is None:
        ldq = (K + 15) // 16 * 16
        out = torch.empty((M, ldq), dtype=torch.int8, device=x.device)[:, :K]
    ldq_ = _rowmajor(out, "out", torch.int8)
    scale = torch.empty(M, dtype=torch.float32, device=x.device)
    zero = torch.empty(M, dtype=torch.float32, device=x.device)
    qsum = torch.empty(M, dtype=torch.int32, device=x.device)
    _check(raw.qg_quantize_rowwise_asym_int8(_ptr(x), ldx, _ptr(out), ldq_, _ptr(scale), _ptr(zero),
                                             _ptr(qsum), M, K, _stream()), "qg_quantize_rowwise_asym_int8")
    return out, scale, zero, qsum


def gemm_w8a8_zp(xq: torch.Tensor, x_scale, x_zero, x_qsum, wq: torch.Tensor, w_scale, w_zero, w_qsum,
                 bias: torch.Tensor | None = None, out_dtype: torch.dtype = torch.float16,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """W8A8 with optional per-row zero points on either operand (see qg_gemm_w8a8_zp)."""
    ldx = _rowmajor(xq, "xq", torch.int8)
    ldw = _rowmajor(wq, "wq", torch.int8)
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"wq must be [N, K] = [*, {K}], got {tuple(wq.shape)}")
    y = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=xq.device)
    ldy = _rowmajor(y, "out", out_dtype)
    for t, name, n, dt in ((x_scale, "x_scale", M, torch.float32), (x_zero, "x_zero", M, torch.float32),
                           (x_qsum, "x_qsum", M, torch.int32), (w_scale, "w_scale", N, torch.float32),
                           (w_zero, "w_zero", N, torch.float32), (w_qsum, "w_qsum", N, torch.int32),
                           (bias, "bias", N, torch.float32)):
        _vec(t, name, dt, n)
    _check(raw.qg_gemm_w8a8_zp(_ptr(xq), ldx, _ptr(x_scale), _ptr(x_zero), _ptr(x_qsum), _ptr(wq), ldw,
                               _ptr(w_scale), _ptr(w_zero), _ptr(w_qsum), _ptr(bias), _ptr(y),
                               _DTYPE_CODE[out_dtype], ldy, M, N, K, _stream()), "qg_gemm_w8a8_zp")
    return y


def quantize_gemm_w8a8(x: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor | None,
                       bias: torch.Tensor | None = None, out_dtype: torch.dtype = torch.float16,
                       out: torch.Tensor | None = None, xq_out: torch.Tensor | None = None,
                       x_scale_out: torch.Tensor | None = None) -> torch.Tensor:
    """Per-row int8 quantization of fp16 X fused with the W8A8 GEMM (M <= 64):
    bit-identical to quantize_rowwise_int8 followed by gemm_w8a8."""
    ldx = _rowmajor(x, "x", torch.float16)
    ldw = _rowmajor(wq, "wq", torch.int8)
    M, K = x.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"wq must be [N, K] = [*, {K}], got {tuple(wq.shape)}")
    y = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=x.device)
    ldy = _rowmajor(y, "out", out_dtype)
    _vec(w_scale, "w_scale", torch.float32, N)
    _vec(bias, "bias", torch.float32, N)
    ldq = 0
    if xq_out is not None:
        ldq = _rowmajor(xq_out, "xq_out", torch.int8)
        if tuple(xq_out.shape) != (M, K):
            raise ValueError(f"xq_out must be [M, K] = [{M}, {K}]")
    _vec(x_scale_out, "x_scale_out", torch.float32, M)
    _check(raw.qg_quantize_gemm_w8a8(_ptr(x), ldx, _ptr(wq), ldw, _ptr(w_scale), _ptr(bias), _ptr(y),
                                     _DTYPE_CODE[out_dtype], ldy, _ptr(xq_out), ldq, _ptr(x_scale_out),
                                     M, N, K, _stream()), "qg_quantize_gemm_w8a8")
    return y


def _w8a16_args(x, wq, w_scale, bias, out, workspace):
    """(y, workspace tensor or None, the C arguments but flags and stream) of qg_gemm_w8a16_ex."""
    ldx = _rowmajor(x, "x", torch.float16)
    ldw = _rowmajor(wq, "wq", torch.int8)
    M, K = x.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"wq must be [N, K] = [*, {K}], got {tuple(wq.shape)}")
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    ldy = _rowmajor(y, "out", torch.float16)
    _vec(w_scale, "w_scale", torch.float32, N)
    _vec(bias, "bias", torch.float32, N)
    wst, wsp, wsn = _ws_args(workspace, M, N, K, x.device)
    return y, wst, (_ptr(x), ldx, _ptr(wq), ldw, _ptr(w_scale), _ptr(bias), _ptr(y), ldy, M, N, K, wsp, wsn)


def gemm_w8a16(x: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
               bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
               workspace=None, static_weights: bool = False) -> torch.Tensor:
    """static_weights=True calls qg_gemm_w8a16_ex with QG_FLAG_STATIC_WEIGHTS."""
    y, _, a = _w8a16_args(x, wq, w_scale, bias, out, workspace)
    if static_weights:
        _check(raw.qg_gemm_w8a16_ex(*a, QG_FLAG_STATIC_WEIGHTS, _stream()), "qg_gemm_w8a16_ex")
    else:
        _check(raw.qg_gemm_w8a16(*a, _stream()), "qg_gemm_w8a16")
    return y


def _w4a16_args(x, qweight, scale, zero, group, bias, out, workspace):
    """(y, workspace tensor or None, the C arguments but flags and stream) of qg_gemm_w4a16_ex."""
    ldx = _rowmajor(x, "x", torch.float16)
    M, K = x.shape
    N = qweight.shape[0]
    if qweight.dtype != torch.int32 or tuple(qweight.shape) != (N, K // 8) or not qweight.is_contiguous():
        raise ValueError(f"qweight must be contiguous int32 [N, K/8] = [{N}, {K // 8}]")
    for name, t in (("scale", scale), ("zero", zero)):
        if t.dtype != torch.float16 or tuple(t.shape) != (K // group, N) or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous fp16 [K/group, N] = [{K // group}, {N}]")
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    ldy = _rowmajor(y, "out", torch.float16)
    _vec(bias, "bias", torch.float32, N)
    wst, wsp, wsn = _ws_args(workspace, M, N, K, x.device)
    return y, wst, (_ptr(x), ldx, _ptr(qweight), _ptr(scale), _ptr(zero), group, _ptr(bias), _ptr(y), ldy,
                    M, N, K, wsp, wsn)


def gemm_w4a16(x: torch.Tensor, qweight: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
               group: int = 64, bias: torch.Tensor | None = None,
               out: torch.Tensor | None = None, workspace=None, static_weights: bool = False) -> torch.Tensor:
    """static_weights=True calls qg_gemm_w4a16_ex with QG_FLAG_STATIC_WEIGHTS."""
    y, _, a = _w4a16_args(x, qweight, scale, zero, group, bias, out, workspace)
    if static_weights:
        _check(raw.qg_gemm_w4a16_ex(*a, QG_FLAG_STATIC_WEIGHTS, _stream()), "qg_gemm_w4a16_ex")
    else:
        _check(raw.qg_gemm_w4a16(*a, _stream()), "qg_gemm_w4a16")
    return y


def gemm_w4a16_noalloc(x: torch.Tensor, qweight: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
                       group: int = 64, bias: torch.Tensor | None = None,
                       out: torch.Tensor | None = None) -> torch.Tensor:
    """W4A16 for M <= 16 whose scratch is the library's static device array.

    For callers that may not allocate device memory: pass `out`, and the call
    itself allocates nothing (without `out` this wrapper allocates the result).
    Calls that may overlap on the GPU share the scratch and race."""
    ldx = _rowmajor(x, "x", torch.float16)
    M, K = x.shape
    N = qweight.shape[0]
    if qweight.dtype != torch.int32 or tuple(qweight.shape) != (N, K // 8) or not qweight.is_contiguous():
        raise ValueError(f"qweight must be contiguous int32 [N, K/8] = [{N}, {K // 8}]")
    for name, t in (("scale", scale), ("zero", zero)):
        if t.dtype != torch.float16 or tuple(t.shape) != (K // group, N) or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous fp16 [K/group, N] = [{K // group}, {N}]")
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    ldy = _rowmajor(y, "out", torch.float16)
    _vec(bias, "bias", torch.float32, N)
    _check(raw.qg_gemm_w4a16_noalloc(_ptr(x), ldx, _ptr(qweight), _ptr(scale), _ptr(zero), group,
                                     _ptr(bias), _ptr(y), ldy, M, N, K, _stream()), "qg_gemm_w4a16_noalloc")
    return y


# ---------------------------------------------------------------------------
# Launch plans (qg_plan_*): one call's arguments bound once, launched many times
# ---------------------------------------------------------------------------
class Plan:
    """A bound call: the arguments of one quantize / GEMM call (tensors, shapes,
    flags) checked and marshalled once, for issuing the same call on the same
    buffers many times, e.g. once per decode step with new activations written
    into the bound input tensors in place.  ``out`` is the bound output (the
    result tensor; (xq, x_scale) for the quantizer).  The plan keeps every bound
    tensor alive; the C side re-checks the arguments at every launch.  Dropping
    a plan releases those references at once, so, as for any tensor used on a
    stream other than the one it was allocated on, keep the tensors (or the
    plan) until launches issued on other streams have finished.  close() is
    for one thread; launch() may be called from several."""

    __slots__ = ("_h", "_keep", "out")

    def __init__(self, handle: int, keep: tuple, out):
        self._h, self._keep, self.out = handle, keep, out

    def launch(self, stream=None) -> None:
        """Issue the call on `stream` (a torch.cuda.Stream or a raw handle;
        default: the current stream)."""
        s = _stream() if stream is None else getattr(stream, "cuda_stream", stream)
        st = raw.qg_plan_launch(self._h, s)
        if st != QG_OK:
            raise QGError(st, "qg_plan_launch")

    __call__ = launch

    def close(self) -> None:
        """Free the C plan (launches already issued are unaffected)."""
        h, self._h = self._h, None
        if h and raw is not None:
            raw.qg_plan_destroy(h)

    def __del__(self):
        self.close()


def _new_plan(fn, args, keep, out, where: str) -> Plan:
    h = ctypes.c_void_p()
    _check(fn(ctypes.byref(h), *args), where)
    return Plan(h.value, keep, out)


def _plan_workspace(workspace):
    if isinstance(workspace, str):
        raise ValueError("a plan takes workspace=None or a CUDA uint8 tensor (kept by the plan), not 'auto'")
    return workspace


def plan_quantize_rowwise_int8(x: torch.Tensor, out: torch.Tensor | None = None,
                               scale_out: torch.Tensor | None = None) -> Plan:
    """qg_plan_quantize_rowwise_int8: quantize_rowwise_int8 bound to x and its outputs."""
    xq, xs, a = _quantize_rowwise_args(x, out, scale_out)
    return _new_plan(raw.qg_plan_quantize_rowwise_int8, a, (x, xq, xs), (xq, xs), "qg_plan_quantize_rowwise_int8")


def plan_gemm_w8a8(xq: torch.Tensor, wq: torch.Tensor, x_scale: torch.Tensor | None,
                   w_scale: torch.Tensor | None, bias: torch.Tensor | None = None,
                   out_dtype: torch.dtype = torch.float16, out: torch.Tensor | None = None,
                   workspace=None, static_weights: bool = False) -> Plan:
    """qg_plan_gemm_w8a8: gemm_w8a8 bound to its operands and output."""
    y, wst, a = _w8a8_args(xq, wq, x_scale, w_scale, bias, out_dtype, out, _plan_workspace(workspace))
    flags = QG_FLAG_STATIC_WEIGHTS if static_weights else 0
    return _new_plan(raw.qg_plan_gemm_w8a8, a + (flags,), (xq, wq, x_scale, w_scale, bias, y, wst), y,
                     "qg_plan_gemm_w8a8")


def plan_gemm_w8a16(x: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                    bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                    workspace=None, static_weights: bool = False) -> Plan:
    """qg_plan_gemm_w8a16: gemm_w8a16 bound to its operands and output."""
    y, wst, a = _w8a16_args(x, wq, w_scale, bias, out, _plan_workspace(workspace))
    flags = QG_FLAG_STATIC_WEIGHTS if static_weights else 0
    return _new_plan(raw.qg_plan_gemm_w8a16, a + (flags,), (x, wq, w_scale, bias, y, wst), y, "qg_plan_gemm_w8a16")


def plan_gemm_w4a16(x: torch.Tensor, qweight: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
                    group: int = 64, bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                    workspace=None, static_weights: bool = False) -> Plan:
    """qg_plan_gemm_w4a16: gemm_w4a16 bound to its operands and output."""
    y, wst, a = _w4a16_args(x, qweight, scale, zero, group, bias, out, _plan_workspace(workspace))
    flags = QG_FLAG_STATIC_WEIGHTS if static_weights else 0
    return _new_plan(raw.qg_plan_gemm_w4a16, a + (flags,), (x, qweight, scale, zero, bias, y, wst), y,
                     "qg_plan_gemm_w4a16")
