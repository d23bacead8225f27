"""CPU oracle for the quantized-GEMM hot path (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product (``int4_quantized_gemm_b200``) never
does, and shares no code with it: the arithmetic lives in ``qg_oracle.c``,
plain C compiled with gcc (IEEE binary32/binary64, no FMA contraction, no
fast-math), and this module only marshals numpy arrays through ctypes.

Every function names the page passage it follows in ``qg_oracle.c``.
Pins (checks against things other than the oracle itself) live in
``tests/test_oracle_pins.py``.  Functions without an independent pin: none.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qg_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-shared", "-fPIC", "-Wall", "-Wextra"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile qg_oracle.c into oracle/_build/liboracle.so (gcc)."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, vp, d = ctypes.c_int64, ctypes.c_void_p, ctypes.c_double
            sig = {
                "ref_quantize_rowwise_int8": [vp, i64, i64, i64, vp, i64, vp],
                "ref_quantize_block_asym4": [vp, i64, i64, i64, i64, vp, vp, vp, vp],
                "ref_gemm_i8_i64": [vp, i64, vp, i64, i64, i64, i64, vp],
                "ref_w8a8_epilogue_f64": [vp, vp, vp, vp, i64, i64, vp],
                "ref_w8a8_f64": [vp, i64, vp, i64, vp, vp, vp, i64, i64, i64, vp],
                "ref_w8a16_f64": [vp, i64, vp, i64, vp, vp, i64, i64, i64, vp],
                "ref_w4a16_f64": [vp, i64, vp, vp, vp, i64, vp, i64, i64, i64, vp],
                "ref_w4_dequant": [vp, vp, vp, i64, i64, i64, i64, i64],
                "ref_quantize_rowwise_asym_int8": [vp, i64, i64, i64, vp, i64, vp, vp, vp],
                "ref_w8a8_zp_f64": [vp, i64, vp, vp, vp, i64, vp, vp, vp, i64, i64, i64, vp],
                "ref_gelu_f64": [vp, i64, vp],
                "ref_quantize_block_sym4": [vp, i64, i64, i64, i64, vp, vp, vp],
                "ref_quantize_channel_sym4": [vp, i64, i64, i64, vp, vp, vp],
                "ref_w4a8_f64": [vp, i64, vp, vp, vp, vp, i64, i64, i64, vp],
                "ref_w4a16_sym_f64": [vp, i64, vp, vp, i64, vp, i64, i64, i64, vp],
                "ref_round_f16": [vp, i64, vp],
                "ref_round_bf16": [vp, i64, vp],
                "oracle_f16_decode_array": [vp, i64, vp],
                "oracle_f32_to_f16_array": [vp, i64, vp],
                "oracle_bf16_decode_array": [vp, i64, vp],
                "oracle_set_threads": [ctypes.c_int],
                "oracle_max_threads": [],
            }
            for name, args in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = None
            lib.ref_w4_dequant.restype = d
            lib.oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _f16bits(a) -> np.ndarray:
    """fp16 array (or its uint16 bit pattern) -> contiguous uint16 bits."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a)
    return np.ascontiguousarray(a, dtype=np.float16).view(np.uint16)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


# --- codecs -----------------------------------------------------------------

def f16_decode(bits: np.ndarray) -> np.ndarray:
    b = _c(bits, np.uint16).ravel()
    out = np.empty(b.size, np.float64)
    _load().oracle_f16_decode_array(_p(b), b.size, _p(out))
    return out.reshape(np.shape(bits))


def f32_to_f16(values: np.ndarray) -> np.ndarray:
    """binary32 -> binary16 bit patterns, nearest even."""
    v = _c(values, np.float32).ravel()
    out = np.empty(v.size, np.uint16)
    _load().oracle_f32_to_f16_array(_p(v), v.size, _p(out))
    return out.reshape(np.shape(values))


def bf16_decode(bits: np.ndarray) -> np.ndarray:
    b = _c(bits, np.uint16).ravel()
    out = np.empty(b.size, np.float64)
    _load().oracle_bf16_decode_array(_p(b), b.size, _p(out))
    return out.reshape(np.shape(bits))


def round_f16(y: np.ndarray) -> np.ndarray:
    """fp64 -> binary16 bit patterns (uint16), nearest even."""
    v = _c(y, np.float64).ravel()
    out = np.empty(v.size, np.uint16)
    _load().ref_round_f16(_p(v), v.size, _p(out))
    return out.reshape(np.shape(y))


def round_bf16(y: np.ndarray) -> np.ndarray:
    """fp64 -> bfloat16 bit patterns (uint16), nearest even."""
    v = _c(y, np.float64).ravel()
    out = np.empty(v.size, np.uint16)
    _load().ref_round_bf16(_p(v), v.size, _p(out))
    return out.reshape(np.shape(y))


# --- a1 / a2: quantizers ----------------------------------------------------

def quantize_rowwise_int8(x: np.ndarray):
    """Symmetric per-row int8 quantization of fp16 X [M,K] -> (q int8 [M,K], scale f32 [M])."""
    xb = _f16bits(x)
    M, K = xb.shape
    q = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    _load().ref_quantize_rowwise_int8(_p(xb), M, K, K, _p(q), K, _p(s))
    return q, s


def quantize_rowwise_asym_int8(x: np.ndarray):
    """Asymmetric per-row int8 quantization of fp16 X [R,K] ->
    (q int8 [R,K], scale f32 [R], zero f32 [R], qsum int32 [R])."""
    xb = _f16bits(x)
    M, K = xb.shape
    q = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    z = np.empty(M, np.float32)
    qs = np.empty(M, np.int32)
    _load().ref_quantize_rowwise_asym_int8(_p(xb), M, K, K, _p(q), K, _p(s), _p(z), _p(qs))
    return q, s, z, qs


def quantize_block_asym4(w: np.ndarray, group: int = 64):
    """Block-asymmetric 4-bit quantization of fp16 W [N,K] (storage of column-major [K,N]).

    Returns (qweight uint32 [N,K/8], scale fp16 [K/group,N], zero fp16 [K/group,N], q uint8 [N,K]).
    """
    wb = _f16bits(w)
    N, K = wb.shape
    assert K % group == 0 and K % 8 == 0
    qw = np.empty((N, K // 8), np.uint32)
    sc = np.empty((K // group, N), np.uint16)
    ze = np.empty((K // group, N), np.uint16)
    q = np.empty((N, K), np.uint8)
    _load().ref_quantize_block_asym4(_p(wb), N, K, K, group, _p(qw), _p(sc), _p(ze), _p(q))
    return qw, sc.view(np.float16), ze.view(np.float16), q


# --- a3 .. a6: products -------------------------------------------------------

def gemm_i8_i64(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """acc[m,n] = sum_k xq[m,k] * wq[n,k] in int64 (wq is the [N,K] storage)."""
    a = _c(xq, np.int8)
    b = _c(wq, np.int8)
    M, K = a.shape
    N = b.shape[0]
    acc = np.empty((M, N), np.int64)
    _load().ref_gemm_i8_i64(_p(a), K, _p(b), K, M, N, K, _p(acc))
    return acc


def w8a8_epilogue_f64(acc, x_scale, w_scale, bias=None) -> np.ndarray:
    acc = _c(acc, np.int64)
    M, N = acc.shape
    xs, ws = _c(x_scale, np.float32), _c(w_scale, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.float64)
    _load().ref_w8a8_epilogue_f64(_p(acc), _p(xs), _p(ws), _p(b), M, N, _p(y))
    return y


def w8a8_f64(xq, wq, x_scale, w_scale, bias=None) -> np.ndarray:
    a, b_ = _c(xq, np.int8), _c(wq, np.int8)
    M, K = a.shape
    N = b_.shape[0]
    xs, ws = _c(x_scale, np.float32), _c(w_scale, np.float32)
    bb = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.float64)
    _load().ref_w8a8_f64(_p(a), K, _p(b_), K, _p(xs), _p(ws), _p(bb), M, N, K, _p(y))
    return y


def w8a8_zp_f64(xq, x_scale, x_zero, wq, w_scale, w_zero, bias=None) -> np.ndarray:
    """Zero-point W8A8 from the definition: sum_k xs(xq - xz) * ws(wq - wz) + bias, fp64.
    x_zero / w_zero None: that operand is symmetric."""
    a, b_ = _c(xq, np.int8), _c(wq, np.int8)
    M, K = a.shape
    N = b_.shape[0]
    xs, ws = _c(x_scale, np.float32), _c(w_scale, np.float32)
    xz = None if x_zero is None else _c(x_zero, np.float32)
    wz = None if w_zero is None else _c(w_zero, np.float32)
    bb = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.float64)
    _load().ref_w8a8_zp_f64(_p(a), K, _p(xs), _p(xz), _p(b_), K, _p(ws), _p(wz), _p(bb), M, N, K, _p(y))
    return y


def quantize_block_sym4(w: np.ndarray, group: int = 64):
    """Block-wise symmetric int4 of fp16 W [N,K] -> (qweight uint32 [N,K/8], scale fp16 [K/group,N],
    q int8 [N,K]); nibbles are two's complement, nibble j of word p is k = 8p + j."""
    wb = _f16bits(w)
    N, K = wb.shape
    assert K % group == 0 and K % 8 == 0
    qw = np.empty((N, K // 8), np.uint32)
    sc = np.empty((K // group, N), np.uint16)
    q = np.empty((N, K), np.int8)
    _load().ref_quantize_block_sym4(_p(wb), N, K, K, group, _p(qw), _p(sc), _p(q))
    return qw, sc.view(np.float16), q


def quantize_channel_sym4(w: np.ndarray):
    """Per-output-column symmetric int4 of fp16 W [N,K] -> (qweight uint32 [N,K/8], scale f32 [N], q int8 [N,K])."""
    wb = _f16bits(w)
    N, K = wb.shape
    assert K % 8 == 0
    qw = np.empty((N, K // 8), np.uint32)
    sc = np.empty(N, np.float32)
    q = np.empty((N, K), np.int8)
    _load().ref_quantize_channel_sym4(_p(wb), N, K, K, _p(qw), _p(sc), _p(q))
    return qw, sc, q


def w4a8_f64(xq, qweight, x_scale, w_scale, bias=None) -> np.ndarray:
    a = _c(xq, np.int8)
    qw = _c(qweight, np.uint32)
    M, K = a.shape
    N = qw.shape[0]
    assert qw.shape[1] * 8 == K
    xs, ws = _c(x_scale, np.float32), _c(w_scale, np.float32)
    bb = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.float64)
    _load().ref_w4a8_f64(_p(a), K, _p(qw), _p(xs), _p(ws), _p(bb), M, N, K, _p(y))
    return y


def w4a16_sym_f64(x, qweight, scale, group: int = 64, bias=None) -> np.ndarray:
    xb = _f16bits(x)
    qw = _c(qweight, np.uint32)
    sc = _f16bits(scale)
    M, K = xb.shape
    N = qw.shape[0]
    assert qw.shape[1] * 8 == K and sc.shape == (K // group, N)
    bb = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.float64)
    _load().ref_w4a16_sym_f64(_p(xb), K, _p(qw), _p(sc), group, _p(bb), M, N, K, _p(y))
    return y


def gelu_f64(y: np.ndarray) -> np.ndarray:
    """gelu(y) = 0.5 y (1 + erf(y / sqrt 2)), elementwise in fp64."""
    v = _c(y, np.float64).ravel()
    out = np.empty(v.size, np.float64)
    _load().ref_gelu_f64(_p(v), v.size, _p(out))
    return out.reshape(np.shape(y))


def w8a16_f64(x, wq, w_scale, bias=None) -> np.ndarray:
    xb = _f16bits(x)
    b_ = _c(wq, np.int8)
    M, K = xb.shape
    N = b_.shape[0]
    ws = _c(w_scale, np.float32)
    bb = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.float64)
    _load().ref_w8a16_f64(_p(xb), K, _p(b_), K, _p(ws), _p(bb), M, N, K, _p(y))
    return y


def w4a16_f64(x, qweight, scale, zero, group: int = 64, bias=None) -> np.ndarray:
    xb = _f16bits(x)
    qw = _c(qweight, np.uint32)
    sc = _f16bits(scale)
    ze = _f16bits(zero)
    M, K = xb.shape
    N = qw.shape[0]
    assert qw.shape[1] * 8 == K and sc.shape == (K // group, N) == ze.shape
    bb = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.float64)
    _load().ref_w4a16_f64(_p(xb), K, _p(qw), _p(sc), _p(ze), group, _p(bb), M, N, K, _p(y))
    return y


def w4_dequant(qweight, scale, zero, group: int, k: int, n: int) -> float:
    qw = _c(qweight, np.uint32)
    sc = _f16bits(scale)
    ze = _f16bits(zero)
    N, K = qw.shape[0], qw.shape[1] * 8
    return float(_load().ref_w4_dequant(_p(qw), _p(sc), _p(ze), N, K, group, k, n))
