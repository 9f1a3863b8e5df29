"""CPU oracle for FP4 (ExMy) weight quantization and the W4A16 product.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it; the product library never does.
This module is argument marshalling over ``fp4_oracle.c`` (numpy in, numpy
out).  bf16 and fp16 tensors travel as uint16 bit patterns.

The C file states each reading of the LLM-FP4 summary page it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4_oracle.c")
_HDR = os.path.join(_HERE, "fp4_oracle.h")
_LIB = os.path.join(_HERE, "libfp4_oracle.so")

E1M2, E2M1, E3M0, AUTO = 0, 1, 2, -1
ACT_NONE, ACT_SILU, ACT_GELU, ACT_SILU_GATE = 0, 1, 2, 3
SCALE_F32, SCALE_F16 = 0, 1
GRAN_GROUP, GRAN_CHANNEL, GRAN_HEAD = 0, 1, 2
FORMAT_NAMES = ("E1M2", "E2M1", "E3M0")

_ERRORS = {1: "invalid argument", 2: "non-finite input", 3: "stored scale not finite", 4: "allocation failed"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
               "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i, f, d = ctypes.c_int, ctypes.c_float, ctypes.c_double
        sig = {
            "orc_format_bias": (i, [i]),
            "orc_code_value": (d, [i, i]),
            "orc_format_table": (None, [i, P, P]),
            "orc_bias_factor": (f, [i]),
            "orc_f32_to_bf16": (ctypes.c_uint16, [f]),
            "orc_f32_to_f16": (ctypes.c_uint16, [f]),
            "orc_f16_to_f32": (f, [ctypes.c_uint16]),
            "orc_nearest_index": (i, [d, P]),
            "orc_quantize_fixed": (i, [P, i, i, i, i, i, P, i, P, P, P]),
            "orc_quantize": (i, [P, i, i, i, i, i, P, i, P, P, P, P]),
            "orc_dequantize": (i, [P, P, i, i, i, i, i, P]),
            "orc_gemm": (i, [P, P, P, i, i, i, i, i, i, f, P]),
            "orc_gemm_sampled": (i, [P, P, P, i, i, i, i, i, i, f, i, P, P, P]),
            "orc_preshift_calibrate": (i, [P, i, i, P, P]),
            "orc_preshift_apply": (i, [P, i, i, P, f, P]),
            "orc_block_count": (i, [i, i, i, i, i]),
            "orc_quantize_blocks": (i, [P, i, i, i, i, i, i, i, P, P, i, P, P, P, P]),
            "orc_act_quantize": (i, [P, i, i, P, f, i, i, P, P]),
            "orc_gemm_w4a4": (i, [P, i, f, P, P, i, i, i, i, i, i, P]),
            "orc_gemm_w4a4_sampled": (i, [P, i, f, P, P, i, i, i, i, i, i, i, P, P, P]),
            "orc_num_threads": (i, []),
            "orc_set_num_threads": (None, [i]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc):
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, "error %d" % rc))


def _sdt(scale_dtype):
    return SCALE_F16 if scale_dtype in ("f16", "fp16", SCALE_F16, np.float16) else SCALE_F32


def num_threads() -> int:
    return _L().orc_num_threads()


def set_num_threads(n: int) -> None:
    _L().orc_set_num_threads(int(n))


def format_bias(fmt: int) -> int:
    return _L().orc_format_bias(fmt)


def code_value(fmt: int, code: int) -> float:
    return _L().orc_code_value(fmt, code)


def format_table(fmt: int):
    mags = np.zeros(8, np.float64)
    q = np.zeros(1, np.float64)
    _L().orc_format_table(fmt, _p(mags), _p(q))
    return mags, float(q[0])


def bias_factor(j: int) -> np.float32:
    return np.float32(_L().orc_bias_factor(j))


def f32_to_bf16(x) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32).ravel()
    fn = _L().orc_f32_to_bf16
    return np.array([fn(float(v)) for v in x], np.uint16)


def f32_to_f16(x) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32).ravel()
    fn = _L().orc_f32_to_f16
    return np.array([fn(float(v)) for v in x], np.uint16)


def nearest_index(a: float, fmt: int) -> int:
    mags, _ = format_table(fmt)
    return _L().orc_nearest_index(float(a), _p(mags))


def _shift_arr(shift, K):
    if shift is None:
        return None
    s = np.ascontiguousarray(shift, np.int8)
    assert s.shape == (K,)
    return s


def quantize_fixed(W, group, fmt, j=0, shift=None, scale_dtype="f16", want_codes=True):
    """Quantize with a forced (format, bias index) choice.

    Returns (packed uint8 [N][K/2], scales [N][K/group] as float16/float32
    array, sse float)."""
    W = np.ascontiguousarray(W, np.float32)
    N, K = W.shape
    sdt = _sdt(scale_dtype)
    packed = np.zeros((N, K // 2), np.uint8) if want_codes else None
    scales = (np.zeros((N, K // group), np.float16 if sdt else np.float32) if want_codes else None)
    sse = np.zeros(1, np.float64)
    s = _shift_arr(shift, K)
    _check(_L().orc_quantize_fixed(_p(W), N, K, group, fmt, j, _p(s), sdt, _p(packed), _p(scales), _p(sse)))
    return packed, scales, float(sse[0])


def quantize(W, group=128, fmt=E2M1, bias_search=False, shift=None, scale_dtype="f16"):
    """Full quantizer: optional format/bias search, then codes, scales, pack.

    Returns dict(packed, scales, choice=(fmt, j), sse=float64[24] with NaN
    for candidates that were not evaluated)."""
    W = np.ascontiguousarray(W, np.float32)
    N, K = W.shape
    sdt = _sdt(scale_dtype)
    packed = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // group), np.float16 if sdt else np.float32)
    choice = np.zeros(2, np.int32)
    sse = np.zeros(24, np.float64)
    s = _shift_arr(shift, K)
    _check(_L().orc_quantize(_p(W), N, K, group, fmt, 1 if bias_search else 0, _p(s), sdt,
                             _p(packed), _p(scales), _p(choice), _p(sse)))
    return {"packed": packed, "scales": scales, "choice": (int(choice[0]), int(choice[1])), "sse": sse}


def dequantize(packed, scales, fmt, group):
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales)
    N, Kh = packed.shape
    K = 2 * Kh
    sdt = SCALE_F16 if scales.dtype == np.float16 else SCALE_F32
    out = np.zeros((N, K), np.float64)
    _check(_L().orc_dequantize(_p(packed), _p(scales), sdt, fmt, N, K, group, _p(out)))
    return out


def gemm(X_bf16, packed, scales, fmt, group, rho=1.0):
    """Y = rho * X . dequant(W)^T in fp64.  X_bf16: uint16 [M][K]."""
    X = np.ascontiguousarray(X_bf16, np.uint16)
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales)
    M, K = X.shape
    N = packed.shape[0]
    assert packed.shape[1] * 2 == K
    sdt = SCALE_F16 if scales.dtype == np.float16 else SCALE_F32
    Y = np.zeros((M, N), np.float64)
    _check(_L().orc_gemm(_p(X), _p(packed), _p(scales), sdt, fmt, M, N, K, group, float(rho), _p(Y)))
    return Y


def activation(Y, act):
    """The output activation of the fused epilogue, elementwise in fp64 on
    the finished product Y (HiFloat4 page, section 5 "性能优化实战案例": the
    fused Quant-GeLU-Dequant operator).  SiLU y / (1 + e^-y); GeLU in its
    erf form y * (1 + erf(y / sqrt 2)) / 2 (Python's math.erf, double)."""
    import math
    Y = np.asarray(Y, np.float64)
    if act == ACT_NONE:
        return Y.copy()
    if act == ACT_SILU:
        with np.errstate(over="ignore"):
            return Y / (1.0 + np.exp(-Y))
    if act == ACT_GELU:
        erf = np.vectorize(math.erf, otypes=[np.float64])
        return 0.5 * Y * (1.0 + erf(Y / math.sqrt(2.0)))
    raise OracleError("unknown activation %r" % (act,))


def silu_gate(Y):
    """Gate/up pairs of the fused MLP epilogue: column i of the result is
    silu(Y[:, 2i]) * Y[:, 2i+1] (gate and up rows interleaved), in fp64."""
    Y = np.asarray(Y, np.float64)
    g, u = Y[:, 0::2], Y[:, 1::2]
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u


def gemm_act(X_bf16, packed, scales, fmt, group, act, rho=1.0):
    """act(rho * X . dequant(W)^T) in fp64: gemm() followed by activation(),
    or by silu_gate() for ACT_SILU_GATE."""
    Y = gemm(X_bf16, packed, scales, fmt, group, rho)
    return silu_gate(Y) if act == ACT_SILU_GATE else activation(Y, act)


def gemm_sampled(X_bf16, packed, scales, fmt, group, ms, ns, rho=1.0):
    X = np.ascontiguousarray(X_bf16, np.uint16)
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales)
    M, K = X.shape
    N = packed.shape[0]
    ms = np.ascontiguousarray(ms, np.int32)
    ns = np.ascontiguousarray(ns, np.int32)
    out = np.zeros(len(ms), np.float64)
    sdt = SCALE_F16 if scales.dtype == np.float16 else SCALE_F32
    _check(_L().orc_gemm_sampled(_p(X), _p(packed), _p(scales), sdt, fmt, M, N, K, group, float(rho),
                                 len(ms), _p(ms), _p(ns), _p(out)))
    return out


def preshift_calibrate(X_bf16):
    X = np.ascontiguousarray(X_bf16, np.uint16)
    M, K = X.shape
    shift = np.zeros(K, np.int8)
    rho = np.zeros(1, np.float32)
    _check(_L().orc_preshift_calibrate(_p(X), M, K, _p(shift), _p(rho)))
    return shift, np.float32(rho[0])


def preshift_apply(X_bf16, shift, rho):
    X = np.ascontiguousarray(X_bf16, np.uint16)
    M, K = X.shape
    shift = np.ascontiguousarray(shift, np.int8)
    Xt = np.zeros((M, K), np.uint16)
    _check(_L().orc_preshift_apply(_p(X), M, K, _p(shift), float(rho), _p(Xt)))
    return Xt


def block_count(N, K, group, gran, heads=0):
    return _L().orc_block_count(N, K, group, gran, heads)


def quantize_blocks(W, group, gran, fmt, j=0, heads=0, shift=None, scale_dtype="f16", jforce=None):
    """Quantize with the scale's absmax taken over a block (reading R11):
    GRAN_GROUP (group elements of a row), GRAN_CHANNEL (a row) or GRAN_HEAD
    (N/heads rows).  j = None searches the bias index per block; jforce
    (int8 [blocks]) imposes one per block.  Scales come out in the
    [N][K/group] layout, a block's scale in every slot it covers.

    Returns dict(packed, scales, jmap int8 [blocks], sse float)."""
    W = np.ascontiguousarray(W, np.float32)
    N, K = W.shape
    sdt = _sdt(scale_dtype)
    nb = block_count(N, K, group, gran, heads)
    packed = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // group), np.float16 if sdt else np.float32)
    jmap = np.zeros(max(nb, 0), np.int8)
    jf = None if jforce is None else np.ascontiguousarray(jforce, np.int8)
    if jf is not None:
        assert jf.shape == (nb,)
    sse = np.zeros(1, np.float64)
    s = _shift_arr(shift, K)
    _check(_L().orc_quantize_blocks(_p(W), N, K, group, gran, heads, fmt, -1 if j is None else j, _p(jf), _p(s),
                                    sdt, _p(packed), _p(scales), _p(jmap), _p(sse)))
    return {"packed": packed, "scales": scales, "jmap": jmap, "sse": float(sse[0])}


def act_quantize(X_bf16, rho, fmt=E2M1, j=0, shift=None):
    """4-bit activation codes with the pre-shifted bias (reading R10).

    Returns (packed uint8 [M][K/2], s_a float32): X' = X * 2^-shift coded
    against the per-tensor scale s_a = fl32(fl32(rho * c_j) / Qmax)."""
    X = np.ascontiguousarray(X_bf16, np.uint16)
    M, K = X.shape
    packed = np.zeros((M, K // 2), np.uint8)
    s_a = np.zeros(1, np.float32)
    s = _shift_arr(shift, K)
    _check(_L().orc_act_quantize(_p(X), M, K, _p(s), float(rho), fmt, j, _p(packed), _p(s_a)))
    return packed, np.float32(s_a[0])


def gemm_w4a4(apacked, afmt, s_a, packed, scales, fmt, group):
    """Y = s_a * v_a(A) . dequant(W)^T in fp64 (reading R10)."""
    apacked = np.ascontiguousarray(apacked, np.uint8)
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales)
    M, K = apacked.shape[0], apacked.shape[1] * 2
    N = packed.shape[0]
    assert packed.shape[1] * 2 == K
    sdt = SCALE_F16 if scales.dtype == np.float16 else SCALE_F32
    Y = np.zeros((M, N), np.float64)
    _check(_L().orc_gemm_w4a4(_p(apacked), afmt, float(s_a), _p(packed), _p(scales), sdt, fmt, M, N, K, group,
                              _p(Y)))
    return Y


def gemm_w4a4_sampled(apacked, afmt, s_a, packed, scales, fmt, group, ms, ns):
    apacked = np.ascontiguousarray(apacked, np.uint8)
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales)
    M, K = apacked.shape[0], apacked.shape[1] * 2
    N = packed.shape[0]
    ms = np.ascontiguousarray(ms, np.int32)
    ns = np.ascontiguousarray(ns, np.int32)
    out = np.zeros(len(ms), np.float64)
    sdt = SCALE_F16 if scales.dtype == np.float16 else SCALE_F32
    _check(_L().orc_gemm_w4a4_sampled(_p(apacked), afmt, float(s_a), _p(packed), _p(scales), sdt, fmt, M, N, K,
                                      group, len(ms), _p(ms), _p(ns), _p(out)))
    return out
