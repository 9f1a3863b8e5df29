"""ctypes binding of libfp4w4a16.so (C interface in include/fp4w4a16.h).

Argument marshalling only: every step of quantization and the GEMM runs in
the CUDA library.  PyTorch provides device memory (output and workspace
allocation) and the current CUDA stream.  There is no fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp4w4a16.so")

E1M2, E2M1, E3M0, AUTO = 0, 1, 2, -1
SCALE_F32, SCALE_F16 = 0, 1
ENGINE_AUTO, ENGINE_DECODE, ENGINE_TENSOR = 0, 1, 2
ACT_NONE, ACT_SILU, ACT_GELU, ACT_SILU_GATE = 0, 1, 2, 3
GRAN_GROUP, GRAN_CHANNEL, GRAN_HEAD = 0, 1, 2
DEV_NONFINITE_INPUT, DEV_SCALE_OVERFLOW, DEV_WAIT_TIMEOUT, DEV_LAYOUT = 1, 2, 4, 8

STATUS = {0: "FP4_OK", 1: "FP4_ERR_INVALID_ARG", 2: "FP4_ERR_UNSUPPORTED_SHAPE", 3: "FP4_ERR_MISALIGNED",
          4: "FP4_ERR_WORKSPACE", 5: "FP4_ERR_CUDA", 6: "FP4_ERR_DEVICE_STATUS"}

EXPORTS = ("fp4_abi_version", "fp4_status_string", "fp4_quantize_workspace_size", "fp4_quantize",
           "fp4_dequantize", "fp4_preshift_workspace_size", "fp4_preshift_calibrate", "fp4_preshift_apply",
           "fp4_gemm_workspace_size", "fp4_gemm", "fp4_gemm_ex", "fp4_gemm_act", "fp4_get_device_status",
           "fp4_set_wait_timeout_us", "fp4_selftest_bounded_wait", "fp4_preshift_calibrate_noalloc",
           "fp4_gemm_engine_for", "fp4_quantize_blocks_workspace_size", "fp4_quantize_blocks",
           "fp4_act_quantize", "fp4_gemm_w4a4_workspace_size", "fp4_gemm_w4a4")


class Fp4Error(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (where, STATUS.get(code, "?"), code))


_lib = None
_lock = threading.Lock()


def lib():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError("libfp4w4a16.so is not built (run python -m w4a16_gemm_fp4_b200.build); "
                                   "there is no CPU fallback")
            L = ctypes.CDLL(LIB_PATH)
            P, i, sz, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong
            sigs = {
                "fp4_abi_version": (i, []),
                "fp4_status_string": (ctypes.c_char_p, [i]),
                "fp4_quantize_workspace_size": (sz, [i, i, i, i, i]),
                "fp4_quantize": (i, [P, i, i, i, i, i, P, i, P, P, P, P, P, sz, P]),
                "fp4_dequantize": (i, [P, P, i, i, i, i, i, P, P]),
                "fp4_preshift_workspace_size": (sz, [i, i]),
                "fp4_preshift_calibrate": (i, [P, i, i, P, P, P, sz, P]),
                "fp4_preshift_apply": (i, [P, i, i, P, P, P, P]),
                "fp4_gemm_workspace_size": (sz, [i, i, i]),
                "fp4_gemm": (i, [P, P, P, i, i, i, i, i, i, P, P, P, sz, P]),
                "fp4_gemm_ex": (i, [P, P, P, i, i, i, i, i, i, P, P, P, sz, i, i, P]),
                "fp4_gemm_act": (i, [P, P, P, i, i, i, i, i, i, P, i, P, P, sz, i, i, P]),
                "fp4_get_device_status": (i, [ctypes.POINTER(ctypes.c_int32), i, P]),
                "fp4_set_wait_timeout_us": (None, [ll]),
                "fp4_selftest_bounded_wait": (i, [ll, P]),
                "fp4_preshift_calibrate_noalloc": (i, [P, i, i, P, P, P]),
                "fp4_gemm_engine_for": (i, [i, i, i, i]),
                "fp4_quantize_blocks_workspace_size": (sz, [i, i, i, i, i, i]),
                "fp4_quantize_blocks": (i, [P, i, i, i, i, i, i, i, P, i, P, P, P, P, sz, P]),
                "fp4_act_quantize": (i, [P, i, i, P, P, i, i, P, P, P]),
                "fp4_gemm_w4a4_workspace_size": (sz, [i, i, i]),
                "fp4_gemm_w4a4": (i, [P, i, P, P, P, i, i, i, i, i, i, i, P, P, sz, P]),
            }
            for name, (res, args) in sigs.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(code, where):
    if code != 0:
        raise Fp4Error(code, where)


def _sdt(scale_dtype):
    if scale_dtype in ("f16", "fp16", torch.float16, SCALE_F16):
        return SCALE_F16
    if scale_dtype in ("f32", "fp32", torch.float32, SCALE_F32):
        return SCALE_F32
    raise ValueError("scale dtype must be f16 or f32")


def _bits(t):
    """bf16 tensors travel as their 16-bit patterns."""
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


# ------------------------------------------------------------------ workspaces

class Workspace:
    """A zero-filled device buffer reused across calls (grown on demand)."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = None

    def get(self, nbytes):
        if nbytes == 0:
            return None, 0
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=self.device)
        return self.buf, self.buf.numel()


_ws = {}


def _workspace(device, kind="scratch"):
    """Per-device grow-only buffers, one per kind: "gemm" holds fp4_gemm's
    f16 activations, "scratch" serves quantize and calibrate.  Calls on one
    stream reuse them in order; calls on concurrent streams need their own
    (pass ``workspace=``)."""
    key = (device.type, device.index, kind)
    if key not in _ws:
        _ws[key] = Workspace(device)
    return _ws[key]


# ------------------------------------------------------------------- quantize

def quantize(W, group=128, fmt=E2M1, bias_search=False, chan_shift=None, scale_dtype="f16", want_sse=False,
             stream=None):
    """FP4 quantize a [N][K] fp32 CUDA tensor.

    Returns dict(packed uint8 [N][K/2], scales [N][K/group] fp16/fp32,
    choice int32[2] (device), sse float64[24] (device) or None)."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2
    N, K = W.shape
    sdt = _sdt(scale_dtype)
    dev = W.device
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // group), dtype=torch.float16 if sdt else torch.float32, device=dev)
    choice = torch.empty(2, dtype=torch.int32, device=dev)
    sse = torch.empty(24, dtype=torch.float64, device=dev) if want_sse else None
    L = lib()
    need = L.fp4_quantize_workspace_size(N, K, group, fmt, 1 if bias_search else 0)
    ws, wsb = _workspace(dev).get(need)
    if chan_shift is not None:
        assert chan_shift.dtype == torch.int8 and chan_shift.numel() == K and chan_shift.is_cuda
    _check(L.fp4_quantize(_ptr(W), N, K, group, fmt, 1 if bias_search else 0, _ptr(chan_shift), sdt, _ptr(packed),
                          _ptr(scales), _ptr(choice), _ptr(sse), _ptr(ws), wsb, _stream(stream)), "fp4_quantize")
    return {"packed": packed, "scales": scales, "choice": choice, "sse": sse}


def quantize_into(W, packed, scales, choice, group=128, fmt=E2M1, bias_search=False, chan_shift=None,
                  sse=None, workspace=None, stream=None):
    """In-place variant over preallocated outputs (no allocation)."""
    N, K = W.shape
    sdt = SCALE_F16 if scales.dtype == torch.float16 else SCALE_F32
    L = lib()
    if workspace is None:
        need = L.fp4_quantize_workspace_size(N, K, group, fmt, 1 if bias_search else 0)
        workspace, wsb = _workspace(W.device).get(need)
    else:
        wsb = workspace.numel() * workspace.element_size()
    _check(L.fp4_quantize(_ptr(W), N, K, group, fmt, 1 if bias_search else 0, _ptr(chan_shift), sdt, _ptr(packed),
                          _ptr(scales), _ptr(choice), _ptr(sse), _ptr(workspace), wsb, _stream(stream)),
           "fp4_quantize")


def block_count(N, K, group, gran, heads=0):
    if gran == GRAN_GROUP:
        return N * (K // group)
    return N if gran == GRAN_CHANNEL else heads


def quantize_blocks(W, group=128, gran=GRAN_CHANNEL, heads=0, fmt=E2M1, bias_index=0, chan_shift=None,
                    scale_dtype="f16", want_jmap=True, stream=None):
    """FP4 quantize with the scale's absmax over a group, a row (output
    channel) or N/heads rows (attention head); bias_index -1 searches the
    bias per block.  Returns dict(packed, scales [N][K/group], jmap int8
    [blocks] or None), all on the device."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2
    N, K = W.shape
    sdt = _sdt(scale_dtype)
    dev = W.device
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // group), dtype=torch.float16 if sdt else torch.float32, device=dev)
    jmap = torch.empty(max(block_count(N, K, group, gran, heads), 1), dtype=torch.int8, device=dev) \
        if want_jmap else None
    L = lib()
    need = L.fp4_quantize_blocks_workspace_size(N, K, group, gran, heads, bias_index)
    ws, wsb = _workspace(dev).get(need)
    _check(L.fp4_quantize_blocks(_ptr(W), N, K, group, gran, heads, fmt, bias_index, _ptr(chan_shift), sdt,
                                 _ptr(packed), _ptr(scales), _ptr(jmap), _ptr(ws), wsb, _stream(stream)),
           "fp4_quantize_blocks")
    return {"packed": packed, "scales": scales, "jmap": jmap}


def dequantize(packed, scales, fmt, group=128, stream=None):
    N, Kh = packed.shape
    K = 2 * Kh
    sdt = SCALE_F16 if scales.dtype == torch.float16 else SCALE_F32
    out = torch.empty((N, K), dtype=torch.float32, device=packed.device)
    _check(lib().fp4_dequantize(_ptr(packed), _ptr(scales), sdt, fmt, N, K, group, _ptr(out), _stream(stream)),
           "fp4_dequantize")
    return out


# ------------------------------------------------------------------ pre-shift

def preshift_calibrate(X, stream=None):
    """X: [M][K] bf16 CUDA tensor -> (shift int8 [K], rho float32 [1]), on device."""
    M, K = X.shape
    shift = torch.empty(K, dtype=torch.int8, device=X.device)
    rho = torch.empty(1, dtype=torch.float32, device=X.device)
    L = lib()
    ws, wsb = _workspace(X.device).get(L.fp4_preshift_workspace_size(M, K))
    _check(L.fp4_preshift_calibrate(_ptr(_bits(X)), M, K, _ptr(shift), _ptr(rho), _ptr(ws), wsb, _stream(stream)),
           "fp4_preshift_calibrate")
    return shift, rho


def preshift_apply(X, shift, rho, out=None, stream=None):
    M, K = X.shape
    if out is None:
        out = torch.empty_like(X)
    _check(lib().fp4_preshift_apply(_ptr(_bits(X)), M, K, _ptr(shift), _ptr(rho), _ptr(_bits(out)),
                                    _stream(stream)), "fp4_preshift_apply")
    return out


# ----------------------------------------------------------------------- GEMM

def gemm_workspace_size(M, N, K):
    return lib().fp4_gemm_workspace_size(M, N, K)


def gemm_engine_for(M, N, K, group=128):
    """Engine the automatic choice runs for this shape (ENGINE_DECODE or ENGINE_TENSOR)."""
    return lib().fp4_gemm_engine_for(M, N, K, group)


def gemm(X, packed, scales, fmt=E2M1, group=128, x_scale=None, out=None, engine=ENGINE_AUTO, splits=0,
         workspace=None, stream=None, act=ACT_NONE):
    """Y = bf16(act(x_scale * X . dequant(W)^T)).  X: [M][K] bf16 CUDA tensor.

    ``workspace`` defaults to a per-device zero-filled buffer of
    fp4_gemm_workspace_size bytes (tile counters, partial tiles, prepared
    activations); a smaller one makes the automatic choice take the tensor
    engine's bf16 path.  ``engine``/``splits`` force an engine or a split
    count (0: automatic).  ``act``: ACT_NONE, ACT_SILU or ACT_GELU, applied
    in the epilogue, or ACT_SILU_GATE: rows 2i / 2i+1 of the weights are the
    gate / up rows of output column i, and Y is [M][N/2]."""
    M, K = X.shape
    N = packed.shape[0]
    assert packed.shape[1] * 2 == K
    sdt = SCALE_F16 if scales.dtype == torch.float16 else SCALE_F32
    if out is None:
        out = torch.empty((M, N // 2 if act == ACT_SILU_GATE else N), dtype=torch.bfloat16, device=X.device)
    L = lib()
    if workspace is None:
        need = L.fp4_gemm_workspace_size(M, N, K)
        ws, wsb = _workspace(X.device, "gemm").get(need)
    else:
        ws, wsb = workspace, workspace.numel() * workspace.element_size()
    _check(L.fp4_gemm_act(_ptr(_bits(X)), _ptr(packed), _ptr(scales), sdt, fmt, M, N, K, group, _ptr(x_scale),
                          act, _ptr(_bits(out)), _ptr(ws), wsb, engine, splits, _stream(stream)), "fp4_gemm")
    return out


# ---------------------------------------------------------- 4-bit activations

def act_quantize(X, rho, fmt=E2M1, j=0, shift=None, out=None, a_scale=None, stream=None):
    """4-bit activation codes of X [M][K] bf16 against the per-tensor scale
    s_a = fl32(fl32(rho * c_j) / Qmax) after the per-channel shift.
    Returns (packed uint8 [M][K/2], a_scale float32 [1]) on the device."""
    M, K = X.shape
    if out is None:
        out = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device)
    if a_scale is None:
        a_scale = torch.empty(1, dtype=torch.float32, device=X.device)
    _check(lib().fp4_act_quantize(_ptr(_bits(X)), M, K, _ptr(shift), _ptr(rho), fmt, j, _ptr(out), _ptr(a_scale),
                                  _stream(stream)), "fp4_act_quantize")
    return out, a_scale


def gemm_w4a4_workspace_size(M, N, K):
    return lib().fp4_gemm_w4a4_workspace_size(M, N, K)


def gemm_w4a4(apacked, a_scale, packed, scales, afmt=E2M1, fmt=E2M1, group=128, act=ACT_NONE, out=None,
              workspace=None, stream=None):
    """Y = bf16(act(s_a * v_a(A) . dequant(W)^T)) from 4-bit activation codes."""
    M, K = apacked.shape[0], apacked.shape[1] * 2
    N = packed.shape[0]
    assert packed.shape[1] * 2 == K
    sdt = SCALE_F16 if scales.dtype == torch.float16 else SCALE_F32
    if out is None:
        out = torch.empty((M, N // 2 if act == ACT_SILU_GATE else N), dtype=torch.bfloat16, device=apacked.device)
    L = lib()
    if workspace is None:
        ws, wsb = _workspace(apacked.device, "w4a4").get(L.fp4_gemm_w4a4_workspace_size(M, N, K))
    else:
        ws, wsb = workspace, workspace.numel() * workspace.element_size()
    _check(L.fp4_gemm_w4a4(_ptr(apacked), afmt, _ptr(a_scale), _ptr(packed), _ptr(scales), sdt, fmt, M, N, K, group,
                           act, _ptr(_bits(out)), _ptr(ws), wsb, _stream(stream)), "fp4_gemm_w4a4")
    return out


# --------------------------------------------------------------------- status

def device_status(clear=True, stream=None):
    v = ctypes.c_int32(0)
    code = lib().fp4_get_device_status(ctypes.byref(v), 1 if clear else 0, _stream(stream))
    if code not in (0, 6):
        raise Fp4Error(code, "fp4_get_device_status")
    return v.value


def set_wait_timeout_us(us):
    lib().fp4_set_wait_timeout_us(int(us))


def selftest_bounded_wait(timeout_us, stream=None):
    _check(lib().fp4_selftest_bounded_wait(int(timeout_us), _stream(stream)), "fp4_selftest_bounded_wait")
