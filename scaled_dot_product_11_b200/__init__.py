"""B200-native fused scaled-dot-product attention forward.

Python binding of ``libsdpa_b200.so`` (C ABI in ``include/sdpa.h``).  The
functions with the C names take raw device pointers and sizes and only
marshal arguments; :func:`attention` and :func:`attention_fp8` add the torch
conveniences a user wants (output allocation with torch, the current stream,
error translation).  Every step of the computation runs in the library's
CUDA kernels; there is no fallback, and importing this package fails loudly
when the library has not been built.
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "SDPA_BF16", "SDPA_FP16", "SDPA_OK", "SDPA_ERR_INVALID_ARG", "SDPA_ERR_UNSUPPORTED",
    "SDPA_ERR_CUDA", "SDPA_ERR_DEVICE_TIMEOUT", "SDPA_ERR_DEVICE_LAYOUT", "SDPA_ERR_SCRATCH_LIMIT",
    "SDPA_BWD_NOALLOC_MAX_ROWS", "sdpa_bwd_noalloc", "SdpaError", "LIB_PATH",
    "SDPA_NO_MASK", "SDPA_CAUSAL", "SDPA_CAUSAL_BOTTOM_RIGHT",
    "sdpa_fwd", "sdpa_fwd_strided", "sdpa_fwd_fp8", "sdpa_bwd", "attention_backward", "sdpa_strerror", "sdpa_device_status",
    "sdpa_launches_per_call", "attention", "attention_fp8", "sdpa_selftest_wait",
    "sdpa_selftest_exp2", "sdpa_selftest_fastdiv", "sdpa_bwd_fp8", "sdpa_bwd_fp8_workspace_bytes",
    "attention_backward_fp8",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsdpa_b200.so")

SDPA_BF16, SDPA_FP16 = 0, 1
(SDPA_OK, SDPA_ERR_INVALID_ARG, SDPA_ERR_UNSUPPORTED, SDPA_ERR_CUDA, SDPA_ERR_DEVICE_TIMEOUT,
 SDPA_ERR_DEVICE_LAYOUT, SDPA_ERR_SCRATCH_LIMIT) = range(7)
SDPA_BWD_NOALLOC_MAX_ROWS = 1 << 21    # B*Hq*Sq limit of sdpa_bwd_noalloc


class SdpaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        super().__init__("%s%s (status %d)" % (what + ": " if what else "",
                                                sdpa_strerror(self.status), self.status))


from . import build as _build  # noqa: E402  (mtime checks; compiles nothing by itself)

# A library missing or older than its sources (a new entry point, say) is
# compiled first, when nvcc is here, so that what loads matches the header.
if _build.needs_build() and _build.nvcc_available():
    _build.build()
if not os.path.exists(LIB_PATH):
    raise ImportError("libsdpa_b200.so is not built at %s; run "
                      "`python -m scaled_dot_product_11_b200.build` (nvcc, sm_100a)" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_lib.sdpa_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp]
_lib.sdpa_fwd.restype = _i
_ll3 = ctypes.c_longlong * 3
_lib.sdpa_fwd_strided.argtypes = ([_vp] * 5 + [_i] * 6 + [ctypes.POINTER(ctypes.c_longlong)] * 4
                                  + [_f, _i, _i, _vp])
_lib.sdpa_fwd_strided.restype = _i
_lib.sdpa_bwd.argtypes = [_vp] * 10 + [_i] * 6 + [_f, _i, _i, _vp]
_lib.sdpa_bwd.restype = _i
_lib.sdpa_bwd_noalloc.argtypes = [_vp] * 9 + [_i] * 6 + [_f, _i, _i, _vp]
_lib.sdpa_bwd_noalloc.restype = _i
_lib.sdpa_fwd_fp8.argtypes = [_vp, _vp, _vp, _f, _f, _f, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]
_lib.sdpa_fwd_fp8.restype = _i
_lib.sdpa_strerror.argtypes = [_i]
_lib.sdpa_strerror.restype = ctypes.c_char_p
_lib.sdpa_device_status.argtypes = [ctypes.POINTER(_i), ctypes.POINTER(_i), _i]
_lib.sdpa_device_status.restype = _i
_lib.sdpa_launches_per_call.argtypes = []
_lib.sdpa_launches_per_call.restype = _i
_lib.sdpa_bwd_fp8_workspace_bytes.argtypes = [_i] * 6
_lib.sdpa_bwd_fp8_workspace_bytes.restype = ctypes.c_size_t
_lib.sdpa_bwd_fp8.argtypes = [_vp] * 6 + [_f] * 4 + [_vp] * 4 + [ctypes.c_size_t] + [_i] * 6 + [_f, _i, _vp]
_lib.sdpa_bwd_fp8.restype = _i
_lib.sdpa_selftest_wait.argtypes = [ctypes.c_uint, _vp, _vp]
_lib.sdpa_selftest_wait.restype = _i
_lib.sdpa_selftest_exp2.argtypes = [_vp, _vp, _vp, _i, _vp]
_lib.sdpa_selftest_fastdiv.argtypes = [_vp, _vp, _i, _vp]
_lib.sdpa_selftest_fastdiv.restype = _i
_lib.sdpa_selftest_exp2.restype = _i


# ---- the C entry points, same names, raw arguments ------------------------

def sdpa_fwd(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal, dtype, stream) -> int:
    """Raw call: pointers are ints (device addresses, lse may be 0/None),
    stream an int cudaStream_t (0 = default stream).  Returns the status."""
    return int(_lib.sdpa_fwd(q, k, v, o, lse or None, B, Hq, Hkv, Sq, Sk, d, float(scale),
                             int(causal), int(dtype), stream or None))


def sdpa_fwd_strided(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, q_strides, k_strides, v_strides,
                     o_strides, scale, causal, dtype, stream) -> int:
    """Raw call with element strides (batch, head, row) per tensor, each a
    sequence of three ints."""
    st = [_ll3(*[int(x) for x in t]) for t in (q_strides, k_strides, v_strides, o_strides)]
    return int(_lib.sdpa_fwd_strided(q, k, v, o, lse or None, B, Hq, Hkv, Sq, Sk, d, *st,
                                     float(scale), int(causal), int(dtype), stream or None))


def sdpa_fwd_fp8(q8, k8, v8, descale_q, descale_k, descale_v, o, lse, B, Hq, Hkv, Sq, Sk, d,
                 scale, causal, stream) -> int:
    return int(_lib.sdpa_fwd_fp8(q8, k8, v8, float(descale_q), float(descale_k), float(descale_v),
                                 o, lse or None, B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal),
                                 stream or None))


def sdpa_bwd(q, k, v, o, dout, lse, dq, dk, dv, delta, B, Hq, Hkv, Sq, Sk, d, scale, causal,
             dtype, stream) -> int:
    """Raw backward call: device addresses as ints (delta: a [B,Hq,Sq] float32
    workspace), stream an int."""
    return int(_lib.sdpa_bwd(q, k, v, o, dout, lse, dq, dk, dv, delta, B, Hq, Hkv, Sq, Sk, d,
                             float(scale), int(causal), int(dtype), stream or None))


def sdpa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Sq, Sk, d, scale, causal,
                     dtype, stream) -> int:
    """Raw call of the backward that allocates nothing (its workspace is a
    static device array, B*Hq*Sq <= SDPA_BWD_NOALLOC_MAX_ROWS), for callers
    that cannot allocate device memory.  Device addresses as ints, stream an
    int; calls on one device must not overlap on the GPU."""
    return int(_lib.sdpa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Sq, Sk, d,
                                     float(scale), int(causal), int(dtype), stream or None))


def sdpa_bwd_fp8_workspace_bytes(B, Hq, Hkv, Sq, Sk, d) -> int:
    """Bytes of device workspace sdpa_bwd_fp8 needs (0 for invalid sizes)."""
    return int(_lib.sdpa_bwd_fp8_workspace_bytes(B, Hq, Hkv, Sq, Sk, d))


def sdpa_bwd_fp8(q8, k8, v8, o, dout8, lse, descale_q, descale_k, descale_v, descale_do,
                 dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, Sq, Sk, d, scale, causal,
                 stream) -> int:
    """Raw FP8 backward call: device addresses as ints (E4M3 q8/k8/v8, bf16 o,
    E5M2 dout8, fp32 lse; bf16 dq/dk/dv; a 256-byte aligned workspace)."""
    return int(_lib.sdpa_bwd_fp8(q8, k8, v8, o, dout8, lse, float(descale_q), float(descale_k),
                                 float(descale_v), float(descale_do), dq, dk, dv, workspace,
                                 int(workspace_bytes), B, Hq, Hkv, Sq, Sk, d, float(scale),
                                 int(causal), stream or None))


def sdpa_strerror(status: int) -> str:
    return _lib.sdpa_strerror(int(status)).decode()


def sdpa_device_status(clear: bool = True):
    """(status, detail) of the current device; synchronises the device."""
    st, dt = _i(0), _i(0)
    rc = _lib.sdpa_device_status(ctypes.byref(st), ctypes.byref(dt), int(bool(clear)))
    if rc != SDPA_OK:
        raise SdpaError(rc, "sdpa_device_status")
    return st.value, dt.value


def sdpa_launches_per_call() -> int:
    return int(_lib.sdpa_launches_per_call())


def sdpa_selftest_wait(limit_us, out, stream) -> int:
    """Raw call: the kernels' bounded wait on a barrier nothing completes;
    out is the device address of 4 uint32 (see include/sdpa.h)."""
    return int(_lib.sdpa_selftest_wait(int(limit_us), out, stream or None))


def sdpa_selftest_fastdiv(n, d, count, q) -> int:
    """Raw call (host memory, no GPU): q[i] = n[i] // d[i] by the schedule's
    multiply-and-shift division (host addresses as ints)."""
    return int(_lib.sdpa_selftest_fastdiv(n, d, int(count), q))


def sdpa_selftest_exp2(x, poly, mufu, n, stream) -> int:
    """Raw call: 2^x for n device floats by the FMA-pipe polynomial and by
    ex2.approx (device addresses as ints)."""
    return int(_lib.sdpa_selftest_exp2(x, poly, mufu, int(n), stream or None))


# ---- torch conveniences -------------------------------------------------------

SDPA_NO_MASK, SDPA_CAUSAL, SDPA_CAUSAL_BOTTOM_RIGHT = 0, 1, 2


def _causal_code(causal) -> int:
    """False/0: no mask; True/1: key j <= query i (Sq == Sk); 2 or
    "bottom_right": key j <= i + Sk - Sq (Sq <= Sk, queries at the end)."""
    if causal in (2, "bottom_right"):
        return SDPA_CAUSAL_BOTTOM_RIGHT
    if causal in (True, False, 0, 1):
        return int(bool(causal))
    raise ValueError("causal must be False, True, 2 or 'bottom_right'")

def _dims(q, k, v, allow_views=False):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, S, d]")
    B, Hq, Sq, d = q.shape
    Bk, Hkv, Sk, dk = k.shape
    if tuple(v.shape) != (Bk, Hkv, Sk, dk) or Bk != B or dk != d:
        raise ValueError("shape mismatch: q %s k %s v %s" % (tuple(q.shape), tuple(k.shape),
                                                              tuple(v.shape)))
    for t in (q, k, v):
        if not t.is_cuda or t.device != q.device:
            raise ValueError("q, k, v must be CUDA tensors on one device")
        if not (t.is_contiguous() or (allow_views and t.stride(3) == 1)):
            raise ValueError("q, k, v must be contiguous CUDA tensors%s" % (
                " or views whose last dimension is contiguous" if allow_views else ""))
    return int(B), int(Hq), int(Hkv), int(Sq), int(Sk), int(d)


def _check_buffer(t, name, shape, dtype, device, contiguous=True):
    """A tensor the kernels read or write through a raw pointer, `shape`
    elements of it: size, type, device and layout are checked here because
    the C ABI cannot see them.  contiguous=False accepts any view whose last
    dimension is contiguous."""
    layout_ok = t.is_contiguous() if contiguous else t.stride(-1) == 1
    if (tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_cuda or t.device != device
            or not layout_ok):
        raise ValueError("%s must be a %s CUDA tensor of shape %s on %s, %s" % (
            name, dtype, tuple(shape), device,
            "contiguous" if contiguous else "with a contiguous last dimension"))


def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream(torch.cuda.current_device())
    return int(s.cuda_stream)


def attention(q, k, v, causal=False, scale: float | None = None, out=None, lse=None,
              return_lse: bool = True, stream=None):
    """O (and LSE) = softmax(q k^T * scale [causal]) v for bf16 / fp16 CUDA
    tensors q [B,Hq,Sq,d], k/v [B,Hkv,Sk,d].  They may be strided views
    whose last dimension is contiguous, e.g. BTNH data passed as
    x.transpose(1, 2): those go through sdpa_fwd_strided, in place.  `out`
    defaults to a tensor laid out like q.  Enqueued on `stream` (default:
    torch's current stream); raises SdpaError on a refused call."""
    import torch
    B, Hq, Hkv, Sq, Sk, d = _dims(q, k, v, allow_views=True)
    causal = _causal_code(causal)
    if q.dtype not in (torch.bfloat16, torch.float16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype bfloat16 or float16")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is not None:
        _check_buffer(out, "out", (B, Hq, Sq, d), q.dtype, q.device, contiguous=False)
    if lse is not None:
        _check_buffer(lse, "lse", (B, Hq, Sq), torch.float32, q.device)
    with torch.cuda.device(q.device):
        if out is None:
            out = torch.empty_like(q)
        if lse is None and return_lse:
            lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
        dt = SDPA_BF16 if q.dtype == torch.bfloat16 else SDPA_FP16
        lp = lse.data_ptr() if lse is not None else 0
        if all(t.is_contiguous() for t in (q, k, v, out)):
            what = "sdpa_fwd"
            rc = sdpa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lp,
                          B, Hq, Hkv, Sq, Sk, d, scale, causal, dt, _stream_handle(stream))
        else:
            what = "sdpa_fwd_strided"
            if tuple(out.shape) != (B, Hq, Sq, d) or out.stride(3) != 1:
                raise ValueError("out must be [B, Hq, Sq, d] with a contiguous last dimension")
            rc = sdpa_fwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lp,
                                  B, Hq, Hkv, Sq, Sk, d, q.stride()[:3], k.stride()[:3],
                                  v.stride()[:3], out.stride()[:3], scale, causal, dt,
                                  _stream_handle(stream))
    if rc != SDPA_OK:
        raise SdpaError(rc, what)
    return (out, lse) if return_lse else out


def attention_fp8(q8, k8, v8, descales, causal=False, scale: float | None = None,
                  out=None, lse=None, stream=None):
    """FP8 E4M3 forward: q8/k8/v8 torch.float8_e4m3fn CUDA tensors holding
    codes, descales = (dq, dk, dv) so that value = code * descale.  Returns
    (O bf16, LSE fp32)."""
    import torch
    B, Hq, Hkv, Sq, Sk, d = _dims(q8, k8, v8)
    causal = _causal_code(causal)
    for t in (q8, k8, v8):
        if t.dtype != torch.float8_e4m3fn:
            raise ValueError("q8, k8, v8 must be float8_e4m3fn")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is not None:
        _check_buffer(out, "out", (B, Hq, Sq, d), torch.bfloat16, q8.device)
    if lse is not None:
        _check_buffer(lse, "lse", (B, Hq, Sq), torch.float32, q8.device)
    with torch.cuda.device(q8.device):
        if out is None:
            out = torch.empty((B, Hq, Sq, d), dtype=torch.bfloat16, device=q8.device)
        if lse is None:
            lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q8.device)
        rc = sdpa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), descales[0], descales[1],
                          descales[2], out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Sq, Sk, d,
                          scale, causal, _stream_handle(stream))
    if rc != SDPA_OK:
        raise SdpaError(rc, "sdpa_fwd_fp8")
    return out, lse


def attention_backward(q, k, v, o, lse, dout, causal=False, scale: float | None = None,
                       stream=None):
    """(dQ, dK, dV) for contiguous bf16 / fp16 CUDA tensors: q, o, dout
    [B,Hq,Sq,d], k, v [B,Hkv,Sk,d], lse [B,Hq,Sq] float32 from attention()
    with the same causal and scale."""
    import torch
    B, Hq, Hkv, Sq, Sk, d = _dims(q, k, v)
    causal = _causal_code(causal)
    _check_buffer(o, "o", (B, Hq, Sq, d), q.dtype, q.device)
    _check_buffer(dout, "dout", (B, Hq, Sq, d), q.dtype, q.device)
    _check_buffer(lse, "lse", (B, Hq, Sq), torch.float32, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    with torch.cuda.device(q.device):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        delta = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)   # workspace
        rc = sdpa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                      lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), delta.data_ptr(),
                      B, Hq, Hkv, Sq, Sk, d, scale, causal,
                      SDPA_BF16 if q.dtype == torch.bfloat16 else SDPA_FP16, _stream_handle(stream))
    if rc != SDPA_OK:
        raise SdpaError(rc, "sdpa_bwd")
    return dq, dk, dv


def attention_backward_fp8(q8, k8, v8, o, lse, dout8, descales, causal=False,
                           scale: float | None = None, stream=None):
    """(dQ, dK, dV) bf16 for the FP8 forward: q8/k8/v8 float8_e4m3fn codes,
    o (bf16) and lse from attention_fp8 with the same causal and scale,
    dout8 float8_e5m2 codes, descales = (dq, dk, dv, ddo) with value =
    code * descale.  The workspace is allocated with torch."""
    import torch
    B, Hq, Hkv, Sq, Sk, d = _dims(q8, k8, v8)
    causal = _causal_code(causal)
    for t in (q8, k8, v8):
        if t.dtype != torch.float8_e4m3fn:
            raise ValueError("q8, k8, v8 must be float8_e4m3fn")
    _check_buffer(o, "o", (B, Hq, Sq, d), torch.bfloat16, q8.device)
    _check_buffer(dout8, "dout8", (B, Hq, Sq, d), torch.float8_e5m2, q8.device)
    _check_buffer(lse, "lse", (B, Hq, Sq), torch.float32, q8.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    with torch.cuda.device(q8.device):
        dq = torch.empty((B, Hq, Sq, d), dtype=torch.bfloat16, device=q8.device)
        dk = torch.empty((B, Hkv, Sk, d), dtype=torch.bfloat16, device=q8.device)
        dv = torch.empty((B, Hkv, Sk, d), dtype=torch.bfloat16, device=q8.device)
        nbytes = sdpa_bwd_fp8_workspace_bytes(B, Hq, Hkv, Sq, Sk, d)
        ws = torch.empty(nbytes + 256, dtype=torch.uint8, device=q8.device)
        base = (ws.data_ptr() + 255) // 256 * 256
        rc = sdpa_bwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), o.data_ptr(), dout8.data_ptr(),
                          lse.data_ptr(), descales[0], descales[1], descales[2], descales[3],
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), base, nbytes,
                          B, Hq, Hkv, Sq, Sk, d, scale, causal, _stream_handle(stream))
    if rc != SDPA_OK:
        raise SdpaError(rc, "sdpa_bwd_fp8")
    return dq, dk, dv
