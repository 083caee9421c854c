"""fp64 CPU oracle for the fused SDPA forward -- test infrastructure.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it and shares no code with it.

The arithmetic lives in ``sdpa_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only compiles it with gcc and marshals numpy / torch CPU arrays.
See that file's header for the formula and the passages it follows.

Parity status of each function (what pins it, in ``tests/test_oracle.py``):
  sdpa_fwd         pinned: closed forms (Sk=1, Sk=2 logistic, d=1, first causal
                   row), invariants (rows of weights sum to 1, constant V,
                   affine V, key permutation, LSE shift, GQA == repeated-KV
                   MHA, causal prefix independence), a dominant key, and a
                   40-digit mpmath evaluation on tiny inputs.  The mask
                   aligned to the end of the keys (causal=2) is pinned by
                   equality with the causal mask when Sq == Sk, with no mask
                   when Sq == 1, and row by row with unmasked attention over
                   the visible key prefix.
  sdpa_bwd         pinned: central differences of sdpa_fwd (no mask, causal,
                   end-aligned causal, GQA) to 1e-8, the single-key closed
                   form, invariance to a common key shift, GQA == summed
                   repeated-KV MHA.
  sdpa_rows        pinned: equals sdpa_fwd on the same rows (same per-row code
                   reached through a different index path) and the pins above.
  sdpa_bruteforce  pinned: mpmath evaluation, weights-sum, V = identity.
  sdpa_bwd_fp8     pinned: equals sdpa_bwd on the decoded values (the same
                   code path reached with E4M3 / E5M2 loads and descales),
                   a power-of-two descale scaling each gradient exactly, and
                   central differences of sdpa_fwd on the decoded inputs.
  decode_*         pinned: all 256 e4m3 and e5m2 codes and all 65536 fp16 /
                   bf16 codes against torch's own casts.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sdpa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F64, BF16, F16, E4M3, E5M2 = 0, 1, 2, 3, 4

_lib = None


def build(force: bool = False) -> str:
    """Compile sdpa_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        vp, i32, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        lib.oracle_sdpa_fwd.argtypes = [vp, vp, vp, i32, f64, f64, f64, vp, vp,
                                        i32, i32, i32, i32, i32, i32, f64, i32, i32]
        lib.oracle_sdpa_rows.argtypes = [vp, vp, vp, i32, f64, f64, f64, vp, ctypes.c_int64,
                                         vp, vp, i32, i32, i32, i32, i32, i32, f64, i32, i32]
        lib.oracle_sdpa_bruteforce.argtypes = [vp, vp, vp, i32, f64, f64, f64, vp, vp, vp,
                                               i32, i32, i32, i32, i32, i32, f64, i32]
        lib.oracle_sdpa_bwd.argtypes = [vp, vp, vp, vp, i32, vp, vp, vp,
                                        i32, i32, i32, i32, i32, i32, f64, i32, i32]
        lib.oracle_sdpa_bwd.restype = i32
        lib.oracle_sdpa_bwd_fp8.argtypes = [vp, vp, vp, vp, f64, f64, f64, f64, vp, vp, vp,
                                            i32, i32, i32, i32, i32, i32, f64, i32, i32]
        lib.oracle_sdpa_bwd_fp8.restype = i32
        lib.oracle_decode_bf16.argtypes = [ctypes.c_uint16]
        lib.oracle_decode_bf16.restype = f64
        lib.oracle_decode_f16.argtypes = [ctypes.c_uint16]
        lib.oracle_decode_f16.restype = f64
        lib.oracle_decode_e4m3.argtypes = [ctypes.c_uint8]
        lib.oracle_decode_e4m3.restype = f64
        lib.oracle_decode_e5m2.argtypes = [ctypes.c_uint8]
        lib.oracle_decode_e5m2.restype = f64
        for fn in (lib.oracle_sdpa_fwd, lib.oracle_sdpa_rows, lib.oracle_sdpa_bruteforce):
            fn.restype = i32
        lib.oracle_max_threads.restype = i32
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _raw(x):
    """(contiguous numpy array of the storage bits, dtype code)."""
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        x = x.detach().contiguous().cpu()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), BF16
        if x.dtype == torch.float16:
            return x.view(torch.int16).numpy().view(np.uint16), F16
        if x.dtype == torch.float8_e4m3fn:
            return x.view(torch.uint8).numpy(), E4M3
        if x.dtype == torch.float8_e5m2:
            return x.view(torch.uint8).numpy(), E5M2
        return x.to(torch.float64).numpy(), F64
    a = np.ascontiguousarray(x)
    if a.dtype != np.float64:
        a = a.astype(np.float64)
    return a, F64


def _shape(q, k):
    B, Hq, Sq, d = (int(s) for s in q.shape)
    Bk, Hkv, Sk, dk = (int(s) for s in k.shape)
    if Bk != B or dk != d:
        raise ValueError("q and k shapes disagree")
    return B, Hq, Hkv, Sq, Sk, d


def _check(rc):
    if rc == 1:
        raise ValueError("oracle: invalid arguments")
    if rc == 2:
        raise ValueError("oracle: causal attention needs Sq == Sk (bottom-right: Sq <= Sk)")
    if rc != 0:
        raise MemoryError("oracle: allocation failed")


def _mask(causal) -> int:
    """0 no mask, 1 causal (key j <= query i, Sq == Sk), 2 causal aligned to
    the end of the keys (j <= i + Sk - Sq, Sq <= Sk).  True means 1."""
    if causal in ("bottom_right", 2):
        return 2
    return 1 if causal else 0


def _prep(q, k, v):
    qa, tq = _raw(q)
    ka, tk = _raw(k)
    va, tv = _raw(v)
    if not (tq == tk == tv):
        raise ValueError("q, k, v must share one storage type")
    return qa, ka, va, tq


def sdpa_fwd(q, k, v, scale: float, causal: bool = False, descales=(1.0, 1.0, 1.0),
             nthreads: int | None = None):
    """Full forward.  q [B,Hq,Sq,d], k/v [B,Hkv,Sk,d] (torch CPU tensors in bf16,
    fp16, float8_e4m3fn or any float, or numpy).  Returns (O, LSE) as float64
    numpy arrays [B,Hq,Sq,d] and [B,Hq,Sq]."""
    lib = _load()
    qa, ka, va, t = _prep(q, k, v)
    B, Hq, Hkv, Sq, Sk, d = _shape(q, k)
    o = np.empty((B, Hq, Sq, d), np.float64)
    lse = np.empty((B, Hq, Sq), np.float64)
    nt = nthreads or max_threads()
    _check(lib.oracle_sdpa_fwd(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, t,
                               float(descales[0]), float(descales[1]), float(descales[2]),
                               o.ctypes.data, lse.ctypes.data,
                               B, Hq, Hkv, Sq, Sk, d, float(scale), _mask(causal), nt))
    return o, lse


def sdpa_rows(q, k, v, rows, scale: float, causal: bool = False, descales=(1.0, 1.0, 1.0),
              nthreads: int | None = None):
    """Selected rows: rows are flat indices (b*Hq + hq)*Sq + i.  Returns
    (O_rows [n,d], LSE_rows [n]) float64."""
    lib = _load()
    qa, ka, va, t = _prep(q, k, v)
    B, Hq, Hkv, Sq, Sk, d = _shape(q, k)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.empty((r.size, d), np.float64)
    lse = np.empty((r.size,), np.float64)
    nt = nthreads or max_threads()
    _check(lib.oracle_sdpa_rows(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, t,
                                float(descales[0]), float(descales[1]), float(descales[2]),
                                r.ctypes.data, r.size, o.ctypes.data, lse.ctypes.data,
                                B, Hq, Hkv, Sq, Sk, d, float(scale), _mask(causal), nt))
    return o, lse


def sdpa_bwd(q, k, v, dout, scale: float, causal=False, nthreads: int | None = None):
    """Gradients (dQ, dK, dV) as float64 arrays of q's, k's and v's shapes
    for the loss whose gradient with respect to O is `dout` (q's shape and
    storage type; bf16, fp16 or float)."""
    lib = _load()
    qa, ka, va, t = _prep(q, k, v)
    da, td = _raw(dout)
    if td != t:
        raise ValueError("dout must share q's storage type")
    B, Hq, Hkv, Sq, Sk, d = _shape(q, k)
    if tuple(da.shape) != (B, Hq, Sq, d):
        raise ValueError("dout must have q's shape")
    dq = np.empty((B, Hq, Sq, d), np.float64)
    dk = np.empty((B, Hkv, Sk, d), np.float64)
    dv = np.empty((B, Hkv, Sk, d), np.float64)
    nt = nthreads or max_threads()
    _check(lib.oracle_sdpa_bwd(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data, t,
                               dq.ctypes.data, dk.ctypes.data, dv.ctypes.data,
                               B, Hq, Hkv, Sq, Sk, d, float(scale), _mask(causal), nt))
    return dq, dk, dv


def sdpa_bwd_fp8(q8, k8, v8, dout8, descales, scale: float, causal=False,
                 nthreads: int | None = None):
    """Gradients (dQ, dK, dV) float64 for the FP8 hybrid recipe: q8, k8, v8
    float8_e4m3fn codes, dout8 float8_e5m2 codes, descales = (dq, dk, dv, ddo)
    so that value = code * descale."""
    lib = _load()
    qa, ka, va, t = _prep(q8, k8, v8)
    da, td = _raw(dout8)
    if t != E4M3 or td != E5M2:
        raise ValueError("q8, k8, v8 must be float8_e4m3fn and dout8 float8_e5m2")
    B, Hq, Hkv, Sq, Sk, d = _shape(q8, k8)
    if tuple(da.shape) != (B, Hq, Sq, d):
        raise ValueError("dout8 must have q8's shape")
    dq = np.empty((B, Hq, Sq, d), np.float64)
    dk = np.empty((B, Hkv, Sk, d), np.float64)
    dv = np.empty((B, Hkv, Sk, d), np.float64)
    nt = nthreads or max_threads()
    _check(lib.oracle_sdpa_bwd_fp8(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data,
                                   *(float(x) for x in descales), dq.ctypes.data, dk.ctypes.data,
                                   dv.ctypes.data, B, Hq, Hkv, Sq, Sk, d, float(scale),
                                   _mask(causal), nt))
    return dq, dk, dv


def sdpa_bruteforce(q, k, v, scale: float, causal: bool = False, descales=(1.0, 1.0, 1.0),
                    return_weights: bool = False):
    """Explicit-matrix forward for tiny inputs.  Returns (O, LSE) or
    (O, LSE, W) with W the [B,Hq,Sq,Sk] attention weights."""
    lib = _load()
    qa, ka, va, t = _prep(q, k, v)
    B, Hq, Hkv, Sq, Sk, d = _shape(q, k)
    o = np.empty((B, Hq, Sq, d), np.float64)
    lse = np.empty((B, Hq, Sq), np.float64)
    w = np.empty((B, Hq, Sq, Sk), np.float64) if return_weights else None
    _check(lib.oracle_sdpa_bruteforce(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, t,
                                      float(descales[0]), float(descales[1]), float(descales[2]),
                                      o.ctypes.data, lse.ctypes.data,
                                      None if w is None else w.ctypes.data,
                                      B, Hq, Hkv, Sq, Sk, d, float(scale), _mask(causal)))
    return (o, lse, w) if return_weights else (o, lse)


def decode_bf16(bits: int) -> float:
    return float(_load().oracle_decode_bf16(int(bits)))


def decode_f16(bits: int) -> float:
    return float(_load().oracle_decode_f16(int(bits)))


def decode_e4m3(code: int) -> float:
    return float(_load().oracle_decode_e4m3(int(code)))


def decode_e5m2(code: int) -> float:
    return float(_load().oracle_decode_e5m2(int(code)))
