"""Host-side checks of the C-ABI library (no GPU, no kernel launch): the .so
loads, exports every entry point include/sdpa.h declares, and refuses bad
arguments with the documented status before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdpa.h")


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"SDPA_API\s+[\w\s\*]+?\b(sdpa_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    assert set(declared_symbols()) == {"sdpa_fwd", "sdpa_fwd_strided", "sdpa_fwd_fp8",
                                       "sdpa_bwd", "sdpa_bwd_noalloc", "sdpa_strerror",
                                       "sdpa_device_status", "sdpa_launches_per_call",
                                       "sdpa_selftest_wait", "sdpa_selftest_exp2", "sdpa_selftest_fastdiv",
                                       "sdpa_bwd_fp8", "sdpa_bwd_fp8_workspace_bytes"}


def test_library_exports_every_declared_symbol():
    import scaled_dot_product_11_b200 as sdpa
    lib = ctypes.CDLL(sdpa.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", sdpa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(declared_symbols()) <= exported
    # nothing else of ours leaks out of the library
    assert not [s for s in exported if s.startswith("_ZN4sdpa")]


def test_strerror_and_launch_count():
    import scaled_dot_product_11_b200 as sdpa
    assert sdpa.sdpa_strerror(0) == "success"
    assert "invalid" in sdpa.sdpa_strerror(1)
    assert "unsupported" in sdpa.sdpa_strerror(2)
    assert "timed out" in sdpa.sdpa_strerror(4)
    assert "layout" in sdpa.sdpa_strerror(5)
    assert "static workspace" in sdpa.sdpa_strerror(6)
    assert sdpa.sdpa_strerror(99) == "unknown status"
    assert sdpa.sdpa_launches_per_call() == 1


# Fake, never dereferenced device addresses: every call below is refused by
# the argument checks, which run before any CUDA call.
P = 0x10000
GOOD = dict(B=1, Hq=4, Hkv=2, Sq=128, Sk=128, d=128, scale=0.088, causal=0, dtype=0)


def call(**kw):
    import scaled_dot_product_11_b200 as sdpa
    a = dict(GOOD)
    a.update(kw)
    ptrs = a.pop("ptrs", (P, P + 0x1000, P + 0x2000, P + 0x3000, P + 0x4000))
    return sdpa.sdpa_fwd(*ptrs, a["B"], a["Hq"], a["Hkv"], a["Sq"], a["Sk"], a["d"], a["scale"],
                         a["causal"], a["dtype"], 0)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=(0, P, P, P, P)), 1),
    (dict(ptrs=(P, P, P, 0, P)), 1),
    (dict(B=0), 1), (dict(Hq=-1), 1), (dict(Sq=0), 1), (dict(Sk=0), 1), (dict(d=0), 1),
    (dict(Hq=3, Hkv=2), 1),
    (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1), (dict(scale=0.0), 1),
    (dict(scale=-1.0), 1),
    (dict(ptrs=(P + 8, P, P, P, P)), 1),
    (dict(ptrs=(P, P, P, P + 4, P)), 1),
    (dict(ptrs=(P, P, P, P, P + 2)), 1),
    (dict(causal=3), 1), (dict(causal=-1), 1),
    (dict(B=1 << 16, Hq=1 << 16, Hkv=1 << 16), 1),
    (dict(d=96), 2), (dict(d=256), 2), (dict(d=16), 2), (dict(d=48), 2),
    (dict(causal=1, Sq=128, Sk=256), 2),
    (dict(causal=2, Sq=257, Sk=256), 2),
    (dict(dtype=2), 2), (dict(dtype=-1), 2),
])
def test_argument_checks(kw, code):
    assert call(**kw) == code


def test_fp8_argument_checks():
    import scaled_dot_product_11_b200 as sdpa

    def fp8(dq=1.0, dk=1.0, dv=1.0, d=128, causal=0, Sq=128, Sk=128):
        return sdpa.sdpa_fwd_fp8(P, P, P, dq, dk, dv, P, P, 1, 2, 2, Sq, Sk, d, 0.088, causal, 0)
    assert fp8(dq=0.0) == 1
    assert fp8(dk=float("nan")) == 1
    assert fp8(dv=-2.0) == 1
    assert fp8(d=64) == 2
    assert fp8(causal=1, Sk=64) == 2


def test_torch_wrapper_rejects_cpu_tensors():
    import torch
    import scaled_dot_product_11_b200 as sdpa
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sdpa.attention(q, q, q)


def test_strided_argument_checks():
    """sdpa_fwd_strided refuses views the kernel cannot address: strides that
    are not positive or whose byte size is not a multiple of 16."""
    import scaled_dot_product_11_b200 as sdpa
    B, H, S, d = 2, 4, 256, 128
    btnh = (S * H * d, d, H * d)            # [B, T, N, d] viewed as [B, N, T, d]

    def strided(qs=btnh, ks=btnh, vs=btnh, os_=btnh, d=d, dtype=0):
        return sdpa.sdpa_fwd_strided(P, P + 0x1000, P + 0x2000, P + 0x3000, P + 0x4000,
                                     B, H, H, S, S, d, qs, ks, vs, os_, 0.088, 0, dtype, 0)
    for bad in ((0, d, H * d), (S * H * d, -d, H * d), (S * H * d, d, H * d + 4),
                (S * H * d + 2, d, H * d), (1 << 41, d, H * d)):
        assert strided(qs=bad) == 1, bad
        assert strided(os_=bad) == 1, bad
    assert strided(ks=(S * H * d, d, 100)) == 1
    assert strided(d=96) == 2          # unsupported head dim before the strides
    assert strided(dtype=3) == 2
    assert sdpa.sdpa_fwd_strided(P, P, P, 0, 0, B, H, H, S, S, d, btnh, btnh, btnh, btnh,
                                 0.088, 0, 0, 0) == 1


def test_torch_wrapper_rejects_views_with_strided_last_dim():
    import torch
    import scaled_dot_product_11_b200 as sdpa
    x = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sdpa.attention(x[..., ::2], x[..., ::2], x[..., ::2])


def test_backward_argument_checks():
    import scaled_dot_product_11_b200 as sdpa

    def bwd(ptrs=None, d=128, causal=0, dtype=0, B=1, Hq=2, Hkv=2, Sq=128, Sk=128):
        ptrs = ptrs or tuple(P + 0x1000 * i for i in range(10))
        return sdpa.sdpa_bwd(*ptrs, B, Hq, Hkv, Sq, Sk, d, 0.088, causal, dtype, 0)
    good = tuple(P + 0x1000 * i for i in range(10))
    for i in range(10):            # every pointer required, lse and delta included
        ptrs = list(good)
        ptrs[i] = 0
        assert bwd(tuple(ptrs)) == 1, i
    ptrs = list(good)
    ptrs[6] += 8                   # dq misaligned
    assert bwd(tuple(ptrs)) == 1
    ptrs = list(good)
    ptrs[9] += 2                   # delta not 4-byte aligned
    assert bwd(tuple(ptrs)) == 1
    assert bwd(d=96) == 2
    assert bwd(dtype=2) == 2
    assert bwd(causal=1, Sq=64) == 2
    assert bwd(causal=3) == 1
    assert bwd(B=300, Hq=256, Hkv=256) == 1   # grid rows


class _FakeCudaTensor:
    """Duck-typed stand-in for a CUDA tensor (none can be made without a
    GPU): just what the binding's buffer check looks at."""

    def __init__(self, shape, dtype, device, strides=None, cuda=True):
        import torch
        self.shape, self.dtype, self.is_cuda = tuple(shape), dtype, cuda
        self.device = torch.device(device)
        if strides is None:
            strides, acc = [], 1
            for n in reversed(self.shape):
                strides.insert(0, acc)
                acc *= n
        self._strides = tuple(strides)

    def stride(self, i=None):
        return self._strides if i is None else self._strides[i]

    def is_contiguous(self):
        acc = 1
        for n, st in zip(reversed(self.shape), reversed(self._strides)):
            if n != 1 and st != acc:
                return False
            acc *= n
        return True


def test_wrapper_buffer_check_accepts_matching_buffers():
    import torch
    from scaled_dot_product_11_b200 import _check_buffer
    dev = torch.device("cuda", 0)
    _check_buffer(_FakeCudaTensor((2, 4, 100, 64), torch.bfloat16, dev), "o", (2, 4, 100, 64),
                  torch.bfloat16, dev)
    # a BTNH view: contiguous last dimension only, accepted where views are
    btnh = _FakeCudaTensor((2, 4, 100, 64), torch.bfloat16, dev, strides=(4 * 100 * 64, 64, 256, 1))
    _check_buffer(btnh, "out", (2, 4, 100, 64), torch.bfloat16, dev, contiguous=False)
    with pytest.raises(ValueError):
        _check_buffer(btnh, "o", (2, 4, 100, 64), torch.bfloat16, dev)


@pytest.mark.parametrize("bad", ["shape", "dtype", "device", "host", "last_stride"])
def test_wrapper_buffer_check_refuses_mismatches(bad):
    """Outputs and backward inputs reach the kernels as raw pointers: a short,
    mistyped, host or other-device buffer is refused before any launch."""
    import torch
    from scaled_dot_product_11_b200 import _check_buffer
    dev = torch.device("cuda", 0)
    shape, dtype, device, strides, cuda = (2, 4, 100, 64), torch.bfloat16, dev, None, True
    if bad == "shape":
        shape = (2, 4, 99, 64)
    elif bad == "dtype":
        dtype = torch.float16
    elif bad == "device":
        device = torch.device("cuda", 1)
    elif bad == "host":
        cuda = False
    else:
        strides = (4 * 100 * 128, 100 * 128, 128, 2)
    t = _FakeCudaTensor(shape, dtype, device, strides, cuda)
    with pytest.raises(ValueError):
        _check_buffer(t, "out", (2, 4, 100, 64), torch.bfloat16, dev, contiguous=False)


def test_fp8_backward_workspace_size_and_argument_checks():
    """sdpa_bwd_fp8: the workspace holds widened Q, K, V, dO (bf16) and D
    (fp32), each part 256-byte aligned; bad arguments are refused before any
    device call."""
    import scaled_dot_product_11_b200 as sdpa
    up = lambda x: (x + 255) // 256 * 256
    B, Hq, Hkv, Sq, Sk, d = 2, 8, 2, 300, 500, 128
    want = 2 * up(B * Hq * Sq * d * 2) + 2 * up(B * Hkv * Sk * d * 2) + up(B * Hq * Sq * 4)
    assert sdpa.sdpa_bwd_fp8_workspace_bytes(B, Hq, Hkv, Sq, Sk, d) == want
    assert sdpa.sdpa_bwd_fp8_workspace_bytes(0, Hq, Hkv, Sq, Sk, d) == 0
    p = 1 << 20          # an aligned stand-in address; never dereferenced
    ws = 1 << 24
    args = dict(q8=p, k8=p, v8=p, o=p, dout8=p, lse=p, descale_q=0.01, descale_k=0.01,
                descale_v=0.01, descale_do=1e-4, dq=p, dk=p, dv=p, workspace=ws,
                workspace_bytes=want, B=B, Hq=Hq, Hkv=Hkv, Sq=Sq, Sk=Sk, d=d, scale=0.088,
                causal=0, stream=0)
    bad = [dict(dout8=0), dict(workspace=0), dict(workspace=ws + 16), dict(workspace_bytes=want - 1),
           dict(descale_do=0.0), dict(descale_q=float("inf")), dict(descale_v=-1.0), dict(lse=0)]
    for b in bad:
        assert sdpa.sdpa_bwd_fp8(**{**args, **b}) == sdpa.SDPA_ERR_INVALID_ARG, b
    w64 = sdpa.sdpa_bwd_fp8_workspace_bytes(B, Hq, Hkv, Sq, Sk, 64)
    assert sdpa.sdpa_bwd_fp8(**{**args, "d": 64, "workspace_bytes": w64}) == sdpa.SDPA_ERR_UNSUPPORTED
