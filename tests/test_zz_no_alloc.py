"""sdpa_bwd_noalloc: the backward for callers that cannot allocate device
memory (a host framework that owns every device allocation, or a path where
cudaMalloc's possible device synchronisation is not allowed).  Its workspace
is a static device array; these checks compare it, through the C ABI, with
sdpa_bwd given a workspace the test allocates, on several calls in a row (each
one finds the previous one's values in the shared array).  Both entry points
launch the same deterministic kernels, so the gradients must agree bit for
bit: a row of D read from a wrong offset of the shared array, or left over
from the previous call, cannot hide inside a tolerance.

The file is named to be collected last, so that a run stopping at the first
failure has run every other test before it.
"""
import pytest
import torch

from sdpa_workloads import Workload, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sdpa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import scaled_dot_product_11_b200 as lib
    lib.sdpa_device_status(clear=True)
    return lib


def problem(B, Hq, Hkv, Sq, Sk, d, causal, dtype, seed):
    w = Workload("noalloc", B, Hq, Hkv, Sq, Sk, d, causal, dtype=dtype, seed=seed)
    q, k, v = make_qkv(w, "cuda")
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    dout = torch.randn(q.shape, generator=g).to(q.dtype).cuda()
    return w, q, k, v, dout


def run(sdpa, entry, w, q, k, v, o, lse, dout, with_workspace):
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dims = (w.B, w.Hq, w.Hkv, w.Sq, w.Sk, w.d, w.scale, int(w.causal),
            sdpa.SDPA_BF16 if q.dtype == torch.bfloat16 else sdpa.SDPA_FP16, 0)
    ptrs = [t.data_ptr() for t in (q, k, v, o, dout, lse, dq, dk, dv)]
    if with_workspace:
        delta = torch.empty(w.B, w.Hq, w.Sq, dtype=torch.float32, device="cuda")
        rc = entry(*ptrs, delta.data_ptr(), *dims)
    else:
        rc = entry(*ptrs, *dims)
    assert rc == sdpa.SDPA_OK, sdpa.sdpa_strerror(rc)
    return dq, dk, dv


def test_noalloc_backward_matches_sdpa_bwd_calls_in_a_row(sdpa):
    cases = [
        # the larger problem first, so the later calls meet its D values
        (2, 8, 2, 1000, 1000, 128, 1, "bf16", 31),
        (1, 4, 4, 300, 500, 64, 0, "fp16", 32),
        (1, 4, 2, 100, 700, 128, 2, "bf16", 33),   # mask aligned to the end of the keys
        (1, 2, 2, 77, 77, 32, 1, "fp16", 34),      # head dim 32 (CUDA-core kernels)
    ]
    for B, Hq, Hkv, Sq, Sk, d, causal, dtype, seed in cases:
        w, q, k, v, dout = problem(B, Hq, Hkv, Sq, Sk, d, causal, dtype, seed)
        o, lse = sdpa.attention(q, k, v, causal=causal, scale=w.scale)
        got = run(sdpa, sdpa.sdpa_bwd_noalloc, w, q, k, v, o, lse, dout, False)
        ref = run(sdpa, sdpa.sdpa_bwd, w, q, k, v, o, lse, dout, True)
        torch.cuda.synchronize()
        st, detail = sdpa.sdpa_device_status(clear=True)
        assert st == 0, "device status %d detail %#x" % (st, detail)
        for name, a, b in zip(("dQ", "dK", "dV"), got, ref):
            assert torch.equal(a, b), "%s differs for %r: max |diff| %.3g" % (
                name, (B, Hq, Hkv, Sq, Sk, d, causal), float((a.float() - b.float()).abs().max()))


def test_noalloc_backward_refuses_more_rows_than_its_workspace(sdpa):
    # null buffers: the size limit is checked before anything else, and even
    # a call that got past it would stop at the null pointers, unlaunched
    rows = sdpa.SDPA_BWD_NOALLOC_MAX_ROWS
    rc = sdpa.sdpa_bwd_noalloc(0, 0, 0, 0, 0, 0, 0, 0, 0, 4, 8, 8, rows // 32 + 1, 128, 128,
                               0.088, 0, sdpa.SDPA_BF16, 0)
    assert rc == sdpa.SDPA_ERR_SCRATCH_LIMIT
    assert "static workspace" in sdpa.sdpa_strerror(rc)
