"""GPU parity of the backward kernels (sdpa_bwd) against the fp64 oracle.

Inputs are seeded (sdpa_workloads); dO is drawn from its own seed.  The
forward runs on the GPU (its O and LSE feed the backward, as in training) and
the oracle recomputes everything from Q, K, V, dO in fp64.

Tolerance: the kernels work in fp32; the inputs they take from the forward
are O rounded to 16 bits (relative 2^-9, entering through D = dO . O) and the
fp32 LSE.  Each gradient is compared element by element with
|g - g_ref| <= 1e-2 * max(1, max|g_ref|) + ulp(g_ref)/2 in the output format.
"""
import numpy as np
import pytest
import torch

import oracle
from sdpa_workloads import Workload, make_qkv

pytestmark = pytest.mark.gpu

MANT = {"bf16": 7, "fp16": 10}


@pytest.fixture(scope="module")
def sdpa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import scaled_dot_product_11_b200 as lib
    lib.sdpa_device_status(clear=True)
    return lib


def half_ulp(ref, dtype):
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -14.0 if dtype == "fp16" else -126.0)
    return np.where(a > 0, 2.0 ** (e - MANT[dtype]) / 2.0, 0.0)


def check(got, ref, dtype, what):
    tol = 1e-2 * max(1.0, float(np.abs(ref).max()))
    err = np.abs(got - ref) - half_ulp(ref, dtype)
    i = int(np.argmax(err))
    assert err.flat[i] <= tol, "%s: |d| %.4g at %d (ref %.5g got %.5g), tol %.3g" % (
        what, abs(got.flat[i] - ref.flat[i]), i, ref.flat[i], got.flat[i], tol)


CASES = [
    # (B, Hq, Hkv, Sq, Sk, d, causal, dtype)
    (1, 2, 2, 128, 128, 64, 0, "bf16"),
    (1, 2, 2, 200, 200, 128, 1, "bf16"),
    (2, 4, 2, 150, 300, 128, 0, "bf16"),     # GQA, ragged tiles
    (1, 4, 1, 100, 300, 64, 2, "bf16"),      # MQA, end-aligned causal
    (1, 2, 2, 77, 77, 32, 1, "fp16"),        # head dim 32
    (1, 3, 3, 65, 190, 128, 0, "fp16"),
    (1, 4, 4, 1024, 1024, 128, 1, "bf16"),   # many tiles
    # the tensor-core kernels walk 64-row steps through a ring of 4 (d=128)
    # or 8 (d=64) slots, with S and dP double-buffered
    (1, 2, 2, 40, 40, 128, 0, "bf16"),       # one partial step
    (1, 2, 2, 33, 33, 64, 1, "fp16"),        # one partial causal step
    (1, 2, 2, 320, 320, 128, 1, "bf16"),     # causal starts on 64-row steps inside 128-key tiles
    (1, 8, 2, 257, 257, 128, 1, "bf16"),     # GQA: steps of four query heads wrap the ring
    (1, 2, 2, 190, 450, 128, 2, "bf16"),     # end-aligned causal, Sk > Sq
    (2, 2, 2, 130, 131, 64, 2, "fp16"),      # ragged rows and keys, d=64, end-aligned causal
    (1, 2, 1, 1536, 1536, 64, 0, "bf16"),    # long: the 8-slot ring wraps many times
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_hq%d_hkv%d_sq%d_sk%d_d%d_c%d_%s" % c)
def test_backward_matches_oracle(sdpa, case):
    B, Hq, Hkv, Sq, Sk, d, causal, dtype = case
    w = Workload("bwd", B, Hq, Hkv, Sq, Sk, d, causal, dtype=dtype, seed=Sq * 3 + Sk + d)
    q, k, v = make_qkv(w, "cuda")
    g = torch.Generator(device="cpu").manual_seed(w.seed + 1)
    dout = torch.randn(B, Hq, Sq, d, generator=g).to(q.dtype).cuda()
    o, lse = sdpa.attention(q, k, v, causal=causal, scale=w.scale)
    dq, dk, dv = sdpa.attention_backward(q, k, v, o, lse, dout, causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    st, detail = sdpa.sdpa_device_status(clear=True)
    assert st == 0, "device status %d detail %#x" % (st, detail)
    rq, rk, rv = oracle.sdpa_bwd(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), w.scale, causal)
    check(dq.double().cpu().numpy(), rq, dtype, "dQ")
    check(dk.double().cpu().numpy(), rk, dtype, "dK")
    check(dv.double().cpu().numpy(), rv, dtype, "dV")


def test_backward_is_deterministic(sdpa):
    w = Workload("det", 1, 4, 2, 300, 300, 128, 1, seed=8)
    q, k, v = make_qkv(w, "cuda")
    dout = q.flip(2).contiguous()             # any fixed gradient of O
    o, lse = sdpa.attention(q, k, v, causal=True)
    a = sdpa.attention_backward(q, k, v, o, lse, dout, causal=True)
    b = sdpa.attention_backward(q, k, v, o, lse, dout, causal=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_writes_row_statistic_to_workspace(sdpa):
    """The raw call's workspace holds D_i = dO_i . O_i on return (head dims 64
    and 128), computed here in fp64 from the same 16-bit O and dO."""
    w = Workload("delta", 2, 4, 2, 200, 200, 128, 0, seed=11)
    q, k, v = make_qkv(w, "cuda")
    g = torch.Generator(device="cpu").manual_seed(12)
    dout = torch.randn(q.shape, generator=g).to(q.dtype).cuda()
    o, lse = sdpa.attention(q, k, v, scale=w.scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    delta = torch.full((2, 4, 200), float("nan"), device="cuda")
    rc = sdpa.sdpa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                       lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), delta.data_ptr(),
                       2, 4, 2, 200, 200, 128, w.scale, 0, sdpa.SDPA_BF16, 0)
    assert rc == 0
    torch.cuda.synchronize()
    ref = (dout.double() * o.double()).sum(-1).cpu().numpy()
    got = delta.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= 1e-5 * max(1.0, float(np.abs(ref).max()))
