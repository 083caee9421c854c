"""GPU parity of the FP8 backward (sdpa_bwd_fp8) against the fp64 oracle.

The codelab's hybrid recipe (section 10): E4M3 for the forward tensors, E5M2
for the gradient.  Q, K, V are drawn as fp32 N(0,1) and quantised to E4M3 with
per-tensor current scaling (amax / 448), dO likewise to E5M2 (amax / 57344);
the FP8 forward (sdpa_fwd_fp8) supplies O (bf16) and LSE, as in training; the
oracle computes the exact gradients from the decoded codes.

Tolerance: |g - g_ref| <= 2e-2 * max(1, max|g_ref|) + ulp(g_ref)/2 (bf16) per
element.  The kernels run the 16-bit backward's arithmetic on codes widened
exactly to bf16 (P and dS rounded to bf16, fp32 accumulation), whose bound is
1e-2 * max(1, max|g_ref|); what is new is that O enters D_i = dO_i . O_i from
the FP8 forward, whose own O error bound is 6e-2 (six times the bf16 one):
the error it adds to dS_ij = P_ij (dP_ij - D_i) is P_ij dO_i . dO_err, of the
order of the 16-bit path's own dS rounding for these inputs, so the bound is
doubled.
"""
import numpy as np
import pytest
import torch

import oracle
from sdpa_workloads import Workload, make_dout_e5m2, make_qkv_fp8

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module")
def sdpa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import scaled_dot_product_11_b200 as lib
    lib.sdpa_device_status(clear=True)
    return lib


def half_ulp_bf16(ref):
    a = np.abs(ref)
    e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), -126.0)
    return np.where(a > 0, 2.0 ** (e - 7) / 2.0, 0.0)


CASES = [
    # (B, Hq, Hkv, Sq, Sk, causal)
    (1, 2, 2, 200, 200, 1),
    (2, 4, 2, 150, 300, 0),        # GQA, ragged tiles
    (1, 4, 1, 100, 300, 2),        # MQA, mask aligned to the end of the keys
    (1, 2, 2, 1024, 1024, 1),      # many tiles
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_hq%d_hkv%d_sq%d_sk%d_c%d" % c)
def test_fp8_backward_matches_oracle(sdpa, case):
    B, Hq, Hkv, Sq, Sk, causal = case
    w = Workload("bwd8", B, Hq, Hkv, Sq, Sk, 128, causal, dtype="e4m3", seed=Sq * 3 + Sk + causal)
    q8, k8, v8, (dq_, dk_, dv_), _ = make_qkv_fp8(w, "cuda")
    do8, ddo, _ = make_dout_e5m2(w, "cuda")
    o, lse = sdpa.attention_fp8(q8, k8, v8, (dq_, dk_, dv_), causal=causal, scale=w.scale)
    grads = sdpa.attention_backward_fp8(q8, k8, v8, o, lse, do8, (dq_, dk_, dv_, ddo),
                                        causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    st, detail = sdpa.sdpa_device_status(clear=True)
    assert st == 0, "device status %d detail %#x" % (st, detail)
    refs = oracle.sdpa_bwd_fp8(q8.cpu(), k8.cpu(), v8.cpu(), do8.cpu(), (dq_, dk_, dv_, ddo),
                               w.scale, causal)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, refs):
        got = g.double().cpu().numpy()
        assert np.isfinite(got).all(), name
        tol = TOL * max(1.0, float(np.abs(r).max()))
        err = np.abs(got - r) - half_ulp_bf16(r)
        i = int(np.argmax(err))
        assert err.flat[i] <= tol, "%s: |d| %.4g at %d (ref %.5g got %.5g), tol %.3g" % (
            name, abs(got.flat[i] - r.flat[i]), i, r.flat[i], got.flat[i], tol)


def test_fp8_backward_is_deterministic(sdpa):
    w = Workload("bwd8d", 1, 4, 2, 300, 300, 128, 1, dtype="e4m3", seed=77)
    q8, k8, v8, ds, _ = make_qkv_fp8(w, "cuda")
    do8, ddo, _ = make_dout_e5m2(w, "cuda")
    o, lse = sdpa.attention_fp8(q8, k8, v8, ds, causal=True, scale=w.scale)
    a = sdpa.attention_backward_fp8(q8, k8, v8, o, lse, do8, (*ds, ddo), causal=True, scale=w.scale)
    b = sdpa.attention_backward_fp8(q8, k8, v8, o, lse, do8, (*ds, ddo), causal=True, scale=w.scale)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
