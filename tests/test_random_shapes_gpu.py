"""GPU parity on seeded random shapes, forward and backward, against the fp64
oracle.

The hand-picked cases of test_parity_gpu.py and test_backward_gpu.py aim at
known edges; these draw (batch, query and K/V heads, both lengths, head dim,
mask, dtype) at random within the library's range, so that combinations no
one listed -- ragged rows and keys together with GQA, end-aligned causal masks
with Sk just above Sq, lengths one past a tile, several heads per schedule
group -- are exercised too.  The draws are fixed by one seed, and each case is
small enough for the oracle to compute every element.  Bounds are those of the
two parity files.
"""
import random

import numpy as np
import pytest
import torch

import oracle
from sdpa_workloads import Workload, make_qkv
from test_backward_gpu import check as check_grad
from test_parity_gpu import LSE_TOL, O_TOL, check_o

pytestmark = pytest.mark.gpu


def draw(n, seed, max_len):
    rng = random.Random(seed)
    cases = []
    while len(cases) < n:
        hkv = rng.choice([1, 1, 2, 3])
        group = rng.choice([1, 2, 4])
        B = rng.choice([1, 1, 2, 3])
        d = rng.choice([32, 64, 64, 128, 128])
        causal = rng.choice([0, 1, 2])
        # lengths: uniform, or one either side of a tile edge
        def length():
            if rng.random() < 0.4:
                return max(1, 128 * rng.randrange(1, max_len // 128 + 1) + rng.choice([-1, 0, 1]))
            return rng.randrange(1, max_len + 1)
        Sq = length()
        Sk = Sq if causal == 1 else length()
        if causal == 2 and Sk < Sq:
            Sq, Sk = Sk, Sq
        dtype = rng.choice(["bf16", "fp16"])
        cases.append((B, hkv * group, hkv, Sq, Sk, d, causal, dtype, rng.randrange(1 << 20)))
    return cases


def case_id(c):
    return "b%d_hq%d_hkv%d_sq%d_sk%d_d%d_c%d_%s" % c[:8]


@pytest.fixture(scope="module")
def sdpa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import scaled_dot_product_11_b200 as lib
    lib.sdpa_device_status(clear=True)
    return lib


@pytest.mark.parametrize("case", draw(24, 2024, 700), ids=case_id)
def test_forward_random_shape(sdpa, case):
    B, Hq, Hkv, Sq, Sk, d, causal, dtype, seed = case
    w = Workload("rand", B, Hq, Hkv, Sq, Sk, d, causal, dtype=dtype, seed=seed)
    q, k, v = make_qkv(w, "cuda")
    o, lse = sdpa.attention(q, k, v, causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    st, detail = sdpa.sdpa_device_status(clear=True)
    assert st == 0, "device status %d detail %#x" % (st, detail)
    ro, rl = oracle.sdpa_fwd(q.cpu(), k.cpu(), v.cpu(), w.scale, causal)
    go, gl = o.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.isfinite(go).all() and np.isfinite(gl).all()
    check_o(go, ro, O_TOL, dtype, case_id(case))
    assert np.abs(gl - rl).max() <= LSE_TOL


@pytest.mark.parametrize("case", draw(12, 77, 400), ids=case_id)
def test_backward_random_shape(sdpa, case):
    B, Hq, Hkv, Sq, Sk, d, causal, dtype, seed = case
    w = Workload("rand", B, Hq, Hkv, Sq, Sk, d, causal, dtype=dtype, seed=seed)
    q, k, v = make_qkv(w, "cuda")
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    dout = torch.randn(B, Hq, Sq, d, generator=g).to(q.dtype).cuda()
    o, lse = sdpa.attention(q, k, v, causal=causal, scale=w.scale)
    dq, dk, dv = sdpa.attention_backward(q, k, v, o, lse, dout, causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    st, detail = sdpa.sdpa_device_status(clear=True)
    assert st == 0, "device status %d detail %#x" % (st, detail)
    rq, rk, rv = oracle.sdpa_bwd(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), w.scale, causal)
    check_grad(dq.double().cpu().numpy(), rq, dtype, "dQ")
    check_grad(dk.double().cpu().numpy(), rk, dtype, "dK")
    check_grad(dv.double().cpu().numpy(), rv, dtype, "dV")
