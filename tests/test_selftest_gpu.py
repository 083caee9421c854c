"""GPU checks of the kernels' device-side machinery through the library's
self-test entry points (include/sdpa.h, sdpa_selftest_*).

Bounded waits.  Every wait of the attention kernels gives up after a time
limit instead of hanging: the waiting warp raises its CTA's abort flag,
records SDPA_ERR_DEVICE_TIMEOUT and a location code in the device status word
and returns, and every other warp of the CTA leaves its own wait when it sees
the flag.  The self-test runs exactly that path on a barrier nothing ever
completes, with a limit of a few milliseconds; the kernel returns by design
(no trap, no fault), the status comes back through sdpa_device_status, and a
forward on the same device afterwards is still parity-green: a refusal is
raised to the caller, never turned into a silent fallback (the codelab's
cuDNN back-end raises likewise, section 6).

The FMA-pipe exponential.  The softmax can evaluate part of its 2^x on the
FMA pipe instead of the MUFU: x = n + f with n = rint(x) (the 1.5 * 2^23
rounding trick) and f in [-1/2, 1/2], 2^f by a cubic fitted to the relative
error on that interval (max 1.0e-4 in exact arithmetic), and 2^n added to the
exponent bits.  It is checked over the whole range the softmax feeds it,
[-126, 64], against exact 2^x (float64) and against ex2.approx.
"""
import numpy as np
import pytest
import torch

import oracle
from sdpa_workloads import Workload, make_qkv

pytestmark = pytest.mark.gpu

SELFTEST_WHERE = 0x7E000
# the cubic's own max relative error is 1.0e-4; its float32 evaluation
# (three fma steps, the range reduction exact) adds at most a few ulps
POLY_REL_TOL = 1.2e-4


@pytest.fixture(scope="module")
def sdpa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import scaled_dot_product_11_b200 as lib
    lib.sdpa_device_status(clear=True)
    return lib


def test_bounded_wait_gives_up_records_status_and_leaves_a_usable_context(sdpa):
    out = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    rc = sdpa.sdpa_selftest_wait(2000, out.data_ptr(), 0)     # 2 ms limit
    assert rc == sdpa.SDPA_OK, sdpa.sdpa_strerror(rc)
    torch.cuda.synchronize()
    st, detail = sdpa.sdpa_device_status(clear=True)
    assert st == sdpa.SDPA_ERR_DEVICE_TIMEOUT, (st, hex(detail))
    assert detail == SELFTEST_WHERE, hex(detail)
    # warp 0 gave up and raised the abort flag; warp 1 (one-second limit)
    # gave up on seeing it
    assert out.tolist() == [0, 1, 0, 1]
    # the status word is clear again and the context still computes
    w = Workload("after_timeout", 1, 4, 2, 300, 300, 128, True, seed=17)
    q, k, v = make_qkv(w, "cuda")
    o, lse = sdpa.attention(q, k, v, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert sdpa.sdpa_device_status(clear=True)[0] == sdpa.SDPA_OK
    ro, rl = oracle.sdpa_fwd(q.cpu(), k.cpu(), v.cpu(), w.scale, True)
    assert np.abs(o.double().cpu().numpy() - ro).max() <= 1e-2
    assert np.abs(lse.double().cpu().numpy() - rl).max() <= 1e-3


def test_bounded_wait_refuses_bad_arguments(sdpa):
    out = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert sdpa.sdpa_selftest_wait(0, out.data_ptr(), 0) == sdpa.SDPA_ERR_INVALID_ARG
    assert sdpa.sdpa_selftest_wait(1000001, out.data_ptr(), 0) == sdpa.SDPA_ERR_INVALID_ARG
    assert sdpa.sdpa_selftest_wait(100, 0, 0) == sdpa.SDPA_ERR_INVALID_ARG


def test_fma_pipe_exp2_against_exact_and_ex2_approx(sdpa):
    rng = np.random.default_rng(2)
    grid = np.linspace(-126.0, 64.0, 1_900_001)
    special = np.concatenate([np.arange(-126, 65), np.arange(-126, 64) + 0.5,
                              np.arange(-126, 64) + 0.5 - 2.0 ** -20, [0.0, -1e-7, 1e-7]])
    x = np.concatenate([grid, rng.uniform(-126.0, 64.0, 500_001), special]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    poly = torch.empty_like(xd)
    mufu = torch.empty_like(xd)
    rc = sdpa.sdpa_selftest_exp2(xd.data_ptr(), poly.data_ptr(), mufu.data_ptr(), x.size, 0)
    assert rc == sdpa.SDPA_OK, sdpa.sdpa_strerror(rc)
    torch.cuda.synchronize()
    exact = np.exp2(x.astype(np.float64))
    p = poly.cpu().numpy().astype(np.float64)
    m = mufu.cpu().numpy().astype(np.float64)
    assert np.isfinite(p).all()
    rel_poly = np.abs(p - exact) / exact
    rel_mufu = np.abs(m - exact) / exact
    i = int(np.argmax(rel_poly))
    assert rel_poly[i] <= POLY_REL_TOL, "poly: rel err %.3g at x = %r" % (rel_poly[i], float(x[i]))
    # the MUFU instruction is far more accurate: both agree to the poly's bound
    assert rel_mufu.max() <= 1e-6
    assert (np.abs(p - m) / m).max() <= POLY_REL_TOL + 1e-6
    # exact at integers: the range reduction leaves f = 0 and the cubic gives 1
    ints = np.isin(x, np.arange(-126, 65).astype(np.float32))
    assert np.array_equal(p[ints], exact[ints])


def test_exp2_refuses_bad_arguments(sdpa):
    x = torch.zeros(4, device="cuda")
    assert sdpa.sdpa_selftest_exp2(0, x.data_ptr(), x.data_ptr(), 4, 0) == sdpa.SDPA_ERR_INVALID_ARG
    assert sdpa.sdpa_selftest_exp2(x.data_ptr(), x.data_ptr(), x.data_ptr(), 0, 0) == \
        sdpa.SDPA_ERR_INVALID_ARG
