"""The forward's schedule divides by run-time constants with one multiply and
a shift (host-computed magic numbers, Granlund and Montgomery's round-up
method for 31-bit numerators).  sdpa_selftest_fastdiv runs that arithmetic on
the host (no GPU); here it is held to Python's integer division on the edge
cases of the method (divisor 1, powers of two and their neighbours, the
largest numerators and divisors, numerators next to multiples of the divisor)
and on random pairs."""
import random

import numpy as np
import pytest

import scaled_dot_product_11_b200 as sdpa

INT_MAX = 2**31 - 1


def fastdiv(n, d):
    n = np.ascontiguousarray(n, dtype=np.int32)
    d = np.ascontiguousarray(d, dtype=np.int32)
    q = np.full(n.shape, -1, dtype=np.int32)
    rc = sdpa.sdpa_selftest_fastdiv(n.ctypes.data, d.ctypes.data, n.size, q.ctypes.data)
    return rc, q


def pairs():
    rng = random.Random(31)
    divisors = [1, 2, 3, 5, 7, 127, 128, 129, 148, 255, 256, 257, 1000, 4095, 4096, 4097,
                65535, 65536, 65537, 2**30 - 1, 2**30, 2**30 + 1, INT_MAX - 1, INT_MAX]
    divisors += [rng.randrange(1, INT_MAX) for _ in range(200)]
    divisors += [rng.randrange(1, 5000) for _ in range(200)]
    ns, ds = [], []
    for d in divisors:
        cand = {0, 1, d - 1, d, d + 1, INT_MAX, INT_MAX - 1, INT_MAX // d * d, INT_MAX // d * d - 1}
        for k in (2, 3, 1000, 2**20):
            cand.update({k * d - 1, k * d, k * d + 1})
        cand.update(rng.randrange(0, INT_MAX + 1) for _ in range(50))
        for n in cand:
            if 0 <= n <= INT_MAX:
                ns.append(n)
                ds.append(d)
    return ns, ds


def test_fastdiv_matches_integer_division():
    ns, ds = pairs()
    rc, q = fastdiv(ns, ds)
    assert rc == 0
    want = np.array([n // d for n, d in zip(ns, ds)], dtype=np.int64)
    bad = np.nonzero(q.astype(np.int64) != want)[0]
    assert bad.size == 0, [(ns[i], ds[i], int(q[i]), int(want[i])) for i in bad[:5]]


def test_fastdiv_every_numerator_for_small_divisors():
    # all numerators below 4 d for d < 300: covers every remainder class
    ns, ds = [], []
    for d in range(1, 300):
        for n in range(0, 4 * d):
            ns.append(n)
            ds.append(d)
    rc, q = fastdiv(ns, ds)
    assert rc == 0
    assert np.array_equal(q, np.array(ns) // np.array(ds))


@pytest.mark.parametrize("n,d", [(-1, 3), (5, 0), (5, -2)])
def test_fastdiv_rejects_pairs_out_of_range(n, d):
    rc, _ = fastdiv([n], [d])
    assert rc == sdpa.SDPA_ERR_INVALID_ARG


def test_fastdiv_rejects_null_pointers():
    assert sdpa.sdpa_selftest_fastdiv(0, 0, 1, 0) == sdpa.SDPA_ERR_INVALID_ARG
