"""Pins for the fp64 CPU oracle (no GPU).

Each test ties the oracle to something other than itself: closed forms worked
out by hand, invariants of softmax attention, the pages' own statements
(codelab 'JAX on GPU, Lab 5: attention on GPU', sections 5-9), torch's casts
for the storage formats, and a 40-digit mpmath evaluation on tiny inputs.
"""
import json
import math
import os

import mpmath
import numpy as np
import pytest
import torch

import oracle
from sdpa_workloads import quantize_e4m3, quantize_e5m2

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(20261202)


def rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


# --------------------------------------------------------------------------
# storage-format decoding against torch's own casts
# --------------------------------------------------------------------------

def test_decode_e4m3_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.decode_e4m3(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2                      # 0x7f and 0xff only
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7e] == 448.0 and got[0x01] == 2.0 ** -9


def test_decode_e5m2_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e5m2).to(torch.float64).numpy()
    got = np.array([oracle.decode_e5m2(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 6                      # 0x7d-0x7f and 0xfd-0xff
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7b] == 57344.0 and got[0x7c] == np.inf and got[0x01] == 2.0 ** -16


def test_decode_bf16_and_f16_all_codes():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    for tdt, dec in ((torch.bfloat16, oracle.decode_bf16), (torch.float16, oracle.decode_f16)):
        ref = bits.view(tdt).to(torch.float64).numpy()
        got = np.array([dec(b & 0xFFFF) for b in range(65536)])
        nan = np.isnan(ref)
        assert np.array_equal(nan, np.isnan(got))
        assert np.array_equal(ref[~nan], got[~nan])


def test_storage_dtypes_widen_exactly():
    """The oracle on bf16 / fp16 / e4m3 storage equals the oracle on the same
    values handed over as fp64 (so the decode step is the only difference)."""
    q, k, v = rand(1, 2, 9, 16), rand(1, 2, 11, 16), rand(1, 2, 11, 16)
    for dt in (torch.bfloat16, torch.float16):
        tq, tk, tv = (torch.from_numpy(x).to(dt) for x in (q, k, v))
        o1, l1 = oracle.sdpa_fwd(tq, tk, tv, 0.25)
        o2, l2 = oracle.sdpa_fwd(*(t.to(torch.float64).numpy() for t in (tq, tk, tv)), 0.25)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    (q8, dq), (k8, dk), (v8, dv) = (quantize_e4m3(torch.from_numpy(x).float()) for x in (q, k, v))
    o1, l1 = oracle.sdpa_fwd(q8, k8, v8, 0.25, descales=(dq, dk, dv))
    o2, l2 = oracle.sdpa_fwd(q8.to(torch.float64).numpy() * dq, k8.to(torch.float64).numpy() * dk,
                             v8.to(torch.float64).numpy() * dv, 0.25)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

def test_single_key_closed_form():
    """Sk = 1: the only weight is 1, so O = V[0] and LSE = scale * q . k0."""
    q, k, v = rand(2, 3, 5, 8), rand(2, 3, 1, 8), rand(2, 3, 1, 8)
    o, lse = oracle.sdpa_fwd(q, k, v, 0.7)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, 0.7 * np.einsum("bhid,bhd->bhi", q, k[:, :, 0]),
                               rtol=1e-14, atol=1e-14)


def test_two_key_logistic_closed_form():
    """Sk = 2: softmax of two scores is a logistic function of their
    difference D = scale * q . (k1 - k0):  O = v0 + sigmoid(D) (v1 - v0),
    LSE = s0 + log(1 + e^D)."""
    q, k, v = rand(1, 4, 6, 5), rand(1, 4, 2, 5), rand(1, 4, 2, 5)
    sc = 0.45
    o, lse = oracle.sdpa_fwd(q, k, v, sc)
    for h in range(4):
        for i in range(6):
            s0 = sc * float(q[0, h, i] @ k[0, h, 0])
            D = sc * float(q[0, h, i] @ (k[0, h, 1] - k[0, h, 0]))
            sig = 1.0 / (1.0 + math.exp(-D))
            np.testing.assert_allclose(o[0, h, i], v[0, h, 0] + sig * (v[0, h, 1] - v[0, h, 0]),
                                       rtol=0, atol=1e-14)
            assert abs(lse[0, h, i] - (s0 + math.log1p(math.exp(D)))) < 1e-13


def test_d1_hand_worked_example():
    """d = 1, scale = 1, q = 1, keys (0, ln 2, ln 3): weights 1/6, 2/6, 3/6.
    With V = (6, 0, 12): O = 1 + 0 + 6 = 7 and LSE = ln(1 + 2 + 3) = ln 6."""
    q = np.array([1.0]).reshape(1, 1, 1, 1)
    k = np.array([0.0, math.log(2.0), math.log(3.0)]).reshape(1, 1, 3, 1)
    v = np.array([6.0, 0.0, 12.0]).reshape(1, 1, 3, 1)
    for fn in (oracle.sdpa_fwd, oracle.sdpa_bruteforce):
        o, lse = fn(q, k, v, 1.0)
        assert abs(o[0, 0, 0, 0] - 7.0) < 1e-14
        assert abs(lse[0, 0, 0] - math.log(6.0)) < 1e-15


def test_first_causal_row_is_v0():
    """Codelab section 7: with the causal mask the first position attends only
    to itself, so O[0] = V[0] and LSE[0] = scale * q0 . k0."""
    q, k, v = rand(2, 2, 7, 6), rand(2, 2, 7, 6), rand(2, 2, 7, 6)
    o, lse = oracle.sdpa_fwd(q, k, v, 0.3, causal=True)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[:, :, 0], 0.3 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]),
                               rtol=1e-14, atol=1e-15)


def test_codelab_causal_first_and_last_rows():
    """Codelab section 7 on its default shape: the first row changes a lot
    under the mask, the last row does not change at all."""
    g = json.load(open(os.path.join(GOLDEN, "codelab_causal.json")))
    B, T, N, H = g["shape_btnh"]
    q, k, v = (rand(B, N, T, H) for _ in range(3))
    sc = 1.0 / math.sqrt(H)
    oc, lc = oracle.sdpa_fwd(q, k, v, sc, causal=True)
    of, lf = oracle.sdpa_fwd(q, k, v, sc, causal=False)
    assert np.abs(oc[:, :, 0] - of[:, :, 0]).max() > 0.5
    np.testing.assert_allclose(oc[:, :, -1], of[:, :, -1], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lc[:, :, -1], lf[:, :, -1], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------

def test_weights_sum_to_one_via_identity_values():
    """Codelab section 1 step 2: the weights of a row sum to 1.  With
    V = identity (Sk = d) the output row is the weight row itself."""
    n = 12
    q, k = rand(1, 3, 5, n), rand(1, 3, n, n)
    v = np.broadcast_to(np.eye(n), (1, 3, n, n)).copy()
    o, _ = oracle.sdpa_fwd(q, k, v, 0.5)
    assert (o >= 0).all()
    np.testing.assert_allclose(o.sum(-1), 1.0, rtol=0, atol=1e-14)
    _, _, w = oracle.sdpa_bruteforce(q, k, v, 0.5, return_weights=True)
    np.testing.assert_allclose(o, w, rtol=0, atol=1e-15)


def test_constant_and_affine_values():
    q, k, v = rand(2, 2, 9, 8), rand(2, 2, 13, 8), rand(2, 2, 13, 8)
    for causal in (False,):
        o, _ = oracle.sdpa_fwd(q, k, np.full_like(v, -2.5), 0.4, causal)
        np.testing.assert_allclose(o, -2.5, rtol=0, atol=1e-14)
        o1, l1 = oracle.sdpa_fwd(q, k, v, 0.4, causal)
        o2, l2 = oracle.sdpa_fwd(q, k, 3.0 * v + 1.25, 0.4, causal)
        np.testing.assert_allclose(o2, 3.0 * o1 + 1.25, rtol=0, atol=1e-13)
        np.testing.assert_array_equal(l1, l2)


def test_key_permutation_invariance():
    q, k, v = rand(1, 2, 6, 8), rand(1, 2, 10, 8), rand(1, 2, 10, 8)
    perm = rng.permutation(10)
    o1, l1 = oracle.sdpa_fwd(q, k, v, 0.35)
    o2, l2 = oracle.sdpa_fwd(q, k[:, :, perm], v[:, :, perm], 0.35)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-14)


def test_lse_shift_by_common_key_offset():
    """Adding u to every key adds scale * q.u to every score: weights and O are
    unchanged and LSE moves by exactly that amount."""
    q, k, v = rand(1, 2, 6, 8), rand(1, 2, 10, 8), rand(1, 2, 10, 8)
    u = rand(8)
    o1, l1 = oracle.sdpa_fwd(q, k, v, 0.35)
    o2, l2 = oracle.sdpa_fwd(q, k + u, v, 0.35)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l2 - l1, 0.35 * (q @ u), rtol=0, atol=1e-13)


def test_scale_is_applied_to_scores():
    """(c q, scale / c) gives the same result as (q, scale); doubling the scale
    is not the same as doubling nothing (catches a dropped scale)."""
    q, k, v = rand(1, 2, 6, 8), rand(1, 2, 10, 8), rand(1, 2, 10, 8)
    o1, l1 = oracle.sdpa_fwd(q, k, v, 0.35)
    o2, l2 = oracle.sdpa_fwd(4.0 * q, k, v, 0.35 / 4.0)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)
    o3, _ = oracle.sdpa_fwd(q, k, v, 0.7)
    assert np.abs(o3 - o1).max() > 1e-3


def test_causal_prefix_independence():
    """A causal row i depends on keys 0..i only: changing later keys and
    values leaves rows 0..i untouched, and does change later rows."""
    q, k, v = rand(1, 2, 12, 8), rand(1, 2, 12, 8), rand(1, 2, 12, 8)
    o1, l1 = oracle.sdpa_fwd(q, k, v, 0.4, causal=True)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 7:] += 5.0
    v2[:, :, 7:] -= 3.0
    o2, l2 = oracle.sdpa_fwd(q, k2, v2, 0.4, causal=True)
    np.testing.assert_array_equal(o1[:, :, :7], o2[:, :, :7])
    np.testing.assert_array_equal(l1[:, :, :7], l2[:, :, :7])
    assert np.abs(o1[:, :, 7:] - o2[:, :, 7:]).min() > 0


def test_dominant_key_selects_its_value_row():
    """If key j* matches q_i far better than every other key (score gap > 40),
    the weight mass sits on j*, so O_i = V[j*] up to e^-40."""
    q, k, v = rand(1, 1, 4, 16), rand(1, 1, 9, 16) * 0.1, rand(1, 1, 9, 16)
    for i, jstar in enumerate((0, 3, 8, 5)):
        kk = k.copy()
        kk[0, 0, jstar] = 60.0 * q[0, 0, i] / np.linalg.norm(q[0, 0, i]) ** 2
        o, _ = oracle.sdpa_fwd(q[:, :, i:i + 1], kk, v, 1.0)
        np.testing.assert_allclose(o[0, 0, 0], v[0, 0, jstar], rtol=0, atol=1e-12)


def test_gqa_equals_repeated_kv_mha():
    """Codelab section 9: KV heads are shared by groups of query heads.
    Reading: contiguous groups, hk = hq // (Hq / Hkv).  GQA on (q, k, v) must
    equal MHA on K/V heads repeated Hq/Hkv times in place."""
    for hkv in (4, 2, 1):
        q, k, v = rand(2, 8, 7, 8), rand(2, hkv, 9, 8), rand(2, hkv, 9, 8)
        rep = 8 // hkv
        o1, l1 = oracle.sdpa_fwd(q, k, v, 0.3)
        o2, l2 = oracle.sdpa_fwd(q, np.repeat(k, rep, axis=1), np.repeat(v, rep, axis=1), 0.3)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)


def test_gqa_contiguous_group_mapping():
    """Hq = 4, Hkv = 2 with V constant per KV head (-3 on head 0, +5 on head 1):
    query heads 0, 1 must read KV head 0 and heads 2, 3 KV head 1."""
    q, k = rand(1, 4, 5, 8), rand(1, 2, 6, 8)
    v = np.empty((1, 2, 6, 8))
    v[:, 0], v[:, 1] = -3.0, 5.0
    o, _ = oracle.sdpa_fwd(q, k, v, 0.3)
    np.testing.assert_allclose(o[0, :2], -3.0, atol=1e-14)
    np.testing.assert_allclose(o[0, 2:], 5.0, atol=1e-14)


def test_codelab_mha_gqa_mqa_shapes():
    """Codelab section 9: all three variants return Q's shape."""
    g = json.load(open(os.path.join(GOLDEN, "codelab_shapes.json")))
    B, T, N, H = g["q_shape_btnh"]
    q = rand(B, N, T, H)
    for name, kvh in g["kv_heads"].items():
        k, v = rand(B, kvh, T, H), rand(B, kvh, T, H)
        o, lse = oracle.sdpa_fwd(q, k, v, 1.0 / math.sqrt(H))
        Bo, To, No, Ho = g["expected_output_shape_btnh"]
        assert o.shape == (Bo, No, To, Ho), name
        assert lse.shape == (Bo, No, To)
    assert g["kv_heads"]["MHA"] // g["kv_heads"]["GQA"] == g["gqa_group_size_stated"]


def test_large_scores_do_not_overflow():
    """Scores around 1e3 would overflow a one-pass exp; the two-pass form
    subtracts the row max first.  Shifting every score by a constant (via a
    common key offset along q) leaves O unchanged."""
    q, k, v = rand(1, 1, 4, 8), rand(1, 1, 6, 8), rand(1, 1, 6, 8)
    o, lse = oracle.sdpa_fwd(q * 30, k * 30, v, 1.0)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    assert lse.max() > 100


def test_bruteforce_matches_two_pass():
    for causal in (False, True):
        q, k, v = rand(2, 4, 11, 8), rand(2, 2, 11, 8), rand(2, 2, 11, 8)
        o1, l1 = oracle.sdpa_fwd(q, k, v, 0.37, causal)
        o2, l2 = oracle.sdpa_bruteforce(q, k, v, 0.37, causal)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def test_rows_entry_matches_full():
    q, k, v = rand(2, 4, 13, 8), rand(2, 2, 13, 8), rand(2, 2, 13, 8)
    for causal in (False, True):
        o, l = oracle.sdpa_fwd(q, k, v, 0.37, causal)
        rows = [0, 5, 12, 13, 40, 2 * 4 * 13 - 1]
        orow, lrow = oracle.sdpa_rows(q, k, v, rows, 0.37, causal)
        np.testing.assert_array_equal(orow, o.reshape(-1, 8)[rows])
        np.testing.assert_array_equal(lrow, l.reshape(-1)[rows])


def test_mpmath_40_digit_reference():
    """Tiny problems evaluated in 40-digit arithmetic: the oracle's fp64
    result is exact up to fp64 rounding (1e-13)."""
    mpmath.mp.dps = 40
    for causal in (False, True):
        B, Hq, Hkv, S, d = 1, 2, 1, 5, 3
        q, k, v = rand(B, Hq, S, d), rand(B, Hkv, S, d), rand(B, Hkv, S, d)
        sc = 0.61
        o, lse = oracle.sdpa_fwd(q, k, v, sc, causal)
        ob, lb = oracle.sdpa_bruteforce(q, k, v, sc, causal)
        for h in range(Hq):
            for i in range(S):
                keys = range(i + 1) if causal else range(S)
                s = [mpmath.mpf(sc) * mpmath.fsum(mpmath.mpf(q[0, h, i, c]) * mpmath.mpf(k[0, 0, j, c])
                                                  for c in range(d)) for j in keys]
                z = mpmath.fsum(mpmath.exp(x) for x in s)
                ref_lse = mpmath.log(z)
                for c in range(d):
                    ref = mpmath.fsum(mpmath.exp(s[n]) / z * mpmath.mpf(v[0, 0, j, c])
                                      for n, j in enumerate(keys))
                    assert abs(o[0, h, i, c] - float(ref)) < 1e-13
                    assert abs(ob[0, h, i, c] - float(ref)) < 1e-13
                assert abs(lse[0, h, i] - float(ref_lse)) < 1e-13
                assert abs(lb[0, h, i] - float(ref_lse)) < 1e-13


def test_rejects_bad_arguments():
    q, k, v = rand(1, 3, 4, 8), rand(1, 2, 4, 8), rand(1, 2, 4, 8)
    with pytest.raises(ValueError):
        oracle.sdpa_fwd(q, k, v, 1.0)           # Hq % Hkv != 0
    q, k, v = rand(1, 2, 4, 8), rand(1, 2, 5, 8), rand(1, 2, 5, 8)
    with pytest.raises(ValueError):
        oracle.sdpa_fwd(q, k, v, 1.0, causal=True)   # causal needs Sq == Sk


def test_page_tolerance_precedents_recorded():
    g = json.load(open(os.path.join(GOLDEN, "codelab_tolerances.json")))
    assert g["f32_atol"] == 1e-3 and g["bf16_atol"] == 1e-2 and g["bf16_rtol"] == 1e-2


# --------------------------------------------------------------------------
# causal mask aligned to the end of the keys (causal=2): query i of Sq is
# position Sk - Sq + i of the sequence and sees keys 0 .. i + Sk - Sq
# --------------------------------------------------------------------------

def test_bottom_right_equal_lengths_is_the_causal_mask():
    q, k, v = rand(1, 2, 9, 8), rand(1, 2, 9, 8), rand(1, 2, 9, 8)
    o1, l1 = oracle.sdpa_fwd(q, k, v, 0.5, causal=True)
    o2, l2 = oracle.sdpa_fwd(q, k, v, 0.5, causal="bottom_right")
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_bottom_right_single_query_sees_every_key():
    """Sq = 1 (one new token against a cache of Sk keys): no key is masked."""
    q, k, v = rand(2, 4, 1, 8), rand(2, 2, 13, 8), rand(2, 2, 13, 8)
    o1, l1 = oracle.sdpa_fwd(q, k, v, 0.4, causal=False)
    o2, l2 = oracle.sdpa_fwd(q, k, v, 0.4, causal=2)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_bottom_right_rows_are_unmasked_attention_over_a_key_prefix():
    """Row i equals unmasked attention of that one query over keys
    0 .. i + Sk - Sq (sliced K, V), so the offset and its off-by-one are
    pinned by the (independently pinned) unmasked path."""
    Sq, Sk = 5, 12
    q, k, v = rand(1, 2, Sq, 8), rand(1, 1, Sk, 8), rand(1, 1, Sk, 8)
    o, l = oracle.sdpa_fwd(q, k, v, 0.45, causal=2)
    for i in range(Sq):
        n = i + 1 + Sk - Sq
        oi, li = oracle.sdpa_fwd(q[:, :, i:i + 1].copy(), k[:, :, :n].copy(), v[:, :, :n].copy(), 0.45)
        np.testing.assert_allclose(o[:, :, i], oi[:, :, 0], rtol=0, atol=1e-14)
        np.testing.assert_allclose(l[:, :, i], li[:, :, 0], rtol=0, atol=1e-14)
    # and it differs from the top-left reading, under which row 0 sees key 0
    # only and returns V[0]
    assert np.abs(o[:, :, 0] - v[:, :, 0]).max() > 1e-3


def test_bottom_right_bruteforce_and_rows_agree():
    q, k, v = rand(2, 4, 7, 8), rand(2, 2, 11, 8), rand(2, 2, 11, 8)
    o1, l1 = oracle.sdpa_fwd(q, k, v, 0.37, 2)
    o2, l2 = oracle.sdpa_bruteforce(q, k, v, 0.37, 2)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)
    rows = [0, 6, 7, 20, 2 * 4 * 7 - 1]
    orow, lrow = oracle.sdpa_rows(q, k, v, rows, 0.37, 2)
    np.testing.assert_array_equal(orow, o1.reshape(-1, 8)[rows])
    np.testing.assert_array_equal(lrow, l1.reshape(-1)[rows])


def test_bottom_right_rejects_more_queries_than_keys():
    q, k, v = rand(1, 2, 6, 8), rand(1, 2, 5, 8), rand(1, 2, 5, 8)
    with pytest.raises(ValueError):
        oracle.sdpa_fwd(q, k, v, 1.0, causal=2)


# --------------------------------------------------------------------------
# backward: dQ, dK, dV of the loss L = sum(dO * O)
# --------------------------------------------------------------------------

def _loss(q, k, v, dout, scale, causal):
    o, _ = oracle.sdpa_fwd(q, k, v, scale, causal)
    return float((o * dout).sum())


@pytest.mark.parametrize("causal", [0, 1, 2])
def test_backward_matches_finite_differences_of_the_forward(causal):
    """Central differences of the (independently pinned) forward oracle:
    every sampled coordinate of dQ, dK, dV agrees to 1e-8."""
    B, Hq, Hkv, d = 1, 4, 2, 6
    Sq, Sk = (7, 7) if causal != 2 else (5, 9)
    q, k, v = rand(B, Hq, Sq, d), rand(B, Hkv, Sk, d), rand(B, Hkv, Sk, d)
    dout = rand(B, Hq, Sq, d)
    sc = 0.43
    dq, dk, dv = oracle.sdpa_bwd(q, k, v, dout, sc, causal)
    h = 1e-5
    pick = np.random.default_rng(causal + 7)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            idx = tuple(int(pick.integers(0, n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd = (_loss(args_p["q"], args_p["k"], args_p["v"], dout, sc, causal) -
                  _loss(args_m["q"], args_m["k"], args_m["v"], dout, sc, causal)) / (2 * h)
            assert abs(fd - g[idx]) < 1e-8 * max(1.0, abs(fd)), (name, idx, fd, g[idx])


def test_backward_single_key_closed_form():
    """One key: the weights are all 1, so dQ = dK = 0 and dV is the sum of
    dO over the rows and query heads sharing the key."""
    q, k, v = rand(2, 4, 5, 3), rand(2, 2, 1, 3), rand(2, 2, 1, 3)
    dout = rand(2, 4, 5, 3)
    dq, dk, dv = oracle.sdpa_bwd(q, k, v, dout, 0.7)
    assert np.abs(dq).max() < 1e-14 and np.abs(dk).max() < 1e-14
    expect = dout.reshape(2, 2, 2, 5, 3).sum(axis=(2, 3))[:, :, None, :]
    np.testing.assert_allclose(dv, expect, rtol=0, atol=1e-13)


def test_backward_dq_invariant_to_a_common_key_shift():
    """Adding one vector to every key shifts each row's scores by a constant:
    the weights, dS and hence dK and dV are unchanged, and dQ too because
    sum_j ds_j = 0 per row."""
    q, k, v = rand(1, 2, 6, 5), rand(1, 2, 6, 5), rand(1, 2, 6, 5)
    dout = rand(1, 2, 6, 5)
    dq1, dk1, dv1 = oracle.sdpa_bwd(q, k, v, dout, 0.5)
    shift = rand(5)
    # the shift changes the scores by q . shift, constant per row: same weights
    dq2, dk2, dv2 = oracle.sdpa_bwd(q, k + shift, v, dout, 0.5)
    np.testing.assert_allclose(dq1, dq2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk1, dk2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv1, dv2, rtol=0, atol=1e-12)


def test_backward_gqa_equals_summed_repeated_kv_mha():
    B, Hq, Hkv, S, d = 1, 6, 2, 5, 4
    q, k, v = rand(B, Hq, S, d), rand(B, Hkv, S, d), rand(B, Hkv, S, d)
    dout = rand(B, Hq, S, d)
    dq, dk, dv = oracle.sdpa_bwd(q, k, v, dout, 0.6, True)
    g = Hq // Hkv
    kr, vr = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    dq2, dk2, dv2 = oracle.sdpa_bwd(q, kr, vr, dout, 0.6, True)
    np.testing.assert_allclose(dq, dq2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk, dk2.reshape(B, Hkv, g, S, d).sum(axis=2), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(B, Hkv, g, S, d).sum(axis=2), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [0, 1, 2])
def test_backward_matches_autograd_of_the_plain_definition(causal):
    """torch's automatic differentiation of softmax(scale Q K^T + mask) V in
    float64, an independent route to the same derivative: every coordinate of
    dQ, dK, dV agrees to 1e-12."""
    B, Hq, Hkv, d = 2, 4, 2, 5
    Sq, Sk = (6, 6) if causal != 2 else (4, 7)
    q, k, v = rand(B, Hq, Sq, d), rand(B, Hkv, Sk, d), rand(B, Hkv, Sk, d)
    dout = rand(B, Hq, Sq, d)
    sc = 0.61
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    g = Hq // Hkv
    s = sc * tq @ tk.repeat_interleave(g, dim=1).transpose(-1, -2)
    if causal:
        off = Sk - Sq if causal == 2 else 0
        keep = torch.arange(Sk)[None, :] <= torch.arange(Sq)[:, None] + off
        s = s.masked_fill(~keep, float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv.repeat_interleave(g, dim=1)
    (o * torch.tensor(dout)).sum().backward()
    dq, dk, dv = oracle.sdpa_bwd(q, k, v, dout, sc, causal)
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [0, 1])
def test_backward_zero_queries_closed_form(causal):
    """q = 0 makes every visible key equally weighted (1/n_i for row i), so
    dV_j is the average-weighted sum of the dO rows that see key j; dK = 0
    because each row's scores do not depend on the keys."""
    B, H, S, d = 1, 3, 5, 4
    q = np.zeros((B, H, S, d))
    k, v, dout = rand(B, H, S, d), rand(B, H, S, d), rand(B, H, S, d)
    dq, dk, dv = oracle.sdpa_bwd(q, k, v, dout, 0.9, causal)
    assert np.abs(dk).max() < 1e-14
    expect = np.zeros_like(v)
    for i in range(S):
        seen = range(i + 1) if causal else range(S)
        for j in seen:
            expect[:, :, j, :] += dout[:, :, i, :] / len(seen)
    np.testing.assert_allclose(dv, expect, rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# FP8 backward (E4M3 forward tensors, E5M2 output gradient; codelab section 10)
# --------------------------------------------------------------------------

def _fp8_problem(B=1, Hq=2, Hkv=1, Sq=9, Sk=13, d=8, seed=5):
    g = torch.Generator().manual_seed(seed)
    q, ds_q = quantize_e4m3(torch.randn(B, Hq, Sq, d, generator=g))
    k, ds_k = quantize_e4m3(torch.randn(B, Hkv, Sk, d, generator=g))
    v, ds_v = quantize_e4m3(torch.randn(B, Hkv, Sk, d, generator=g))
    do, ds_do = quantize_e5m2(torch.randn(B, Hq, Sq, d, generator=g))
    return (q, k, v, do), (ds_q, ds_k, ds_v, ds_do)


def _decoded(t, ds):
    return t.to(torch.float64).numpy() * ds


@pytest.mark.parametrize("causal", [0, 2])
def test_fp8_backward_matches_finite_differences_of_the_forward(causal):
    """dQ, dK, dV of the FP8 recipe against central differences of the
    pinned forward on the decoded values (the loss is <O, dO>)."""
    (q8, k8, v8, do8), ds = _fp8_problem()
    scale = 0.35
    gq, gk, gv = oracle.sdpa_bwd_fp8(q8, k8, v8, do8, ds, scale, causal)
    q, k, v = _decoded(q8, ds[0]), _decoded(k8, ds[1]), _decoded(v8, ds[2])
    do = _decoded(do8, ds[3])

    def loss(qq, kk, vv):
        o, _ = oracle.sdpa_fwd(qq, kk, vv, scale, causal)
        return float((o * do).sum())

    h = 1e-6
    picks = [(q, gq, (0, 1, 3, 2)), (k, gk, (0, 0, 7, 5)), (v, gv, (0, 0, 12, 1)), (k, gk, (0, 0, 0, 0))]
    for arr, grad, idx in picks:
        plus, minus = arr.copy(), arr.copy()
        plus[idx] += h
        minus[idx] -= h
        args_p = [plus if a is arr else a for a in (q, k, v)]
        args_m = [minus if a is arr else a for a in (q, k, v)]
        fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (idx, fd, grad[idx])


def test_fp8_backward_equals_backward_on_decoded_values():
    (q8, k8, v8, do8), ds = _fp8_problem(B=2, Hq=4, Hkv=2, Sq=20, Sk=31, d=16, seed=9)
    got = oracle.sdpa_bwd_fp8(q8, k8, v8, do8, ds, 0.25, 0)
    ref = oracle.sdpa_bwd(_decoded(q8, ds[0]), _decoded(k8, ds[1]), _decoded(v8, ds[2]),
                          _decoded(do8, ds[3]), 0.25, 0)
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)


def test_fp8_backward_descales_scale_the_gradients_exactly():
    """Doubling dO's descale doubles every gradient; doubling V's doubles dQ
    and dK (through dP) and leaves dV = P^T dO unchanged."""
    (q8, k8, v8, do8), ds = _fp8_problem(seed=11)
    base = oracle.sdpa_bwd_fp8(q8, k8, v8, do8, ds, 0.3, 0)
    two_do = oracle.sdpa_bwd_fp8(q8, k8, v8, do8, (ds[0], ds[1], ds[2], 2 * ds[3]), 0.3, 0)
    two_v = oracle.sdpa_bwd_fp8(q8, k8, v8, do8, (ds[0], ds[1], 2 * ds[2], ds[3]), 0.3, 0)
    for a, b in zip(two_do, base):
        assert np.array_equal(a, 2 * b)
    assert np.array_equal(two_v[0], 2 * base[0]) and np.array_equal(two_v[1], 2 * base[1])
    assert np.array_equal(two_v[2], base[2])
