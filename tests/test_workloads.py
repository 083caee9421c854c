"""The seeded input generators (no GPU): the recipe the parity tests and the
benchmark rely on, checked against what it promises."""
import pytest
import torch

from sdpa_workloads import (WORKLOADS, Workload, batch_sweep, make_inputs, make_qkv,
                            make_qkv_btnh, make_qkv_fp8, quantize_e4m3, sample_rows, sweep)


def visible_pairs(Sq, Sk, causal):
    off = Sk - Sq if causal == 2 else 0
    return sum(1 for i in range(Sq) for j in range(Sk) if not causal or j <= i + off)


@pytest.mark.parametrize("Sq,Sk", [(1, 9), (5, 9), (9, 9), (3, 130)])
def test_flops_count_the_visible_pairs_of_the_end_aligned_mask(Sq, Sk):
    w = Workload("f", 2, 3, 1, Sq, Sk, 8, 2)
    assert w.flops == 4.0 * 2 * 3 * 8 * visible_pairs(Sq, Sk, 2)


def test_flops_causal_is_half_of_full():
    full = Workload("f", 2, 4, 2, 64, 64, 32, 0)
    causal = Workload("f", 2, 4, 2, 64, 64, 32, 1)
    assert full.flops == 4.0 * 2 * 4 * 64 * 64 * 32
    assert causal.flops == full.flops / 2


def test_qkv_drawn_in_order_from_one_seeded_generator():
    w = Workload("r", 2, 4, 2, 33, 47, 64, 0, seed=5)
    q, k, v = make_qkv(w)
    g = torch.Generator(device="cpu").manual_seed(5)
    for t, shape in ((q, (2, 4, 33, 64)), (k, (2, 2, 47, 64)), (v, (2, 2, 47, 64))):
        x = torch.randn(*shape, generator=g, dtype=torch.float32)
        assert t.dtype == torch.bfloat16 and torch.equal(t, x.to(torch.bfloat16))
    a = make_qkv(w)
    assert all(torch.equal(x, y) for x, y in zip(a, (q, k, v)))
    q16 = make_qkv(Workload("r", 2, 4, 2, 33, 47, 64, 0, dtype="fp16", seed=5))[0]
    assert q16.dtype == torch.float16


def test_values_are_standard_normal():
    q, k, v = make_qkv(Workload("n", 4, 8, 8, 256, 256, 64, 0, seed=1))
    x = torch.cat([t.float().flatten() for t in (q, k, v)])
    assert abs(float(x.mean())) < 0.01 and abs(float(x.std()) - 1.0) < 0.01


def test_btnh_views_have_bhsd_shape_and_a_contiguous_head_dim():
    w = Workload("b", 2, 8, 2, 40, 50, 64, 0, seed=3, layout="btnh")
    q, k, v = make_inputs(w)
    assert q.shape == (2, 8, 40, 64) and k.shape == (2, 2, 50, 64)
    assert all(t.stride(3) == 1 and not t.is_contiguous() for t in (q, k, v))
    qb = make_qkv_btnh(w)[0]
    assert torch.equal(q, qb.transpose(1, 2))


def test_e4m3_per_tensor_scaling():
    x = torch.randn(1000, generator=torch.Generator().manual_seed(2))
    codes, descale = quantize_e4m3(x)
    amax = float(x.abs().max())
    assert descale == amax / 448.0
    back = codes.float() * descale
    assert float(back.abs().max()) == pytest.approx(amax, rel=1e-6)   # amax lands on code 448
    # e4m3 keeps 3 mantissa bits: relative rounding error at most 2^-4 (normal range)
    big = x.abs() > 2.0 ** -6 * descale
    assert float(((back - x).abs() / x.abs())[big].max()) <= 2.0 ** -4 + 1e-7
    zero_codes, zero_descale = quantize_e4m3(torch.zeros(8))
    assert zero_descale == 1.0 and not zero_codes.float().any()


def test_fp8_workload_returns_codes_descales_and_the_fp32_draws():
    w = WORKLOADS["fp8"]
    small = Workload("s", 1, 2, 2, 64, 64, 128, 1, dtype="e4m3", seed=w.seed)
    q8, k8, v8, ds, raw = make_qkv_fp8(small)
    assert q8.dtype == torch.float8_e4m3fn and len(ds) == 3
    for codes, d, x in zip((q8, k8, v8), ds, raw):
        assert d == float(x.abs().max()) / 448.0
        assert torch.equal(codes, (x / d).to(torch.float8_e4m3fn))


def test_sample_rows_cover_ends_and_tile_boundaries_of_every_head():
    w = Workload("s", 2, 3, 3, 300, 300, 64, 0)
    rows = sample_rows(w, n_random=50)
    assert rows == sorted(set(rows))
    assert all(0 <= r < 2 * 3 * 300 for r in rows)
    for bh in range(6):
        for i in (0, 127, 128, 129, 255, 256, 257, 299):
            assert bh * 300 + i in rows


def test_codelab_batch_sweep_and_sequence_sweep():
    bs = batch_sweep()
    assert [w.B for w in bs] == [1, 2, 4, 8, 16]
    assert all((w.Hq, w.Hkv, w.Sq, w.Sk, w.d, w.causal, w.layout) == (8, 8, 256, 256, 64, 0, "btnh")
               for w in bs)
    for causal in (False, True):
        ws = sweep(causal)
        assert [w.Sq for w in ws] == [512, 1024, 2048, 4096, 8192, 16384]
        assert all(w.B * w.Sq == 32768 and w.Sq == w.Sk for w in ws)

