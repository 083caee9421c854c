"""The C-ABI calls inside CUDA graphs: a forward or backward call made while
torch captures a stream is recorded as its kernel launches (the host work --
argument checks, tensor-map encoding -- runs at capture time), and replaying
the graph gives exactly the outputs of the eager call on the same inputs.
The kernels are deterministic, so the comparison is bit for bit."""
import pytest
import torch

from sdpa_workloads import Workload, make_qkv, make_qkv_fp8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sdpa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import scaled_dot_product_11_b200 as lib
    lib.sdpa_device_status(clear=True)
    return lib


def capture(fn, replays=2):
    """Eager warm-up, then fn captured once and replayed `replays` times;
    returns what fn returned during the capture (the graph's outputs)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        outs = fn()
    for _ in range(replays):
        g.replay()
    torch.cuda.synchronize()
    return g, outs


FWD = [
    Workload("graph_causal_d128", 2, 4, 2, 700, 700, 128, True, seed=31),
    Workload("graph_vit_d64", 4, 3, 3, 196, 196, 64, False, seed=32),
    Workload("graph_fp16_ragged", 1, 2, 2, 300, 450, 128, False, dtype="fp16", seed=33),
]


@pytest.mark.parametrize("w", FWD, ids=lambda w: w.name)
def test_forward_replays_bit_exact(sdpa, w):
    q, k, v = make_qkv(w, "cuda")
    o_ref, lse_ref = sdpa.attention(q, k, v, causal=w.causal, scale=w.scale)
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(lse_ref)
    g, _ = capture(lambda: sdpa.attention(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse))
    st, detail = sdpa.sdpa_device_status(clear=True)
    assert st == 0, "device status %d detail %#x" % (st, detail)
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    # new inputs copied into the captured buffers: the replay follows them
    q2, k2, v2 = make_qkv(Workload(w.name, w.B, w.Hq, w.Hkv, w.Sq, w.Sk, w.d, w.causal,
                                   dtype=w.dtype, seed=w.seed + 100), "cuda")
    q.copy_(q2), k.copy_(k2), v.copy_(v2)
    g.replay()
    o2, lse2 = sdpa.attention(q2, k2, v2, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_fp8_forward_replays_bit_exact(sdpa):
    w = Workload("graph_fp8", 1, 4, 4, 512, 512, 128, True, dtype="e4m3", seed=34)
    q, k, v, ds, _ = make_qkv_fp8(w, "cuda")
    o_ref, lse_ref = sdpa.attention_fp8(q, k, v, ds, causal=True, scale=w.scale)
    o, lse = torch.empty_like(o_ref), torch.empty_like(lse_ref)
    capture(lambda: sdpa.attention_fp8(q, k, v, ds, causal=True, scale=w.scale, out=o, lse=lse))
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_backward_replays_bit_exact(sdpa):
    w = Workload("graph_bwd", 1, 4, 2, 384, 384, 128, True, seed=35)
    q, k, v = make_qkv(w, "cuda")
    g0 = torch.Generator(device="cpu").manual_seed(36)
    dout = torch.randn(q.shape, generator=g0).to(q.dtype).cuda()
    o, lse = sdpa.attention(q, k, v, causal=True, scale=w.scale)
    ref = sdpa.attention_backward(q, k, v, o, lse, dout, causal=True, scale=w.scale)
    _, got = capture(lambda: sdpa.attention_backward(q, k, v, o, lse, dout, causal=True,
                                                     scale=w.scale))
    st, detail = sdpa.sdpa_device_status(clear=True)
    assert st == 0, "device status %d detail %#x" % (st, detail)
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
