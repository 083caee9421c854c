"""Seeded synthetic workloads for the fused SDPA forward.

This module only draws inputs: it holds none of the attention arithmetic, and
both sides of every parity check (the CUDA library and the CPU oracle) receive
the same tensors from it.  Shapes and value distributions stand in for the
workloads on the pages (the codelab's B/T/S/N/H sweeps, section 3 and 8; its
MHA/GQA/MQA comparison, section 9; its FP8 check, section 10; the article's
ViT-B/16 example, 196 tokens and 12 heads, section 1).  No dataset is used.

Recipe: ``torch.Generator('cpu').manual_seed(seed)``, then Q, K, V drawn in
that order as fp32 N(0,1) and rounded to the storage dtype by torch's cast
(round to nearest even).  FP8 inputs: fp32 N(0,1) per tensor, per-tensor
descale = amax(|x|) / 448, codes = e4m3fn(x / descale) by torch's cast;
output gradients for the FP8 backward: per-tensor descale = amax(|x|) / 57344,
codes = e5m2(x / descale).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Sk: int
    d: int
    causal: int             # 0 none, 1 causal (Sq == Sk), 2 aligned to the end of the keys
    dtype: str = "bf16"     # "bf16", "fp16" or "e4m3"
    seed: int = 0
    layout: str = "bhsd"    # "bhsd": [B,H,S,d] tensors; "btnh": [B,S,H,d] data passed as views

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs of the two contractions, 4*B*Hq*Sq*Sk*d, halved
        when causal (the masked half of the score matrix is not work); for
        the mask aligned to the end of the keys (causal == 2) the visible
        (query, key) pairs are counted exactly."""
        if self.causal == 2:
            pairs = self.Sq * (self.Sk - self.Sq) + self.Sq * (self.Sq + 1) / 2.0
            return 4.0 * self.B * self.Hq * pairs * self.d
        f = 4.0 * self.B * self.Hq * self.Sq * self.Sk * self.d
        return f / 2.0 if self.causal else f

    @property
    def elem_bytes(self) -> int:
        return 1 if self.dtype == "e4m3" else 2

    @property
    def min_hbm_bytes(self) -> int:
        """Q, K, V read once, O (2-byte) and LSE (fp32) written once."""
        eb = self.elem_bytes
        q = self.B * self.Hq * self.Sq * self.d * eb
        kv = 2 * self.B * self.Hkv * self.Sk * self.d * eb
        o = self.B * self.Hq * self.Sq * self.d * 2
        lse = self.B * self.Hq * self.Sq * 4
        return q + kv + o + lse

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "Hq": self.Hq, "Hkv": self.Hkv,
                "Sq": self.Sq, "Sk": self.Sk, "d": self.d, "causal": self.causal,
                "dtype": self.dtype, "seed": self.seed}


WORKLOADS = {
    "tiny": Workload("tiny_b1_h2_s128_d64", 1, 2, 2, 128, 128, 64, False, seed=0),
    "vit": Workload("vit_b16_b32_h12_s196_d64", 32, 12, 12, 196, 196, 64, False, seed=196),
    "lm_causal": Workload("lm_causal_b8_h16_s4096_d128", 8, 16, 16, 4096, 4096, 128, True,
                          seed=4096),
    "gqa": Workload("gqa_b4_hq32_hkv8_s8192_d128_causal", 4, 32, 8, 8192, 8192, 128, True,
                    seed=42),
    "mqa": Workload("mqa_b4_hq32_hkv1_s8192_d128_causal", 4, 32, 1, 8192, 8192, 128, True,
                    seed=42),
    "fp8": Workload("fp8_b2_h32_s16384_d128_causal", 2, 32, 32, 16384, 16384, 128, True,
                    dtype="e4m3", seed=9000),
    # decode-shaped GQA: one new token per sequence against an 8192-key cache
    # (the codelab's KV-cache motivation, section 9); query heads packed
    "decode_gqa": Workload("decode_gqa_b64_hq32_hkv8_sq1_sk8192_d128", 64, 32, 8, 1, 8192, 128, 2,
                           seed=8192),
    # profiling-sized cases: inputs above the 126 MB L2, a few hundred MB in all
    "lm_causal_b4": Workload("lm_causal_b4_h16_s4096_d128", 4, 16, 16, 4096, 4096, 128, True,
                             seed=4096),
    "lm_full_b4": Workload("lm_full_b4_h16_s4096_d128", 4, 16, 16, 4096, 4096, 128, False,
                           seed=4096),
}


def sweep(causal: bool, tokens: int = 32768, heads: int = 16, d: int = 128):
    """Fixed B*S = tokens sweep over S in {512 .. 16384} (the codelab's
    sequence sweep, section 8, scaled to B200 sizes)."""
    out = []
    for s in (512, 1024, 2048, 4096, 8192, 16384):
        out.append(Workload("sweep_s%d_%s" % (s, "causal" if causal else "full"),
                            tokens // s, heads, heads, s, s, d, causal, seed=s))
    return out


def batch_sweep():
    """The codelab's batch-size sweep (section 8): B in {1, 2, 4, 8, 16},
    T = S = 256, N = 8 heads, head dim 64, no mask, seed B + 100, inputs in
    its [batch, time, heads, head_dim] layout."""
    return [Workload("bsweep_b%d_t256_n8_h64" % b, b, 8, 8, 256, 256, 64, False, seed=b + 100,
                     layout="btnh") for b in (1, 2, 4, 8, 16)]


WORKLOADS.update({"bsweep_b%d" % w.B: w for w in batch_sweep()})
# the sequence sweep's points by name (e.g. sweep_s16384_full), so that
# bench.py --workload can select one
WORKLOADS.update({w.name: w for causal in (False, True) for w in sweep(causal)})


def with_shape(w: Workload, **kw) -> Workload:
    return replace(w, **kw)


_TORCH_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}


def make_qkv(w: Workload, device="cpu"):
    """(q, k, v) for a bf16/fp16 workload, drawn on the CPU from w.seed and
    then moved to `device`."""
    if w.dtype not in _TORCH_DTYPES:
        raise ValueError("make_qkv: use make_qkv_fp8 for %s" % w.dtype)
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    dt = _TORCH_DTYPES[w.dtype]
    q = torch.randn(w.B, w.Hq, w.Sq, w.d, generator=g, dtype=torch.float32).to(dt)
    k = torch.randn(w.B, w.Hkv, w.Sk, w.d, generator=g, dtype=torch.float32).to(dt)
    v = torch.randn(w.B, w.Hkv, w.Sk, w.d, generator=g, dtype=torch.float32).to(dt)
    return q.to(device), k.to(device), v.to(device)


def make_inputs(w: Workload, device="cpu"):
    """(q, k, v) as [B,H,S,d] tensors for a bf16/fp16 workload: contiguous
    for layout "bhsd", transposed views of [B,S,H,d] data for "btnh"."""
    if w.layout == "btnh":
        return tuple(t.transpose(1, 2) for t in make_qkv_btnh(w, device))
    return make_qkv(w, device)


def make_qkv_btnh(w: Workload, device="cpu"):
    """(q, k, v) in the codelab's [batch, time, heads, head_dim] layout
    (q [B,Sq,Hq,d], k/v [B,Sk,Hkv,d]), drawn on the CPU from w.seed."""
    if w.dtype not in _TORCH_DTYPES:
        raise ValueError("make_qkv_btnh: bf16 / fp16 only, not %s" % w.dtype)
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    dt = _TORCH_DTYPES[w.dtype]
    q = torch.randn(w.B, w.Sq, w.Hq, w.d, generator=g, dtype=torch.float32).to(dt)
    k = torch.randn(w.B, w.Sk, w.Hkv, w.d, generator=g, dtype=torch.float32).to(dt)
    v = torch.randn(w.B, w.Sk, w.Hkv, w.d, generator=g, dtype=torch.float32).to(dt)
    return q.to(device), k.to(device), v.to(device)


E4M3_MAX = 448.0
E5M2_MAX = 57344.0


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor current scaling: descale = amax/448, codes = e4m3fn(x/descale)."""
    amax = float(x.abs().max())
    descale = amax / E4M3_MAX if amax > 0 else 1.0
    codes = (x / descale).to(torch.float8_e4m3fn)
    return codes, descale


def quantize_e5m2(x: torch.Tensor):
    """Per-tensor current scaling for gradients (the FP8 hybrid recipe's E5M2
    format): descale = amax/57344, codes = e5m2(x/descale) by torch's cast."""
    amax = float(x.abs().max())
    descale = amax / E5M2_MAX if amax > 0 else 1.0
    codes = (x / descale).to(torch.float8_e5m2)
    return codes, descale


def make_dout_e5m2(w: Workload, device="cpu"):
    """(do8, descale_do, do32): an output gradient of q's shape drawn as fp32
    N(0,1) from w.seed + 1 and quantised to e5m2."""
    g = torch.Generator(device="cpu").manual_seed(w.seed + 1)
    do = torch.randn(w.B, w.Hq, w.Sq, w.d, generator=g, dtype=torch.float32)
    do8, dd = quantize_e5m2(do)
    return do8.to(device), dd, do


def make_qkv_fp8(w: Workload, device="cpu"):
    """(q8, k8, v8, (dq, dk, dv), (q32, k32, v32)) for an e4m3 workload."""
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    q = torch.randn(w.B, w.Hq, w.Sq, w.d, generator=g, dtype=torch.float32)
    k = torch.randn(w.B, w.Hkv, w.Sk, w.d, generator=g, dtype=torch.float32)
    v = torch.randn(w.B, w.Hkv, w.Sk, w.d, generator=g, dtype=torch.float32)
    q8, dq = quantize_e4m3(q)
    k8, dk = quantize_e4m3(k)
    v8, dv = quantize_e4m3(v)
    return (q8.to(device), k8.to(device), v8.to(device), (dq, dk, dv), (q, k, v))


def sample_rows(w: Workload, n_random: int = 256, seed: int = 1234, tile: int = 128):
    """Flat row indices (b*Hq + hq)*Sq + i for sampled parity checks: for
    every (b, hq) the first and last rows and the rows around each multiple of
    the tile height, plus `n_random` seeded random rows overall."""
    rows = set()
    special = {0, w.Sq - 1}
    for t in range(tile, w.Sq, tile):
        special.update((t - 1, t, t + 1))
    special = sorted(i for i in special if 0 <= i < w.Sq)
    # keep the per-(b,h) set small at long sequence lengths
    if len(special) > 8:
        g = torch.Generator().manual_seed(seed + 1)
        pick = torch.randperm(len(special), generator=g)[:6].tolist()
        special = sorted({special[0], special[-1]} | {special[p] for p in pick})
    for bh in range(w.B * w.Hq):
        for i in special:
            rows.add(bh * w.Sq + i)
    g = torch.Generator().manual_seed(seed)
    total = w.B * w.Hq * w.Sq
    for r in torch.randint(0, total, (n_random,), generator=g).tolist():
        rows.add(int(r))
    return sorted(rows)
