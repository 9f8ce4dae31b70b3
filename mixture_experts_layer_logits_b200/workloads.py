"""Seeded synthetic inputs for the MoE layer forward.

This module only draws random numbers: it holds none of the layer's arithmetic,
and it is the one piece of code that both the CUDA path's callers and the CPU
oracle's callers share.

Workloads (shapes and value distributions of the layer problem):

=================  =====  =====  =====  =====  =====  ==========================================
name                 T      E      k      H      I     logits
=================  =====  =====  =====  =====  =====  ==========================================
tiny                 16      8      2    256    512    N(0,1)
decode                8    128      8   2048    768    N(0,1)
skewed_decode        64    256      8   7168   2048    N(0,1) + 2*ln(Zipf(s=1.2) weight of expert)
routing_stress    16384   1024      8      -      -    N(0,1), 1% of entries copied from the same row
prefill            8192    128      8   4096   1536    N(0,1)
=================  =====  =====  =====  =====  =====  ==========================================

x ~ N(0,1) rounded to bf16; w13 [E,2I,H] ~ N(0, std=1/sqrt(H)) and w2 [E,H,I] ~
N(0, std=1/sqrt(I)), drawn in fp32 then rounded to bf16.  Every tensor has its
own torch.Generator on the target device, seeded from (seed, tensor tag), so a
tensor does not depend on which others were drawn.  Values therefore depend on
the device type (CPU and CUDA generators differ); the oracle is always handed
host copies of the exact tensors the GPU path consumed.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    E: int
    k: int
    H: int = 0           # 0: routing-only workload (no expert FFN)
    I: int = 0
    zipf_s: float = 0.0  # > 0: add 2*ln(Zipf(s) weight of the expert's rank) to every logit
    dup_frac: float = 0.0
    notes: str = field(default="", compare=False)

    @property
    def R(self) -> int:
        return self.T * self.k

    @property
    def has_ffn(self) -> bool:
        return self.H > 0 and self.I > 0

    def as_dict(self) -> dict:
        d = dict(workload=self.name, T=self.T, E=self.E, top_k=self.k)
        if self.has_ffn:
            d.update(H=self.H, I=self.I)
        if self.zipf_s:
            d["logit_bias"] = f"2*ln(Zipf(s={self.zipf_s}))"
        if self.dup_frac:
            d["dup_frac"] = self.dup_frac
        return d


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 16, 8, 2, 256, 512),
        Workload("decode", 8, 128, 8, 2048, 768),
        Workload("skewed_decode", 64, 256, 8, 7168, 2048, zipf_s=1.2),
        Workload("routing_stress", 16384, 1024, 8, dup_frac=0.01),
        Workload("prefill", 8192, 128, 8, 4096, 1536),
    ]
}

_TAG_LOGITS, _TAG_DUP, _TAG_X, _TAG_W13, _TAG_W2 = 1, 2, 3, 4, 5


def _gen(device, seed: int, tag: int) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed) * 1_000_003 + tag)
    return g


def zipf_bias(E: int, s: float) -> torch.Tensor:
    """2*ln(p_e) with p_e = (e+1)^-s / sum_r r^-s (expert 0 is the hottest)."""
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p = ranks.pow(-s)
    p = p / p.sum()
    return (2.0 * torch.log(p)).to(torch.float32)


def make_logits(w: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """fp32 [T,E] router logits."""
    g = _gen(device, seed, _TAG_LOGITS)
    logits = torch.randn(w.T, w.E, generator=g, device=device, dtype=torch.float32)
    if w.zipf_s:
        logits += zipf_bias(w.E, w.zipf_s).to(device)
    if w.dup_frac:
        gd = _gen(device, seed, _TAG_DUP)
        pick = torch.rand(w.T, w.E, generator=gd, device=device) < w.dup_frac
        # source column drawn uniformly from the other E-1 columns of the same row
        src = torch.randint(0, w.E - 1, (w.T, w.E), generator=gd, device=device)
        col = torch.arange(w.E, device=device).expand(w.T, w.E)
        src = src + (src >= col).to(src.dtype)
        logits = torch.where(pick, torch.gather(logits, 1, src), logits)
    return logits.contiguous()


def make_x(w: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """bf16 [T,H] activations."""
    g = _gen(device, seed, _TAG_X)
    return torch.randn(w.T, w.H, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def make_expert_weights(w: Workload, e: int, seed: int = 0, device="cpu"):
    """(w13[e] bf16 [2I,H], w2[e] bf16 [H,I]) of one expert; each expert has its own
    generator, so one expert can be drawn without the others."""
    g13 = _gen(device, seed * 65_537 + e, _TAG_W13)
    g2 = _gen(device, seed * 65_537 + e, _TAG_W2)
    a = (torch.randn(2 * w.I, w.H, generator=g13, device=device) / math.sqrt(w.H))
    b = (torch.randn(w.H, w.I, generator=g2, device=device) / math.sqrt(w.I))
    return a.to(torch.bfloat16), b.to(torch.bfloat16)


def make_weights(w: Workload, seed: int = 0, device="cpu"):
    """(w13 bf16 [E,2I,H], w2 bf16 [E,H,I]), drawn one expert at a time."""
    w13 = torch.empty(w.E, 2 * w.I, w.H, dtype=torch.bfloat16, device=device)
    w2 = torch.empty(w.E, w.H, w.I, dtype=torch.bfloat16, device=device)
    for e in range(w.E):
        w13[e], w2[e] = make_expert_weights(w, e, seed, device)
    return w13, w2


E4M3_MAX = 448.0  # largest finite E4M3 (E4M3FN) value


def quantize_e4m3_rows(t: torch.Tensor):
    """Symmetric per-row E4M3 quantisation of a [..., rows, cols] weight tensor:
    scale = max|row| / 448 (1 for an all-zero row), codes = the E4M3 value nearest
    to w / scale.  Returns (codes uint8 [..., rows, cols], scales float32
    [..., rows]).  Input preparation only: the layer reads codes and scales."""
    tf = t.float()
    amax = tf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    q = (tf / scale.unsqueeze(-1)).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), scale


def make_weights_w8(w: Workload, seed: int = 0, device="cpu"):
    """FP8 copies of make_weights' draws, quantised one expert at a time:
    (q13 uint8 [E,2I,H], s13 f32 [E,2I], q2 uint8 [E,H,I], s2 f32 [E,H])."""
    q13 = torch.empty(w.E, 2 * w.I, w.H, dtype=torch.uint8, device=device)
    s13 = torch.empty(w.E, 2 * w.I, dtype=torch.float32, device=device)
    q2 = torch.empty(w.E, w.H, w.I, dtype=torch.uint8, device=device)
    s2 = torch.empty(w.E, w.H, dtype=torch.float32, device=device)
    for e in range(w.E):
        a, b = make_expert_weights(w, e, seed, device)
        q13[e], s13[e] = quantize_e4m3_rows(a)
        q2[e], s2[e] = quantize_e4m3_rows(b)
    return q13, s13, q2, s2


def make_inputs(w: Workload, seed: int = 0, device="cpu", weights: bool = True) -> dict:
    d = dict(logits=make_logits(w, seed, device))
    if w.has_ffn:
        d["x"] = make_x(w, seed, device)
        if weights:
            d["w13"], d["w2"] = make_weights(w, seed, device)
    return d


def custom(name: str, T: int, E: int, k: int, H: int = 0, I: int = 0, zipf_s: float = 0.0,
           dup_frac: float = 0.0) -> Workload:
    """An ad-hoc shape (edge cases in tests) with the same distributions."""
    return Workload(name, T, E, k, H, I, zipf_s, dup_frac)


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor's bit patterns (for the oracle)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
