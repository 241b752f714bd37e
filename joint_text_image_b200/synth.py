"""Seeded synthetic inputs for the attention workloads.

This module holds no attention, mask or RoPE arithmetic: it only draws
sequence lengths and bf16 normal tensors from a seeded torch CPU generator.
Both the CUDA path (tests, bench) and the oracle (tests) are fed from here.

Shapes follow the HunyuanImage-3.0 pages: the cache contract lays a sample out
as prefix (ending in <timestep>) + h*w image tokens + suffix, right-padded to
the batch maximum; 1024px images give 64x64 = 4096 tokens through the 16x
VAE; aspect ratios span 1:4 to 4:1; the classifier-free-guidance prefix is a
run of <cfg> tokens.  No dataset is used: the pages train on private image
caches, so these draws stand in for them.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass
class Workload:
    name: str
    samples: list            # per batch row: (prefix, img_h, img_w, suffix) or (images, suffix)
    Hq: int
    Hkv: int
    D: int
    S: int                   # padded length = max over samples of prefix + h*w + suffix
    base: float = 10000.0
    backward: bool = False
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def B(self):
        return len(self.samples)

    @property
    def scale(self):
        return self.D ** -0.5


def _draw(gen, lo, hi, n):
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=gen)]


def _length(x):
    """Valid length of a sample: (prefix, h, w, suffix), or (images, suffix)
    with images a list of (text_before, h, w)."""
    if len(x) == 2:
        return sum(t + h * w for (t, h, w) in x[0]) + x[1]
    p, h, w, s = x
    return p + h * w + s


def _finish(name, samples, Hq, Hkv, D, **kw):
    S = max(_length(x) for x in samples) if samples else 0
    return Workload(name=name, samples=samples, Hq=Hq, Hkv=Hkv, D=D, S=S, **kw)


def workload(name: str, seed: int = 0) -> Workload:
    """The synthetic workloads; lengths drawn from torch.Generator(seed)."""
    gen = torch.Generator().manual_seed(seed)
    if name == "tiny":
        # 15 text + <timestep> = prefix 16; 8x8 image; suffix 2; no padding.
        return _finish(name, [(16, 8, 8, 2)], 4, 1, 64, note="S=82")
    if name == "256px":
        # prefixes U[64,256] for three rows; one row uses a 32-token <cfg>
        # unconditional prefix (+ <timestep> = 33); 16x16 image; suffix 2.
        pre = _draw(gen, 64, 256, 3)
        samples = [(pre[0], 16, 16, 2), (33, 16, 16, 2), (pre[1], 16, 16, 2), (pre[2], 16, 16, 2)]
        return _finish(name, samples, 32, 8, 128)
    if name == "1024px":
        pre = _draw(gen, 512, 1536, 2)
        return _finish(name, [(p, 64, 64, 2) for p in pre], 32, 8, 128)
    if name == "mixed":
        # grids 32x128 (1:4), 128x32 (4:1), 48x80, plus a text-only 2048 row.
        pre = _draw(gen, 128, 1024, 3)
        samples = [(pre[0], 32, 128, 2), (pre[1], 128, 32, 2), (pre[2], 48, 80, 2),
                   (2048, 0, 0, 0)]
        return _finish(name, samples, 32, 8, 128)
    if name == "1024px_bwd":
        return _finish(name, [(1024, 64, 64, 2)], 32, 8, 128, backward=True)
    if name == "multi_image":
        # two generated images per sample: prefix U[256,768], a 512px image
        # (32x32 tokens, in context for what follows), a 64-token caption,
        # a 1024px image (64x64), suffix 2.
        pre = _draw(gen, 256, 768, 2)
        samples = [([(p, 32, 32), (64, 64, 64)], 2) for p in pre]
        return _finish(name, samples, 32, 8, 128, backward=True)
    raise KeyError(name)


WORKLOADS = ("tiny", "256px", "1024px", "mixed", "1024px_bwd", "multi_image")


def tensors(wl: Workload, seed: int = 0, grad: bool = False):
    """bf16 ~N(0,1) q [B,S,Hq,D], k, v [B,S,Hkv,D] (and dout [B,S,Hq,D]) on CPU."""
    gen = torch.Generator().manual_seed(seed + 1)
    B, S = wl.B, wl.S
    q = torch.randn(B, S, wl.Hq, wl.D, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, S, wl.Hkv, wl.D, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, S, wl.Hkv, wl.D, generator=gen).to(torch.bfloat16)
    if not grad:
        return q, k, v
    do = torch.randn(B, S, wl.Hq, wl.D, generator=gen).to(torch.bfloat16)
    return q, k, v, do


def custom(samples, Hq, Hkv, D, S=None, name="custom") -> Workload:
    wl = _finish(name, list(samples), Hq, Hkv, D)
    if S is not None:
        wl.S = S
    return wl


# ---------------------------------------------------------------- MoE feed-forward
@dataclass
class MoeWorkload:
    """Sizes of one MoE feed-forward call: T tokens, hidden H, expert
    intermediate I, E routed experts of which topk per token, plus the shared
    expert.  The pages fix E = 64 and topk = 8 (technical report summary
    3.1.1); they give neither H nor I: H = 4096 is the attention's 32 heads x
    128, and I = 3072 is a reading (with 32 layers it matches both the 80B
    total and the 13B active parameters the pages quote)."""
    name: str
    T: int
    H: int
    I: int
    E: int
    topk: int
    note: str = ""


def moe_workload(name: str, seed: int = 0) -> MoeWorkload:
    if name == "moe_tiny":
        return MoeWorkload(name, 300, 256, 128, 8, 2, note="every shape one or two tiles, ragged token count")
    if name == "moe_mid":
        return MoeWorkload(name, 1000, 512, 256, 64, 8, note="the pages' routing (64 experts, top-8), small dims")
    if name == "moe_e16":
        # the benchmark's H and I with 16 experts, top-4, 4096 tokens: 1.3 GB of
        # weights (still well above L2), small enough for a full profiler capture
        return MoeWorkload(name, 4096, 4096, 3072, 16, 4, note="profiling size: bench dims, fewer experts")
    if name == "moe_1024px":
        # the valid tokens of the 1024px attention workload's batch (two
        # samples: prefix + 64x64 image + 2 suffix tokens each), packed
        wl = workload("1024px", seed)
        T = sum(p + h * w + s for (p, h, w, s) in wl.samples)
        return MoeWorkload(name, T, 4096, 3072, 64, 8, note="tokens of the 1024px batch, packed")
    raise KeyError(name)


MOE_WORKLOADS = ("moe_tiny", "moe_mid", "moe_e16", "moe_1024px")


def moe_tensors(mw: MoeWorkload, seed: int = 0):
    """x bf16 [T, H] ~ N(0, 1) (the block's RMS-normed hidden states have unit
    RMS); router weight fp32 [E, H] ~ N(0, 1/H), so logits ~ N(0, 1); w13 bf16
    [E + 1, 2I, H] ~ N(0, 1/H) and w2 bf16 [E + 1, H, I] ~ N(0, 1/I) (index E:
    the shared expert), so every projection keeps unit scale.  CPU tensors
    from a seeded generator, one expert at a time."""
    gen = torch.Generator().manual_seed(seed + 101)
    x = torch.randn(mw.T, mw.H, generator=gen).to(torch.bfloat16)
    wg = torch.randn(mw.E, mw.H, generator=gen) * mw.H ** -0.5
    w13 = torch.empty(mw.E + 1, 2 * mw.I, mw.H, dtype=torch.bfloat16)
    w2 = torch.empty(mw.E + 1, mw.H, mw.I, dtype=torch.bfloat16)
    for e in range(mw.E + 1):
        w13[e] = (torch.randn(2 * mw.I, mw.H, generator=gen) * mw.H ** -0.5).to(torch.bfloat16)
        w2[e] = (torch.randn(mw.H, mw.I, generator=gen) * mw.I ** -0.5).to(torch.bfloat16)
    return x, wg, w13, w2
