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
