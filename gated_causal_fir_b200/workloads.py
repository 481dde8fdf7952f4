"""Seeded synthetic workloads for the gated causal FIR (Hyena-SE / Hyena-MR forward).

This module holds the workload table and the seeded input generators, and nothing of the
convolution itself: both the CUDA path's tests/bench and the fp64 oracle receive the tensors
it makes.  It imports neither side.

Recipes (StripedHyena 2 operator classes; the pages fix no distributions, so these are the
stated synthetic ones):

* q, k, v ~ N(0, 1), drawn in fp32 and rounded to nearest-even bf16 (fp32 kept for ``tiny``).
* short explicit filters (SE, tiny): h ~ N(0, 1/l_h), the second argument read as a variance.
* medium regularised filters (MR): h[g, t] = w[g, t] * exp(-alpha_g * t), t = 0 .. l_h-1, with
  w ~ N(0, 1/sqrt(l_h)) (variance) and alpha_g ~ U[0.01, 0.1] drawn once per group.
* filters are fp32, shape [G = D / d_g, l_h], natural tap order.

Draw order is q, k, v, then the filter tensors, from one ``torch.Generator`` seeded with the
workload's seed on the device the tensors are made on.
"""
from dataclasses import dataclass, asdict
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int
    D: int
    d_g: int
    l_h: int
    l_b: int
    dtype: str          # "f32" or "bf16" for q, k, v, y
    filt: str           # "se" (Gaussian) or "mr" (decayed Gaussian)
    seed: int

    @property
    def G(self) -> int:
        return self.D // self.d_g

    @property
    def tokens(self) -> int:
        return self.B * self.L

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def algorithmic_bytes(self) -> int:
        """Bytes the method must move once: q, k, v read, y written, plus the filters."""
        return 4 * self.B * self.L * self.D * self.elem_bytes + self.G * self.l_h * 4

    def algorithmic_flops(self) -> int:
        """Direct-form flops: l_h multiply-adds per output, plus the k*v and q gates."""
        return (2 * self.l_h + 2) * self.B * self.L * self.D

    def describe(self) -> str:
        return ("%s: B=%d L=%d D=%d d_g=%d l_h=%d l_b=%d %s"
                % (self.name, self.B, self.L, self.D, self.d_g, self.l_h, self.l_b, self.dtype))

    def as_dict(self):
        return asdict(self)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1024, 64, 16, 7, 16, "f32", "se", 0),
    "se": Workload("se", 1, 8192, 4096, 16, 7, 16, "bf16", "se", 1),
    "mr": Workload("mr", 1, 8192, 4096, 64, 128, 64, "bf16", "mr", 2),
    "mr_batched": Workload("mr_batched", 8, 32768, 4096, 64, 128, 64, "bf16", "mr", 3),
    "mr_1m": Workload("mr_1m", 1, 1 << 20, 4096, 64, 128, 64, "bf16", "mr", 4),
    # long filters (the Hyena-LI class): filter as long as the sequence, decayed like MR's
    "li": Workload("li", 1, 8192, 4096, 64, 8192, 64, "bf16", "mr", 5),
}


def torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def make_filters(G: int, l_h: int, kind: str, gen: torch.Generator, device) -> torch.Tensor:
    """Filters [G, l_h] fp32 by the recipe named ``kind`` ("se" or "mr")."""
    if kind == "se":
        return torch.randn(G, l_h, generator=gen, device=device) * math.sqrt(1.0 / l_h)
    if kind == "mr":
        w = torch.randn(G, l_h, generator=gen, device=device) * (l_h ** -0.25)
        alpha = torch.rand(G, 1, generator=gen, device=device) * 0.09 + 0.01
        t = torch.arange(l_h, device=device, dtype=torch.float32)[None, :]
        return (w * torch.exp(-alpha * t)).contiguous()
    raise ValueError("unknown filter recipe %r" % kind)


def make_inputs(wl: Workload, device="cpu", seed=None, l_slice: int = 0):
    """q, k, v [B, L, D] in the workload's dtype and h [G, l_h] fp32, seeded.

    ``l_slice`` > 0 draws q, k, v in slices of that many time rows (each slice from its own
    generator seeded (seed, slice)), which bounds the fp32 temporaries for the 1M-token case.
    """
    seed = wl.seed if seed is None else seed
    dt = torch_dtype(wl.dtype)
    shape = (wl.B, wl.L, wl.D)
    if l_slice <= 0 or l_slice >= wl.L:
        gen = torch.Generator(device=device).manual_seed(seed)
        q, k, v = (torch.randn(shape, generator=gen, device=device).to(dt) for _ in range(3))
    else:
        q, k, v = (torch.empty(shape, dtype=dt, device=device) for _ in range(3))
        gen = torch.Generator(device=device)
        for s, t0 in enumerate(range(0, wl.L, l_slice)):
            t1 = min(wl.L, t0 + l_slice)
            gen.manual_seed(seed * 1000003 + s)
            for dst in (q, k, v):
                dst[:, t0:t1].copy_(torch.randn((wl.B, t1 - t0, wl.D), generator=gen,
                                                device=device))
        gen.manual_seed(seed)
    h = make_filters(wl.G, wl.l_h, wl.filt, gen, device)
    return q, k, v, h


def make_grad(wl: Workload, device="cpu", seed=None):
    """Upstream gradient dy [B, L, D] in the workload's dtype, standard normal, seeded apart
    from the forward inputs (seed + 7919)."""
    seed = (wl.seed if seed is None else seed) + 7919
    gen = torch.Generator(device=device).manual_seed(seed)
    return torch.randn((wl.B, wl.L, wl.D), generator=gen, device=device).to(
        torch_dtype(wl.dtype))


def make_integer_inputs(wl: Workload, device="cpu", seed=None):
    """q, k, v, dy with integer values in [-2, 2] and h with integers in [-3, 3], seeded.

    Every product and partial sum of the forward and backward is then an integer well inside
    the fp16/fp32 exact range (for B * L * d_g * 16 < 2**24), so any correct summation order
    gives the exact result and the GPU path must match the oracle bit for bit.
    """
    seed = wl.seed if seed is None else seed
    gen = torch.Generator(device=device).manual_seed(seed + 104729)
    shape = (wl.B, wl.L, wl.D)
    dt = torch_dtype(wl.dtype)
    q, k, v, dy = (torch.randint(-2, 3, shape, generator=gen, device=device).to(dt)
                   for _ in range(4))
    h = torch.randint(-3, 4, (wl.G, wl.l_h), generator=gen, device=device).to(torch.float32)
    return q, k, v, dy, h


def custom(name="custom", B=1, L=256, D=128, d_g=64, l_h=16, l_b=16, dtype="bf16", filt="se",
           seed=7) -> Workload:
    """A workload outside the table (edge cases in the tests)."""
    return Workload(name, B, L, D, d_g, l_h, l_b, dtype, filt, seed)
