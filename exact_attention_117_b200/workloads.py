"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module holds shapes and random draws only -- none of the attention
arithmetic -- so that the CUDA path and the CPU oracle can consume the very
same tensors without sharing any computation.

Workloads (the pages measure no public dataset; every input is i.i.d.
N(0, 1) drawn in float32 and rounded to bf16):

* ``c1``  B=1,  H=1,  N=256,   d=64,  non-causal, plus the page-3 scalar case
  and a +500 logit-shift copy.
* ``c2``  B=4,  H=16, N=2048,  d=64,  full and causal; also N=1000 (ragged).
* ``c3``  B=2,  H=16, N=4096,  d=128, causal forward + backward.
* ``c4``  B=1,  H=32, N=16384, d=128, causal forward + backward, Q times 4.
* ``c5``  d in {64, 128}, N in {512 .. 8192}, B*H*N = 2**20 with H=16.

Seeds: Q=0, K=1, V=2, dO=3, each offset by 100 * (config index).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = ["Workload", "WORKLOADS", "sweep_workloads", "make_inputs",
           "scalar_case", "shift_copy", "sample_slices", "SHIFT"]

# logit shift of the stability test (page 2, section 动手实现, item 3)
SHIFT = 500.0


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: tuple = (False,)
    q_mult: float = 1.0
    seed_base: int = 0
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> str:
        c = "/".join("causal" if x else "full" for x in self.causal)
        qm = f" Q*{self.q_mult:g}" if self.q_mult != 1.0 else ""
        return f"B={self.B} H={self.H} N={self.N} d={self.d} {c}{qm}"


WORKLOADS = {
    "c1": Workload("c1", 1, 1, 256, 64, (False,), seed_base=0),
    "c2": Workload("c2", 4, 16, 2048, 64, (False, True), seed_base=100),
    "c2r": Workload("c2r", 4, 16, 1000, 64, (False, True), seed_base=100),
    "c3": Workload("c3", 2, 16, 4096, 128, (True,), seed_base=200),
    "c4": Workload("c4", 1, 32, 16384, 128, (True,), q_mult=4.0, seed_base=300),
}


def sweep_workloads():
    """The B*H*N = 2**20 sweep (H = 16) for d in {64, 128}."""
    out = []
    for d in (64, 128):
        for n in (512, 1024, 2048, 4096, 8192):
            b = (1 << 20) // (16 * n)
            out.append(Workload(f"c5_d{d}_n{n}", b, 16, n, d, (False, True),
                                seed_base=400))
    return out


def _randn(shape, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def make_inputs(w: Workload, device="cpu", with_do: bool = True, n: int | None = None):
    """bf16 ``q, k, v`` (and ``do``) of shape ``[B, H, N, d]``, contiguous."""
    n = w.N if n is None else n
    shape = (w.B, w.H, n, w.d)
    q = _randn(shape, w.seed_base + 0, device)
    if w.q_mult != 1.0:
        q = q * w.q_mult                      # a power of two: exact in bf16
    out = {"q": q.contiguous(),
           "k": _randn(shape, w.seed_base + 1, device),
           "v": _randn(shape, w.seed_base + 2, device)}
    if with_do:
        out["do"] = _randn(shape, w.seed_base + 3, device)
    return out


def scalar_case(d: int = 64, device="cpu"):
    """The page-3 scalar example embedded in a d-wide, N=2 problem.

    One query ``e0``; keys ``0`` and ``e0``; scale ``ln 2`` -> scores
    ``[0, ln 2]``.  Values ``10 e0`` and ``20 e0``.  Returns q, k, v of shape
    ``[1, 1, 2, d]`` (the second query row repeats the first) and the scale.
    """
    q = torch.zeros(1, 1, 2, d)
    k = torch.zeros(1, 1, 2, d)
    v = torch.zeros(1, 1, 2, d)
    q[0, 0, :, 0] = 1.0
    k[0, 0, 1, 0] = 1.0
    v[0, 0, 0, 0] = 10.0
    v[0, 0, 1, 0] = 20.0
    bf = torch.bfloat16
    return (q.to(bf).to(device), k.to(bf).to(device), v.to(bf).to(device),
            math.log(2.0))


def shift_copy(q: torch.Tensor, k: torch.Tensor, scale: float, shift: float = SHIFT):
    """Base and shifted copies whose logits differ by exactly ``shift``.

    Column d-1 is zeroed in the base copy; the shifted copy sets
    ``K[..., d-1] = 1`` and ``Q[..., d-1] = shift / scale``, which is exact in
    bf16 for the workloads used (500 * 8 = 4000).
    """
    qb, kb = q.clone(), k.clone()
    qb[..., -1] = 0
    kb[..., -1] = 0
    qs, ks = qb.clone(), kb.clone()
    qs[..., -1] = shift / scale
    ks[..., -1] = 1.0
    if float(qs[..., -1].flatten()[0]) != shift / scale:
        raise ValueError("shift / scale is not exact in bf16")
    return (qb, kb), (qs, ks)


def sample_slices(bh: int, count: int, seed: int = 1234):
    """Seeded subset of (batch*head) slice indices for the large configs."""
    import numpy as np
    rng = np.random.default_rng(seed)
    count = min(count, bh)
    return sorted(int(x) for x in rng.choice(bh, size=count, replace=False))
