"""Seeded synthetic workloads for segmented chunkwise gated linear attention.

This module only draws random inputs; it holds none of the method's arithmetic.  Both the
CUDA path and the fp64 oracle consume the exact tensors it returns (the oracle reads a host
copy of the already-rounded values).

The workloads follow the ZeCO operator benchmarks' setting (ZeCO review, referee major
comment 1 and Table 2: 16k tokens per device, H = 16, d_k = 128) with the sequence cut into
P segments on one GPU.  Distributions:

* ``toy``  -- q, k, v ~ N(0,1)/sqrt(d_k); log_g = logsigmoid(N(0,1)) / 16.
* ``gla``  -- q, k ~ N(0,1) then L2-normalised over d_k per (b, h, t) (fp32, eps 1e-12);
              v ~ N(0,1); log_g = logsigmoid(N(0,1) + 4), one gate per key dimension.
* ``weak`` -- as ``gla`` but log_g divided by 64, so that the decay over a 4096-token
              segment is about e^-1.9 and the state a segment receives matters.
* ``dO``   -- N(0,1) upstream gradient (backward workloads).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    dk: int
    dv: int
    P: int
    chunk: int
    dtype: str          # "f32" or "bf16": dtype of q, k, v, log_g, o and the gradients
    dist: str           # "toy", "gla" or "weak"
    backward: bool = False
    seed: int = 0

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def describe(self) -> str:
        return (f"{self.name}: {self.dtype} {'fwd+bwd' if self.backward else 'fwd'} B={self.B} "
                f"H={self.H} L={self.L} dk={self.dk} dv={self.dv} P={self.P} "
                f"({self.L // self.P} tok/segment) chunk={self.chunk} dist={self.dist}")

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "C0": Workload("C0", 1, 2, 256, 32, 32, 4, 16, "f32", "toy"),
    "C1": Workload("C1", 1, 16, 16384, 128, 128, 1, 64, "bf16", "gla"),
    "C2": Workload("C2", 1, 16, 131072, 128, 128, 8, 64, "bf16", "gla"),
    "C3": Workload("C3", 1, 16, 4194304, 128, 128, 256, 64, "bf16", "gla"),
    "C4": Workload("C4", 2, 16, 131072, 128, 128, 8, 64, "bf16", "gla", backward=True),
    # not benchmark workloads: the cross-segment scan under weak decay (tests), and a 16k-token
    # fwd+bwd case for kernel profiles (inputs larger than L2, a few hundred MB in all)
    "WEAK": Workload("WEAK", 1, 4, 16384, 128, 128, 4, 64, "bf16", "weak"),
    "BWD16K": Workload("BWD16K", 1, 16, 16384, 128, 128, 1, 64, "bf16", "gla", backward=True),
}


def _draw(gen, shape, device, mean=0.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return x + mean if mean else x


def make_inputs(w: Workload, device="cpu", with_s0: bool = False, slab_tokens: int = 1 << 20):
    """Return dict(q, k, v, log_g[, S0][, dO]) on ``device`` in the workload's dtype.

    Tensors are drawn per (b, h) slab of at most ``slab_tokens`` tokens in a fixed order from
    one torch.Generator seeded with ``w.seed``, so large workloads never hold an fp32 copy of
    a whole tensor.  S0 (fp32 [B,H,dk,dv], N(0,1)/sqrt(dk)) is drawn only when asked for.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.torch_dtype
    B, H, L, dk, dv = w.B, w.H, w.L, w.dk, w.dv
    out = {name: torch.empty((B, H, L, d), dtype=dt, device=device)
           for name, d in (("q", dk), ("k", dk), ("v", dv), ("log_g", dk))}
    if w.backward:
        out["dO"] = torch.empty((B, H, L, dv), dtype=dt, device=device)
    for b in range(B):
        for h in range(H):
            for t0 in range(0, L, slab_tokens):
                t1 = min(L, t0 + slab_tokens)
                n = t1 - t0
                if w.dist == "toy":
                    s = 1.0 / math.sqrt(dk)
                    out["q"][b, h, t0:t1] = (_draw(gen, (n, dk), device) * s).to(dt)
                    out["k"][b, h, t0:t1] = (_draw(gen, (n, dk), device) * s).to(dt)
                    out["v"][b, h, t0:t1] = (_draw(gen, (n, dv), device) * s).to(dt)
                    out["log_g"][b, h, t0:t1] = (F.logsigmoid(_draw(gen, (n, dk), device)) / 16).to(dt)
                else:
                    out["q"][b, h, t0:t1] = F.normalize(_draw(gen, (n, dk), device), dim=-1, eps=1e-12).to(dt)
                    out["k"][b, h, t0:t1] = F.normalize(_draw(gen, (n, dk), device), dim=-1, eps=1e-12).to(dt)
                    out["v"][b, h, t0:t1] = _draw(gen, (n, dv), device).to(dt)
                    lg = F.logsigmoid(_draw(gen, (n, dk), device, mean=4.0))
                    if w.dist == "weak":
                        lg = lg / 64
                    out["log_g"][b, h, t0:t1] = lg.to(dt)
                if w.backward:
                    out["dO"][b, h, t0:t1] = _draw(gen, (n, dv), device).to(dt)
    if with_s0:
        out["S0"] = torch.randn((B, H, dk, dv), generator=gen, device=device,
                                dtype=torch.float32) / math.sqrt(dk)
    return out
