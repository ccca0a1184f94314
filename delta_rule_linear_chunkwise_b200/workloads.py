"""Seeded synthetic inputs for the chunkwise gated delta-rule operator.

This module only draws random numbers; it holds none of the operator's
arithmetic, so both the CUDA path and the fp64 oracle can be fed from it.

Recipe (the workloads the ReWY / GDN / KDA / KLA abstracts are about, sized as
below): q and k ~ N(0, 1), L2-normalised per token (k left raw for the
Kaczmarz workload); v ~ N(0, 1); beta (or eta) = sigmoid(N(0, 1)); log-gate
g = logsigmoid(N(mu, 1)) with mu = 3 (mu = 4 for the long-context Kaczmarz
workload), one per head and token (scalar gate) or per key channel (KDA);
dO ~ N(0, 1); optional initial state S0 ~ N(0, 0.1) (0.1 is the standard
deviation).  The SFDA phase gate (one rotation-decay per key pair) draws the
pair decays log alpha = logsigmoid(N(mu, 1)) and then the phases theta ~
U(-pi, pi) (a phase per pair and token; the explainer's cyclic counter uses
2 pi / 5), interleaved as g[..., 2j] = log alpha_j, g[..., 2j+1] = theta_j.
Values are drawn in fp32 from ``torch.Generator(seed)`` in the fixed
order q, k, v, beta-logits, g-logits (then phases), dO, S0, then q/k/v/dO are rounded to
bf16 (round-to-nearest-even) for bf16 workloads; beta, g and S0 stay fp32.  The
oracle receives exactly these rounded values, upcast to fp64.

L2 normalisation is x / max(||x||, 1e-12); it is part of the input recipe, not
of the operator, and receives no gradient.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    dk: int = 128
    dv: int = 128
    chunk: int = 64
    dtype: str = "bf16"          # "f32" or "bf16": storage type of q, k, v, o, dO
    gate: str = "scalar"         # "none" | "scalar" | "channel" | "phase"
    beta_mode: str = "direct"    # "direct" | "kaczmarz"
    g_mean: float = 3.0
    eps: float = 1e-6
    normalize_k: bool = True
    s0_std: float = 0.0          # 0 -> zero initial state
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.B * self.T

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five synthetic workloads of the operator, named by what they are.
WORKLOADS = {
    "gdn_f32_b1h2t256d64": Workload("gdn_f32_b1h2t256d64", B=1, H=2, T=256, dk=64, dv=64,
                                    dtype="f32", gate="scalar", seed=0),
    "deltanet_bf16_b4h8t2048": Workload("deltanet_bf16_b4h8t2048", B=4, H=8, T=2048,
                                        gate="none", s0_std=0.1, seed=1),
    "gdn_bf16_b4h8t2048": Workload("gdn_bf16_b4h8t2048", B=4, H=8, T=2048,
                                   gate="scalar", s0_std=0.1, seed=1),
    "gdn_bf16_b8h16t4096": Workload("gdn_bf16_b8h16t4096", B=8, H=16, T=4096,
                                    gate="scalar", seed=2),
    "kda_bf16_b4h16t8192": Workload("kda_bf16_b4h16t8192", B=4, H=16, T=8192,
                                    gate="channel", seed=3),
    "kla_bf16_b1h16t65536": Workload("kla_bf16_b1h16t65536", B=1, H=16, T=65536,
                                     gate="scalar", beta_mode="kaczmarz", g_mean=4.0,
                                     normalize_k=False, seed=4),
    # SFDA: the KDA sizes with the rotation-decay gate (forward and decode only)
    "sfda_bf16_b4h16t8192": Workload("sfda_bf16_b4h16t8192", B=4, H=16, T=8192,
                                     gate="phase", seed=5),
}

# The headline benchmark workload (KDA per-channel gate, B4 H16 T8192 d128).
HEADLINE = "kda_bf16_b4h16t8192"


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_inputs(w: Workload, seed: int | None = None, device="cpu") -> dict:
    """Draw one batch of inputs for workload ``w`` on the CPU.

    Returns a dict of CPU tensors: q, k, v, dO in the storage dtype; beta (eta
    in Kaczmarz mode), g (or None), S0 (or None), dST (None) in fp32.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed if seed is None else seed)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv

    def normal(*shape, mean=0.0, std=1.0):
        x = torch.randn(*shape, generator=gen, dtype=torch.float32)
        return x * std + mean

    q = _l2norm(normal(B, T, H, dk))
    k = normal(B, T, H, dk)
    if w.normalize_k:
        k = _l2norm(k)
    v = normal(B, T, H, dv)
    beta = torch.sigmoid(normal(B, T, H))
    if w.gate == "phase":
        logalpha = torch.nn.functional.logsigmoid(normal(B, T, H, dk // 2, mean=w.g_mean))
        theta = (torch.rand(B, T, H, dk // 2, generator=gen, dtype=torch.float32) * 2 - 1) \
            * torch.pi
        g = torch.stack([logalpha, theta], dim=-1).reshape(B, T, H, dk).contiguous()
    else:
        g_shape = (B, T, H, dk) if w.gate == "channel" else (B, T, H)
        g_logit = normal(*g_shape, mean=w.g_mean)
        g = None if w.gate == "none" else torch.nn.functional.logsigmoid(g_logit)
    dO = normal(B, T, H, dv)
    S0 = normal(B, H, dv, dk, std=w.s0_std) if w.s0_std > 0 else None
    sdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    out = dict(q=q.to(sdt), k=k.to(sdt), v=v.to(sdt), beta=beta.contiguous(), g=g,
               dO=dO.to(sdt), S0=S0, dST=None)
    if device != "cpu":
        out = {n: (None if x is None else x.to(device)) for n, x in out.items()}
    return out


def random_state(w: Workload, seed: int, std: float = 1.0) -> torch.Tensor:
    """A seeded fp32 state-shaped tensor [B, H, dv, dk] (e.g. an upstream dS_T)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return torch.randn(w.B, w.H, w.dv, w.dk, generator=gen, dtype=torch.float32) * std
