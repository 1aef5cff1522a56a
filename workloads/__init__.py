"""Seeded synthetic inputs for the verification path (shared by tests and bench).

This module only draws inputs; it holds none of the verification arithmetic.
Each configuration restates one of the five workloads the verifier is
measured on (logit shapes, value distributions, temperatures, how the draft
tokens are drawn).  Inputs are generated with torch on the requested device
from a generator seeded with ``1000 * config_index + step``; the oracle side
copies the same bits to the host.

Configurations (names by what they are):
  c0_single_b1_g4_v32000_f32       B=1,   gamma=4, V=32000,  fp32, 1 step
  c1_b16_g5_v32000_bf16            B=16,  gamma=5, V=32000,  bf16, 100 steps
  c2_b64_g8_v128256_bf16           B=64,  gamma=8, V=128256, bf16, 50 steps
  c3_multidraft_b8_k4_l5_v32000    B=8, K=4, L=5,  V=32000,  bf16, 100 steps
  c4_b256_g4_v151936_bf16          B=256, gamma=4, V=151936, bf16, 200 steps
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Config:
    index: int
    name: str
    B: int
    gamma: int  # draft length (L for the multi-draft workload)
    V: int
    dtype: str  # "f32" | "bf16"
    steps: int
    K: int = 0  # drafts per sequence (multi-draft workload only)
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def multidraft(self) -> bool:
        return self.K > 0

    @property
    def rows_per_step(self) -> int:
        """Verified draft rows per step: B*gamma, or B*K*L for multi-draft."""
        return self.B * self.gamma * (self.K if self.multidraft else 1)


CONFIGS = [
    Config(0, "c0_single_b1_g4_v32000_f32", B=1, gamma=4, V=32000, dtype="f32", steps=1,
           notes="target ~ N(0, 2.0); draft = target + N(0, 0.5); tokens ~ draft softmax at "
                 "T=1.0; T=1.0"),
    Config(1, "c1_b16_g5_v32000_bf16", B=16, gamma=5, V=32000, dtype="bf16", steps=100,
           notes="target ~ N(0, 3.0) with 20 distinct peak ids per row boosted by +8; "
                 "draft = target + N(0, 0.7); T alternates 0.7 / 1.0 by sequence"),
    Config(2, "c2_b64_g8_v128256_bf16", B=64, gamma=8, V=128256, dtype="bf16", steps=50,
           notes="target ~ N(0, 2.5); draft = 0.8 * target + N(0, 1.0); T=1.0"),
    Config(3, "c3_multidraft_b8_k4_l5_v32000", B=8, gamma=5, V=32000, dtype="bf16", steps=100,
           K=4, notes="target [B, L+1, V] ~ N(0, 2.0); draft [B, L, V] = target + N(0, 0.6), "
                      "shared by the K drafts; K drafts drawn independently; T cycles "
                      "0.1 / 0.4 / 0.7 by sequence"),
    Config(4, "c4_b256_g4_v151936_bf16", B=256, gamma=4, V=151936, dtype="bf16", steps=200,
           notes="target ~ N(0, 2.5) - 1.1 ln(v + 1) (Zipf s=1.1 bias over token ids); "
                 "draft = target + N(0, 0.5); per-sequence T drawn once from "
                 "{0, 0.1, 0.4, 0.7, 1.0}"),
]
BY_NAME = {c.name: c for c in CONFIGS}


def get(cfg) -> Config:
    if isinstance(cfg, Config):
        return cfg
    if isinstance(cfg, int):
        return CONFIGS[cfg]
    if cfg in BY_NAME:
        return BY_NAME[cfg]
    for c in CONFIGS:
        if c.name.startswith(cfg):
            return c
    raise KeyError(cfg)


# ------------------------------------------------------------------ helpers
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even) and return the raw 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    """Host copy of a logit tensor as the oracle wants it (fp32, or bf16 bits)."""
    t = t.detach().contiguous()
    if t.dtype == torch.bfloat16:
        return t.cpu().view(torch.int16).numpy().view(np.uint16)
    return t.cpu().numpy()


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def temperatures(cfg: Config, device="cpu") -> torch.Tensor:
    B = cfg.B
    if cfg.index == 1:
        t = [0.7 if b % 2 == 0 else 1.0 for b in range(B)]
    elif cfg.index == 3:
        t = [(0.1, 0.4, 0.7)[b % 3] for b in range(B)]
    elif cfg.index == 4:
        g = np.random.default_rng(1000 * cfg.index)  # drawn once, fixed across steps
        t = list(g.choice(np.array([0.0, 0.1, 0.4, 0.7, 1.0], dtype=np.float32), size=B))
    else:
        t = [1.0] * B
    return torch.tensor(t, dtype=torch.float32, device=device)


def sample_tokens(draft: torch.Tensor, temps: torch.Tensor, n: int, gen) -> torch.Tensor:
    """Draw n independent draft tokens per (b, position) from softmax(draft / T);
    the draft argmax where T == 0.  draft [B, P, V] -> tokens [B, n, P]."""
    B, P, V = draft.shape
    z = draft.float()
    out = torch.empty((B, n, P), dtype=torch.int32, device=draft.device)
    for b in range(B):
        T = float(temps[b])
        if T == 0.0:
            out[b] = z[b].argmax(dim=-1).to(torch.int32)[None, :].expand(n, P)
        else:
            prob = torch.softmax(z[b] / T, dim=-1)  # [P, V]
            s = torch.multinomial(prob, n, replacement=True, generator=gen)  # [P, n]
            out[b] = s.t().to(torch.int32)
    return out


@dataclass
class Step:
    target: torch.Tensor  # [B, gamma+1, V]
    draft: torch.Tensor   # [B, gamma, V]
    tokens: torch.Tensor  # [B, gamma] int32, or [B, K, L] for multi-draft
    temps: torch.Tensor   # [B] float32
    step: int


def make_step(cfg, step: int, device="cpu", B: int | None = None) -> Step:
    """Inputs of one step of a configuration (optionally with a smaller batch)."""
    cfg = get(cfg)
    Bn = cfg.B if B is None else B
    g = _gen(device, 1000 * cfg.index + step)
    gam, V = cfg.gamma, cfg.V
    shape_t = (Bn, gam + 1, V)
    if cfg.index == 0:
        tgt = torch.randn(shape_t, generator=g, device=device) * 2.0
        drf = tgt[:, :gam] + torch.randn((Bn, gam, V), generator=g, device=device) * 0.5
    elif cfg.index == 1:
        tgt = torch.randn(shape_t, generator=g, device=device) * 3.0
        keys = torch.rand(shape_t, generator=g, device=device)
        peaks = keys.topk(20, dim=-1).indices  # 20 distinct ids per row, uniform
        tgt.scatter_add_(-1, peaks, torch.full(peaks.shape, 8.0, device=device))
        drf = tgt[:, :gam] + torch.randn((Bn, gam, V), generator=g, device=device) * 0.7
    elif cfg.index == 2:
        tgt = torch.randn(shape_t, generator=g, device=device) * 2.5
        drf = 0.8 * tgt[:, :gam] + torch.randn((Bn, gam, V), generator=g, device=device) * 1.0
    elif cfg.index == 3:
        tgt = torch.randn(shape_t, generator=g, device=device) * 2.0
        drf = tgt[:, :gam] + torch.randn((Bn, gam, V), generator=g, device=device) * 0.6
    elif cfg.index == 4:
        bias = -1.1 * torch.log(torch.arange(V, device=device, dtype=torch.float32) + 1.0)
        tgt = torch.randn(shape_t, generator=g, device=device) * 2.5 + bias
        drf = tgt[:, :gam] + torch.randn((Bn, gam, V), generator=g, device=device) * 0.5
    else:
        raise KeyError(cfg.index)
    if cfg.dtype == "bf16":
        tgt = tgt.to(torch.bfloat16)
        drf = drf.to(torch.bfloat16)
    tgt = tgt.contiguous()
    drf = drf.contiguous()
    temps = temperatures(cfg, device)[:Bn].contiguous()
    if cfg.multidraft:
        toks = sample_tokens(drf, temps, cfg.K, g).contiguous()  # [B, K, L]
    else:
        toks = sample_tokens(drf, temps, 1, g)[:, 0].contiguous()  # [B, gamma]
    return Step(tgt, drf, toks, temps, step)


def make_custom(B, gamma, V, dtype="bf16", seed=0, T=1.0, K=0, device="cpu",
                target_scale=2.0, noise=0.5) -> Step:
    """Small seeded inputs of arbitrary shape (edge-case and property tests)."""
    g = _gen(device, seed)
    tgt = torch.randn((B, gamma + 1, V), generator=g, device=device) * target_scale
    drf = tgt[:, :gamma] + torch.randn((B, gamma, V), generator=g, device=device) * noise
    if dtype == "bf16":
        tgt = tgt.to(torch.bfloat16)
        drf = drf.to(torch.bfloat16)
    if isinstance(T, (list, tuple)):
        temps = torch.tensor([T[b % len(T)] for b in range(B)], dtype=torch.float32,
                             device=device)
    else:
        temps = torch.full((B,), float(T), dtype=torch.float32, device=device)
    if K:
        toks = sample_tokens(drf, temps, K, g).contiguous()
    else:
        toks = sample_tokens(drf, temps, 1, g)[:, 0].contiguous()
    return Step(tgt.contiguous(), drf.contiguous(), toks, temps, 0)


def host_inputs(st: Step):
    """numpy copies of a step (logits as fp32 or bf16 bits) for the oracle."""
    return (to_host_bits(st.target), to_host_bits(st.draft), st.tokens.cpu().numpy(),
            st.temps.cpu().numpy())
