"""Seeded synthetic inputs for the MoE expert-FFN layer.

This module is shared by the CPU oracle's tests and by the CUDA path's tests
and benchmark. It only draws random numbers and lays them out in the layer's
input formats. It holds none of the layer's arithmetic (no routing, no
softmax, no GEMM, no dequantisation).

Workloads (shapes and distributions follow the problem statement of the
InfiniLM PR #500 Qwen3-MoE report, §2.1 and §2.2, which fixes
Qwen3-30B-A3B at 128 experts and top-8, and the FlashInfer PR #7196 analysis
for the W4A16 format):

  tiny           T=16,   H=128,  I=64,   E=8,   k=2   bf16 weights
  qwen3_decode   T=64,   H=2048, I=768,  E=128, k=8   bf16 weights
  qwen3_prefill  T=8192, H=2048, I=768,  E=128, k=8   bf16, logits + N(0,0.5) per-expert bias
  skewed         T=4096, H=4096, I=1536, E=64,  k=6   bf16, logits + 3 ln Zipf(1.2)
  w4a16_decode   T=256,  H=7168, I=2048, E=256, k=8   int4 weights, 1 bf16 scale / 128 K
  mxfp8_decode   T=64,   H=2048, I=768,  E=128, k=8   MXFP8 weights (E4M3, 1 E8M0 scale / 32 K)
  mxfp4_decode   T=64,   H=2048, I=768,  E=128, k=8   MXFP4 weights (E2M1, 1 E8M0 scale / 32 K)
  shared_decode  T=64,   H=2048, I=768,  E=64,  k=6   bf16, plus 2 shared experts

Draw recipe. Every tensor has its own torch CPU generator, seeded from
(seed, stream id), so a single expert's weights can be regenerated alone:
  stream 1           hidden  [T,H]     N(0,1) fp32 -> bf16 (round to nearest even)
  stream 2           logits  [T,E]     N(0,1) fp32
  stream 3           per-expert bias [E] N(0,0.5) fp32 (qwen3_prefill only)
  stream 16+2e       expert e gate/up weights [2I,H]
  stream 17+2e       expert e down weights    [H,I]
bf16 weights are N(0,0.02) fp32 draws rounded to bf16. int4 weights are
uniform bytes (each nibble uniform on [0,15], read as two's complement
[-8,7]; the low nibble holds the even K index) followed, from the same
generator, by scales U(0.002,0.02) fp32 rounded to bf16, one per 128
consecutive K elements of a row. MXFP8 weights are E4M3 codes with a uniform
sign, an exponent field uniform on 4..7 and a uniform mantissa, followed by
E8M0 scale codes uniform on 120..122, one per 32 consecutive K elements.
MXFP4 weights are E2M1 codes with a uniform sign and a magnitude code
uniform on 1..7, two per byte (the even K index in the low nibble), followed
by E8M0 scale codes uniform on 119..121, one per 32 consecutive K elements.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable, Optional

import torch

__all__ = [
    "MoeConfig",
    "CONFIGS",
    "get_config",
    "generator_for",
    "gen_hidden",
    "gen_logits",
    "gen_expert_weights",
    "gen_inputs",
]


@dataclasses.dataclass(frozen=True)
class MoeConfig:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    fmt: str = "bf16"          # "bf16", "int4_g128", "mxfp8" or "mxfp4"
    logit_extra: str = "none"  # "none", "bias0.5" or "zipf1.2"
    weight_std: float = 0.02
    n_shared: int = 0          # shared experts: weight arrays hold E + n_shared experts

    def with_(self, **kw) -> "MoeConfig":
        return dataclasses.replace(self, **kw)

    @property
    def P(self) -> int:
        """(token, expert) pairs: k routed slots plus n_shared shared slots per token."""
        return self.T * (self.k + self.n_shared)

    def describe(self) -> str:
        shared = f" n_shared={self.n_shared}" if self.n_shared else ""
        return (f"{self.name}: T={self.T} H={self.H} I={self.I} E={self.E} "
                f"top_k={self.k}{shared} fmt={self.fmt} logits+={self.logit_extra}")


CONFIGS: Dict[str, MoeConfig] = {
    c.name: c
    for c in [
        MoeConfig("tiny", 16, 128, 64, 8, 2),
        MoeConfig("qwen3_decode", 64, 2048, 768, 128, 8),
        MoeConfig("qwen3_prefill", 8192, 2048, 768, 128, 8, logit_extra="bias0.5"),
        MoeConfig("skewed", 4096, 4096, 1536, 64, 6, logit_extra="zipf1.2"),
        MoeConfig("w4a16_decode", 256, 7168, 2048, 256, 8, fmt="int4_g128"),
        # beyond the five workloads above: the Qwen3 decode shape with MXFP8
        # weights, and a decode layer with two shared experts
        MoeConfig("mxfp8_decode", 64, 2048, 768, 128, 8, fmt="mxfp8"),
        MoeConfig("mxfp4_decode", 64, 2048, 768, 128, 8, fmt="mxfp4"),
        MoeConfig("shared_decode", 64, 2048, 768, 64, 6, n_shared=2),
    ]
}


def get_config(name: str, **overrides) -> MoeConfig:
    cfg = CONFIGS[name]
    return cfg.with_(**overrides) if overrides else cfg


_MASK63 = (1 << 63) - 1


def generator_for(seed: int, stream: int) -> torch.Generator:
    """A CPU generator for one input tensor, from (seed, stream id)."""
    s = (seed * 0x9E3779B97F4A7C15 + stream * 0xBF58476D1CE4E5B9 + 0x94D049BB133111EB) & _MASK63
    return torch.Generator().manual_seed(s)


def gen_hidden(cfg: MoeConfig, seed: int = 0) -> torch.Tensor:
    g = generator_for(seed, 1)
    return torch.randn(cfg.T, cfg.H, generator=g, dtype=torch.float32).to(torch.bfloat16)


def gen_logits(cfg: MoeConfig, seed: int = 0) -> torch.Tensor:
    g = generator_for(seed, 2)
    logits = torch.randn(cfg.T, cfg.E, generator=g, dtype=torch.float32)
    if cfg.logit_extra == "bias0.5":
        bias = torch.randn(cfg.E, generator=generator_for(seed, 3), dtype=torch.float32) * 0.5
        logits = logits + bias[None, :]
    elif cfg.logit_extra == "zipf1.2":
        # Expert e has popularity rank e+1; p_e = (e+1)^-1.2 / sum_j (j+1)^-1.2.
        ranks = [(e + 1) ** -1.2 for e in range(cfg.E)]
        z = math.fsum(ranks)
        term = torch.tensor([3.0 * math.log(r / z) for r in ranks], dtype=torch.float64)
        logits = logits + term.to(torch.float32)[None, :]
    elif cfg.logit_extra != "none":
        raise ValueError(f"unknown logit_extra {cfg.logit_extra!r}")
    return logits.contiguous()


def gen_expert_weights(cfg: MoeConfig, e: int, seed: int = 0) -> Dict[str, torch.Tensor]:
    """Weights of expert e.

    bf16:      {"w_gu": [2I,H] bf16, "w_d": [H,I] bf16}
    int4_g128: {"w_gu": [2I,H/2] uint8, "w_gu_scales": [2I,H/128] bf16,
                "w_d":  [H,I/2]  uint8, "w_d_scales":  [H,I/128]  bf16}
    Rows [0,I) of w_gu are the gate projection, rows [I,2I) the up projection.
    """
    g_gu = generator_for(seed, 16 + 2 * e)
    g_d = generator_for(seed, 17 + 2 * e)
    H, I = cfg.H, cfg.I
    if cfg.fmt == "bf16":
        w_gu = (torch.randn(2 * I, H, generator=g_gu, dtype=torch.float32) * cfg.weight_std).to(torch.bfloat16)
        w_d = (torch.randn(H, I, generator=g_d, dtype=torch.float32) * cfg.weight_std).to(torch.bfloat16)
        return {"w_gu": w_gu, "w_d": w_d}
    if cfg.fmt == "int4_g128":
        if H % 128 or I % 128:
            raise ValueError("int4_g128 needs H and I multiples of 128")
        out = {}
        for name, g, rows, K in (("w_gu", g_gu, 2 * I, H), ("w_d", g_d, H, I)):
            q = torch.randint(0, 256, (rows, K // 2), generator=g, dtype=torch.uint8)
            s = torch.rand(rows, K // 128, generator=g, dtype=torch.float32) * 0.018 + 0.002
            out[name] = q
            out[name + "_scales"] = s.to(torch.bfloat16)
        return out
    if cfg.fmt == "mxfp8":
        if H % 32 or I % 32:
            raise ValueError("mxfp8 needs H and I multiples of 32")
        out = {}
        for name, g, rows, K in (("w_gu", g_gu, 2 * I, H), ("w_d", g_d, H, I)):
            # E4M3 codes: sign, exponent field uniform on 4..7, mantissa uniform;
            # E8M0 scale codes uniform on 120..122 (2^-7 .. 2^-5)
            sign = torch.randint(0, 2, (rows, K), generator=g, dtype=torch.int32) << 7
            expo = torch.randint(4, 8, (rows, K), generator=g, dtype=torch.int32) << 3
            mant = torch.randint(0, 8, (rows, K), generator=g, dtype=torch.int32)
            out[name] = (sign | expo | mant).to(torch.uint8)
            out[name + "_scales"] = torch.randint(120, 123, (rows, K // 32), generator=g, dtype=torch.int32).to(torch.uint8)
        return out
    if cfg.fmt == "mxfp4":
        if H % 32 or I % 32:
            raise ValueError("mxfp4 needs H and I multiples of 32")
        out = {}
        for name, g, rows, K in (("w_gu", g_gu, 2 * I, H), ("w_d", g_d, H, I)):
            # E2M1 codes: sign uniform, magnitude code uniform on 1..7 (0.5 .. 6),
            # two per byte with the even K index in the low nibble; E8M0 scale
            # codes uniform on 119..121 (2^-8 .. 2^-6)
            sign = torch.randint(0, 2, (rows, K), generator=g, dtype=torch.int32) << 3
            mag = torch.randint(1, 8, (rows, K), generator=g, dtype=torch.int32)
            nib = sign | mag
            out[name] = (nib[:, 0::2] | (nib[:, 1::2] << 4)).to(torch.uint8)
            out[name + "_scales"] = torch.randint(119, 122, (rows, K // 32), generator=g, dtype=torch.int32).to(torch.uint8)
        return out
    raise ValueError(f"unknown weight format {cfg.fmt!r}")


def gen_inputs(cfg: MoeConfig, seed: int = 0, experts: Optional[Iterable[int]] = None,
               pin_memory: bool = False) -> Dict[str, torch.Tensor]:
    """All inputs of one layer call as CPU tensors.

    Weights are stacked over experts: w_gu [E,2I,H] (or packed [E,2I,H/2] with
    scales [E,2I,H/128]) and w_d [E,H,I] (or [E,H,I/2] with [E,H,I/128]); with
    n_shared shared experts the arrays hold E + n_shared experts, the shared
    ones last (expert e's weights always come from streams 16+2e, 17+2e).
    If `experts` is given, only those experts' weights are drawn and the rest
    are left zero (used to keep tests of large configs cheap).
    """
    hidden = gen_hidden(cfg, seed)
    logits = gen_logits(cfg, seed)
    E, H, I = cfg.E + cfg.n_shared, cfg.H, cfg.I       # routed experts, then the shared ones
    if cfg.fmt == "bf16":
        shapes = {"w_gu": ((E, 2 * I, H), torch.bfloat16), "w_d": ((E, H, I), torch.bfloat16)}
    elif cfg.fmt == "mxfp4":
        shapes = {
            "w_gu": ((E, 2 * I, H // 2), torch.uint8),
            "w_gu_scales": ((E, 2 * I, H // 32), torch.uint8),
            "w_d": ((E, H, I // 2), torch.uint8),
            "w_d_scales": ((E, H, I // 32), torch.uint8),
        }
    elif cfg.fmt == "mxfp8":
        shapes = {
            "w_gu": ((E, 2 * I, H), torch.uint8),
            "w_gu_scales": ((E, 2 * I, H // 32), torch.uint8),
            "w_d": ((E, H, I), torch.uint8),
            "w_d_scales": ((E, H, I // 32), torch.uint8),
        }
    else:
        shapes = {
            "w_gu": ((E, 2 * I, H // 2), torch.uint8),
            "w_gu_scales": ((E, 2 * I, H // 128), torch.bfloat16),
            "w_d": ((E, H, I // 2), torch.uint8),
            "w_d_scales": ((E, H, I // 128), torch.bfloat16),
        }
    out = {"hidden": hidden, "logits": logits}
    for name, (shape, dt) in shapes.items():
        out[name] = torch.zeros(shape, dtype=dt, pin_memory=pin_memory)
    todo = range(E) if experts is None else sorted(set(int(e) for e in experts))
    for e in todo:
        for name, t in gen_expert_weights(cfg, e, seed).items():
            out[name][e].copy_(t)
    return out
