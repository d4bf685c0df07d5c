"""Seeded synthetic KV-cache tensors shared by the tests, the smoke check and the benchmark.

This module holds no codec arithmetic: it only draws random tensors with the
shapes and value distributions of the workloads the codec is measured on.  The
models the SplitZip project page names (FAQ "Which models were tested?":
Qwen3-32B, Qwen3-30B-A3B, Llama-3-8B, Phi-2) supply the shapes only; no trained
weights or prompts are used, so the values are synthetic:

  x[t, h, d] = z * s[h, d] * L
    z ~ N(0, 1) per element, s[h, d] = exp(N(0, 1)) per channel,
    max(1, round(0.001 * H * D)) channels (drawn without replacement) get s *= 100,
    L = exp(U(-2, 2)) per (layer, K/V) for the Llama-3-8B and Qwen3-32B shapes, else 1.
  computed in fp32, rounded to bf16 (round to nearest even); then at the bit
  level each element is set to +0.0 with p = 0.01, and to a bf16 subnormal
  (random sign, exponent 0, mantissa uniform in 1..127) with p = 1e-4.
  The FP8 workload casts that bf16 tensor to float8_e5m2 (round to nearest even).

Escape-stress tensors draw exponents by an exact integer inverse CDF: with
rare fraction p (0, 1, 10 or 50 percent), exponents 113..127 each have
probability (1-p)/15 and exponents 81..112 each p/32; sign and mantissa are
uniform.  The worst case is uniformly random 16-bit patterns.

Random streams come from torch.Generator; CPU and CUDA generators give
different (equally distributed) values for the same seed, so every consumer
that needs both sides to see the same tensor copies one tensor to the other.
"""
from dataclasses import dataclass
import math

import torch

__all__ = ["KVConfig", "CONFIGS", "kv_seed", "kv_tensor", "kv_batch", "stress_case",
           "stress_tensor", "STRESS_SIZES", "STRESS_RARE_PERCENT"]


@dataclass(frozen=True)
class KVConfig:
    name: str
    config_id: int
    layers: int
    tokens: int
    heads: int
    head_dim: int
    layer_scale: bool      # per-(layer, K/V) scale L = exp(U(-2, 2))
    fp8: bool = False      # cast to float8_e5m2 after the bf16 draw

    @property
    def shape(self):
        return (self.tokens, self.heads, self.head_dim)

    @property
    def numel(self) -> int:
        return self.tokens * self.heads * self.head_dim

    @property
    def tensors(self) -> int:
        return 2 * self.layers


CONFIGS = {
    "phi2": KVConfig("phi2", 1, 1, 1024, 32, 80, layer_scale=False),
    "llama3-8b": KVConfig("llama3-8b", 2, 32, 8192, 8, 128, layer_scale=True),
    "qwen3-32b": KVConfig("qwen3-32b", 3, 64, 131072, 8, 128, layer_scale=True),
    "qwen3-30b-a3b-e5m2": KVConfig("qwen3-30b-a3b-e5m2", 5, 48, 32768, 4, 128,
                                   layer_scale=False, fp8=True),
}


def kv_seed(cfg: KVConfig, layer: int, kv: int) -> int:
    """Seed of one (layer, K/V) tensor; kv = 0 for K, 1 for V.  Phi-2 uses base seed 0."""
    base = 0 if cfg.config_id == 1 else 1_000_000 * cfg.config_id
    return base + 2 * layer + kv


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def kv_tensor(cfg: KVConfig, layer: int, kv: int, device="cpu") -> torch.Tensor:
    """One K or V tensor [tokens, heads, head_dim] in bf16 (or float8_e5m2)."""
    T, H, D = cfg.shape
    g = _gen(kv_seed(cfg, layer, kv), device)
    z = torch.randn((T, H, D), generator=g, device=device, dtype=torch.float32)
    s = torch.exp(torch.randn((H, D), generator=g, device=device, dtype=torch.float32))
    k = max(1, int(round(0.001 * H * D)))
    outliers = torch.randperm(H * D, generator=g, device=device)[:k]
    s.view(-1)[outliers] *= 100.0
    if cfg.layer_scale:
        u = torch.rand((1,), generator=g, device=device, dtype=torch.float32)
        scale = torch.exp(u * 4.0 - 2.0)
    else:
        scale = torch.ones((1,), device=device, dtype=torch.float32)
    z.mul_(s).mul_(scale)
    x = z.to(torch.bfloat16)
    del z
    bits = x.view(torch.int16)
    zero = torch.rand((T, H, D), generator=g, device=device) < 0.01
    bits.masked_fill_(zero, 0)
    del zero
    sub = torch.rand((T, H, D), generator=g, device=device) < 1e-4
    cnt = int(sub.sum().item())
    sign = torch.randint(0, 2, (cnt,), generator=g, device=device, dtype=torch.int32)
    mant = torch.randint(1, 128, (cnt,), generator=g, device=device, dtype=torch.int32)
    sub_bits = ((sign << 15) | mant).to(torch.int32)
    sub_bits = torch.where(sub_bits >= 32768, sub_bits - 65536, sub_bits).to(torch.int16)
    bits[sub] = sub_bits
    if cfg.fp8:
        return x.to(torch.float8_e5m2)
    return x


def kv_batch(cfg: KVConfig, device="cpu", layers=None):
    """All (or the given) layers' K and V tensors, in order K0, V0, K1, V1, ..."""
    out = []
    for layer in (range(cfg.layers) if layers is None else layers):
        for kv in (0, 1):
            out.append(kv_tensor(cfg, layer, kv, device))
    return out


# Escape-stress workload: flat bf16 tensors of 1 MB, 64 MB, 1 GB and 4 GB.
STRESS_SIZES = (1 << 19, 1 << 25, 1 << 29, 1 << 31)
STRESS_RARE_PERCENT = (0, 1, 10, 50, None)  # None = uniformly random 16-bit patterns
_STRESS_CHUNK = 1 << 26


def stress_case(size_index: int, rare_index: int) -> int:
    """Case number of (size, rare fraction); the seed is 4_000_000 + case."""
    return size_index * len(STRESS_RARE_PERCENT) + rare_index


def stress_tensor(n: int, rare_percent, seed: int, device="cpu") -> torch.Tensor:
    """Flat bf16 tensor of n elements; rare_percent in (0, 1, 10, 50) or None (uniform bits)."""
    g = _gen(seed, device)
    out = torch.empty(n, dtype=torch.int16, device=device)
    for lo in range(0, n, _STRESS_CHUNK):
        m = min(_STRESS_CHUNK, n - lo)
        if rare_percent is None:
            w = torch.randint(0, 65536, (m,), generator=g, device=device, dtype=torch.int32)
        else:
            P = int(rare_percent)
            # r uniform in [0, 48000): the first 480*P values are rare (32 buckets of
            # 15*P), the rest common (15 buckets of 32*(100-P)).  All bucket sizes are
            # integers, so the probabilities are exact.
            r = torch.randint(0, 48000, (m,), generator=g, device=device, dtype=torch.int32)
            rare = r < 480 * P
            if P > 0:
                e_rare = 81 + torch.div(r, 15 * P, rounding_mode="floor")
            else:
                e_rare = torch.zeros_like(r)
            e_common = 113 + torch.div(r - 480 * P, 32 * (100 - P), rounding_mode="floor")
            e = torch.where(rare, e_rare, e_common)
            sign = torch.randint(0, 2, (m,), generator=g, device=device, dtype=torch.int32)
            mant = torch.randint(0, 128, (m,), generator=g, device=device, dtype=torch.int32)
            w = (sign << 15) | (e << 7) | mant
        w = torch.where(w >= 32768, w - 65536, w)
        out[lo:lo + m] = w.to(torch.int16)
    return out.view(torch.bfloat16)


def describe() -> str:
    lines = []
    for c in CONFIGS.values():
        gb = c.tensors * c.numel * (1 if c.fp8 else 2) / 1e9
        lines.append("%s: %d x {K,V} x %s = %.3f GB" % (c.name, c.layers, c.shape, gb))
    return "\n".join(lines)


if __name__ == "__main__":
    print(describe())
    print(math.prod(CONFIGS["llama3-8b"].shape))
