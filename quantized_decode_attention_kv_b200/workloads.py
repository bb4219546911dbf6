"""Seeded synthetic workloads shaped like the pages' models (no method arithmetic here).

The pages describe per-layer, per-KV-head caches of [T x d] keys and values
("Why the KV Cache Exists", What's in the KV Cache: Llama-3.1-8B, 32 layers x 8 KV heads,
d = 128), keys whose norms dwarf the values' ("What the Paper Doesn't Tell You", Finding 1),
GPT-2's head_dim 64 (Finding 2), 128K contexts, and 70B-class asymmetric K/V bit-widths with
the first and last two layers kept at higher precision (Finding 1). No dataset or trained
weight is used: every tensor is drawn from torch generators with a fixed seed, and these
shapes stand in for the real models.

Recipe per workload (seed 1000 + index): K ~ N(0,1) (optionally: `k_outliers` channels
chosen by a CPU randperm are multiplied by 20, then each token by U(0.5, 2); or the whole of
K by `k_scale`), V ~ N(0,1), one query per head q ~ N(0,1); cast to `dtype`.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

MSE, PROD = 0, 1


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int
    k_bits: int
    v_bits: int
    k_mode: int = MSE
    v_mode: int = MSE
    qjl_m: int = 0
    dtype: torch.dtype = torch.bfloat16
    k_outliers: int = 0      # channels scaled x20
    k_jitter: bool = False   # per-token x U(0.5, 2)
    k_scale: float = 1.0
    layers: int = 1
    bf16_layers: tuple = ()  # layer indices kept unquantised
    seed: int = 0            # rotation seed
    qjl_seed: int = 1

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return self.d ** -0.5


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_single_head_fp32", 0, B=1, Hq=1, Hkv=1, d=128, T=1024, k_bits=4, v_bits=4,
                 dtype=torch.float32),
        Workload("llama3_8b_decode_32k", 1, B=16, Hq=32, Hkv=8, d=128, T=32768, k_bits=4,
                 v_bits=2, k_outliers=4, k_jitter=True),
        Workload("gpt2_prod_2bit", 2, B=64, Hq=12, Hkv=12, d=64, T=8192, k_bits=2, v_bits=2,
                 k_mode=PROD, v_mode=PROD, qjl_m=64),
        Workload("llama3_8b_128k_3bit", 3, B=4, Hq=32, Hkv=8, d=128, T=131072, k_bits=3,
                 v_bits=3, k_outliers=4, k_jitter=True, layers=32),
        Workload("llama70b_asym_16k", 4, B=32, Hq=64, Hkv=8, d=128, T=16384, k_bits=4, v_bits=2,
                 k_scale=50.0, layers=80, bf16_layers=(0, 1, 78, 79)),
        # the pages' 3.5-bit operating point read as 4-bit keys and 3-bit values (3.5 bits per
        # cached coordinate on average) on the Llama-3.1-8B shape
        Workload("llama3_8b_32k_3p5bit", 5, B=16, Hq=32, Hkv=8, d=128, T=32768, k_bits=4,
                 v_bits=3, k_outliers=4, k_jitter=True),
    ]
}


def make_inputs(w: Workload, device="cpu", B: int | None = None, T: int | None = None,
                Hkv: int | None = None, Hq: int | None = None, layer: int = 0):
    """K, V [B, Hkv, T, d] and q [B, Hq, d] for workload ``w`` (optionally scaled down in B, T or
    heads). The same (w, sizes, layer, device) always gives the same tensors."""
    B = B or w.B
    T = T or w.T
    Hkv = Hkv or w.Hkv
    Hq = Hq or (w.G * Hkv)
    seed = 1000 + w.index + 7919 * layer
    cpu = torch.Generator(device="cpu").manual_seed(seed)
    g = torch.Generator(device=device).manual_seed(seed)
    K = torch.randn(B, Hkv, T, w.d, generator=g, device=device, dtype=torch.float32)
    if w.k_outliers:
        ch = torch.randperm(w.d, generator=cpu)[: w.k_outliers].to(device)
        K[..., ch] *= 20.0
    if w.k_jitter:
        K *= torch.empty(B, Hkv, T, 1, device=device).uniform_(0.5, 2.0, generator=g)
    if w.k_scale != 1.0:
        K *= w.k_scale
    V = torch.randn(B, Hkv, T, w.d, generator=g, device=device, dtype=torch.float32)
    q = torch.randn(B, Hq, w.d, generator=g, device=device, dtype=torch.float32)
    return K.to(w.dtype), V.to(w.dtype), q.to(w.dtype)


def random_kv(B, Hkv, T, d, dtype=torch.float32, seed=0, device="cpu", scale=1.0):
    """Plain N(0, scale^2) K, V for small parity cases."""
    g = torch.Generator(device=device).manual_seed(seed)
    K = torch.randn(B, Hkv, T, d, generator=g, device=device) * scale
    V = torch.randn(B, Hkv, T, d, generator=g, device=device)
    return K.to(dtype), V.to(dtype)
