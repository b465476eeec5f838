"""Seeded synthetic workloads for tiled attention.

This module only draws inputs.  It holds none of the attention arithmetic, so
both the fp64 oracle tests and the CUDA path can take their inputs from here
without sharing any computation.

Recipe (one ``torch.Generator`` on the CPU per workload, seeded):
  Q, K, V, dO are drawn in that order as fp32 ``randn`` of their shapes,
  multiplied by their standard deviation, then rounded to bf16 (RNE).
Shapes are [B, H, N, D] contiguous; K and V carry ``Hkv`` heads (GQA when
Hkv < Hq), Q and dO carry ``Hq`` heads.  scale defaults to 1/sqrt(D).

The five named workloads are the Llama-shaped attention problems the pages
talk about (FlashAttention V2 deep dive, "实测性能数据" and "生产环境部署建议";
Ascend ops-transformer article, section 五): a tiny case, a Llama-2-7B layer
(B8 H32 N2048 D128), the long N=8192 case where standard attention runs out
of memory, a Llama-2-70B GQA layer (64 query heads over 8 K/V heads) and an
N=65536 stability stress case with large logits.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    causal: bool
    seed: int
    sigma_qk: float = 1.0
    sigma_vdo: float = 1.0
    scale: float | None = None  # None -> 1/sqrt(D)

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.D)

    def flops_fwd(self) -> float:
        """4*B*Hq*N^2*D, halved when causal (matmul flop convention)."""
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.D
        return f / 2 if self.causal else f

    def flops_bwd(self) -> float:
        """10*B*Hq*N^2*D (five GEMMs), halved when causal."""
        f = 10.0 * self.B * self.Hq * self.N * self.N * self.D
        return f / 2 if self.causal else f

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hq=2, Hkv=2, N=128, D=64, causal=False, seed=0),
    "llama7b": Workload("llama7b", B=8, Hq=32, Hkv=32, N=2048, D=128, causal=True, seed=1),
    "long": Workload("long", B=2, Hq=32, Hkv=32, N=8192, D=128, causal=True, seed=2),
    "gqa70b": Workload("gqa70b", B=1, Hq=64, Hkv=8, N=4096, D=128, causal=True, seed=3),
    "stress": Workload("stress", B=1, Hq=16, Hkv=16, N=65536, D=128, causal=True, seed=4,
                       sigma_qk=3.0, sigma_vdo=1.0),
}


def make_inputs(wl: Workload):
    """Return (q, k, v, do) as contiguous bf16 CPU tensors for ``wl``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed)
    shapes = [
        ((wl.B, wl.Hq, wl.N, wl.D), wl.sigma_qk),
        ((wl.B, wl.Hkv, wl.N, wl.D), wl.sigma_qk),
        ((wl.B, wl.Hkv, wl.N, wl.D), wl.sigma_vdo),
        ((wl.B, wl.Hq, wl.N, wl.D), wl.sigma_vdo),
    ]
    out = []
    for shape, sigma in shapes:
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if sigma != 1.0:
            x.mul_(sigma)
        out.append(x.to(torch.bfloat16).contiguous())
    return tuple(out)


@dataclass(frozen=True)
class KvWorkload:
    """Nq new queries over an Nk-long K/V history (query i at position Nk - Nq + i)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    D: int
    causal: bool
    seed: int
    sigma_qk: float = 1.0

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def kv_bytes(self) -> int:
        """Bytes of the K and V history (bf16), the traffic the work is bound by."""
        return 2 * 2 * self.B * self.Hkv * self.Nk * self.D


# Decoding one token per sequence against a 32K-token cache of a Llama-2-70B
# shaped layer (64 query heads over 8 K/V heads).
KV_WORKLOADS = {
    "decode70b": KvWorkload("decode70b", B=8, Hq=64, Hkv=8, Nq=1, Nk=32768, D=128, causal=True, seed=5),
    # the same layer with 2 sequences at 16K: 134 MB of history (above L2), for profiling
    "decode_small": KvWorkload("decode_small", B=2, Hq=64, Hkv=8, Nq=1, Nk=16384, D=128, causal=True, seed=6),
}


def make_kv_inputs(wl: KvWorkload):
    """(q [B,Hq,Nq,D], k, v [B,Hkv,Nk,D]) bf16 CPU tensors: fp32 randn drawn in
    the order q, k, v from one generator seeded with wl.seed, q and k times
    sigma_qk, rounded to bf16."""
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed)
    out = []
    for shape, sigma in (((wl.B, wl.Hq, wl.Nq, wl.D), wl.sigma_qk), ((wl.B, wl.Hkv, wl.Nk, wl.D), wl.sigma_qk),
                         ((wl.B, wl.Hkv, wl.Nk, wl.D), 1.0)):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if sigma != 1.0:
            x.mul_(sigma)
        out.append(x.to(torch.bfloat16).contiguous())
    return tuple(out)


E4M3_MAX = 448.0


def make_fp8_inputs(wl: Workload):
    """FP8 forward inputs for ``wl``: the fp32 draws of ``make_inputs``'s
    recipe (same generator, seed and order) encoded per tensor as e4m3 with
    descale = amax / 448, the largest finite e4m3 magnitude.  Returns
    (q8, k8, v8, q_scale, k_scale, v_scale); element x of q8 stands for
    float(x) * q_scale."""
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed)
    shapes = [((wl.B, wl.Hq, wl.N, wl.D), wl.sigma_qk), ((wl.B, wl.Hkv, wl.N, wl.D), wl.sigma_qk),
              ((wl.B, wl.Hkv, wl.N, wl.D), wl.sigma_vdo)]
    tens, scales = [], []
    for shape, sigma in shapes:
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if sigma != 1.0:
            x.mul_(sigma)
        s = float(x.abs().max()) / E4M3_MAX
        s = s if s > 0 else 1.0
        tens.append((x / s).to(torch.float8_e4m3fn).contiguous())
        scales.append(s)
    return tens[0], tens[1], tens[2], scales[0], scales[1], scales[2]


def sample_indices(n: int, count: int, seed: int, must=()):
    """Seeded sorted sample of ``count`` distinct indices in [0, n), always
    including the valid entries of ``must`` (e.g. first/last rows, tile edges)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    chosen = {i for i in must if 0 <= i < n}
    if count >= n:
        return list(range(n))
    perm = torch.randperm(n, generator=g).tolist()
    for i in perm:
        if len(chosen) >= count:
            break
        chosen.add(i)
    return sorted(chosen)
