"""Seeded synthetic inputs for the GQE forward pass.

This module only draws random numbers and names workload shapes. It holds none
of the layer's arithmetic, so the fp64 oracle (``oracle/``) and the CUDA path
(``moe_gqa_query_gqe_b200``) can both be fed from it without sharing any code
that computes the method.

Recipe (identical for every workload):
  * one ``torch.Generator`` seeded with ``seed``;
  * draw order x, Wq, Wk, Wv, Wr, Wo, Wo_dense;
  * x ~ N(0, 1); every weight ~ N(0, 0.02^2); drawn in fp32, then rounded to
    bf16 (round-to-nearest-even);
  * router bias br is fp32 zeros, except ``bias0`` added on expert 0 of every
    group (the skewed-routing workload uses +2.0).

Weights are stored [in, out] row-major:
  x        [B*T, D]
  Wq       [D, (G*M + 1) * dh]    routed heads h = g*M + e, then the shared head
  Wk, Wv   [D, G * dh]
  Wr       [D, G * M]
  br       [G * M]                fp32
  Wo       [(G*k + G + 1) * dh, D] rows: concat (g-major, slot j), slot g, shared
  Wo_dense [G * M * dh, D]        output projection of the all-heads baseline
"""
from dataclasses import dataclass, asdict, replace

import torch


@dataclass(frozen=True)
class Dims:
    B: int
    T: int
    D: int
    G: int
    M: int
    k: int
    dh: int = 64
    bias0: float = 0.0

    @property
    def n_tokens(self) -> int:
        return self.B * self.T

    @property
    def wq_cols(self) -> int:
        return (self.G * self.M + 1) * self.dh

    @property
    def wo_rows(self) -> int:
        return (self.G * self.k + self.G + 1) * self.dh

    def with_(self, **kw) -> "Dims":
        return replace(self, **kw)

    def as_dict(self) -> dict:
        return asdict(self)


# The workloads, each named by what it is. Sizes follow the layer the method
# was measured on (16 query heads over 8 KV groups, k = 1, one shared head).
CONFIGS = {
    # 2 sequences of 256 tokens: small enough for the full fp64 oracle.
    "tiny_b2_t256": Dims(B=2, T=256, D=1024, G=8, M=2, k=1),
    # 8 sequences of 2048 tokens: the main layer.
    "main_b8_t2048": Dims(B=8, T=2048, D=1024, G=8, M=2, k=1),
    # one sequence of 32768 tokens, near-balanced routing.
    "long_b1_t32768": Dims(B=1, T=32768, D=1024, G=8, M=2, k=1),
    # 131072 tokens, pool of 4 experts per group, k = 2, skewed router.
    "skewed_b1_t131072_m4k2": Dims(B=1, T=131072, D=2048, G=8, M=4, k=2, bias0=2.0),
    # one sequence of 8192 tokens: mid-size case for profiling captures.
    "mid_b1_t8192": Dims(B=1, T=8192, D=1024, G=8, M=2, k=1),
    # one sequence of 1,048,576 tokens.
    "million_b1_t1048576": Dims(B=1, T=1048576, D=1024, G=8, M=2, k=1),
}


def _normal(gen: torch.Generator, shape, std: float, device) -> torch.Tensor:
    t = torch.randn(*shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def make_inputs(dims: Dims, seed: int = 0, device: str = "cpu") -> dict:
    """Draw the layer's inputs and weights. Returns bf16 tensors (br fp32).

    ``device`` chooses where the generator runs; CPU and CUDA generators give
    different (but each reproducible) values for the same seed.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    d = dims
    out = {}
    out["x"] = _normal(gen, (d.B * d.T, d.D), 1.0, device)
    out["Wq"] = _normal(gen, (d.D, d.wq_cols), 0.02, device)
    out["Wk"] = _normal(gen, (d.D, d.G * d.dh), 0.02, device)
    out["Wv"] = _normal(gen, (d.D, d.G * d.dh), 0.02, device)
    out["Wr"] = _normal(gen, (d.D, d.G * d.M), 0.02, device)
    out["Wo"] = _normal(gen, (d.wo_rows, d.D), 0.02, device)
    out["Wo_dense"] = _normal(gen, (d.G * d.M * d.dh, d.D), 0.02, device)
    br = torch.zeros(d.G * d.M, dtype=torch.float32, device=device)
    if d.bias0 != 0.0:
        br[0::d.M] = d.bias0
    out["br"] = br
    return out


def make_x(dims: Dims, seed: int, device: str = "cpu") -> torch.Tensor:
    """Only the activations of ``make_inputs`` (same first draw)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return _normal(gen, (dims.B * dims.T, dims.D), 1.0, device)


def make_decode_inputs(dims: Dims, cache_len, seed: int = 0, device: str = "cpu") -> dict:
    """One decode step of the layer: weights as ``make_inputs`` (dims.T is the
    cache capacity), the new tokens x_new [B, D] ~ N(0, 1), and K/V caches
    [B, T, G, dh] ~ N(0, (0.02*sqrt(D))^2) -- the spread of x Wk for x ~ N(0, 1)
    and weights ~ N(0, 0.02^2) -- with the rows at and past cache_len[b]
    zeroed. cache_len ([B] ints, each < T) is returned as an int32 tensor."""
    d = dims
    out = make_inputs(Dims(B=d.B, T=1, D=d.D, G=d.G, M=d.M, k=d.k, dh=d.dh, bias0=d.bias0), seed, device)
    out["x_new"] = out.pop("x")
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 7919)
    std = 0.02 * d.D ** 0.5
    lens = torch.as_tensor(list(cache_len), dtype=torch.int32)
    keep = (torch.arange(d.T)[None, :] < lens[:, None]).to(device)[:, :, None, None]
    for key in ("K_cache", "V_cache"):
        c = torch.randn((d.B, d.T, d.G, d.dh), generator=gen, device=device, dtype=torch.float32) * std
        out[key] = (c * keep).to(torch.bfloat16)
    out["cache_len"] = lens.to(device)
    return out
