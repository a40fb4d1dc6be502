"""Seeded synthetic inputs for the ternary MoE block.

This module draws random numbers and rounds them to their storage dtypes; it
holds none of the block's arithmetic (no packing, no routing, no matmul).  The
same draws feed the CUDA library and the CPU oracle.

Shapes and distributions (the pages' model families; dims the pages leave open
are chosen here and named as such):

* ``tiny``              d=256, 8 experts, top-2, ffn=128, no shared expert,
                        PQ2_0, fp32 router N(0,0.02) + delta N(0,0.002),
                        rank-32 correction, T=16.
* ``a3b_decode``        35B-A3B-class: d=2048, 256 experts, top-8 + 1 shared,
                        ffn=512, PQ2_0, bf16 router, rank-512 correction,
                        T in {1,8,32,64}, 40 independent layers.
* ``a3b_prefill``       the same layer at T=4096.
* ``flashnext_decode``  FlashNext-class: d=3072, 512 experts, top-10 + 1
                        shared, ffn=768, PTQ1_0, rank-512 correction,
                        T in {1,16,64}, 48 independent layers.
* ``flashnext_prefill`` the same layer at T=16384 with a router bias whose
                        expert popularity follows Zipf(1.2) over a seeded
                        permutation of the experts.

Expert codes are iid with P(0)=0.4 and P(-1)=P(+1)=0.3; group scales are
U[0.005, 0.02] rounded to fp16; activations x ~ N(0,1) rounded to bf16; the
bf16 router has std 1/sqrt(d) (router logits ~ N(0,1)) and its delta a tenth
of that; shared-expert and correction weights are N(0, 0.02) in bf16.

bf16 and fp16 values are returned as their uint16 bit patterns (numpy) or as
torch bf16/fp16 tensors (device generators).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

PQ2_0 = 0
PTQ1_0 = 1


@dataclass(frozen=True)
class Config:
    name: str
    index: int            # seeds are 1000*index + layer
    d: int
    n_experts: int
    top_k: int
    ffn: int
    shared_ffn: int
    fmt: int
    rank: int
    router_f32: bool
    tokens: List[int] = field(default_factory=list)
    n_layers: int = 1
    zipf_s: Optional[float] = None


CONFIGS: Dict[str, Config] = {
    c.name: c
    for c in [
        Config("tiny", 1, 256, 8, 2, 128, 0, PQ2_0, 32, True, [16], 1),
        Config("a3b_decode", 2, 2048, 256, 8, 512, 512, PQ2_0, 512, False, [1, 8, 32, 64], 40),
        Config("a3b_prefill", 3, 2048, 256, 8, 512, 512, PQ2_0, 512, False, [4096], 2),
        Config("flashnext_decode", 4, 3072, 512, 10, 768, 768, PTQ1_0, 512, False, [1, 16, 64], 48),
        Config("flashnext_prefill", 5, 3072, 512, 10, 768, 768, PTQ1_0, 512, False, [16384], 2, 1.2),
    ]
}


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def layer_seed(cfg: Config, layer: int) -> int:
    return 1000 * cfg.index + layer


def x_seed(cfg: Config, T: int, stream: int = 0) -> int:
    return 1_000_000 + 1000 * cfg.index + 97 * T + stream


# ----------------------------------------------------------- dtype rounding
def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round-to-nearest-even, by torch) -> uint16 bit patterns."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def to_f16_bits(a: np.ndarray) -> np.ndarray:
    """Round to fp16 (numpy, round-to-nearest-even) -> uint16 bit patterns."""
    return np.ascontiguousarray(a).astype(np.float16).view(np.uint16)


# ---------------------------------------------------------- host generators
_CODE_OF_DIGIT = np.array([0, 0, 0, 0, 1, 1, 1, -1, -1, -1], dtype=np.int8)


def ternary_codes(rng: np.random.Generator, shape) -> np.ndarray:
    """iid codes: a uniform decimal digit maps 0-3 -> 0, 4-6 -> +1, 7-9 -> -1."""
    return _CODE_OF_DIGIT[rng.integers(0, 10, size=shape, dtype=np.uint8)]


def group_scales(rng: np.random.Generator, shape) -> np.ndarray:
    return to_f16_bits(rng.uniform(0.005, 0.02, size=shape))


def normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std))


def zipf_router_column(cfg: Config, seed: int) -> np.ndarray:
    """ln p_{pi(e)} with p_i proportional to i^-s over a seeded permutation pi (float32)."""
    rng = rng_for(seed + 7)
    ranks = np.arange(1, cfg.n_experts + 1, dtype=np.float64)
    p = ranks ** (-cfg.zipf_s)
    p /= p.sum()
    perm = rng.permutation(cfg.n_experts)
    return np.log(p[perm]).astype(np.float32)


def layer_host(cfg: Config, layer: int = 0) -> dict:
    """All weights of one layer as numpy arrays (codes int8, fp16/bf16 as uint16)."""
    seed = layer_seed(cfg, layer)
    rng = rng_for(seed)
    d, E, F, Fs, r = cfg.d, cfg.n_experts, cfg.ffn, cfg.shared_ffn, cfg.rank
    out = {}
    if cfg.router_f32:
        out["w_router"] = (rng.standard_normal((E, d), dtype=np.float32) * np.float32(0.02))
        out["w_delta"] = (rng.standard_normal((E, d), dtype=np.float32) * np.float32(0.002))
    else:
        std = 1.0 / np.sqrt(d)
        wr = rng.standard_normal((E, d), dtype=np.float32) * np.float32(std)
        wd = rng.standard_normal((E, d), dtype=np.float32) * np.float32(0.1 * std)
        if cfg.zipf_s is not None:
            wr[:, 0] = zipf_router_column(cfg, seed)
            wd[:, 0] = 0.0
        out["w_router"] = to_bf16_bits(wr)
        out["w_delta"] = to_bf16_bits(wd)
    out["gate_codes"] = ternary_codes(rng, (E, F, d))
    out["gate_scales"] = group_scales(rng, (E, F, d // 128))
    out["up_codes"] = ternary_codes(rng, (E, F, d))
    out["up_scales"] = group_scales(rng, (E, F, d // 128))
    out["down_codes"] = ternary_codes(rng, (E, d, F))
    out["down_scales"] = group_scales(rng, (E, d, F // 128))
    if Fs:
        out["sh_gate"] = normal_bf16(rng, (Fs, d), 0.02)
        out["sh_up"] = normal_bf16(rng, (Fs, d), 0.02)
        out["sh_down"] = normal_bf16(rng, (d, Fs), 0.02)
    if r:
        out["corr_a"] = normal_bf16(rng, (r, d), 0.02)
        out["corr_b"] = normal_bf16(rng, (d, r), 0.02)
    return out


def x_host(cfg: Config, T: int, stream: int = 0) -> np.ndarray:
    """Activations bf16 [T, d] (uint16 bits); channel 0 is 1.0 for the Zipf config."""
    rng = rng_for(x_seed(cfg, T, stream))
    x = rng.standard_normal((T, cfg.d), dtype=np.float32)
    if cfg.zipf_s is not None:
        x[:, 0] = 1.0
    return to_bf16_bits(x)


def x_rows_host(cfg: Config, n: int, seed: int) -> np.ndarray:
    """Fresh replacement rows (for resampling tokens), same distribution as x_host."""
    rng = rng_for(seed)
    x = rng.standard_normal((n, cfg.d), dtype=np.float32)
    if cfg.zipf_s is not None:
        x[:, 0] = 1.0
    return to_bf16_bits(x)


# -------------------------------------------------------- device generators
def layer_device(cfg: Config, layer: int, device) -> dict:
    """Same distributions as layer_host, drawn on the GPU by torch (different stream of
    random numbers; used where host generation of tens of GB would dominate)."""
    import torch

    g = torch.Generator(device=device)
    seed = layer_seed(cfg, layer)
    g.manual_seed(seed)
    d, E, F, Fs, r = cfg.d, cfg.n_experts, cfg.ffn, cfg.shared_ffn, cfg.rank
    lut = torch.tensor([0, 0, 0, 0, 1, 1, 1, -1, -1, -1], dtype=torch.int8, device=device)

    def codes(shape):
        return lut[torch.randint(0, 10, shape, generator=g, device=device)]

    def scales(shape):
        return torch.empty(shape, device=device).uniform_(0.005, 0.02, generator=g).half()

    def nbf16(shape, std):
        return (torch.randn(shape, generator=g, device=device) * std).bfloat16()

    out = {}
    if cfg.router_f32:
        out["w_router"] = torch.randn((E, d), generator=g, device=device) * 0.02
        out["w_delta"] = torch.randn((E, d), generator=g, device=device) * 0.002
    else:
        std = 1.0 / float(np.sqrt(d))
        wr = torch.randn((E, d), generator=g, device=device) * std
        wd = torch.randn((E, d), generator=g, device=device) * (0.1 * std)
        if cfg.zipf_s is not None:
            wr[:, 0] = torch.from_numpy(zipf_router_column(cfg, seed)).to(device)
            wd[:, 0] = 0.0
        out["w_router"] = wr.bfloat16()
        out["w_delta"] = wd.bfloat16()
    out["gate_codes"] = codes((E, F, d))
    out["gate_scales"] = scales((E, F, d // 128))
    out["up_codes"] = codes((E, F, d))
    out["up_scales"] = scales((E, F, d // 128))
    out["down_codes"] = codes((E, d, F))
    out["down_scales"] = scales((E, d, F // 128))
    if Fs:
        out["sh_gate"] = nbf16((Fs, d), 0.02)
        out["sh_up"] = nbf16((Fs, d), 0.02)
        out["sh_down"] = nbf16((d, Fs), 0.02)
    if r:
        out["corr_a"] = nbf16((r, d), 0.02)
        out["corr_b"] = nbf16((d, r), 0.02)
    return out


def x_device(cfg: Config, T: int, device, stream: int = 0):
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(x_seed(cfg, T, stream))
    x = torch.randn((T, cfg.d), generator=g, device=device)
    if cfg.zipf_s is not None:
        x[:, 0] = 1.0
    return x.bfloat16()
