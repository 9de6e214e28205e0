"""Seeded synthetic inputs shared by the tests, the smoke entry and the bench.

This module draws random numbers only; it holds none of the attention or cache arithmetic.
Both the CUDA library and the oracle consume the tensors it returns. Draw order per
workload is fixed and documented so that a seed names one input set:
separator flags first, then Q, K, V, dO, each from one torch CPU generator.

The shapes, value distributions and flag patterns follow the workloads described for
SepLLM: a Pythia-160m-shaped training attention, Llama-3-8B-shaped prefill, a SepCache
streaming decode, a 131072-token stress case and a tiny GQA case.
"""

from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class AttnConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    a: int
    n: int
    seed: int
    flags: str        # "bernoulli" or "geometric"
    p: float          # Bernoulli probability, or 1/mean segment length
    bwd: bool
    force0: bool = False   # position 0 forced to be a non-separator

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    S: int
    Hq: int
    Hkv: int
    d: int
    a: int
    s: int
    c: int
    theta: float
    steps: int
    seed: int
    p: float

    @property
    def w(self) -> int:
        return self.c - self.a - self.s

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


TINY = AttnConfig("tiny-gqa-L512-d64", 1, 4, 1, 512, 64, 4, 64, 0, "bernoulli", 0.10, False, True)
PYTHIA160M = AttnConfig("pythia160m-train-B8-H12-L2048-d64", 8, 12, 12, 2048, 64, 4, 64, 1,
                        "geometric", 0.10, True)
LLAMA3_8B_PREFILL = AttnConfig("llama3-8b-prefill-H32-8-L8192-d128", 1, 32, 8, 8192, 128, 4, 256, 2,
                               "bernoulli", 0.08, False)
SEPCACHE_DECODE = DecodeConfig("sepcache-decode-S64-H32-8-d128-c800", 64, 32, 8, 128, 4, 64, 800,
                               500000.0, 65536, 3, 0.10)
LONG_CONTEXT = AttnConfig("long-context-H32-8-L131072-d128", 1, 32, 8, 131072, 128, 4, 256, 4,
                          "bernoulli", 0.10, True)

ATTN_CONFIGS = {c.name: c for c in (TINY, PYTHIA160M, LLAMA3_8B_PREFILL, LONG_CONTEXT)}


def separator_flags(g: torch.Generator, B: int, L: int, kind: str, p: float,
                    force0: bool = False) -> torch.Tensor:
    """uint8 [B, L] separator flags.

    "bernoulli": i.i.d. Bernoulli(p) per position.
    "geometric": segment lengths drawn from Geometric(p) on {1, 2, ...} (mean 1/p); the last
    token of every segment is a separator; the last segment is cut at L.
    """
    if kind == "bernoulli":
        sep = (torch.rand(B, L, generator=g) < p).to(torch.uint8)
    elif kind == "geometric":
        sep = torch.zeros(B, L, dtype=torch.uint8)
        for b in range(B):
            lens = torch.empty(L, dtype=torch.float64).geometric_(p, generator=g).to(torch.int64)
            ends = torch.cumsum(lens, 0) - 1
            ends = ends[ends < L]
            sep[b, ends] = 1
    else:
        raise ValueError(kind)
    if force0:
        sep[:, 0] = 0
    return sep


def _randn_bf16(g, shape, chunk=1 << 26):
    """N(0, 1) drawn in fp32 on the CPU generator, rounded to bf16 (chunked to bound memory)."""
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1)
    for s in range(0, flat.numel(), chunk):
        e = min(flat.numel(), s + chunk)
        flat[s:e] = torch.randn(e - s, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return out


def attn_inputs(cfg: AttnConfig, with_do: bool | None = None):
    """CPU tensors for one attention config: sep [B,L] u8, q [B,L,Hq,d], k/v [B,L,Hkv,d], dO."""
    g = torch.Generator().manual_seed(cfg.seed)
    sep = separator_flags(g, cfg.B, cfg.L, cfg.flags, cfg.p, cfg.force0)
    q = _randn_bf16(g, (cfg.B, cfg.L, cfg.Hq, cfg.d))
    k = _randn_bf16(g, (cfg.B, cfg.L, cfg.Hkv, cfg.d))
    v = _randn_bf16(g, (cfg.B, cfg.L, cfg.Hkv, cfg.d))
    want_do = cfg.bwd if with_do is None else with_do
    do = _randn_bf16(g, (cfg.B, cfg.L, cfg.Hq, cfg.d)) if want_do else None
    return dict(sep=sep, q=q, k=k, v=v, do=do)


def small_attn_inputs(seed, B, L, Hq, Hkv, d, p=0.1, kind="bernoulli", with_do=True):
    """Inputs for ad-hoc small shapes (ragged L, other head counts) in the tests."""
    g = torch.Generator().manual_seed(seed)
    sep = separator_flags(g, B, L, kind, p)
    q = _randn_bf16(g, (B, L, Hq, d))
    k = _randn_bf16(g, (B, L, Hkv, d))
    v = _randn_bf16(g, (B, L, Hkv, d))
    do = _randn_bf16(g, (B, L, Hq, d)) if with_do else None
    return dict(sep=sep, q=q, k=k, v=v, do=do)


def decode_chunk(cfg: DecodeConfig, first_step: int, nsteps: int, S: int | None = None,
                 device="cpu"):
    """Per-step decode inputs for steps [first_step, first_step + nsteps).

    Each 256-step chunk has its own generator seeded (seed, chunk index), so any chunk can be
    regenerated alone. Draw order inside a chunk: flags [256, S], q [256, S, Hq, d],
    k [256, S, Hkv, d], v [256, S, Hkv, d]. The generator runs on `device` (CPU by default;
    "cuda" for the full 65536-step stream, where a CPU draw would take minutes).
    """
    S = cfg.S if S is None else S
    CH = 256
    outs = {"sep": [], "q": [], "k": [], "v": []}
    c0 = first_step // CH
    c1 = (first_step + nsteps - 1) // CH
    for ci in range(c0, c1 + 1):
        g = torch.Generator(device=device).manual_seed(cfg.seed * 1_000_003 + ci)
        sep = (torch.rand(CH, S, generator=g, device=device) < cfg.p).to(torch.uint8)
        q = torch.randn(CH, S, cfg.Hq, cfg.d, generator=g, device=device).to(torch.bfloat16)
        k = torch.randn(CH, S, cfg.Hkv, cfg.d, generator=g, device=device).to(torch.bfloat16)
        v = torch.randn(CH, S, cfg.Hkv, cfg.d, generator=g, device=device).to(torch.bfloat16)
        lo = max(first_step, ci * CH) - ci * CH
        hi = min(first_step + nsteps, (ci + 1) * CH) - ci * CH
        outs["sep"].append(sep[lo:hi])
        outs["q"].append(q[lo:hi])
        outs["k"].append(k[lo:hi])
        outs["v"].append(v[lo:hi])
    return {key: torch.cat(val, 0) for key, val in outs.items()}
