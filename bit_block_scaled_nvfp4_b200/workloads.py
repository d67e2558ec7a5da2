"""Seeded synthetic inputs shaped like the long-context attention workloads.

This module draws random numbers and nothing else: it holds none of the method's arithmetic,
so both the CUDA library's tests/benchmarks and the CPU oracle can be fed from it.

Recipe (all draws on the CPU from one ``torch.Generator`` per workload, in float32, then
rounded once to fp16 or bf16):

* Q, V ~ N(0, 1).
* K = N(0, 1) + mu_c, with mu_c ~ N(0, 0.5^2) per (KV head, channel), shared by all tokens.
* Outlier channels: per KV head, ``outliers`` channels drawn without replacement; the whole
  channel of K (mean included) is multiplied by 10.
* Heavy hitters (mixed-precision workload only): per KV head, ``heavy`` token positions drawn
  without replacement; their whole key vector is multiplied by 4.
* Paged decode: context lengths uniform on [len_lo, len_hi] (integers), a random
  permutation of the physical pages, one generator per sequence for its K/V so a single
  sequence can be regenerated alone; the per-(KV head, channel) means and outlier channels
  are drawn once and shared by every sequence.

The draw order is fixed (q, mu, outlier channels, k noise, heavy positions, v).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

WORKLOADS = {
    "tiny_prefill": dict(B=1, Hq=2, Hkv=2, N=256, d=64, causal=False, dtype="fp16",
                         outliers=2, heavy=0, frac_bp=0, seed=0),
    "prefill_h16_n4096": dict(B=1, Hq=16, Hkv=16, N=4096, d=128, causal=True, dtype="bf16",
                              outliers=4, heavy=0, frac_bp=0, seed=1),
    "prefill_gqa_n32768": dict(B=1, Hq=32, Hkv=8, N=32768, d=128, causal=True, dtype="bf16",
                               outliers=4, heavy=0, frac_bp=0, seed=2),
    "mixed_prefill_n16384": dict(B=1, Hq=32, Hkv=8, N=16384, d=128, causal=True,
                                 dtype="bf16", outliers=4, heavy=64, frac_bp=500, seed=3),
    "paged_decode_s64": dict(S=64, len_lo=8192, len_hi=32768, Hq=32, Hkv=8, d=128, page=64,
                             dtype="bf16", outliers=4, seed=4),
}

_TORCH_DTYPE = {"fp16": torch.float16, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _TORCH_DTYPE[name]


@dataclass
class PrefillInputs:
    q: torch.Tensor            # [B, Hq, N, d]  (fp16 / bf16, CPU)
    k: torch.Tensor            # [B, Hkv, N, d]
    v: torch.Tensor            # [B, Hkv, N, d]
    cfg: dict = field(default_factory=dict)


def make_prefill(name_or_cfg, **override) -> PrefillInputs:
    cfg = dict(WORKLOADS[name_or_cfg]) if isinstance(name_or_cfg, str) else dict(name_or_cfg)
    cfg.update(override)
    B, Hq, Hkv, N, d = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["N"], cfg["d"]
    g = torch.Generator().manual_seed(int(cfg["seed"]))
    q = torch.randn(B, Hq, N, d, generator=g)
    mu = torch.randn(1, Hkv, 1, d, generator=g) * 0.5
    scale = torch.ones(1, Hkv, 1, d)
    for h in range(Hkv):
        ch = torch.randperm(d, generator=g)[: cfg["outliers"]]
        scale[0, h, 0, ch] = 10.0
    k = (torch.randn(B, Hkv, N, d, generator=g) + mu) * scale
    if cfg.get("heavy", 0):
        for h in range(Hkv):
            pos = torch.randperm(N, generator=g)[: cfg["heavy"]]
            k[:, h, pos, :] *= 4.0
    v = torch.randn(B, Hkv, N, d, generator=g)
    dt = torch_dtype(cfg["dtype"])
    return PrefillInputs(q.to(dt), k.to(dt), v.to(dt), cfg)


@dataclass
class DecodeLayout:
    lens: torch.Tensor         # [S] int32 context lengths
    page_table: torch.Tensor   # [S, max_pages] int32 physical page ids (-1 past the end)
    num_pages: int
    cfg: dict = field(default_factory=dict)
    mu: torch.Tensor = None    # [Hkv, d] per-channel means
    chan_scale: torch.Tensor = None  # [Hkv, d] 10 on outlier channels, else 1


def make_decode_layout(name_or_cfg="paged_decode_s64", **override) -> DecodeLayout:
    cfg = dict(WORKLOADS[name_or_cfg]) if isinstance(name_or_cfg, str) else dict(name_or_cfg)
    cfg.update(override)
    S, Hkv, d, page = cfg["S"], cfg["Hkv"], cfg["d"], cfg["page"]
    g = torch.Generator().manual_seed(int(cfg["seed"]))
    lens = torch.randint(cfg["len_lo"], cfg["len_hi"] + 1, (S,), generator=g, dtype=torch.int64)
    pages_per = (lens + page - 1) // page
    num_pages = int(pages_per.sum())
    perm = torch.randperm(num_pages, generator=g)
    max_pages = int(pages_per.max())
    table = torch.full((S, max_pages), -1, dtype=torch.int32)
    off = 0
    for s in range(S):
        n = int(pages_per[s])
        table[s, :n] = perm[off:off + n].to(torch.int32)
        off += n
    mu = torch.randn(Hkv, d, generator=g) * 0.5
    chan = torch.ones(Hkv, d)
    for h in range(Hkv):
        ch = torch.randperm(d, generator=g)[: cfg["outliers"]]
        chan[h, ch] = 10.0
    return DecodeLayout(lens.to(torch.int32), table, num_pages, cfg, mu, chan)


def make_decode_sequence(layout: DecodeLayout, s: int):
    """K, V of sequence ``s``: [len, Hkv, d] each (bf16, CPU), from the sequence's own
    generator."""
    cfg = layout.cfg
    n = int(layout.lens[s])
    g = torch.Generator().manual_seed(int(cfg["seed"]) * 100003 + 17 + s)
    k = (torch.randn(n, cfg["Hkv"], cfg["d"], generator=g) + layout.mu) * layout.chan_scale
    v = torch.randn(n, cfg["Hkv"], cfg["d"], generator=g)
    dt = torch_dtype(cfg["dtype"])
    return k.to(dt), v.to(dt)


def make_decode_query(layout: DecodeLayout, step: int = 0):
    """The step's query: [S, Hq, d] (bf16, CPU)."""
    cfg = layout.cfg
    g = torch.Generator().manual_seed(int(cfg["seed"]) * 7919 + 3 + step)
    q = torch.randn(cfg["S"], cfg["Hq"], cfg["d"], generator=g)
    return q.to(torch_dtype(cfg["dtype"]))


#: Fixed NVFP4 tensor scale of the synthetic K cache (a power of two, so it is exact). With
#: block scales up to 448 and elements up to 6 it covers |k| <= 168; the synthetic keys stay
#: well inside that.
DECODE_K_TENSOR_SCALE = 0.0625
