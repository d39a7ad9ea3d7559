"""Seeded synthetic inputs for shared-index top-k sparse KV attention.

This module only draws inputs.  It holds none of the attention arithmetic, so both
the CUDA library's tests and the fp64 oracle can use it.  Every tensor is drawn in
fp32 from a ``torch.Generator`` on the CPU (or on a given device for large bench
copies) and rounded once to bf16.

Workloads (shapes of the MAGE page's long-context setting -- 8K to 128K context,
top-k of 512 to 2048 tokens, 32 denoising steps per block -- with needle-style
pages in the spirit of the Needle-in-a-Haystack suite the pages evaluate on):

==========  ======================================================================
tiny        1 seq, n=1024, B=4, Hq=4, Hkv=1, d=64, page 16, top-k 128 tokens
            (8 pages), 4 steps; 8 planted pages per KV head.
8k          1 seq, n=8192, B=32, Hq=32, Hkv=8, d=128, page 16, top-k 512 tokens,
            32 steps; 1% of the pages carry a needle.
32k         1 seq, n=32768, B=32, Hq=28, Hkv=4, d=128, page 64, top-k 1024
            tokens, 32 steps; power-law page norms (Zipf exponent 1.1).
128k        1 seq, n=131072, B=32, Hq=32, Hkv=8, d=128, page 16, top-k 1024
            tokens, 32 steps; 0.5% needle pages.
batched     8 seqs, n uniform in [16384, 65536], B=32, Hq=32, Hkv=8, d=128,
            page 16, top-k per seq in {512, 1024, 2048} tokens, 32 steps; key
            temperature per (seq, KV head) uniform in [0.5, 2]; random page table.
==========  ======================================================================

Draw order for one workload: K, V, Q1, the block's own K/V for step 1, then the
structure (needles / page norms / temperatures / page table).  The inputs of
denoising step t >= 2 come from a fresh generator seeded by (seed, t): queries and
the block's K/V are the step-1 values plus N(0, 0.1^2) noise.

A needle at page q of KV head h adds ``strength * mean_{b,g} Q1[b, h*G+g]`` to
every key of that page (computed in fp32 before the single bf16 rounding), so the
block-average query scores those keys higher.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

CONFIG_NAMES = ("tiny", "8k", "32k", "128k", "batched")

# base shapes; every field can be overridden by make(..., **overrides)
_BASE = {
    "tiny": dict(S=1, n=1024, B=4, Hq=4, Hkv=1, d=64, P=16, topk=128, T=4,
                 needle_count=8, needle_strength=3.0),
    "8k": dict(S=1, n=8192, B=32, Hq=32, Hkv=8, d=128, P=16, topk=512, T=32,
               needle_frac=0.01, needle_strength=3.0),
    "32k": dict(S=1, n=32768, B=32, Hq=28, Hkv=4, d=128, P=64, topk=1024, T=32,
                zipf_s=1.1, zipf_scale=4.0),
    "128k": dict(S=1, n=131072, B=32, Hq=32, Hkv=8, d=128, P=16, topk=1024, T=32,
                 needle_frac=0.005, needle_strength=3.0),
    "batched": dict(S=8, n_lo=16384, n_hi=65536, B=32, Hq=32, Hkv=8, d=128, P=16,
                    topk_choices=(512, 1024, 2048), T=32, temp_lo=0.5, temp_hi=2.0,
                    random_page_table=True),
}

STEP_NOISE_STD = 0.1


@dataclass
class Workload:
    name: str
    seed: int
    S: int
    B: int
    Hq: int
    Hkv: int
    d: int
    P: int
    T: int
    n_ctx: torch.Tensor          # [S] int32
    topk: torch.Tensor           # [S] int32, tokens
    max_pages: int
    n_phys: int
    page_table: torch.Tensor | None   # [S, max_pages] int32 (None = identity)
    q1: torch.Tensor             # [S, B, Hq, d] bf16
    k_cache: torch.Tensor        # [n_phys, Hkv, P, d] bf16
    v_cache: torch.Tensor        # [n_phys, Hkv, P, d] bf16
    blk_k1: torch.Tensor         # [S, B, Hkv, d] bf16
    blk_v1: torch.Tensor         # [S, B, Hkv, d] bf16
    planted: dict = field(default_factory=dict)   # (s, h) -> sorted list of logical pages

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def kmax(self) -> int:
        return int(self.topk.max()) // self.P

    def n_pages(self, s: int) -> int:
        return (int(self.n_ctx[s]) + self.P - 1) // self.P

    def step_inputs(self, t: int):
        """(q_t, blk_k_t, blk_v_t) for denoising step t (t = 1 returns the step-1 inputs)."""
        if t <= 1:
            return self.q1, self.blk_k1, self.blk_v1
        g = torch.Generator(device="cpu")
        g.manual_seed(self.seed * 1_000_003 + 7919 * t)
        out = []
        for base in (self.q1, self.blk_k1, self.blk_v1):
            noise = torch.randn(base.shape, generator=g, dtype=torch.float32)
            out.append((base.float() + STEP_NOISE_STD * noise).to(torch.bfloat16))
        return tuple(out)

    def physical_page(self, s: int, lp: int) -> int:
        if self.page_table is None:
            return s * self.max_pages + lp
        return int(self.page_table[s, lp])


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> its raw bit patterns as a uint16 numpy array (no rounding)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def config(name: str, **overrides) -> dict:
    if name not in _BASE:
        raise KeyError(f"unknown workload {name!r}; known: {CONFIG_NAMES}")
    cfg = dict(_BASE[name])
    cfg.update(overrides)
    return cfg


def make(name: str, seed: int = 0, **overrides) -> Workload:
    """Draw the seeded inputs of workload `name` (shapes overridable for small tests)."""
    cfg = config(name, **overrides)
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    S, B, Hq, Hkv, d, P = (cfg[x] for x in ("S", "B", "Hq", "Hkv", "d", "P"))
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv

    # prefix lengths and budgets
    if "n_lo" in cfg:
        n = torch.randint(cfg["n_lo"], cfg["n_hi"] + 1, (S,), generator=g, dtype=torch.int64)
        choices = torch.tensor(cfg["topk_choices"], dtype=torch.int64)
        topk = choices[torch.randint(0, len(choices), (S,), generator=g)]
    else:
        n = torch.full((S,), int(cfg["n"]), dtype=torch.int64)
        tk = cfg["topk"]
        topk = torch.tensor(tk if isinstance(tk, (list, tuple)) else [tk] * S, dtype=torch.int64)
    n_ctx = n.to(torch.int32)
    topk = topk.to(torch.int32)
    nps = [(int(x) + P - 1) // P for x in n]
    max_pages = max(nps)
    total_pages = sum(nps)

    # K, V drawn per sequence in logical page order, then Q1 and the block's K/V
    k_log = [torch.randn((nps[s], Hkv, P, d), generator=g, dtype=torch.float32) for s in range(S)]
    v_log = [torch.randn((nps[s], Hkv, P, d), generator=g, dtype=torch.float32) for s in range(S)]
    q1 = torch.randn((S, B, Hq, d), generator=g, dtype=torch.float32)
    blk_k1 = torch.randn((S, B, Hkv, d), generator=g, dtype=torch.float32)
    blk_v1 = torch.randn((S, B, Hkv, d), generator=g, dtype=torch.float32)
    q1_bf = q1.to(torch.bfloat16)

    planted: dict = {}
    # needles: K += strength * mean over the block's queries of the KV head's group
    if "needle_count" in cfg or "needle_frac" in cfg:
        strength = float(cfg["needle_strength"])
        qmean = q1_bf.float().view(S, B, Hkv, G, d).mean(dim=(1, 3))  # [S, Hkv, d]
        for s in range(S):
            count = (int(cfg["needle_count"]) if "needle_count" in cfg
                     else max(1, int(round(cfg["needle_frac"] * nps[s]))))
            if count > nps[s] - 1:
                raise ValueError("too many needles for the prefix")
            for h in range(Hkv):
                pages = torch.randperm(nps[s] - 1, generator=g)[:count].sort().values
                k_log[s][pages, h] += strength * qmean[s, h]
                planted[(s, h)] = [int(x) for x in pages]
    # power-law page norms: page of rank r scaled by zipf_scale * r^-s
    if "zipf_s" in cfg:
        for s in range(S):
            rank = torch.randperm(nps[s], generator=g).to(torch.float32) + 1.0
            scale = cfg["zipf_scale"] * rank.pow(-float(cfg["zipf_s"]))
            k_log[s] *= scale.view(-1, 1, 1, 1)
    # per-(seq, KV head) key temperature
    if "temp_lo" in cfg:
        for s in range(S):
            tau = cfg["temp_lo"] + (cfg["temp_hi"] - cfg["temp_lo"]) * torch.rand(
                (Hkv,), generator=g, dtype=torch.float32)
            k_log[s] /= tau.view(1, Hkv, 1, 1)

    # physical layout
    if cfg.get("random_page_table", False):
        n_phys = total_pages
        perm = torch.randperm(n_phys, generator=g).to(torch.int32)
        page_table = torch.full((S, max_pages), -1, dtype=torch.int32)
        off = 0
        for s in range(S):
            page_table[s, : nps[s]] = perm[off: off + nps[s]]
            off += nps[s]
        k_cache = torch.empty((n_phys, Hkv, P, d), dtype=torch.bfloat16)
        v_cache = torch.empty((n_phys, Hkv, P, d), dtype=torch.bfloat16)
        for s in range(S):
            rows = page_table[s, : nps[s]].long()
            k_cache[rows] = k_log[s].to(torch.bfloat16)
            v_cache[rows] = v_log[s].to(torch.bfloat16)
    else:
        page_table = None
        n_phys = S * max_pages
        k_cache = torch.zeros((n_phys, Hkv, P, d), dtype=torch.bfloat16)
        v_cache = torch.zeros((n_phys, Hkv, P, d), dtype=torch.bfloat16)
        for s in range(S):
            k_cache[s * max_pages: s * max_pages + nps[s]] = k_log[s].to(torch.bfloat16)
            v_cache[s * max_pages: s * max_pages + nps[s]] = v_log[s].to(torch.bfloat16)

    return Workload(
        name=name, seed=seed, S=S, B=B, Hq=Hq, Hkv=Hkv, d=d, P=P, T=int(cfg["T"]),
        n_ctx=n_ctx, topk=topk, max_pages=max_pages, n_phys=n_phys, page_table=page_table,
        q1=q1_bf, k_cache=k_cache, v_cache=v_cache,
        blk_k1=blk_k1.to(torch.bfloat16), blk_v1=blk_v1.to(torch.bfloat16), planted=planted)


def with_page_table(w: Workload, seed: int) -> Workload:
    """The same logical data laid out through a random page table (an invariance check)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    nps = [w.n_pages(s) for s in range(w.S)]
    n_phys = sum(nps) + 3  # a few unused physical pages
    perm = torch.randperm(n_phys, generator=g).to(torch.int32)
    pt = torch.full((w.S, w.max_pages), -1, dtype=torch.int32)
    k = torch.zeros((n_phys, w.Hkv, w.P, w.d), dtype=torch.bfloat16)
    v = torch.zeros_like(k)
    off = 0
    for s in range(w.S):
        pt[s, : nps[s]] = perm[off: off + nps[s]]
        off += nps[s]
        for lp in range(nps[s]):
            src = w.physical_page(s, lp)
            k[int(pt[s, lp])] = w.k_cache[src]
            v[int(pt[s, lp])] = w.v_cache[src]
    return Workload(
        name=w.name + "+pt", seed=w.seed, S=w.S, B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, P=w.P,
        T=w.T, n_ctx=w.n_ctx.clone(), topk=w.topk.clone(), max_pages=w.max_pages,
        n_phys=n_phys, page_table=pt, q1=w.q1, k_cache=k, v_cache=v, blk_k1=w.blk_k1,
        blk_v1=w.blk_v1, planted=dict(w.planted))
