"""Seeded synthetic decode workloads for Slow-Fast Inference (SFI).

This module only draws inputs: paged K/V caches, page tables, per-step
queries and new tokens, and the boundary-token stream that drives the
slow/fast trigger.  It computes nothing of the method itself (no attention,
no scoring, no selection), so both the CUDA path and the CPU oracle can be
fed from it without sharing any of the method's arithmetic.

The pages measure SFI on Qwen3 models over LongBench / long-CoT traces
(Slow-Fast Inference summaries, gist.science/es "4. Resultados Principales",
gist.science/zh "4. 实验结果").  Neither weights nor datasets are used here;
these synthetic caches stand in for them with the head layout of the named
Qwen3 shapes:

* K and V entries are N(0, 1).  Every key row is scaled by a per-token
  LogNormal(0, 0.5) factor; with ``outlier_frac`` > 0 that fraction of rows is
  scaled by a further 10x (large-norm keys, the case the key-norm prior is
  meant to damp).
* A query is  q_h = beta * sum_{m in P_h(t)} k_m / ||k_m||  +  N(0, 0.3^2)
  with beta = 8, i.e. a few "planted" support positions per head plus noise.
  ``planted`` mode: 3 fixed positions per (batch, query head).
  ``clusters`` mode: 8 clusters of 8 positions per (batch, KV head); query
  head h uses a fixed 3-subset of the active cluster, and the active cluster
  changes at every boundary token (or on its own Bernoulli stream).
* The cache is paged, 16 tokens per page, with a seeded random permutation as
  page table.  Positions at or beyond ``context`` start as zeros; decode
  step t appends the token at position ``context + t``.
* The boundary stream is Bernoulli(p) per step (or a fixed pattern).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np
import torch

PAGE = 16
BETA = 8.0
Q_NOISE = 0.3
KEY_LOGNORMAL_SIGMA = 0.5
OUTLIER_SCALE = 10.0


@dataclasses.dataclass(frozen=True)
class SFIConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    context: int                 # cache length before the first decode step
    steps: int                   # decode steps T
    n_layers: int = 1
    n_sink: int = 4
    n_recent: int = 128
    k_fixed: int = 0             # >0: fixed K per query head; else floor(budget_frac * L)
    budget_frac: float = 0.2
    lam: float = 0.2
    lam_clip: float = 0.5
    alpha_soft: float = 0.5
    alpha_cross: float = 0.5
    nms_window: int = 32
    refresh_budget: int = 32
    evidence_window: int = 1           # queries whose attention the Selector's evidence averages
    boundary_mode: str = "bernoulli"   # "none" | "bernoulli" | "slow_prefix"
    boundary_p: float = 1.0 / 16.0
    slow_prefix: int = 0               # "slow_prefix": steps [0, slow_prefix) are slow
    query_mode: str = "planted"        # "planted" | "clusters"
    cluster_switch: str = "boundary"   # "boundary" | "bernoulli"
    outlier_frac: float = 0.0
    seed: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def pages_per_seq(self) -> int:
        return -(-(self.context + self.steps) // PAGE)

    @property
    def num_pages(self) -> int:
        return self.B * self.pages_per_seq

    @property
    def capacity(self) -> int:
        return self.pages_per_seq * PAGE

    def seq_len(self, t: int) -> int:
        """Context length L at decode step t (the new token included)."""
        return self.context + t + 1

    def replace(self, **kw) -> "SFIConfig":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny one the oracle finishes in seconds and four
# shaped after the attention layers of Qwen3-0.6B, Qwen3-4B (32K and 128K x
# 36 layers) and Qwen3-235B-A22B.
CONFIGS: List[SFIConfig] = [
    SFIConfig("tiny-gqa2-d64-1k", B=1, Hq=4, Hkv=2, D=64, context=1024, steps=32,
              n_recent=64, k_fixed=128, refresh_budget=8, boundary_mode="none",
              query_mode="planted", seed=0),
    SFIConfig("qwen3-0.6b-8k", B=4, Hq=16, Hkv=8, D=128, context=8192, steps=256,
              n_recent=128, budget_frac=0.20, refresh_budget=32,
              boundary_mode="bernoulli", query_mode="planted", seed=1),
    SFIConfig("qwen3-4b-32k", B=8, Hq=32, Hkv=8, D=128, context=32768, steps=512,
              n_recent=256, budget_frac=0.15, refresh_budget=32,
              boundary_mode="bernoulli", query_mode="clusters", outlier_frac=0.005,
              seed=2),
    SFIConfig("qwen3-4b-128k-36l", B=2, Hq=32, Hkv=8, D=128, context=131072, steps=256,
              n_layers=36, n_recent=256, budget_frac=0.15, refresh_budget=32,
              boundary_mode="bernoulli", query_mode="clusters", outlier_frac=0.005,
              seed=3),
    SFIConfig("qwen3-235b-a22b-64k", B=16, Hq=64, Hkv=4, D=128, context=65536, steps=512,
              n_recent=256, budget_frac=0.20, nms_window=32, refresh_budget=1 << 30,
              boundary_mode="slow_prefix", slow_prefix=64, query_mode="clusters",
              cluster_switch="bernoulli", outlier_frac=0.005, seed=4),
]

CONFIG_BY_NAME = {c.name: c for c in CONFIGS}

_TAGS = {"page_table": 1, "k": 2, "v": 3, "kscale": 4, "outlier": 5, "planted": 6,
         "qnoise": 7, "knew": 8, "vnew": 9, "boundary": 10, "clusters": 11,
         "switch": 12, "boundary_rows": 13}


def _seed(cfg: SFIConfig, layer: int, what: str, extra: int = 0) -> int:
    ss = np.random.SeedSequence([cfg.seed, layer, _TAGS[what], extra])
    return int(ss.generate_state(1, np.uint64)[0] & np.uint64(0x7FFF_FFFF_FFFF_FFFF))


def _np_rng(cfg, layer, what, extra=0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(_seed(cfg, layer, what, extra)))


def _torch_gen(cfg, layer, what, device, extra=0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(cfg, layer, what, extra))
    return g


def boundary_stream(cfg: SFIConfig) -> np.ndarray:
    """int8[T]: 1 where decode step t emitted a boundary token (". ? !" etc.)."""
    T = cfg.steps
    if cfg.boundary_mode == "none":
        return np.zeros(T, np.int8)
    if cfg.boundary_mode == "slow_prefix":
        b = np.zeros(T, np.int8)
        b[: max(cfg.slow_prefix - 1, 0)] = 1
        return b
    rng = _np_rng(cfg, 0, "boundary")
    return (rng.random(T) < cfg.boundary_p).astype(np.int8)


def boundary_rows(cfg: SFIConfig) -> np.ndarray:
    """int8[B, T]: boundary tokens of every sequence of the batch, drawn
    independently (Bernoulli(boundary_p) per sequence and step), for decoding
    with a trigger per sequence."""
    T, B = cfg.steps, cfg.B
    if cfg.boundary_mode != "bernoulli":
        return np.broadcast_to(boundary_stream(cfg), (B, T)).copy()
    rng = _np_rng(cfg, 0, "boundary_rows")
    return (rng.random((B, T)) < cfg.boundary_p).astype(np.int8)


def page_table(cfg: SFIConfig, layer: int) -> np.ndarray:
    """int32[B, pages_per_seq]: a seeded random permutation of the pool."""
    rng = _np_rng(cfg, layer, "page_table")
    perm = rng.permutation(cfg.num_pages).astype(np.int32)
    return perm.reshape(cfg.B, cfg.pages_per_seq)


def _key_rows(cfg, layer, what, shape, device, gen_extra=0):
    """Key rows: N(0,1) entries, each row scaled by LogNormal(0, 0.5), and an
    ``outlier_frac`` share of rows scaled by a further 10x."""
    g = _torch_gen(cfg, layer, what, device, gen_extra)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    gs = _torch_gen(cfg, layer, "kscale", device, gen_extra * 2 + (1 if what == "knew" else 0))
    scale = torch.exp(KEY_LOGNORMAL_SIGMA *
                      torch.randn(*shape[:-1], generator=gs, device=device, dtype=torch.float32))
    if cfg.outlier_frac > 0:
        go = _torch_gen(cfg, layer, "outlier", device, gen_extra * 2 + (1 if what == "knew" else 0))
        out = torch.rand(*shape[:-1], generator=go, device=device) < cfg.outlier_frac
        scale = torch.where(out, scale * OUTLIER_SCALE, scale)
    return x * scale.unsqueeze(-1)


@dataclasses.dataclass
class LayerInputs:
    k_pool: torch.Tensor       # bf16 [num_pages, Hkv, 16, D]
    v_pool: torch.Tensor       # bf16 [num_pages, Hkv, 16, D]
    page_table: torch.Tensor   # int32 [B, pages_per_seq]
    q: torch.Tensor            # bf16 [T, B, Hq, D]
    k_new: torch.Tensor        # bf16 [T, B, Hkv, D]
    v_new: torch.Tensor        # bf16 [T, B, Hkv, D]
    planted: np.ndarray        # int64 [T, B, Hq, 3] planted positions per step


def _planted_positions(cfg: SFIConfig, layer: int, boundary: np.ndarray) -> np.ndarray:
    """int64[T, B, Hq, 3] planted support positions for every step."""
    T, B, Hq, G = cfg.steps, cfg.B, cfg.Hq, cfg.G
    lo, hi = cfg.n_sink, cfg.context - cfg.n_recent
    rng = _np_rng(cfg, layer, "planted")
    if cfg.query_mode == "planted":
        p = np.stack([rng.choice(np.arange(lo, hi), size=3, replace=False)
                      for _ in range(B * Hq)]).reshape(B, Hq, 3)
        return np.broadcast_to(p, (T, B, Hq, 3)).copy()
    # clusters: 8 clusters x 8 positions per (b, kv head)
    Hkv = cfg.Hkv
    clusters = np.stack([rng.choice(np.arange(lo, hi), size=64, replace=False)
                         for _ in range(B * Hkv)]).reshape(B, Hkv, 8, 8)
    subsets = np.stack([rng.choice(8, size=3, replace=False)
                        for _ in range(B * Hq)]).reshape(B, Hq, 3)
    crng = _np_rng(cfg, layer, "clusters")
    if cfg.cluster_switch == "bernoulli":
        switch = (_np_rng(cfg, layer, "switch").random(T) < (1.0 / 16.0)).astype(np.int8)
    else:
        switch = boundary
    active = np.zeros((T, B, Hkv), np.int64)
    cur = crng.integers(0, 8, size=(B, Hkv))
    for t in range(T):
        if t > 0 and switch[t - 1]:
            step = crng.integers(1, 8, size=(B, Hkv))
            cur = (cur + step) % 8
        active[t] = cur
    out = np.empty((T, B, Hq, 3), np.int64)
    for h in range(Hq):
        g = h // G
        cl = clusters[:, g][np.arange(B)[None, :], active[:, :, g]]   # [T, B, 8]
        out[:, :, h, :] = np.take_along_axis(
            cl, np.broadcast_to(subsets[None, :, h, :], (T, B, 3)), axis=2)
    return out


def make_layer(cfg: SFIConfig, layer: int = 0, device="cpu",
               boundary: Optional[np.ndarray] = None) -> LayerInputs:
    """Draw one attention layer's cache, queries and new tokens."""
    device = torch.device(device)
    B, Hq, Hkv, D, T = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.steps
    npb, cap, ctx = cfg.pages_per_seq, cfg.capacity, cfg.context
    if boundary is None:
        boundary = boundary_stream(cfg)
    pt_np = page_table(cfg, layer)
    pt = torch.from_numpy(pt_np).to(device)
    k_pool = torch.zeros(cfg.num_pages, Hkv, PAGE, D, dtype=torch.bfloat16, device=device)
    v_pool = torch.zeros_like(k_pool)
    planted = _planted_positions(cfg, layer, boundary)
    q = torch.empty(T, B, Hq, D, dtype=torch.bfloat16, device=device)
    gq = _torch_gen(cfg, layer, "qnoise", device)
    noise = torch.randn(T, B, Hq, D, generator=gq, device=device) * Q_NOISE
    G = cfg.G
    planted_t = torch.from_numpy(planted).to(device)
    for b in range(B):
        kl = _key_rows(cfg, layer, "k", (Hkv, ctx, D), device, gen_extra=b)
        gv = _torch_gen(cfg, layer, "v", device, b)
        vl = torch.randn(Hkv, ctx, D, generator=gv, device=device)
        kb = torch.zeros(Hkv, cap, D, dtype=torch.bfloat16, device=device)
        vb = torch.zeros_like(kb)
        kb[:, :ctx] = kl.to(torch.bfloat16)
        vb[:, :ctx] = vl.to(torch.bfloat16)
        del kl, vl
        pages = pt[b].long()
        k_pool[pages] = kb.view(Hkv, npb, PAGE, D).permute(1, 0, 2, 3)
        v_pool[pages] = vb.view(Hkv, npb, PAGE, D).permute(1, 0, 2, 3)
        # queries: beta * sum of unit planted keys (stored bf16 keys) + noise
        kf = kb.float()
        norms = kf.norm(dim=-1, keepdim=True).clamp_min(1e-30)
        kunit = kf / norms                                   # [Hkv, cap, D]
        for h in range(Hq):
            idx = planted_t[:, b, h, :]                      # [T, 3]
            rows = kunit[h // G][idx]                        # [T, 3, D]
            q[:, b, h, :] = (BETA * rows.sum(dim=1) + noise[:, b, h, :]).to(torch.bfloat16)
        del kb, vb, kf, kunit
    k_new = _key_rows(cfg, layer, "knew", (T, B, Hkv, D), device).to(torch.bfloat16)
    gvn = _torch_gen(cfg, layer, "vnew", device)
    v_new = torch.randn(T, B, Hkv, D, generator=gvn, device=device).to(torch.bfloat16)
    return LayerInputs(k_pool, v_pool, pt, q, k_new, v_new, planted)

