"""The Selector's tolerance model (helpers.selection_bounds / check_selection)
on the CPU: a float32 emulation of the CUDA Selector's arithmetic passes it on
seeded workload groups, with few undecided candidates, and planted mistakes
fail it: a swapped pick, a score moved by a cross-head penalty, and owners
taken by a plain argmax of the rounded scores (no tie tolerance)."""
import math

import numpy as np
import pytest
import torch

from oracle import sfi_oracle as O
from slow_sparse_kv_sfi_b200 import workload as W

import helpers as H


def _emulate(z32, lse32, norms32, L, cfg, K, rounded_owner=False):
    """The CUDA Selector's arithmetic in numpy: x = z - lse_C in fp32, kappa pi
    in fp64 from fp32 norms rounded to fp32, lambda r = that times lambda / Z
    in fp32, s by one fp32 FMA,
    dominance on s, owner with the tie tolerance on l' (or, rounded_owner, a
    plain argmax of the fp32 l'), keys fp32."""
    lo, hi = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
    lam = min(max(cfg.lam, 0.0), cfg.lam_clip)
    w = cfg.nms_window // 2
    n = norms32[lo:hi].astype(np.float64)
    nbar = n.mean()
    kap = np.where(n > 0, np.minimum(1.0, nbar / np.where(n > 0, n, 1.0)), 1.0)
    kp = kap * np.log(1.0 + L - np.arange(lo, hi, dtype=np.float64))
    lam_z = np.float32(lam / kp.sum())          # lambda / Z, rounded once
    x = (z32[:, lo:hi] - lse32[:, None]).astype(np.float32)
    ft = np.exp(x.astype(np.float64)).astype(np.float32)
    lr32 = (kp.astype(np.float32) * lam_z).astype(np.float32)   # fp32 kappa pi times lambda / Z
    s32 = (np.float64(np.float32(1.0 - lam)) * ft.astype(np.float64) + lr32.astype(np.float64)[None]).astype(np.float32)
    key = x if lam <= 0 else s32
    G, nC = x.shape
    dist = np.zeros((G, nC), np.int64)
    for d in range(w, 0, -1):
        hit = np.zeros((G, nC), bool)
        hit[:, d:] |= key[:, :-d] >= key[:, d:]
        hit[:, :-d] |= key[:, d:] > key[:, :-d]
        dist = np.where(hit, d, dist)
    pen = np.where(dist > 0, 1.0 - (dist - 1.0) / w, 0.0).astype(np.float32)
    sv = np.exp(x.astype(np.float64)).astype(np.float32) if lam <= 0 else s32
    l1 = (np.log((sv + np.float32(1e-30)).astype(np.float64)).astype(np.float32)
          - np.float32(cfg.alpha_soft) * pen).astype(np.float32)
    cols = np.arange(nC)
    if rounded_owner:      # a plain argmax on the fp32 scores
        best = np.argmax(l1, axis=0)
    else:                  # the lowest head within the tie tolerance of the largest
        M = l1.max(axis=0)
        thr = (M - np.float32(O.OWNER_TIE)).astype(np.float32)
        best = np.argmax(l1 >= thr[None, :], axis=0)
    sc = (l1 - np.float32(cfg.alpha_cross) * (np.arange(G)[:, None] != best[None]).astype(np.float32)).astype(np.float32)
    sel = np.stack([np.sort(np.lexsort((cols, -sc[h]))[:K]) for h in range(G)]) + lo
    return sel, sc


def _group(cfg, g=0):
    """Oracle float64 and fp32-rounded inputs of one group at the first decode step."""
    li = W.make_layer(cfg, 0, "cpu")
    L = cfg.context + 1
    G = cfg.G
    pages = li.page_table[0, : (L + 15) // 16].long()
    Kb = li.k_pool[pages, g].reshape(-1, cfg.D)[:L].clone()
    Kb[L - 1] = li.k_new[0, 0, g]
    q64 = li.q[0, 0, g * G:(g + 1) * G].double().numpy()
    K64 = Kb.double().numpy()
    _, f, _, z = O.dense_attention(q64, K64, K64)
    lo, hi = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
    z32 = z.astype(np.float32)
    zz = z32.astype(np.float64)[:, lo:hi]
    m = zz.max(axis=1)
    lse32 = (m + np.log(np.exp(zz - m[:, None]).sum(axis=1))).astype(np.float32)
    norms32 = O.key_norms(K64).astype(np.float32)
    K = O.budget(L, cfg.n_sink, cfg.n_recent, cfg.k_fixed, cfg.budget_frac)
    return L, z32, lse32, norms32, K


def _bounds(cfg, L, z32, lse32, norms32):
    """Bounds for a Selector fed the fp32 logits and norms (the oracle takes
    the same values, so only the kernel's own roundings remain)."""
    lo, hi = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
    zz = z32.astype(np.float64)
    m = zz[:, lo:hi].max(axis=1, keepdims=True)
    lse = m + np.log(np.exp(zz[:, lo:hi] - m).sum(axis=1, keepdims=True))
    x = zz[:, lo:hi] - lse
    ft = np.exp(x)
    r = O.prior(norms32.astype(np.float64), L, lo, hi)
    lam_eff = min(max(cfg.lam, 0.0), cfg.lam_clip)
    eps_x = 2.0 ** -23 * (np.abs(x) + np.abs(lse)) + 2.0 ** -21
    return H.selection_bounds(ft, r, lam_eff, cfg.alpha_soft, cfg.alpha_cross, cfg.nms_window, eps_x,
                              1e-12, x=x), lo


CASES = [
    W.CONFIG_BY_NAME["qwen3-0.6b-8k"].replace(B=1, steps=2),
    W.CONFIG_BY_NAME["qwen3-4b-32k"].replace(B=1, steps=2, context=12000),
    W.CONFIG_BY_NAME["qwen3-4b-32k"].replace(B=1, steps=2, context=12000, lam=1.0, lam_clip=1.0),
    W.CONFIG_BY_NAME["qwen3-4b-32k"].replace(B=1, steps=2, context=12000, lam=0.0),
    W.CONFIG_BY_NAME["qwen3-235b-a22b-64k"].replace(B=1, steps=2, context=6000, Hq=16, Hkv=1),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: f"{c.name}-{c.context}-lam{c.lam}-G{c.G}")
def test_emulated_kernel_arithmetic_passes(cfg):
    L, z32, lse32, norms32, K = _group(cfg)
    b, lo = _bounds(cfg, L, z32, lse32, norms32)
    sel, sc = _emulate(z32, lse32, norms32, L, cfg, K)
    H.check_selection(sel, b, K, lo, cfg.name, gpu_scores=sc)


def test_planted_mistakes_fail():
    cfg = CASES[1]
    L, z32, lse32, norms32, K = _group(cfg)
    b, lo = _bounds(cfg, L, z32, lse32, norms32)
    sel, sc = _emulate(z32, lse32, norms32, L, cfg, K)
    # a pick swapped for the worst candidate of the row
    bad = sel.copy()
    worst = int(np.argmin(b["hi"][0])) + lo
    assert worst not in bad[0]
    bad[0, 0] = worst
    with pytest.raises(AssertionError):
        H.check_selection(bad, b, K, lo, "swapped pick")
    # a score moved by the cross-head penalty
    sc2 = sc.copy()
    sc2[1, 10] += cfg.alpha_cross
    with pytest.raises(AssertionError):
        H.check_selection(sel, b, K, lo, "moved score", gpu_scores=sc2)
    # owners by a plain argmax of the rounded scores
    sel3, sc3 = _emulate(z32, lse32, norms32, L, cfg, K, rounded_owner=True)
    with pytest.raises(AssertionError):
        H.check_selection(sel3, b, K, lo, "rounded owner", gpu_scores=sc3)


def test_exact_oracle_passes_with_no_undecided_candidates():
    rng = np.random.default_rng(7)
    G, n, K = 3, 500, 60
    ft = rng.dirichlet(np.ones(n), size=G)
    r = rng.dirichlet(np.ones(n))
    b = H.selection_bounds(ft, r, 0.3, 0.5, 0.5, 16, 0.0, 0.0)
    ora = O.topk(b["ell2"], K)
    H.check_selection(ora, b, K, 0, "oracle itself")
    assert H.SELECTION_RECORD[-1][4] <= 1
