"""Test-side glue: runs the oracle on the same inputs the CUDA path received
and compares the two with the tolerances of the hot path:

* attention outputs: per (b, h) row, max_d |o - o_ref| / max(max_d |o_ref|, 1e-6) <= 2e-3
* probabilities f and lse: absolute 1e-4; key norms: relative 1e-6
* page-table indexing, gathers and compaction: bit-exact
* selections: identical except at elements whose deciding comparisons are
  near-ties (relative gap below NEAR_TIE) in the oracle's float64 values
  (see assert_selection_close).
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import sfi_oracle as O

ATTN_RTOL = 2e-3
PROB_ATOL = 1e-4
NORM_RTOL = 1e-6
NEAR_TIE = 1e-5


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def group_kv(k_pool: np.ndarray, v_pool: np.ndarray, pt: np.ndarray, b: int, g: int, L: int):
    """Logical K, V rows [0, L) of (b, g) read through the page table."""
    pages = pt[b, : (L + 15) // 16]
    K = k_pool[pages, g].reshape(-1, k_pool.shape[-1])[:L]
    V = v_pool[pages, g].reshape(-1, v_pool.shape[-1])[:L]
    return np.asarray(K, np.float64), np.asarray(V, np.float64)


def group_kv_device(layer, b: int, g: int, L: int):
    """Copies only the pages of (b, g) from device pools to host float64."""
    pages = layer.page_table[b, : (L + 15) // 16].long()
    K = layer.k_pool[pages, g].reshape(-1, layer.k_pool.shape[-1])[:L]
    V = layer.v_pool[pages, g].reshape(-1, layer.v_pool.shape[-1])[:L]
    return to64(K), to64(V)


def attn_row_err(o: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per-row max relative error, rows on the leading axes."""
    num = np.abs(o - ref).max(axis=-1)
    den = np.maximum(np.abs(ref).max(axis=-1), 1e-6)
    return num / den


def assert_attn_close(o, ref, what=""):
    e = attn_row_err(np.asarray(o, np.float64), np.asarray(ref, np.float64))
    assert e.max() <= ATTN_RTOL, f"{what}: max row rel err {e.max():.3e}"
    return float(e.max())


def ambiguous_positions(ell: np.ndarray, ell1: np.ndarray, window: int, G: int) -> np.ndarray:
    """bool [G, nC]: elements whose soft-NMS or cross-head decision rests on a
    near-tie (relative gap < NEAR_TIE) in the oracle's float64 scores.

    A head's l'' at position j depends on its own soft-NMS penalty and on the
    owner of j, and the owner depends on every head's l' at j.  So a near-tie
    in any head's dominance test at j (which can move that head's l' by up to
    alpha_soft) or between the top two heads makes all heads at j ambiguous."""
    w = window // 2
    Gh, n = ell.shape
    nms = np.zeros((Gh, n), bool)
    scale = np.maximum(np.abs(ell), 1e-30)
    for d in range(1, w + 1):
        diff = np.abs(ell[:, d:] - ell[:, :-d])
        near = diff < NEAR_TIE * np.maximum(scale[:, d:], scale[:, :-d])
        nms[:, d:] |= near
        nms[:, :-d] |= near
    amb = nms.copy()
    if G > 1:
        s = np.sort(ell1, axis=0)
        top, second = s[-1], s[-2]
        near_owner = np.abs(top - second) < NEAR_TIE * np.maximum(np.abs(top), 1e-30)
        amb |= (near_owner | nms.any(axis=0))[None, :]
    return amb


def oracle_selector_detail(f: np.ndarray, norms: np.ndarray, L: int, cfg, f_window=None):
    """Oracle scores of one group plus the intermediate ell, ell' (float64).
    f_window: the window's distributions (the query's own first), if any."""
    lo, hi = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
    ft = O.evidence(f, lo, hi) if f_window is None else O.evidence_window(f_window, lo, hi)
    r = O.prior(norms, L, lo, hi)
    s = O.fuse(ft, r, cfg.lam, cfg.lam_clip)
    ell = O.log_score(s)
    ell1 = O.soft_nms(ell, cfg.alpha_soft, cfg.nms_window)
    ell2 = O.cross_head(ell1, cfg.alpha_cross)
    return ell, ell1, ell2


def assert_selection_close(gpu_sel: np.ndarray, ora_sel: np.ndarray, ell2: np.ndarray,
                           amb: np.ndarray, lo: int, what="", min_overlap=0.85):
    """gpu_sel, ora_sel: [G, K] absolute positions; ell2: oracle scores.

    Elements whose own soft-NMS dominance or cross-head owner rests on a
    near-tie (amb) may fall either way: a flipped dominance or owner moves a
    score by up to alpha.  Every other element must be decided as the oracle
    decides it: the non-ambiguous part of the GPU's set must be exactly the
    best non-ambiguous candidates by the oracle's scores (ties to the lower
    position), as many as the GPU chose, except for scores within NEAR_TIE of
    that cut.  Also at least `min_overlap` of each set must agree.

    Where the prior dominates s (f~ far below lambda * r), the query heads of
    a group have scores equal to within an ulp, so the cross-head owner and
    many soft-NMS dominances are decided by last-bit rounding (FMA
    contraction, exp/log ulps): a float32 emulation that rounds as numpy does
    reproduces the oracle's sets exactly, the kernel's sets can differ in a
    few percent of such near-tied elements."""
    G, K = ora_sel.shape
    worst = 1.0
    for h in range(G):
        g = np.asarray(gpu_sel[h], np.int64) - lo
        assert len(set(g.tolist())) == K, f"{what}: head {h} has duplicate picks"
        assert g.min() >= 0 and g.max() < ell2.shape[1], f"{what}: head {h} picks outside C"
        in_amb = amb[h, g]
        n_amb = int(in_amb.sum())
        got = set(g[~in_amb].tolist())
        cand = np.flatnonzero(~amb[h])
        v32 = ell2[h, cand].astype(np.float32)
        order = cand[np.lexsort((cand, -v32))]
        m = K - n_amb
        want = set(order[:m].tolist())
        diff = got ^ want
        if diff:
            cut = ell2[h, order[m - 1]] if m > 0 else ell2[h, order[0]]
            for c in diff:
                assert abs(ell2[h, c] - cut) <= NEAR_TIE * max(abs(cut), 1e-30), (
                    f"{what}: head {h} position {c + lo} decided differently from the oracle "
                    f"(score {ell2[h, c]!r}, cut {cut!r}, {n_amb} ambiguous picks)")
        ov = len(set(gpu_sel[h].tolist()) & set(ora_sel[h].tolist())) / K
        worst = min(worst, ov)
    assert worst >= min_overlap, f"{what}: overlap {worst:.5f}"
    return worst


def packed_sets(pos: np.ndarray, hm: np.ndarray, n_rows: int, n_sink: int, G: int):
    """Per-head selected positions recorded in a packed buffer (sinks removed)."""
    p = pos[:n_rows]
    m = hm[:n_rows].astype(np.int64) & 0xFFFFFFFF
    out = []
    for h in range(G):
        sel = p[(m >> h) & 1 == 1]
        out.append(np.asarray(sel[sel >= n_sink], np.int64))
    return out
