"""CPU oracle for the Slow-Fast Inference (SFI) decode hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports, links or calls
this module; only the tests, the package's smoke check and the benchmark's
CPU-baseline leg may use it.  It shares no code with the CUDA path.

Plain, slow, numpy float64.  bf16 inputs are converted to float64 exactly.
Every function cites the passage it follows.  The pages are five summaries of
"Slow-Fast Inference: Training-Free Inference Acceleration via
Within-Sentence Support Stability" (arXiv 2603.12038), cited as

  [ES] gist.science/es/paper/2603.12038, "Resumen técnico"
  [FR] gist.science/fr/paper/2603.12038, "Résumé technique"
  [NL] gist.science/nl/paper/2603.12038, technical summary
  [KO] insight.artgrammer.co.kr/papers/9328, abstract
  [ZH] gist.science/zh/paper/2603.12038, technical summary

Where the pages leave a step open, the plainest reading is taken and marked
READING below.  Soft-NMS dominance is decided as real arithmetic decides it,
from the terms of the fused score (see _score_diff), never from the last bit
of a rounded sum; the cross-head owner treats log-scores within 1e-3 of each
other as tied (see owner); the top-K order is that of the float64 scores.

Pins: every function here is checked in tests/test_oracle_*.py against
closed forms, library routines, brute force or hand-worked fixtures.  Parity
of the prior r, soft-NMS and cross-head exclusivity is pinned only by
hand-worked fixtures and special cases (the pages print no formula for
them): "parity unpinned" by the pages for those three.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

PAGE = 16
LOG_EPS = 1e-30


# ----------------------------------------------------------------------------
# Paged KV cache
# ----------------------------------------------------------------------------

def gather_cache(pool: np.ndarray, page_table: np.ndarray, b: int, h: int,
                 L: int) -> np.ndarray:
    """Logical rows [0, L) of KV head h of sequence b, read through the page
    table: row j lives in page page_table[b, j // 16] at slot j % 16.

    The paged cache is the structure the recent window is read from and the
    packed buffer is gathered from ([NL] "Systeemontwerp en
    Kernel-optimalisatie", Memory-Coalesced Kernel; [ZH] "2.3 系统级优化").
    """
    rows = np.empty((L, pool.shape[-1]), dtype=np.float64)
    for j in range(L):
        rows[j] = pool[page_table[b, j // PAGE], h, j % PAGE]
    return rows


def key_norms(K: np.ndarray) -> np.ndarray:
    """n_j = ||k_j||_2 of each stored key row: the cache statistic the prior
    is built from ([ZH] "2.2", 先验分布, Key 范数因子; [ES] "El Selector",
    Prioridad Estructural)."""
    K = np.asarray(K, dtype=np.float64)
    return np.sqrt(np.sum(K * K, axis=-1))


# ----------------------------------------------------------------------------
# Attention
# ----------------------------------------------------------------------------

def dense_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray):
    """Slow-step dense attention over the whole accessible history.

    ([ES] "2. Metodología", Pasos Lentos; [FR] "A. Le Paradigme
    Lente-Rapide", Étapes Lentes; [ZH] "2.1", 慢步骤.)
    Textbook softmax attention with scale 1/sqrt(D):
      z_{h,j} = q_h . k_j / sqrt(D)
      lse_h   = log sum_j exp(z_{h,j})
      f_{h,j} = exp(z_{h,j} - lse_h)        (the attention distribution f)
      o_h     = sum_j f_{h,j} v_j
    q: [G, D] query heads sharing this KV head; K, V: [L, D].
    Returns (o [G, D], f [G, L], lse [G], z [G, L]).
    """
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    D = q.shape[-1]
    z = (q @ K.T) / math.sqrt(D)
    m = z.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(z - m).sum(axis=1))
    f = np.exp(z - lse[:, None])
    o = f @ V
    return o, f, lse, z


def sparse_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray,
                     sets: Sequence[np.ndarray]) -> np.ndarray:
    """Fast-step attention restricted, per query head h, to the position set
    S_h = sink U selected_h U recent  ([ES] "2. Metodología", Pasos Rápidos;
    [NL] "Methodologie", Fast Steps; [ZH] "2.1", 快步骤):
      o_h = sum_{j in S_h} softmax_{S_h}(z_h)_j v_j.
    sets[h]: positions (any order, no duplicates) into K/V rows.
    """
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    D = q.shape[-1]
    out = np.empty((q.shape[0], V.shape[1]), np.float64)
    for h in range(q.shape[0]):
        S = np.asarray(sets[h], np.int64)
        z = (K[S] @ q[h]) / math.sqrt(D)
        p = np.exp(z - z.max())
        out[h] = (p / p.sum()) @ V[S]
    return out


def sparse_sets(L: int, n_sink: int, n_recent: int,
                selected: Sequence[np.ndarray]) -> List[np.ndarray]:
    """S_h = [0, n_sink) U selected_h U [L - n_recent, L).

    READING: the new token is appended before attention, so it lies inside
    the recent window; selected positions come from the candidate range of a
    slow step at L_slow <= L, hence never overlap the recent window.
    """
    sink = np.arange(0, min(n_sink, L))
    recent = np.arange(max(L - n_recent, 0), L)
    return [np.unique(np.concatenate([sink, np.asarray(s, np.int64), recent]))
            for s in selected]


# ----------------------------------------------------------------------------
# Selector ([ES] "El Selector"; [FR] "B. Le Sélecteur"; [NL] "De Selector";
# [ZH] "2.2 训练无感的 Selector")
# ----------------------------------------------------------------------------

def candidate_range(L: int, n_sink: int, n_recent: int) -> Tuple[int, int]:
    """C = [n_sink, L - n_recent): the long-range positions the Selector may
    choose.  READING: sink and recent tokens are always attended at fast
    steps ([ES] Pasos Rápidos), so the selection excludes them."""
    return n_sink, L - n_recent


def budget(L: int, n_sink: int, n_recent: int, k_fixed: int,
           budget_frac: float) -> int:
    """Per-query-head selection size K.

    READING: k_fixed when given, else floor(budget_frac * L) recomputed at
    every slow step (the pages quote 15-20 % retention: [ES] "4. Resultados",
    [ZH] "4. 实验结果"), clamped to |C|."""
    lo, hi = candidate_range(L, n_sink, n_recent)
    k = k_fixed if k_fixed > 0 else int(math.floor(budget_frac * L))
    return min(k, hi - lo)


def evidence(f: np.ndarray, lo: int, hi: int) -> np.ndarray:
    """Evidence f~: the slow step's attention distribution restricted to the
    candidates and renormalised, f~_{h,j} = f_{h,j} / sum_{i in C} f_{h,i}
    ([ZH] "2.2", 证据分布 (f); [ES] "El Selector", Evidencia).
    READING: the "slow-step window" is the single slow-step query."""
    fc = np.asarray(f, np.float64)[:, lo:hi]
    return fc / fc.sum(axis=1, keepdims=True)


def evidence_window(fs: Sequence[np.ndarray], lo: int, hi: int) -> np.ndarray:
    """Evidence over a window of queries: the mean of the restricted,
    renormalised distributions of the last W queries, f~_{h,j} =
    (1/W) sum_i f_{i,h,j} / sum_{c in C} f_{i,h,c}  ([ES] "2. Metodología", the
    slow step's window; [ZH] "2.2", 证据分布).
    READING: equal weights; fs[i] is the attention distribution of the query
    i steps back over the current cache.  Its positions in C all precede that
    query's own context end (W <= n_recent), so the restriction to C is the
    same either way.  W = 1 is `evidence`."""
    return np.mean([evidence(f, lo, hi) for f in fs], axis=0)


def prior(norms: np.ndarray, L: int, lo: int, hi: int) -> np.ndarray:
    """Prior r from cache statistics, shared by the query heads of one KV head
    ([ZH] "2.2", 先验分布: a key-norm factor that suppresses spuriously high
    logits of large-norm keys and a position factor that keeps attention
    from over-concentrating on recent positions; [ES] "El Selector",
    Prioridad Estructural).

    READING (the pages name the factors but give no formula):
      nbar   = mean_{i in C} n_i
      kappa_j = min(1, nbar / n_j)          (kappa_j = 1 when n_j = 0)
      pi_j    = log(1 + (L - j))
      r_j     = kappa_j pi_j / sum_{i in C} kappa_i pi_i
    """
    n = np.asarray(norms, np.float64)[lo:hi]
    nbar = n.mean()
    kappa = np.ones_like(n)
    pos = n > 0
    kappa[pos] = np.minimum(1.0, nbar / n[pos])
    j = np.arange(lo, hi, dtype=np.float64)
    pi = np.log1p(L - j)
    w = kappa * pi
    return w / w.sum()


def fuse(f_tilde: np.ndarray, r: np.ndarray, lam: float,
         lam_clip: float) -> np.ndarray:
    """Reverse-KL fusion, closed form s_lambda = (1 - lambda) f + lambda r
    ([NL] "De Selector", Gesloten Oplossing; [ZH] "2.2", 融合目标).

    The printed formula is the arithmetic mixture, which minimises
    (1-lambda) KL(f || s) + lambda KL(r || s) over the simplex.
    READING: lambda_clip ([ZH] "4. 实验结果", ablations) clamps lambda:
    lambda_eff = min(max(lambda, 0), lambda_clip)."""
    lam_eff = min(max(lam, 0.0), lam_clip)
    return (1.0 - lam_eff) * np.asarray(f_tilde, np.float64) + lam_eff * np.asarray(r, np.float64)[None, :]


def log_score(s: np.ndarray) -> np.ndarray:
    """l = ln(s + 1e-30): the Selector refines log-scores before Top-K
    ([ZH] "2.2", Log-Score 细化).  READING: natural log, eps = 1e-30."""
    return np.log(np.asarray(s, np.float64) + LOG_EPS)


def _score_diff(ell: np.ndarray, mixture, a: slice, b: slice) -> np.ndarray:
    """l[:, a] - l[:, b] for two equally long column ranges, with the sign of
    the exact difference.

    Without a mixture the log-scores are compared as they are.  With the
    mixture (f~, r, lambda) that l = ln(s + eps) was built from, ln is
    monotone and eps is common, so the sign of l_i - l_j is the sign of
    s_i - s_j = lambda (r_i - r_j) + (1 - lambda)(f~_i - f~_j), formed term
    by term.  Rounding s itself would let its last bit decide comparisons
    that real arithmetic decides by an evidence term far below it (where the
    prior dominates, the group's heads share s to every digit of float64)."""
    if mixture is None:
        return ell[:, a] - ell[:, b]
    ft, r, lam = mixture
    return lam * (r[None, a] - r[None, b]) + (1.0 - lam) * (ft[:, a] - ft[:, b])


def soft_nms_distance(ell: np.ndarray, window: int, mixture=None) -> np.ndarray:
    """Distance to the nearest dominating neighbour within w = window // 2
    (0: none), for every (head, candidate) of ell [G, nC]:
      i dominates j  <=>  l_i > l_j  or  (l_i == l_j and i < j),
    with l_i vs l_j decided exactly (see _score_diff)."""
    ell = np.asarray(ell, np.float64)
    w = window // 2
    G, n = ell.shape
    dist = np.zeros((G, n), np.int64)
    for d in range(w, 0, -1):      # descending: the nearest hit is written last
        hit = np.zeros((G, n), bool)
        # left neighbour i = j - d dominates j when l_i >= l_j
        hit[:, d:] |= _score_diff(ell, mixture, slice(0, n - d), slice(d, n)) >= 0
        # right neighbour i = j + d dominates j when l_i > l_j
        hit[:, :n - d] |= _score_diff(ell, mixture, slice(d, n), slice(0, n - d)) > 0
        dist = np.where(hit, d, dist)
    return dist


def soft_nms_weight(dist: np.ndarray, window: int) -> np.ndarray:
    """Penalty weight of a nearest dominator at distance d: 1 - (d - 1) / w,
    and 0 where there is none (d = 0)."""
    w = window // 2
    d = np.asarray(dist, np.float64)
    return np.where(d > 0, 1.0 - (d - 1.0) / w, 0.0)


def soft_nms(ell: np.ndarray, alpha_soft: float, window: int, mixture=None) -> np.ndarray:
    """Soft non-maximum suppression within each head: penalise tokens whose
    neighbours score higher ([FR] "B. Le Sélecteur", Suppression Non-Maximum
    Douce; [ZH] "2.2", Soft-NMS).

    READING (one pass, data parallel, w = window // 2):
      N(j) = {i in C : 1 <= |i - j| <= w}
      i dominates j  <=>  l_i > l_j  or  (l_i == l_j and i < j)
      l'_j = l_j - alpha_soft * max_{i in N(j), i dominates j} (1 - (|i-j| - 1) / w)
    with max over the empty set = 0.  The weight falls with distance, so the
    max is the weight of the nearest dominator.  ell: [G, nC] over the
    candidate positions in order; mixture: see _score_diff.
    """
    ell = np.asarray(ell, np.float64)
    return ell - alpha_soft * soft_nms_weight(soft_nms_distance(ell, window, mixture), window)


OWNER_TIE = 1e-3


def owner(ell1: np.ndarray, tie: float = OWNER_TIE) -> np.ndarray:
    """owner(j): the lowest-indexed head whose l'_{h,j} is within `tie` of the
    group's largest, M_j = max_h l'_{h,j}:
      owner(j) = min { h : l'_{h,j} >= M_j - tie }.

    READING (the pages name the argmax but no tie rule): heads whose refined
    log-scores agree within 1e-3 (their fused scores within 0.1 %) are tied
    and the lowest one owns the position; the tolerance is thirty times
    below the smallest step of the soft-NMS penalty (alpha_soft / w).
    Where the prior dominates, the group's heads share s to some twenty
    digits; a plain argmax would hand each such position to whichever head
    has the most evidence there, a difference far below anything the scores
    represent, and the ownership of most candidates would then follow it."""
    ell1 = np.asarray(ell1, np.float64)
    M = ell1.max(axis=0)
    return np.argmax(ell1 >= (M - tie)[None, :], axis=0)


def cross_head(ell1: np.ndarray, alpha_cross: float) -> np.ndarray:
    """Cross-head exclusivity within one KV group: discourage the group's
    query heads from choosing the same positions ([FR] "B. Le Sélecteur",
    Exclusivité inter-têtes; [ZH] "2.2", 跨头互斥).

    READING: owner(j) as `owner` gives it (the argmax of l', near-ties to the
    lowest head); l''_{h,j} = l'_{h,j} - alpha_cross * [h != owner(j)].
    """
    ell1 = np.asarray(ell1, np.float64)
    own = owner(ell1)
    G = ell1.shape[0]
    not_owner = np.arange(G)[:, None] != own[None, :]
    return ell1 - alpha_cross * not_owner


def topk(scores: np.ndarray, K: int) -> np.ndarray:
    """Top-K discretisation ([FR] "B. Le Sélecteur", Top-K; [ZH] "2.2",
    Top-K 选择): the K largest scores of each row.

    READING: ties go to the lower index; the result is sorted ascending.
    scores: [G, n] -> [G, K]."""
    s = np.asarray(scores, np.float64)
    G, n = s.shape
    out = np.empty((G, K), np.int64)
    idx = np.arange(n)
    for h in range(G):
        order = np.lexsort((idx, -s[h]))
        out[h] = np.sort(order[:K])
    return out


def selector_detail(ft: np.ndarray, r: np.ndarray, lam: float, lam_clip: float,
                    alpha_soft: float, alpha_cross: float, window: int) -> dict:
    """Every step of the Selector for one KV group from the evidence f~
    [G, nC] and the prior r [nC], in the order the pages give: fusion, log,
    soft-NMS, cross-head.  Returns the intermediates: s, ell (l), dist (the
    soft-NMS nearest-dominator distances), ell1 (l'), owner, ell2 (l'')."""
    lam_eff = min(max(lam, 0.0), lam_clip)
    ft = np.asarray(ft, np.float64)
    r = np.asarray(r, np.float64)
    s = fuse(ft, r, lam, lam_clip)
    ell = log_score(s)
    mixture = (ft, r, lam_eff)
    dist = soft_nms_distance(ell, window, mixture)
    ell1 = ell - alpha_soft * soft_nms_weight(dist, window)
    own = owner(ell1)
    ell2 = ell1 - alpha_cross * (np.arange(ft.shape[0])[:, None] != own[None, :])
    return {"lam_eff": lam_eff, "s": s, "ell": ell, "dist": dist, "ell1": ell1, "owner": own, "ell2": ell2}


def selector_scores(f: np.ndarray, norms: np.ndarray, L: int, n_sink: int,
                    n_recent: int, lam: float, lam_clip: float,
                    alpha_soft: float, alpha_cross: float,
                    window: int) -> np.ndarray:
    """All refined log-scores l'' [G, |C|] of one KV group, in the order the
    pages give: evidence, prior, fusion, log, soft-NMS, cross-head."""
    lo, hi = candidate_range(L, n_sink, n_recent)
    ft = evidence(f, lo, hi)
    r = prior(norms, L, lo, hi)
    return selector_detail(ft, r, lam, lam_clip, alpha_soft, alpha_cross, window)["ell2"]


def select(f: np.ndarray, norms: np.ndarray, L: int, n_sink: int, n_recent: int,
           k_fixed: int, budget_frac: float, lam: float, lam_clip: float,
           alpha_soft: float, alpha_cross: float, window: int) -> np.ndarray:
    """Selector for one (sequence, KV group): absolute positions chosen per
    query head, [G, K] ascending."""
    lo, _ = candidate_range(L, n_sink, n_recent)
    K = budget(L, n_sink, n_recent, k_fixed, budget_frac)
    ell2 = selector_scores(f, norms, L, n_sink, n_recent, lam, lam_clip,
                           alpha_soft, alpha_cross, window)
    return topk(ell2, K) + lo


# ----------------------------------------------------------------------------
# Packed (coalesced) buffer
# ----------------------------------------------------------------------------

def compact(selected: np.ndarray, n_sink: int):
    """Rows of the contiguous packed buffer of one (sequence, KV head): the
    sink tokens, then the union of the group's selected positions, ascending
    ([ES] "3. Optimización del Sistema", item 2; [NL] "Systeemontwerp",
    Memory-Coalesced Kernel; [ZH] "2.3", 显存合并的内核).

    READING: one packed buffer per KV head (the union of its query heads'
    sets); headmask bit h marks rows chosen by query head h; sink rows carry
    every head's bit.  Returns (pos int64 [U], headmask uint32 [U]).
    """
    G = selected.shape[0]
    allbits = (1 << G) - 1
    masks = {}
    for h in range(G):
        for p in np.asarray(selected[h]).tolist():
            masks[p] = masks.get(p, 0) | (1 << h)
    pos = list(range(n_sink)) + sorted(masks)
    hm = [allbits] * n_sink + [masks[p] for p in sorted(masks)]
    return np.asarray(pos, np.int64), np.asarray(hm, np.uint32)


def compact_incremental(prev_pos, n_prev: int, selected: np.ndarray, n_sink: int):
    """Packed rows of one (sequence, KV head) refreshed from the previous
    buffer's rows prev_pos[:n_prev] (n_prev = 0: none) rather than rebuilt.

    READING (the pages name the coalesced buffer and the stability of the
    support across consecutive slow steps — "Slow-Fast Inference",
    within-sentence support stability — but no refresh rule): with U the new
    union (as `compact` forms it) and n_new = n_sink + |U|,
      * a previous row whose position is in U keeps its slot;
      * holes: slots in [n_sink, n_new) holding no kept row, ascending;
      * movers: positions of U not among the previous rows, ascending, then
        the positions of kept rows at slots >= n_new, by slot;
      * the i-th mover goes to the i-th hole.
    Head masks are those of U.  Returns (pos int64 [n_new], headmask uint32
    [n_new], moved: the number of rows written from the cache).
    """
    pos_full, hm_full = compact(selected, n_sink)
    mask_of = dict(zip(pos_full.tolist(), hm_full.tolist()))
    union = [p for p in pos_full.tolist()[n_sink:]]
    n_new = n_sink + len(union)
    if n_prev == 0:
        return pos_full, hm_full, n_new
    prev = [int(p) for p in prev_pos[:n_prev]]
    in_union = set(union)
    layout = {}
    for s_ in range(n_sink):
        layout[s_] = s_
    kept_slots = [s_ for s_ in range(n_sink, n_prev) if prev[s_] in in_union]
    for s_ in kept_slots:
        if s_ < n_new:
            layout[s_] = prev[s_]
    prev_set = set(prev[n_sink:])
    holes = [s_ for s_ in range(n_sink, n_new) if s_ not in layout]
    movers = [p for p in union if p not in prev_set] + [prev[s_] for s_ in kept_slots if s_ >= n_new]
    assert len(movers) == len(holes)
    for s_, p in zip(holes, movers):
        layout[s_] = p
    pos = np.asarray([layout[s_] for s_ in range(n_new)], np.int64)
    hm = np.asarray([mask_of[p] for p in pos.tolist()], np.uint32)
    return pos, hm, len(movers)


# ----------------------------------------------------------------------------
# Trigger
# ----------------------------------------------------------------------------

def trigger(boundary: np.ndarray, refresh_budget: int) -> np.ndarray:
    """Slow-step schedule.  A slow step comes near a semantic boundary (the
    step after a boundary token) or when the reuse budget runs out ([ES]
    "2. Metodología", Pasos Lentos; [ZH] "2.1", 触发机制):
      slow(t) = t == 0  or  boundary[t-1]  or  t - last_slow >= M.
    READING: "budget M" = at most M-1 consecutive fast steps."""
    T = len(boundary)
    slow = np.zeros(T, bool)
    last = 0
    for t in range(T):
        if t == 0 or boundary[t - 1] or t - last >= refresh_budget:
            slow[t] = True
            last = t
    return slow


def trigger_rows(boundary: np.ndarray, refresh_budget: int) -> np.ndarray:
    """Slow-step schedules of a batch whose sequences trigger independently:
    `trigger` applied to every sequence's own boundary stream (boundary
    [B, T] -> bool [B, T]).
    READING: the boundary that makes a step slow is a token of one sequence
    ([ES] "2. Metodología", Pasos Lentos), so in a batch each sequence has its
    own schedule and its own refresh budget."""
    return np.stack([trigger(np.asarray(row), refresh_budget) for row in boundary])


# ----------------------------------------------------------------------------
# A whole decode run (one layer), for end-to-end checks on small workloads
# ----------------------------------------------------------------------------

def decode_run(k_pool, v_pool, page_table, q, k_new, v_new, boundary, context,
               n_sink, n_recent, k_fixed, budget_frac, lam, lam_clip,
               alpha_soft, alpha_cross, window, refresh_budget,
               steps=None):
    """Runs SFI decode for one attention layer ([ES] "2. Metodología").

    Step t appends token context+t, so L_t = context + t + 1.  Slow steps
    return dense attention and refresh the selection from their f; fast
    steps attend to sink U selected_h U recent.  Returns (outputs [T,B,Hq,D],
    slow [T], selections dict t -> [B, Hkv, G, K] absolute positions).
    """
    k_pool = np.array(k_pool, np.float64)
    v_pool = np.array(v_pool, np.float64)
    T = len(boundary) if steps is None else steps
    B, Hq, D = q.shape[1], q.shape[2], q.shape[3]
    Hkv = k_pool.shape[1]
    G = Hq // Hkv
    slow = trigger(boundary, refresh_budget)[:T]
    outs = np.zeros((T, B, Hq, D))
    sel = None
    sels = {}
    for t in range(T):
        L = context + t + 1
        pos = L - 1
        for b in range(B):
            for g in range(Hkv):
                k_pool[page_table[b, pos // PAGE], g, pos % PAGE] = k_new[t, b, g]
                v_pool[page_table[b, pos // PAGE], g, pos % PAGE] = v_new[t, b, g]
        if slow[t]:
            sel = np.zeros((B, Hkv, G, budget(L, n_sink, n_recent, k_fixed, budget_frac)), np.int64)
        for b in range(B):
            for g in range(Hkv):
                K = gather_cache(k_pool, page_table, b, g, L)
                V = gather_cache(v_pool, page_table, b, g, L)
                qg = np.asarray(q[t, b, g * G:(g + 1) * G], np.float64)
                if slow[t]:
                    o, f, _, _ = dense_attention(qg, K, V)
                    sel[b, g] = select(f, key_norms(K), L, n_sink, n_recent, k_fixed,
                                       budget_frac, lam, lam_clip, alpha_soft,
                                       alpha_cross, window)
                else:
                    o = sparse_attention(qg, K, V, sparse_sets(L, n_sink, n_recent, sel[b, g]))
                outs[t, b, g * G:(g + 1) * G] = o
        if slow[t]:
            sels[t] = sel.copy()
    return outs, slow, sels
