"""Pins of the oracle's Selector, compaction and trigger.

The fusion is pinned by its closed form and by an independent numerical
minimisation of the KL objective the pages state; top-K by Python's sorted();
soft-NMS, cross-head exclusivity, the prior, compaction and the trigger by
hand-worked fixtures under tests/golden/ and by their special cases; the
Selector's decisions by a brute-force evaluation in 80-digit decimal
arithmetic (with the owner's tie tolerance).
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.optimize

from oracle import sfi_oracle as O
from conftest import GOLDEN


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


def _kl(p, q):
    return float(np.sum(p * (np.log(p) - np.log(q))))


# ---------------------------------------------------------------- fusion
def test_fuse_closed_form_endpoints_and_simplex():
    rng = np.random.default_rng(0)
    f = rng.dirichlet(np.ones(9), size=3)
    r = rng.dirichlet(np.ones(9))
    np.testing.assert_allclose(O.fuse(f, r, 0.0, 1.0), f, rtol=1e-15)
    np.testing.assert_allclose(O.fuse(f, r, 1.0, 1.0), np.broadcast_to(r, f.shape), rtol=1e-15)
    for lam in (0.1, 0.2, 0.5, 0.9):
        s = O.fuse(f, r, lam, 1.0)
        np.testing.assert_allclose(s.sum(axis=1), 1.0, rtol=1e-14)
        assert np.all(s > 0)


def test_fuse_lambda_clip():
    rng = np.random.default_rng(1)
    f = rng.dirichlet(np.ones(6), size=2)
    r = rng.dirichlet(np.ones(6))
    np.testing.assert_allclose(O.fuse(f, r, 0.9, 0.5), O.fuse(f, r, 0.5, 1.0), rtol=1e-15)
    np.testing.assert_allclose(O.fuse(f, r, -0.3, 0.5), f, rtol=1e-15)
    np.testing.assert_allclose(O.fuse(f, r, 0.2, 0.5), O.fuse(f, r, 0.2, 1.0), rtol=1e-15)


@pytest.mark.parametrize("lam", [0.2, 0.5, 0.8])
def test_fuse_minimises_the_stated_kl_objective(lam):
    """(1-lam) KL(f||s) + lam KL(r||s) minimised over the simplex by an
    independent optimiser lands on the oracle's closed form."""
    rng = np.random.default_rng(int(lam * 10))
    f = rng.dirichlet(np.ones(5))
    r = rng.dirichlet(np.ones(5))

    def obj(x):
        s = np.exp(x - x.max())
        s /= s.sum()
        return (1 - lam) * _kl(f, s) + lam * _kl(r, s)

    res = scipy.optimize.minimize(obj, np.zeros(5), method="BFGS", options={"gtol": 1e-12})
    s_opt = np.exp(res.x - res.x.max())
    s_opt /= s_opt.sum()
    np.testing.assert_allclose(O.fuse(f[None], r, lam, 1.0)[0], s_opt, atol=1e-6)
    # and the closed form beats random feasible perturbations
    s = O.fuse(f[None], r, lam, 1.0)[0]
    best = (1 - lam) * _kl(f, s) + lam * _kl(r, s)
    for _ in range(200):
        d = rng.normal(size=5) * 1e-3
        d -= d.mean()
        t = s + d
        if np.all(t > 0):
            assert (1 - lam) * _kl(f, t) + lam * _kl(r, t) >= best - 1e-15


# ---------------------------------------------------------------- evidence, prior
def test_evidence_restricts_and_renormalises():
    rng = np.random.default_rng(2)
    f = rng.dirichlet(np.ones(20), size=3)
    ft = O.evidence(f, 4, 15)
    np.testing.assert_allclose(ft.sum(axis=1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(ft * f[:, 4:15].sum(axis=1, keepdims=True), f[:, 4:15], rtol=1e-14)


def test_prior_hand_worked():
    g = _golden("prior_example.json")
    lo, hi = O.candidate_range(g["L"], g["n_sink"], g["n_recent"])
    assert list(range(lo, hi)) == g["candidates"]
    r = O.prior(np.array(g["norms_full"]), g["L"], lo, hi)
    w = np.array(g["kappa"]) * np.log(np.array(g["pi_args"], float))
    np.testing.assert_allclose(r, w / w.sum(), rtol=1e-14)


def test_prior_special_cases():
    L, lo, hi = 100, 4, 80
    # equal norms: kappa = 1, r proportional to ln(1 + L - j): decreasing in j
    r = O.prior(np.full(L, 3.0), L, lo, hi)
    assert np.all(np.diff(r) < 0)
    np.testing.assert_allclose(r[0] / r[-1], math.log(1 + L - lo) / math.log(1 + L - (hi - 1)), rtol=1e-14)
    np.testing.assert_allclose(r.sum(), 1.0, rtol=1e-14)
    # a key of norm 10 > mean is damped by nbar / 10 relative to a neighbour
    # whose norm is below the mean
    n = np.ones(L)
    n[40] = 10.0
    nbar = n[lo:hi].mean()
    r = O.prior(n, L, lo, hi)
    pi = np.log1p(L - np.arange(lo, hi))
    np.testing.assert_allclose(r[40 - lo] / r[41 - lo], (nbar / 10.0) * pi[40 - lo] / pi[41 - lo], rtol=1e-13)
    # zero-norm key: factor 1
    n = np.ones(L)
    n[10] = 0.0
    r = O.prior(n, L, lo, hi)
    assert np.isfinite(r).all()


# ---------------------------------------------------------------- soft-NMS
def test_soft_nms_hand_worked():
    g = _golden("soft_nms_8tok.json")
    ell = np.array([g["ell"]])
    for case in g["cases"]:
        got = O.soft_nms(ell, case["alpha_soft"], g["window"])
        np.testing.assert_allclose(got[0], case["expected"], rtol=0, atol=1e-15)


def test_soft_nms_properties():
    rng = np.random.default_rng(3)
    ell = rng.normal(size=(4, 300))
    out = O.soft_nms(ell, 0.5, 32)
    pen = ell - out
    assert np.all(pen >= 0) and np.all(pen <= 0.5 + 1e-15)
    # the row maximum is never penalised
    for h in range(4):
        j = int(np.argmax(ell[h]))
        assert out[h, j] == ell[h, j]
    np.testing.assert_array_equal(O.soft_nms(ell, 0.0, 32), ell)
    # an isolated peak penalises its neighbours by alpha (1 - (d-1)/w)
    x = np.zeros((1, 41))
    x[0, 20] = 5.0
    x[0] -= np.abs(np.arange(41) - 20) * 1e-3   # strictly decreasing away from the peak
    out = O.soft_nms(x, 1.0, 8)
    w = 4
    for d in range(1, w + 1):
        # the nearest dominating neighbour of 20 +- d is at distance 1
        assert out[0, 20 + d] == pytest.approx(x[0, 20 + d] - 1.0)
    assert out[0, 20] == x[0, 20]


# ---------------------------------------------------------------- cross-head
def test_cross_head_hand_worked():
    g = _golden("cross_head_3x4.json")
    got = O.cross_head(np.array(g["ell1"]), g["alpha_cross"])
    np.testing.assert_allclose(got, g["expected"], rtol=0, atol=1e-15)


def test_cross_head_special_cases():
    rng = np.random.default_rng(4)
    e = rng.normal(size=(4, 50))
    np.testing.assert_array_equal(O.cross_head(e, 0.0), e)
    np.testing.assert_array_equal(O.cross_head(e[:1], 0.7), e[:1])    # G = 1
    out = O.cross_head(e, 0.5)
    assert np.all(np.sum(out == e, axis=0) == 1)                       # one owner per column


# ---------------------------------------------------------------- exact decisions
def _selector_decimal(ft, r, lam, alpha_soft, alpha_cross, window, K, prec=80):
    """The Selector's steps (fusion, log, soft-NMS, cross-head, top-K) in
    80-digit decimal arithmetic, by brute force over every pair: the reference
    the float64 oracle's decisions must agree with."""
    from decimal import Decimal as Dc, localcontext
    with localcontext() as ctx:
        ctx.prec = prec
        G, n = ft.shape
        lam_d, one = Dc(lam), Dc(1)
        eps = Dc(O.LOG_EPS)
        ell = [[((one - lam_d) * Dc(ft[h, j]) + lam_d * Dc(r[j]) + eps).ln() for j in range(n)] for h in range(G)]
        w = window // 2
        ell1 = []
        for h in range(G):
            row = []
            for j in range(n):
                wt = Dc(0)
                for d in range(1, w + 1):
                    left = j - d >= 0 and ell[h][j - d] >= ell[h][j]
                    right = j + d < n and ell[h][j + d] > ell[h][j]
                    if left or right:
                        wt = one - Dc(d - 1) / Dc(w)
                        break
                row.append(ell[h][j] - Dc(alpha_soft) * wt)
            ell1.append(row)
        sel = []
        ell2 = [[None] * n for _ in range(G)]
        tie = Dc(O.OWNER_TIE)
        for j in range(n):
            M = max(ell1[h][j] for h in range(G))
            thr = M - tie
            best = min(h for h in range(G) if ell1[h][j] >= thr)
            for h in range(G):
                ell2[h][j] = ell1[h][j] - (Dc(alpha_cross) if h != best else Dc(0))
        for h in range(G):
            sel.append(sorted(sorted(range(n), key=lambda j: (-ell2[h][j], j))[:K]))
        return np.array(sel)


def _prior_dominated_case(seed, n=72, G=3, tiny=1e-24):
    """Evidence many orders of magnitude below the prior (the regime of most
    candidates on the long-context workloads), with a damped prior shape."""
    rng = np.random.default_rng(seed)
    L = n + 20
    kappa = np.minimum(1.0, rng.lognormal(0.0, 0.5, size=n) ** -1 * 1.1)
    pi = np.log1p(L - np.arange(n, dtype=np.float64))
    r = kappa * pi / np.sum(kappa * pi)
    ft = tiny * rng.lognormal(0.0, 2.0, size=(G, n))
    return ft, r


@pytest.mark.parametrize("seed,tiny", [(0, 1e-24), (1, 1e-18), (2, 1e-12), (3, 1e-3), (4, 1.0)])
def test_selector_decisions_agree_with_80_digit_arithmetic(seed, tiny):
    ft, r = _prior_dominated_case(seed, tiny=tiny)
    lam, a_s, a_c, window, K = 0.2, 0.5, 0.5, 8, 20
    det = O.selector_detail(ft, r, lam, 0.5, a_s, a_c, window)
    got = O.topk(det["ell2"], K)
    ref = _selector_decimal(ft, r, lam, a_s, a_c, window, K)
    np.testing.assert_array_equal(got, ref)


def test_owner_tie_tolerance():
    # heads whose l' agree to twenty digits: tied, the lowest head owns
    base = -13.0
    np.testing.assert_array_equal(O.owner(np.array([[base], [base + 1e-14], [base + 2e-14]])), [0])
    # within the tolerance (1e-3): tied; clearly above it: the largest owns
    np.testing.assert_array_equal(O.owner(np.array([[base], [base + 0.9e-3]])), [0])
    np.testing.assert_array_equal(O.owner(np.array([[base], [base + 1.1e-3]])), [1])
    np.testing.assert_array_equal(O.owner(np.array([[base], [base + 0.01], [base + 0.5]])), [2])
    # two heads tie with each other above a third: the lower of the two owns
    np.testing.assert_array_equal(O.owner(np.array([[base], [base + 0.5], [base + 0.5 + 1e-4]])), [1])
    # a plain argmax would take the largest: the tolerance is what differs
    ell1 = np.array([[base], [base + 1e-9]])
    assert list(np.argmax(ell1, axis=0)) == [1] and list(O.owner(ell1)) == [0]
    # cross_head penalises everyone but the owner
    out = O.cross_head(np.array([[base], [base + 1e-14]]), 0.5)
    np.testing.assert_allclose(out[:, 0], [base, base + 1e-14 - 0.5])


def test_soft_nms_exact_dominance_under_equal_prior():
    # two neighbours share the prior; the right one has the larger (tiny)
    # evidence, so it dominates the left one, although their float64 s is equal
    ft = np.array([[1e-30, 2e-30, 0.0]])
    r = np.array([0.5, 0.5, 0.0])
    ell = O.log_score(O.fuse(ft, r, 0.5, 1.0))
    assert ell[0, 0] == ell[0, 1]
    d = O.soft_nms_distance(ell, 2, (ft, r, 0.5))
    assert d[0, 0] == 1 and d[0, 1] == 0
    # without the mixture the rounded tie makes the left one dominate instead
    assert O.soft_nms_distance(ell, 2)[0, 1] == 1


# ---------------------------------------------------------------- top-K
@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_stable_sort(seed):
    rng = np.random.default_rng(seed)
    G, n = 3, 97
    s = rng.integers(0, 12, size=(G, n)).astype(np.float64)   # many ties
    K = int(rng.integers(1, n + 1))
    got = O.topk(s, K)
    for h in range(G):
        ref = sorted(range(n), key=lambda j: (-s[h, j], j))[:K]
        np.testing.assert_array_equal(got[h], sorted(ref))


def test_topk_edge_cases():
    s = np.array([[1.0, 1.0, 1.0, 1.0]])
    np.testing.assert_array_equal(O.topk(s, 2), [[0, 1]])
    np.testing.assert_array_equal(O.topk(s, 4), [[0, 1, 2, 3]])
    np.testing.assert_array_equal(O.topk(np.array([[3.0, -1.0, 7.0]]), 1), [[2]])


def test_budget_rule():
    assert O.budget(1025, 4, 64, 128, 0.2) == 128
    assert O.budget(8193, 4, 128, 0, 0.2) == int(math.floor(0.2 * 8193))
    assert O.budget(200, 4, 128, 0, 0.9) == 200 - 128 - 4          # clamped to |C|


# ---------------------------------------------------------------- whole selector
def test_selector_pure_prior_and_pure_evidence():
    rng = np.random.default_rng(5)
    L, G, ns, nr = 300, 4, 4, 16
    f = rng.dirichlet(np.ones(L), size=G)
    norms = rng.lognormal(size=L)
    lo, hi = O.candidate_range(L, ns, nr)
    K = 37
    # lambda = 1, no refinement: every head picks the top-K of kappa*pi
    sel = O.select(f, norms, L, ns, nr, K, 0, 1.0, 1.0, 0.0, 0.0, 32)
    r = O.prior(norms, L, lo, hi)
    top = np.sort(np.argsort(-r, kind="stable")[:K]) + lo
    for h in range(G):
        np.testing.assert_array_equal(sel[h], top)
    # lambda = 0, no refinement: top-K of f over the candidates
    sel = O.select(f, norms, L, ns, nr, K, 0, 0.0, 0.5, 0.0, 0.0, 32)
    for h in range(G):
        ref = sorted(range(lo, hi), key=lambda j: (-f[h, j], j))[:K]
        np.testing.assert_array_equal(sel[h], sorted(ref))


def test_selector_outputs_are_candidates():
    rng = np.random.default_rng(6)
    L, G = 500, 2
    f = rng.dirichlet(np.ones(L), size=G)
    sel = O.select(f, rng.lognormal(size=L), L, 4, 64, 0, 0.2, 0.2, 0.5, 0.5, 0.5, 32)
    assert sel.shape == (G, 100)
    assert np.all(sel >= 4) and np.all(sel < L - 64)
    assert np.all(np.diff(sel, axis=1) > 0)


# ---------------------------------------------------------------- compaction, trigger
def test_compact_hand_worked():
    g = _golden("compact_example.json")
    pos, hm = O.compact(np.array(g["selected"]), g["n_sink"])
    np.testing.assert_array_equal(pos, g["pos"])
    np.testing.assert_array_equal(hm, g["headmask"])


def test_compact_incremental_hand_worked():
    g = _golden("compact_incremental_example.json")
    for case in g["cases"]:
        prev = np.array(case["prev_pos"])
        pos, hm, moved = O.compact_incremental(prev, len(prev), np.array(case["selected"]), g["n_sink"])
        np.testing.assert_array_equal(pos, case["pos"])
        np.testing.assert_array_equal(hm, case["headmask"])
        assert moved == case["moved"]


def _random_selection(rng, lo, hi, G, K, prev=None, keep=0.9):
    out = []
    for h in range(G):
        base = rng.choice(np.arange(lo, hi), size=K, replace=False) if prev is None else prev[h].copy()
        if prev is not None:
            swap = rng.random(K) > keep
            fresh = rng.choice(np.setdiff1d(np.arange(lo, hi), base), size=int(swap.sum()), replace=False)
            base[swap] = fresh
        out.append(np.sort(base))
    return np.stack(out)


def test_compact_incremental_fresh_equals_full_compaction():
    rng = np.random.default_rng(3)
    sel = _random_selection(rng, 4, 300, 4, 40)
    pos, hm, moved = O.compact_incremental(np.zeros(0), 0, sel, 4)
    ref_pos, ref_hm = O.compact(sel, 4)
    np.testing.assert_array_equal(pos, ref_pos)
    np.testing.assert_array_equal(hm, ref_hm)
    assert moved == len(pos)


@pytest.mark.parametrize("keep", [1.0, 0.95, 0.5, 0.0])
def test_compact_incremental_is_the_union_with_stable_slots(keep):
    """Against the full compaction (pinned above): the same (position, mask)
    rows as a set; every previous row that stays selected and fits below n_new
    keeps its slot; exactly the entering and displaced rows are written."""
    rng = np.random.default_rng(int(keep * 100))
    n_sink, G = 4, 4
    prev_sel = _random_selection(rng, n_sink, 400, G, 30)
    prev_pos, _, _ = O.compact_incremental(np.zeros(0), 0, prev_sel, n_sink)
    for _ in range(6):
        sel = _random_selection(rng, n_sink, 400, G, 30, prev_sel, keep)
        pos, hm, moved = O.compact_incremental(prev_pos, len(prev_pos), sel, n_sink)
        ref_pos, ref_hm = O.compact(sel, n_sink)
        assert sorted(zip(pos.tolist(), hm.tolist())) == sorted(zip(ref_pos.tolist(), ref_hm.tolist()))
        assert len(set(pos.tolist())) == len(pos)
        new = set(ref_pos.tolist())
        same = [s for s in range(min(len(pos), len(prev_pos))) if prev_pos[s] in new and pos[s] == prev_pos[s]]
        should = [s for s in range(min(len(pos), len(prev_pos))) if prev_pos[s] in new]
        assert same == should
        entering = len(new - set(prev_pos.tolist()))
        displaced = sum(1 for s in range(len(pos), len(prev_pos)) if prev_pos[s] in new)
        assert moved == entering + displaced
        assert moved == sum(1 for s in range(n_sink, len(pos)) if s >= len(prev_pos) or pos[s] != prev_pos[s])
        if keep == 1.0:
            assert moved == 0
        prev_pos, prev_sel = pos, sel


def test_evidence_window_hand_worked():
    g = _golden("evidence_window_example.json")
    lo, hi = g["C"]
    got = O.evidence_window([np.array(f) for f in g["f"]], lo, hi)
    np.testing.assert_allclose(got, g["evidence"], rtol=1e-12)


def test_evidence_window_special_cases():
    rng = np.random.default_rng(12)
    fs = [rng.dirichlet(np.ones(50), size=3) for _ in range(4)]
    lo, hi = 5, 40
    # one query: the single-query evidence; repeated queries: the same
    np.testing.assert_allclose(O.evidence_window(fs[:1], lo, hi), O.evidence(fs[0], lo, hi), rtol=1e-14)
    np.testing.assert_allclose(O.evidence_window([fs[1]] * 3, lo, hi), O.evidence(fs[1], lo, hi), rtol=1e-14)
    # a distribution over C per head, inside the hull of the members
    ew = O.evidence_window(fs, lo, hi)
    np.testing.assert_allclose(ew.sum(axis=1), 1.0, rtol=1e-12)
    members = np.stack([O.evidence(f, lo, hi) for f in fs])
    assert np.all(ew <= members.max(axis=0) + 1e-15) and np.all(ew >= members.min(axis=0) - 1e-15)


def test_trigger_rows_hand_worked():
    g = _golden("trigger_rows_example.json")
    got = O.trigger_rows(np.array(g["boundary"], np.int8), g["M"])
    np.testing.assert_array_equal(got.astype(int), g["slow"])


def test_trigger_hand_worked():
    for case in _golden("trigger_example.json")["cases"]:
        got = O.trigger(np.array(case["boundary"], np.int8), case["M"])
        np.testing.assert_array_equal(got.astype(int), case["slow"])


# ---------------------------------------------------------------- end to end
def test_decode_run_full_coverage_equals_dense_over_kept_positions():
    """With K = |C| the slow step selects every candidate.  At fast step t the
    positions that slid out of the recent window since the slow step are the
    only ones missing, so the output is dense attention over the others."""
    from slow_sparse_kv_sfi_b200 import workload as W
    cfg = W.CONFIGS[0].replace(context=200, steps=6, k_fixed=10_000, refresh_budget=4)
    li = W.make_layer(cfg, 0, "cpu")
    outs, slow, sels = O.decode_run(
        li.k_pool.float().numpy(), li.v_pool.float().numpy(), li.page_table.numpy(),
        li.q.float().numpy(), li.k_new.float().numpy(), li.v_new.float().numpy(),
        W.boundary_stream(cfg), cfg.context, cfg.n_sink, cfg.n_recent, cfg.k_fixed,
        cfg.budget_frac, cfg.lam, cfg.lam_clip, cfg.alpha_soft, cfg.alpha_cross,
        cfg.nms_window, cfg.refresh_budget)
    assert slow.tolist() == [True, False, False, False, True, False]
    L_slow = cfg.context + 1
    lo, hi = O.candidate_range(L_slow, cfg.n_sink, cfg.n_recent)
    assert sels[0].shape[-1] == hi - lo
    kp, vp = li.k_pool.float().numpy().copy(), li.v_pool.float().numpy().copy()
    pt = li.page_table.numpy()
    for t in range(3):
        p = cfg.context + t
        kp[pt[0, p // 16], :, p % 16] = li.k_new[t, 0].float().numpy()
        vp[pt[0, p // 16], :, p % 16] = li.v_new[t, 0].float().numpy()
    L = cfg.context + 3
    keep = np.array([j for j in range(L) if not (hi <= j < L - cfg.n_recent)])
    assert len(keep) == L - 2
    for g in range(cfg.Hkv):
        K = O.gather_cache(kp, pt, 0, g, L)[keep]
        V = O.gather_cache(vp, pt, 0, g, L)[keep]
        qg = li.q[2, 0, g * cfg.G:(g + 1) * cfg.G].float().numpy()
        np.testing.assert_allclose(outs[2, 0, g * cfg.G:(g + 1) * cfg.G],
                                   O.dense_attention(qg, K, V)[0], rtol=1e-10, atol=1e-12)
    # at the slow step the output is dense attention over the whole context
    kp0, vp0 = li.k_pool.float().numpy().copy(), li.v_pool.float().numpy().copy()
    p = cfg.context
    kp0[pt[0, p // 16], :, p % 16] = li.k_new[0, 0].float().numpy()
    vp0[pt[0, p // 16], :, p % 16] = li.v_new[0, 0].float().numpy()
    for g in range(cfg.Hkv):
        K = O.gather_cache(kp0, pt, 0, g, L_slow)
        V = O.gather_cache(vp0, pt, 0, g, L_slow)
        qg = li.q[0, 0, g * cfg.G:(g + 1) * cfg.G].float().numpy()
        np.testing.assert_allclose(outs[0, 0, g * cfg.G:(g + 1) * cfg.G],
                                   O.dense_attention(qg, K, V)[0], rtol=1e-10, atol=1e-12)
