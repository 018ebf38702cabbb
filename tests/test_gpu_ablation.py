"""The Selector ablation driver's measurements on a small workload: support
recall is a share of a probability distribution, equals 1 when the selection
covers every candidate (the fast step then attends to everything dense
attention does), selection stability is a share of K, and both agree step
by step with the same quantities recomputed from the oracle's decode."""
import pytest
import torch

from slow_sparse_kv_sfi_b200 import ablation as A
from slow_sparse_kv_sfi_b200 import workload as W

pytestmark = pytest.mark.gpu


def _cfg(**kw):
    base = W.CONFIGS[0].replace(steps=20, boundary_mode="bernoulli", boundary_p=0.25, refresh_budget=6)
    return base.replace(**kw)


def test_full_coverage_recall_is_one():
    res = A.run_setting(_cfg(k_fixed=100_000), torch.device("cuda"))
    assert res["fast_steps"] > 0
    assert abs(res["recall_of_reachable_min"] - 1.0) < 1e-4
    assert 0.9 < res["recall_min"] <= 1.0 + 1e-5


@pytest.mark.parametrize("over", [{}, {"lam": 1.0, "lam_clip": 1.0}, {"alpha_soft": 0.0, "alpha_cross": 0.0}])
def test_recall_and_stability_are_shares(over):
    res = A.run_setting(_cfg(**over), torch.device("cuda"))
    assert res["fast_steps"] > 0 and res["slow_steps"] > 1
    assert 0.0 < res["recall_min"] <= res["recall_p10"] <= res["recall_mean"] <= 1.0 + 1e-5
    assert res["recall_mean"] <= res["recall_of_reachable_mean"] <= 1.0 + 1e-5
    assert 0.0 <= res["stability_mean"] <= 1.0


@pytest.mark.parametrize("over", [{}, {"lam": 0.0}, {"alpha_soft": 0.0, "alpha_cross": 0.0}])
def test_measurements_match_the_oracle(over):
    """Every fast step's recall and every slow step's stability, per (sequence,
    query head), recomputed on the CPU from the oracle's own decode: its dense
    attention distribution at that step and its selections."""
    import numpy as np
    from oracle import sfi_oracle as O
    import helpers as H

    cfg = _cfg(**over)
    res = A.run_setting(cfg, torch.device("cuda"), detail=True)
    li = W.make_layer(cfg, 0, "cuda")          # the tensors run_setting drew
    slow = O.trigger(W.boundary_stream(cfg), cfg.refresh_budget)
    kp, vp, pt = H.to64(li.k_pool), H.to64(li.v_pool), li.page_table.cpu().numpy()
    G = cfg.G
    sel = prev = None
    n_rec = n_stab = 0
    for t in range(cfg.steps):
        L = cfg.seq_len(t)
        p = L - 1
        for b in range(cfg.B):
            kp[pt[b, p // 16], :, p % 16] = H.to64(li.k_new[t, b])
            vp[pt[b, p // 16], :, p % 16] = H.to64(li.v_new[t, b])
        rec = np.zeros(cfg.B * cfg.Hq)
        cur = {}
        for b in range(cfg.B):
            for g in range(cfg.Hkv):
                K, V = H.group_kv(kp, vp, pt, b, g, L)
                _, f, _, _ = O.dense_attention(H.to64(li.q[t, b, g * G:(g + 1) * G]), K, V)
                if slow[t]:
                    cur[(b, g)] = O.select(f, O.key_norms(K), L, cfg.n_sink, cfg.n_recent, cfg.k_fixed,
                                           cfg.budget_frac, cfg.lam, cfg.lam_clip, cfg.alpha_soft,
                                           cfg.alpha_cross, cfg.nms_window)
                else:
                    sets = O.sparse_sets(L, cfg.n_sink, cfg.n_recent, list(sel[(b, g)]))
                    for h in range(G):
                        rec[b * cfg.Hq + g * G + h] = f[h, sets[h]].sum()
        if slow[t]:
            if prev is not None:
                st = [len(set(cur[(b, g)][h]) & set(prev[(b, g)][h])) / len(cur[(b, g)][h])
                      for b in range(cfg.B) for g in range(cfg.Hkv) for h in range(G)]
                np.testing.assert_allclose(res["stability_steps"][t], st, atol=1e-12, err_msg=f"step {t}")
                n_stab += 1
            prev = sel = cur
        else:
            np.testing.assert_allclose(res["recall_steps"][t], rec, atol=1e-3, err_msg=f"step {t}")
            n_rec += 1
    assert n_rec == res["fast_steps"] and n_stab == res["slow_steps"] - 1
