"""The Selector ablation driver's measurements on a small workload: support
recall is a share of a probability distribution, equals 1 when the selection
covers every candidate (the fast step then attends to everything dense
attention does), and selection stability is a share of K."""
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
