"""Incremental compaction on the GPU against the oracle's refresh rule,
bit-exact: a chain of slow-step selections with controlled overlap (all rows
kept, a few swapped, half swapped, none kept, a shrinking and a growing
union), each refreshing the packed buffer in place.  The oracle follows its
own chain (it never reads the GPU's layout); every step compares slot
positions, head masks and n_rows exactly, the packed K/V rows with the cache
rows they name, and the zero rows up to the next multiple of 16."""
import numpy as np
import pytest
import torch

from oracle import sfi_oracle as O
from slow_sparse_kv_sfi_b200 import sfi as S
from slow_sparse_kv_sfi_b200 import workload as W
from slow_sparse_kv_sfi_b200.state import alloc_layer, params_of, shape_of

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cfg(B, Hq, Hkv, D, L, **kw):
    base = dict(context=L, steps=8, n_recent=64, k_fixed=0, budget_frac=0.2,
                query_mode="planted", boundary_mode="none", refresh_budget=8, seed=5)
    base.update(kw)
    return W.SFIConfig(f"inc{B}x{Hq}x{Hkv}x{D}x{L}", B=B, Hq=Hq, Hkv=Hkv, D=D, **base)


def _next_selection(rng, prev, lo, hi, K, keep):
    """Per query head (rows of prev): keep each previous pick with probability
    `keep`, fill up to K with fresh candidates from [lo, hi)."""
    rows = []
    for h in range(prev.shape[0]):
        kept = prev[h][rng.random(prev.shape[1]) < keep][:K]
        pool = np.setdiff1d(np.arange(lo, hi), kept)
        add = rng.choice(pool, size=K - len(kept), replace=False)
        rows.append(np.sort(np.concatenate([kept, add])).astype(np.int32))
    return np.stack(rows)


# (B, Hq, Hkv, D, L, config overrides, keep probability of each refresh)
CASES = [
    (1, 4, 2, 64, 1500, dict(k_fixed=96), [1.0, 0.9, 0.5, 0.0, 0.97]),
    (2, 16, 4, 128, 6000, dict(budget_frac=0.1), [0.95, 1.0, 0.8, 0.3]),
    (1, 32, 2, 128, 4000, dict(budget_frac=0.05), [0.9, 0.6, 0.99]),            # G = 16
    (1, 8, 8, 128, 2000, dict(budget_frac=0.2), [0.9, 0.0, 0.9]),               # G = 1
]


def _check(layer, li, b, g, pos_ref, hm_ref, what):
    n = int(layer.n_rows[b, g])
    assert n == len(pos_ref), what
    np.testing.assert_array_equal(layer.pos[b, g, :n].cpu().numpy(), pos_ref, err_msg=what)
    np.testing.assert_array_equal(layer.headmask[b, g, :n].cpu().numpy().astype(np.uint32), hm_ref, err_msg=what)
    pidx = torch.from_numpy(np.asarray(pos_ref, np.int64))
    pages = li.page_table[b][pidx // 16].long()
    assert torch.equal(layer.pk[b, g, :n].cpu(), li.k_pool[pages, g, pidx % 16]), what
    assert torch.equal(layer.pv[b, g, :n].cpu(), li.v_pool[pages, g, pidx % 16]), what
    pad = (n + 15) // 16 * 16
    assert torch.all(layer.pk[b, g, n:pad] == 0) and torch.all(layer.pv[b, g, n:pad] == 0), what
    assert torch.all(layer.headmask[b, g, n:pad] == 0) and torch.all(layer.pos[b, g, n:pad] == -1), what


@pytest.mark.parametrize("B,Hq,Hkv,D,L,kw,keeps", CASES)
def test_incremental_compaction_chain(B, Hq, Hkv, D, L, kw, keeps):
    cfg = _cfg(B, Hq, Hkv, D, L, **kw)
    li = W.make_layer(cfg, 0, "cpu")
    layer = alloc_layer(cfg, li, DEV)
    shape, params = shape_of(cfg), params_of(cfg)
    ws = torch.zeros(S.sfi_workspace_size(shape, params), dtype=torch.uint8, device=DEV)
    G = cfg.G
    lo, hi = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
    K = S.sfi_budget(params, L)
    rng = np.random.default_rng(L + Hq)
    sel = np.stack([np.sort(rng.choice(np.arange(lo, hi), size=K, replace=False)) for _ in range(B * Hq)])
    sel = sel.reshape(B, Hq, K).astype(np.int32)
    ora = {}
    for step, keep in enumerate([None] + keeps):
        if keep is not None:
            sel = np.stack([_next_selection(rng, sel[b], lo, hi, K, keep) for b in range(B)])
        S.sfi_compact_incremental(shape, params, layer.kv, L, torch.from_numpy(sel).to(DEV), K, K,
                                  layer.packed, step == 0, ws)
        torch.cuda.synchronize()
        assert S.sfi_poll_error(layer.kv) == 0
        for b in range(B):
            for g in range(Hkv):
                prev = ora.get((b, g), np.zeros(0, np.int64))
                pos_ref, hm_ref, _ = O.compact_incremental(prev, len(prev), sel[b, g * G:(g + 1) * G], cfg.n_sink)
                ora[(b, g)] = pos_ref
                _check(layer, li, b, g, pos_ref, hm_ref, f"step {step} keep {keep} b{b} g{g}")
    # the workspace is left in its zero state: a fresh start reproduces the full compaction
    S.sfi_compact_incremental(shape, params, layer.kv, L, torch.from_numpy(sel).to(DEV), K, K, layer.packed, 1, ws)
    torch.cuda.synchronize()
    for b in range(B):
        for g in range(Hkv):
            pos_ref, hm_ref = O.compact(sel[b, g * G:(g + 1) * G], cfg.n_sink)
            _check(layer, li, b, g, pos_ref, hm_ref, f"fresh b{b} g{g}")


def test_incremental_after_full_compaction_and_growing_L():
    """A buffer written by the full compaction at context L is refreshed at a
    longer context (the candidate range grew by two tokens' worth of steps)."""
    cfg = _cfg(1, 16, 4, 128, 3000, budget_frac=0.1)
    li = W.make_layer(cfg, 0, "cpu")
    layer = alloc_layer(cfg, li, DEV)
    shape, params = shape_of(cfg), params_of(cfg)
    ws = torch.zeros(S.sfi_workspace_size(shape, params), dtype=torch.uint8, device=DEV)
    G = cfg.G
    rng = np.random.default_rng(9)
    L0 = 2900
    lo, hi0 = O.candidate_range(L0, cfg.n_sink, cfg.n_recent)
    K0 = S.sfi_budget(params, L0)
    sel0 = np.stack([np.sort(rng.choice(np.arange(lo, hi0), size=K0, replace=False)) for _ in range(16)])
    sel0 = sel0.reshape(1, 16, K0).astype(np.int32)
    S.sfi_compact(shape, params, layer.kv, L0, torch.from_numpy(sel0).to(DEV), K0, K0, layer.packed, ws)
    L1 = 3000
    _, hi1 = O.candidate_range(L1, cfg.n_sink, cfg.n_recent)
    K1 = S.sfi_budget(params, L1)
    sel1 = np.stack([_next_selection(rng, sel0[0], lo, hi1, K1, 0.9)]).astype(np.int32)
    S.sfi_compact_incremental(shape, params, layer.kv, L1, torch.from_numpy(sel1).to(DEV), K1, K1,
                              layer.packed, 0, ws)
    torch.cuda.synchronize()
    assert S.sfi_poll_error(layer.kv) == 0
    for g in range(4):
        prev, _ = O.compact(sel0[0, g * G:(g + 1) * G], cfg.n_sink)
        pos_ref, hm_ref, moved = O.compact_incremental(prev, len(prev), sel1[0, g * G:(g + 1) * G], cfg.n_sink)
        assert moved < len(pos_ref) // 2
        _check(layer, li, 0, g, pos_ref, hm_ref, f"g{g}")
