"""Per-sequence triggers: every sequence of the batch decides its own slow
steps (its own boundary tokens and refresh budget), so a step can run the
dense attention + Selector + compaction on some sequences and the sparse
attention on the others.  Checked against the oracle step by step, as the
batch-wide decode test does: the decisions against `trigger_rows`, slow
sequences' outputs against dense attention and their selections against the
oracle's Selector, fast sequences' outputs against sparse attention over the
sets their own last slow step selected."""
import numpy as np
import pytest
import torch

from oracle import sfi_oracle as O
from slow_sparse_kv_sfi_b200 import sfi as S
from slow_sparse_kv_sfi_b200 import workload as W
from slow_sparse_kv_sfi_b200.state import alloc_layer, params_of, shape_of

import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(cfg, overlap, n_layers, incremental=True):
    shape, params = shape_of(cfg), params_of(cfg)
    lis = [W.make_layer(cfg, l, "cpu") for l in range(n_layers)]
    layers = [alloc_layer(cfg, li, DEV) for li in lis]
    ctx = S.Context(shape, params, n_layers, overlap, incremental=incremental)
    bnd = W.boundary_rows(cfg)
    slow_ref = O.trigger_rows(bnd, cfg.refresh_budget)
    G = cfg.G
    caches = [(H.to64(li.k_pool).copy(), H.to64(li.v_pool).copy()) for li in lis]
    sets = [[None] * (cfg.B * cfg.Hkv) for _ in range(n_layers)]
    worst = 0.0
    mixed = 0
    for t in range(cfg.steps):
        L = cfg.context + t + 1
        prev = bnd[:, t - 1] if t > 0 else None
        outs = []
        for l, (li, layer) in enumerate(zip(lis, layers)):
            out = torch.empty(cfg.B, cfg.Hq, cfg.D, device=DEV)
            got = ctx.decode_step_rows(l, t, prev, L, layer.kv, layer.packed, li.q[t].to(DEV),
                                       li.k_new[t].to(DEV), li.v_new[t].to(DEV), out)
            assert got == [bool(x) for x in slow_ref[:, t]], f"trigger at step {t}"
            outs.append(out)
        mixed += 0 < slow_ref[:, t].sum() < cfg.B
        ctx.join()
        torch.cuda.synchronize()
        K = O.budget(L, cfg.n_sink, cfg.n_recent, cfg.k_fixed, cfg.budget_frac)
        lo, _ = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
        for l, (li, layer) in enumerate(zip(lis, layers)):
            assert S.sfi_poll_error(layer.kv) == 0
            kp, vp = caches[l]
            pt = li.page_table.numpy()
            p = L - 1
            for b in range(cfg.B):
                kp[pt[b, p // 16], :, p % 16] = H.to64(li.k_new[t, b])
                vp[pt[b, p // 16], :, p % 16] = H.to64(li.v_new[t, b])
            qh = H.to64(li.q[t])
            o_gpu = outs[l].cpu().numpy()
            for b in range(cfg.B):
                for g in range(cfg.Hkv):
                    Kc, Vc = H.group_kv(kp, vp, pt, b, g, L)
                    qg = qh[b, g * G:(g + 1) * G]
                    what = f"layer {l} step {t} b{b} g{g}"
                    if slow_ref[b, t]:
                        o, f, _, _ = O.dense_attention(qg, Kc, Vc)
                        sb, _ = H.decode_selection_bounds(qg, Kc, f, L, cfg)
                        n = int(layer.n_rows[b, g])
                        sg = H.packed_sets(layer.pos[b, g].cpu().numpy(), layer.headmask[b, g].cpu().numpy(),
                                           n, cfg.n_sink, G)
                        H.check_selection(np.stack(sg), sb, K, lo, what)
                        sets[l][b * cfg.Hkv + g] = sg
                    else:
                        o = O.sparse_attention(qg, Kc, Vc, O.sparse_sets(L, cfg.n_sink, cfg.n_recent,
                                                                         sets[l][b * cfg.Hkv + g]))
                    worst = max(worst, H.assert_attn_close(o_gpu[b, g * G:(g + 1) * G], o, what))
    ctx.close()
    return worst, mixed


@pytest.mark.parametrize("overlap,incremental", [(True, True), (False, False)])
def test_per_sequence_triggers_two_layers(overlap, incremental):
    cfg = W.CONFIGS[1].replace(steps=20, boundary_p=0.25, refresh_budget=6, context=3000)
    worst, mixed = _run(cfg, overlap, 2, incremental)
    assert mixed >= 5
    assert worst < H.ATTN_RTOL


def test_per_sequence_triggers_group16():
    cfg = W.CONFIG_BY_NAME["qwen3-235b-a22b-64k"].replace(B=3, context=2500, steps=10, boundary_mode="bernoulli",
                                                          boundary_p=0.3, refresh_budget=4)
    worst, mixed = _run(cfg, True, 1)
    assert mixed >= 3
    assert worst < H.ATTN_RTOL
