"""Multi-query evidence window: at a slow step the Selector's evidence is the
mean of the restricted distributions of the last W queries.  The decode-step
driver keeps every layer's recent queries and runs them through one dense
launch (W x G heads per KV group), whose outputs for the step's own queries
are the slow step's attention.  Checked against the oracle step by step:
slow outputs against dense attention of the step's query, selections against
the oracle's Selector on `evidence_window` of the queries the decode has seen
(fewer than W at its start), fast outputs against sparse attention over the
GPU's sets."""
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


def _run(cfg, per_sequence):
    shape, params = shape_of(cfg), params_of(cfg)
    li = W.make_layer(cfg, 0, "cpu")
    layer = alloc_layer(cfg, li, DEV)
    ctx = S.Context(shape, params, 1, True)
    if per_sequence:
        bnd = W.boundary_rows(cfg)
        slow_ref = O.trigger_rows(bnd, cfg.refresh_budget)
    else:
        b1 = W.boundary_stream(cfg)
        bnd = np.broadcast_to(b1, (cfg.B, cfg.steps))
        slow_ref = np.broadcast_to(O.trigger(b1, cfg.refresh_budget), (cfg.B, cfg.steps))
    G, Wn = cfg.G, cfg.evidence_window
    kp, vp = H.to64(li.k_pool).copy(), H.to64(li.v_pool).copy()
    pt = li.page_table.numpy()
    sets = [None] * (cfg.B * cfg.Hkv)
    worst = 0.0
    n_slow_window = 0
    for t in range(cfg.steps):
        L = cfg.context + t + 1
        out = torch.empty(cfg.B, cfg.Hq, cfg.D, device=DEV)
        if per_sequence:
            got = ctx.decode_step_rows(0, t, bnd[:, t - 1] if t > 0 else None, L, layer.kv, layer.packed,
                                       li.q[t].to(DEV), li.k_new[t].to(DEV), li.v_new[t].to(DEV), out)
            assert got == [bool(x) for x in slow_ref[:, t]]
        else:
            slow = ctx.decode_step(0, t, int(bnd[0, t - 1]) if t > 0 else 0, L, layer.kv, layer.packed,
                                   li.q[t].to(DEV), li.k_new[t].to(DEV), li.v_new[t].to(DEV), out)
            assert slow == bool(slow_ref[0, t])
        ctx.join()
        torch.cuda.synchronize()
        assert S.sfi_poll_error(layer.kv) == 0
        p = L - 1
        for b in range(cfg.B):
            kp[pt[b, p // 16], :, p % 16] = H.to64(li.k_new[t, b])
            vp[pt[b, p // 16], :, p % 16] = H.to64(li.v_new[t, b])
        K = O.budget(L, cfg.n_sink, cfg.n_recent, cfg.k_fixed, cfg.budget_frac)
        lo, _ = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
        o_gpu = out.cpu().numpy()
        for b in range(cfg.B):
            for g in range(cfg.Hkv):
                Kc, Vc = H.group_kv(kp, vp, pt, b, g, L)
                hs = slice(g * G, (g + 1) * G)
                what = f"step {t} b{b} g{g}"
                if slow_ref[b, t]:
                    o, f, _, _ = O.dense_attention(H.to64(li.q[t, b, hs]), Kc, Vc)
                    fw = [f] + [O.dense_attention(H.to64(li.q[t - i, b, hs]), Kc, Vc)[1]
                                for i in range(1, min(Wn, t + 1))]
                    n_slow_window += len(fw) > 1
                    qw = [H.to64(li.q[t - i, b, hs]) for i in range(len(fw))]
                    sb, _ = H.decode_selection_bounds(qw[0], Kc, f, L, cfg, f_window=fw, q_window=qw)
                    n = int(layer.n_rows[b, g])
                    sg = H.packed_sets(layer.pos[b, g].cpu().numpy(), layer.headmask[b, g].cpu().numpy(),
                                       n, cfg.n_sink, G)
                    H.check_selection(np.stack(sg), sb, K, lo, what)
                    sets[b * cfg.Hkv + g] = sg
                else:
                    o = O.sparse_attention(H.to64(li.q[t, b, hs]), Kc, Vc,
                                           O.sparse_sets(L, cfg.n_sink, cfg.n_recent, sets[b * cfg.Hkv + g]))
                worst = max(worst, H.assert_attn_close(o_gpu[b, hs], o, what))
    ctx.close()
    return worst, n_slow_window


def test_window_three_queries_per_sequence_triggers():
    """G = 2, W = 3: six query rows per group in the slow launch."""
    cfg = W.CONFIGS[1].replace(steps=16, context=3000, boundary_p=0.25, refresh_budget=5, evidence_window=3)
    worst, n = _run(cfg, per_sequence=True)
    assert n > 0 and worst < H.ATTN_RTOL


def test_window_four_queries_sixteen_rows():
    """G = 4, W = 4: sixteen query rows per group (the two-tile launch plan),
    planted queries."""
    cfg = W.CONFIG_BY_NAME["qwen3-4b-32k"].replace(B=2, context=2600, steps=12, boundary_p=0.3,
                                                   refresh_budget=4, evidence_window=4, query_mode="planted")
    worst, n = _run(cfg, per_sequence=False)
    assert n > 0 and worst < H.ATTN_RTOL
