"""End-to-end parity of the decode-step driver (trigger, append, dense slow
steps with the side-stream Selector + compaction, fast steps) against the
oracle, step by step.  Fast steps are checked with the GPU's own selected
sets fed to the oracle's sparse attention, so set near-ties cannot hide an
attention error; the sets themselves are checked against the oracle's
Selector at every slow step."""
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


def _run(cfg, overlap, n_layers=1):
    shape, params = shape_of(cfg), params_of(cfg)
    lis = [W.make_layer(cfg, l, "cpu") for l in range(n_layers)]
    layers = [alloc_layer(cfg, li, DEV) for li in lis]
    ctx = S.Context(shape, params, n_layers, overlap)
    boundary = W.boundary_stream(cfg)
    slow_ref = O.trigger(boundary, cfg.refresh_budget)
    G = cfg.G
    caches = [(H.to64(li.k_pool).copy(), H.to64(li.v_pool).copy()) for li in lis]
    gpu_sets = [None] * n_layers
    worst = {"attn": 0.0, "overlap": 1.0}
    for t in range(cfg.steps):
        L = cfg.context + t + 1
        outs = []
        for l, (li, layer) in enumerate(zip(lis, layers)):
            out = torch.empty(cfg.B, cfg.Hq, cfg.D, device=DEV)
            slow = ctx.decode_step(l, t, int(boundary[t - 1]) if t > 0 else 0, L, layer.kv,
                                   layer.packed, li.q[t].to(DEV), li.k_new[t].to(DEV),
                                   li.v_new[t].to(DEV), out)
            assert slow == bool(slow_ref[t]), f"trigger at step {t}"
            outs.append(out)
        ctx.join()
        torch.cuda.synchronize()
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
            if slow_ref[t]:
                gpu_sets[l] = []
                K = O.budget(L, cfg.n_sink, cfg.n_recent, cfg.k_fixed, cfg.budget_frac)
                lo, _ = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
            for b in range(cfg.B):
                for g in range(cfg.Hkv):
                    Kc, Vc = H.group_kv(kp, vp, pt, b, g, L)
                    qg = qh[b, g * G:(g + 1) * G]
                    if slow_ref[t]:
                        o, f, _, _ = O.dense_attention(qg, Kc, Vc)
                        sb, _ = H.decode_selection_bounds(qg, Kc, f, L, cfg)
                        n = int(layer.n_rows[b, g])
                        sets = H.packed_sets(layer.pos[b, g].cpu().numpy(),
                                             layer.headmask[b, g].cpu().numpy(), n, cfg.n_sink, G)
                        got = np.stack(sets)
                        ov = H.check_selection(got, sb, K, lo, f"step {t} b{b} g{g}")
                        worst["overlap"] = min(worst["overlap"], ov)
                        gpu_sets[l].append(sets)
                    else:
                        sets = O.sparse_sets(L, cfg.n_sink, cfg.n_recent, gpu_sets[l][b * cfg.Hkv + g])
                        o = O.sparse_attention(qg, Kc, Vc, sets)
                    e = H.assert_attn_close(o_gpu[b, g * G:(g + 1) * G], o, f"step {t} b{b} g{g}")
                    worst["attn"] = max(worst["attn"], e)
    ctx.close()
    return worst


def test_decode_config1_all_steps():
    w = _run(W.CONFIGS[0], overlap=True)
    assert w["attn"] < H.ATTN_RTOL


@pytest.mark.parametrize("overlap", [True, False])
def test_decode_config2_boundary_trigger(overlap):
    cfg = W.CONFIGS[1].replace(steps=40 if overlap else 12)
    w = _run(cfg, overlap)
    assert w["attn"] < H.ATTN_RTOL


def test_decode_two_layers_overlapped_selector():
    """Two stacked layers: the Selector of layer 0 runs on the side stream
    while layer 1 attends; every later step must see both refreshes."""
    cfg = W.CONFIGS[2].replace(B=1, Hq=8, Hkv=2, context=4096, steps=20, refresh_budget=6)
    w = _run(cfg, overlap=True, n_layers=2)
    assert w["attn"] < H.ATTN_RTOL
