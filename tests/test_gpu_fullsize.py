"""Parity at the full sizes of the long-context workloads, in the launch
configuration the benchmark times: one layer of each workload decoded by the
two-stream decode-step driver (fused append, dense slow steps with the
Selector and compaction on the side stream, fast steps), checked against the
oracle on sampled (sequence, KV head) groups.

The oracle's inputs are the seeded generator's tensors only: the sampled
groups' cache rows are copied to the host before the first step, and every
step's appended token is applied on the host from the generator's k_new /
v_new.  Slow steps: dense attention of every head of the group, and the
packed selection against the oracle's Selector (near-tie aware).  Fast steps:
sparse attention over the GPU's own selected sets (checked at the slow step
before), so set near-ties cannot hide an attention error."""
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

CASES = [
    # (workload, steps, overrides, sampled (b, kv head) groups)
    ("qwen3-4b-32k", 3, {}, [(0, 0), (5, 7)]),
    # slow steps 0 and 3: a full build, fast steps, an incremental refresh, a fast step
    ("qwen3-4b-128k-36l", 5, {"boundary_mode": "none", "refresh_budget": 3}, [(0, 3), (1, 6)]),
    # G = 16 Selector stress: nine slow steps in a row (eight incremental refreshes), then fast
    ("qwen3-235b-a22b-64k", 10, {"slow_prefix": 9}, [(3, 1), (15, 3)]),
]


def _host_rows(li, b, g, n):
    """Generator rows [0, n) of (b, kv head g), read through the page table."""
    pages = li.page_table[b, : (n + 15) // 16].long()
    K = li.k_pool[pages, g].reshape(-1, li.k_pool.shape[-1])[:n]
    V = li.v_pool[pages, g].reshape(-1, li.v_pool.shape[-1])[:n]
    return H.to64(K), H.to64(V)


@pytest.mark.parametrize("name,steps,over,groups", CASES)
def test_full_size_decode_sampled(name, steps, over, groups):
    cfg = W.CONFIG_BY_NAME[name].replace(n_layers=1, steps=steps, **over)
    shape, params = shape_of(cfg), params_of(cfg)
    G = cfg.G
    li = W.make_layer(cfg, 0, DEV)
    # host copies of the sampled groups, taken before the device cache is touched
    host = {bg: _host_rows(li, bg[0], bg[1], cfg.context) for bg in groups}
    k_new, v_new, q_all = li.k_new.cpu(), li.v_new.cpu(), li.q.cpu()
    layer = alloc_layer(cfg, W.LayerInputs(**{**li.__dict__, "k_pool": li.k_pool.clone(),
                                              "v_pool": li.v_pool.clone()}), DEV)
    del li
    torch.cuda.empty_cache()
    ctx = S.Context(shape, params, 1, overlap=True)
    boundary = W.boundary_stream(cfg)
    slow_ref = O.trigger(boundary, cfg.refresh_budget)
    sets_gpu = {}
    worst = 0.0
    for t in range(steps):
        L = cfg.context + t + 1
        out = torch.empty(cfg.B, cfg.Hq, cfg.D, device=DEV)
        slow = ctx.decode_step(0, t, int(boundary[t - 1]) if t > 0 else 0, L, layer.kv, layer.packed,
                               q_all[t].to(DEV), k_new[t].to(DEV), v_new[t].to(DEV), out)
        assert slow == bool(slow_ref[t])
        ctx.join()
        torch.cuda.synchronize()
        assert S.sfi_poll_error(layer.kv) == 0
        o_gpu = out.cpu().numpy()
        for (b, g) in groups:
            Kc, Vc = host[(b, g)]
            Kc = np.concatenate([Kc, H.to64(k_new[t, b, g])[None]])
            Vc = np.concatenate([Vc, H.to64(v_new[t, b, g])[None]])
            host[(b, g)] = (Kc, Vc)
            qg = H.to64(q_all[t, b, g * G:(g + 1) * G])
            if slow_ref[t]:
                o, f, _, _ = O.dense_attention(qg, Kc, Vc)
                K = O.budget(L, cfg.n_sink, cfg.n_recent, cfg.k_fixed, cfg.budget_frac)
                lo, _ = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
                sb, _ = H.decode_selection_bounds(qg, Kc, f, L, cfg)
                n = int(layer.n_rows[b, g])
                sets = H.packed_sets(layer.pos[b, g].cpu().numpy(), layer.headmask[b, g].cpu().numpy(),
                                     n, cfg.n_sink, G)
                H.check_selection(np.stack(sets), sb, K, lo, f"{name} step {t} b{b} g{g}")
                # the packed rows are bit-exact copies of the cache rows they name
                pos = layer.pos[b, g, :n].cpu().numpy()
                assert np.array_equal(H.to64(layer.pk[b, g, :n]), Kc[pos])
                assert np.array_equal(H.to64(layer.pv[b, g, :n]), Vc[pos])
                sets_gpu[(b, g)] = sets
            else:
                sets = O.sparse_sets(L, cfg.n_sink, cfg.n_recent, sets_gpu[(b, g)])
                o = O.sparse_attention(qg, Kc, Vc, sets)
            worst = max(worst, H.assert_attn_close(o_gpu[b, g * G:(g + 1) * G], o, f"{name} step {t} b{b} g{g}"))
    ctx.close()
    assert worst < H.ATTN_RTOL
