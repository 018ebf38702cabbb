"""The attention launches that append the step's token themselves
(sfi_dense_attn_append, sfi_fast_attn_append) against the two calls they
replace (sfi_append_kv, then sfi_dense_attn / sfi_fast_attn): every output,
the written cache rows and the key norms must agree bit for bit.  The two-call
path is itself checked against the oracle in test_gpu_kernels.py; the last
case here checks the fused fast step against the oracle directly."""
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


def _cfg(B, Hq, Hkv, D, L, **kw):
    base = dict(context=L, steps=8, n_recent=64, k_fixed=0, budget_frac=0.2,
                query_mode="planted", boundary_mode="none", refresh_budget=8, seed=23)
    base.update(kw)
    return W.SFIConfig(f"f{B}x{Hq}x{Hkv}x{D}x{L}", B=B, Hq=Hq, Hkv=Hkv, D=D, **base)


def _two_layers(cfg):
    li = W.make_layer(cfg, 0, "cpu")
    a = alloc_layer(cfg, li, DEV)
    b = alloc_layer(cfg, li, DEV)
    ws = torch.zeros(S.sfi_workspace_size(shape_of(cfg), params_of(cfg)), dtype=torch.uint8, device=DEV)
    return li, a, b, ws


def _same_cache(a, b):
    assert torch.equal(a.k_pool, b.k_pool)
    assert torch.equal(a.v_pool, b.v_pool)
    assert torch.equal(a.key_norms, b.key_norms)


# the appended row lands mid-page, on the first row of a page, on the last row
@pytest.mark.parametrize("B,Hq,Hkv,D,L0", [
    (1, 4, 2, 64, 1030),
    (2, 32, 8, 128, 4096),
    (1, 32, 2, 128, 2062),
    (2, 8, 8, 64, 95),
])
def test_dense_attn_append_matches_two_calls(B, Hq, Hkv, D, L0):
    cfg = _cfg(B, Hq, Hkv, D, L0)
    li, la, lb, ws = _two_layers(cfg)
    shape = shape_of(cfg)
    ld = L0 + 8
    outs = {}
    for name, layer in (("two", la), ("one", lb)):
        res = []
        for t in range(3):
            L = L0 + t + 1
            kn, vn = li.k_new[t].to(DEV), li.v_new[t].to(DEV)
            q = li.q[t].to(DEV)
            out = torch.empty(B, Hq, D, device=DEV)
            lse = torch.empty(B, Hq, device=DEV)
            lsec = torch.empty(B, Hq, device=DEV)
            logits = torch.empty(B, Hq, ld, device=DEV)
            ex = S.DenseExtras(lse.data_ptr(), logits.data_ptr(), None, ld, lsec.data_ptr(), 4, L - 32)
            if name == "two":
                S.sfi_append_kv(shape, layer.kv, L, kn, vn)
                S.sfi_dense_attn(shape, layer.kv, L, q, out, ws, ex)
            else:
                S.sfi_dense_attn_append(shape, layer.kv, L, kn, vn, q, out, ws, ex)
            res.append((out, lse, lsec, logits[:, :, :L]))
        torch.cuda.synchronize()
        assert S.sfi_poll_error(layer.kv) == 0
        outs[name] = res
    _same_cache(la, lb)
    for ra, rb in zip(outs["two"], outs["one"]):
        for xa, xb in zip(ra, rb):
            assert torch.equal(xa, xb)


@pytest.mark.parametrize("B,Hq,Hkv,D,L0,kw", [
    (1, 4, 2, 64, 1025, dict(k_fixed=128)),
    (2, 32, 8, 128, 4000, dict(budget_frac=0.15, n_recent=256)),
    (1, 32, 2, 128, 3007, dict(budget_frac=0.2)),
])
def test_fast_attn_append_matches_two_calls_and_oracle(B, Hq, Hkv, D, L0, kw):
    cfg = _cfg(B, Hq, Hkv, D, L0, **kw)
    li, la, lb, ws = _two_layers(cfg)
    shape, params = shape_of(cfg), params_of(cfg)
    G = cfg.G
    lo, hi = O.candidate_range(L0, cfg.n_sink, cfg.n_recent)
    K = S.sfi_budget(params, L0)
    rng = np.random.default_rng(L0 + 1)
    sel = np.stack([np.stack([np.sort(rng.choice(np.arange(lo, hi), size=K, replace=False))
                              for _ in range(Hq)]) for _ in range(B)]).astype(np.int32)
    sel_t = torch.from_numpy(sel).to(DEV)
    for layer in (la, lb):
        S.sfi_compact(shape, params, layer.kv, L0, sel_t, K, K, layer.packed, ws)
    outs = {}
    for name, layer in (("two", la), ("one", lb)):
        res = []
        for t in range(4):
            L = L0 + t + 1
            kn, vn = li.k_new[t].to(DEV), li.v_new[t].to(DEV)
            q = li.q[t].to(DEV)
            out = torch.empty(B, Hq, D, device=DEV)
            lse = torch.empty(B, Hq, device=DEV)
            if name == "two":
                S.sfi_append_kv(shape, layer.kv, L, kn, vn)
                S.sfi_fast_attn(shape, params, layer.kv, L, q, layer.packed, out, ws, lse)
            else:
                S.sfi_fast_attn_append(shape, params, layer.kv, L, kn, vn, q, layer.packed, out, ws, lse)
            res.append((out, lse))
        torch.cuda.synchronize()
        assert S.sfi_poll_error(layer.kv) == 0
        outs[name] = res
    _same_cache(la, lb)
    for ra, rb in zip(outs["two"], outs["one"]):
        for xa, xb in zip(ra, rb):
            assert torch.equal(xa, xb)
    # the last fused step against the oracle's sparse attention
    Lt = L0 + 4
    kp, vp = H.to64(lb.k_pool), H.to64(lb.v_pool)
    pt = li.page_table.numpy()
    qh = H.to64(li.q[3])
    out = outs["one"][3][0]
    for b in range(B):
        for g in range(Hkv):
            Kc, Vc = H.group_kv(kp, vp, pt, b, g, Lt)
            sets = O.sparse_sets(Lt, cfg.n_sink, cfg.n_recent, [sel[b, g * G + h] for h in range(G)])
            o = O.sparse_attention(qh[b, g * G:(g + 1) * G], Kc, Vc, sets)
            H.assert_attn_close(out[b, g * G:(g + 1) * G].cpu().numpy(), o, f"fused fast b{b} g{g}")
    # and the appended rows hold the step's tokens
    for t in range(4):
        p = L0 + t
        for b in range(B):
            page = pt[b, p // 16]
            assert torch.equal(lb.k_pool[page, :, p % 16].cpu(), li.k_new[t, b])
            assert torch.equal(lb.v_pool[page, :, p % 16].cpu(), li.v_new[t, b])
            np.testing.assert_allclose(lb.key_norms[b, :, p].cpu().numpy(),
                                       np.linalg.norm(H.to64(li.k_new[t, b]), axis=1), rtol=H.NORM_RTOL)


def test_fused_append_bad_page_is_reported():
    cfg = _cfg(1, 4, 2, 64, 300)
    li = W.make_layer(cfg, 0, "cpu")
    layer = alloc_layer(cfg, li, DEV)
    ws = torch.zeros(S.sfi_workspace_size(shape_of(cfg), params_of(cfg)), dtype=torch.uint8, device=DEV)
    L = 301
    layer.page_table[0, (L - 1) // 16] = 10_000_000
    out = torch.empty(1, 4, 64, device=DEV)
    S.sfi_dense_attn_append(shape_of(cfg), layer.kv, L, li.k_new[0].to(DEV), li.v_new[0].to(DEV),
                            li.q[0].to(DEV), out, ws)
    torch.cuda.synchronize()
    code = S.sfi_poll_error(layer.kv)
    assert code & 0xFF == 5   # SFI_ERR_DEVICE_CHECK
    assert S.sfi_poll_error(layer.kv) == 0
