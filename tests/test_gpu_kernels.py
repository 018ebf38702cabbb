"""Parity of every CUDA kernel of the SFI decode path with the CPU oracle,
called through the C ABI on the same seeded inputs.  Sizes span several
tiles, stages and work items and end in ragged tails."""
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
                query_mode="planted", boundary_mode="none", refresh_budget=8, seed=11)
    base.update(kw)
    return W.SFIConfig(f"t{B}x{Hq}x{Hkv}x{D}x{L}", B=B, Hq=Hq, Hkv=Hkv, D=D, **base)


def _setup(cfg):
    li = W.make_layer(cfg, 0, "cpu")
    layer = alloc_layer(cfg, li, DEV)
    ws = torch.zeros(S.sfi_workspace_size(shape_of(cfg), params_of(cfg)), dtype=torch.uint8, device=DEV)
    return li, layer, ws


ATTN_SHAPES = [
    (1, 4, 2, 64, 1025),      # config 1 layout, one-row tail
    (2, 16, 8, 128, 3000),    # G = 2
    (2, 32, 8, 128, 5001),    # G = 4
    (1, 16, 2, 128, 777),     # G = 8
    (1, 32, 2, 128, 2049),    # G = 16
    (2, 8, 8, 64, 100),       # G = 1, shorter than one stage
    (1, 12, 4, 128, 333),     # G = 3 (padded head tile)
]


@pytest.mark.parametrize("B,Hq,Hkv,D,L", ATTN_SHAPES)
def test_dense_attention_parity(B, Hq, Hkv, D, L):
    cfg = _cfg(B, Hq, Hkv, D, L)
    li, layer, ws = _setup(cfg)
    shape = shape_of(cfg)
    q = li.q[0].to(DEV)
    out = torch.empty(B, Hq, D, device=DEV)
    ld = L + 7
    lse = torch.empty(B, Hq, device=DEV)
    logits = torch.empty(B, Hq, ld, device=DEV)
    probs = torch.empty(B, Hq, ld, device=DEV)
    lsec = torch.empty(B, Hq, device=DEV)
    lo, hi = 4, L - 64
    ex = S.DenseExtras(lse.data_ptr(), logits.data_ptr(), probs.data_ptr(), ld, lsec.data_ptr(), lo, hi)
    S.sfi_dense_attn(shape, layer.kv, L, q, out, ws, ex)
    # the plain full-KV form (no extras) must agree bit for bit on o
    out2 = torch.empty_like(out)
    S.sfi_dense_attn(shape, layer.kv, L, q, out2, ws)
    torch.cuda.synchronize()
    assert S.sfi_poll_error(layer.kv) == 0
    assert torch.equal(out, out2)
    kp, vp, pt = H.to64(li.k_pool), H.to64(li.v_pool), li.page_table.numpy()
    qh = H.to64(li.q[0])
    G = Hq // Hkv
    for b in range(B):
        for g in range(Hkv):
            K, V = H.group_kv(kp, vp, pt, b, g, L)
            o, f, l, z = O.dense_attention(qh[b, g * G:(g + 1) * G], K, V)
            sl = slice(g * G, (g + 1) * G)
            H.assert_attn_close(out[b, sl].cpu().numpy(), o, f"o b{b} g{g}")
            np.testing.assert_allclose(lse[b, sl].cpu().numpy(), l, atol=H.PROB_ATOL, rtol=0)
            np.testing.assert_allclose(probs[b, sl, :L].cpu().numpy(), f, atol=H.PROB_ATOL, rtol=0)
            np.testing.assert_allclose(logits[b, sl, :L].cpu().numpy(), z, atol=1e-4, rtol=1e-5)
            lc = np.log(np.exp(z[:, lo:hi] - l[:, None]).sum(axis=1)) + l
            np.testing.assert_allclose(lsec[b, sl].cpu().numpy(), lc, atol=H.PROB_ATOL, rtol=0)
            # the logit and candidate-lse error budget the Selector's tolerance model assumes
            zb = H.logit_error_bound(qh[b, g * G:(g + 1) * G], K)
            dz = np.abs(logits[b, sl, :L].cpu().numpy().astype(np.float64) - z)
            H.LOGIT_RECORD.append(float((dz / zb).max()) * H.C_Z)
            assert np.all(dz <= zb), f"logit error beyond its bound: {(dz / zb).max():.3f} x the bound"
            dl = np.abs(lsec[b, sl].cpu().numpy().astype(np.float64) - lc)
            lb = H.lse_error_bound(zb[:, lo:hi], O.evidence(f, lo, hi))
            H.LSE_RECORD.append(float((dl / lb).max()))
            assert np.all(dl <= lb), f"candidate lse error {dl.max():.3e} beyond its bound"


def test_dense_attention_masks_garbage_beyond_L():
    """Rows past L in the last page hold NaN: they must not leak into o."""
    cfg = _cfg(1, 8, 2, 128, 200)
    li, layer, ws = _setup(cfg)
    L = 183
    pt = li.page_table.numpy()
    for pos in range(L, 192):
        layer.k_pool[pt[0, pos // 16], :, pos % 16] = float("nan")
        layer.v_pool[pt[0, pos // 16], :, pos % 16] = float("nan")
    out = torch.empty(1, 8, 128, device=DEV)
    S.sfi_dense_attn(shape_of(cfg), layer.kv, L, li.q[0].to(DEV), out, ws)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    kp, vp = H.to64(layer.k_pool), H.to64(layer.v_pool)
    for g in range(2):
        K, V = H.group_kv(kp, vp, pt, 0, g, L)
        o = O.dense_attention(H.to64(li.q[0])[0, g * 4:(g + 1) * 4], K, V)[0]
        H.assert_attn_close(out[0, g * 4:(g + 1) * 4].cpu().numpy(), o)


def test_bad_page_table_entry_is_reported_not_read():
    cfg = _cfg(1, 4, 2, 64, 300)
    li, layer, ws = _setup(cfg)
    layer.page_table[0, 3] = 10_000_000
    out = torch.empty(1, 4, 64, device=DEV)
    S.sfi_dense_attn(shape_of(cfg), layer.kv, 300, li.q[0].to(DEV), out, ws)
    torch.cuda.synchronize()
    code = S.sfi_poll_error(layer.kv)
    assert code & 0xFF == 5   # SFI_ERR_DEVICE_CHECK
    assert S.sfi_poll_error(layer.kv) == 0


@pytest.mark.parametrize("D,Hkv", [(64, 2), (128, 8)])
def test_append_and_key_norms(D, Hkv):
    cfg = _cfg(2, Hkv * 2, Hkv, D, 500)
    li, layer, ws = _setup(cfg)
    shape = shape_of(cfg)
    torch.cuda.synchronize()
    kp = H.to64(li.k_pool)
    pt = li.page_table.numpy()
    norms = layer.key_norms.cpu().numpy()
    for b in range(2):
        for g in range(Hkv):
            K, _ = H.group_kv(kp, kp, pt, b, g, cfg.context)
            np.testing.assert_allclose(norms[b, g, :cfg.context], np.linalg.norm(K, axis=1),
                                       rtol=H.NORM_RTOL, atol=0)
    for t in range(3):
        L = cfg.context + t + 1
        S.sfi_append_kv(shape, layer.kv, L, li.k_new[t].to(DEV), li.v_new[t].to(DEV))
    torch.cuda.synchronize()
    for t in range(3):
        p = cfg.context + t
        for b in range(2):
            page = pt[b, p // 16]
            assert torch.equal(layer.k_pool[page, :, p % 16].cpu(), li.k_new[t, b])
            assert torch.equal(layer.v_pool[page, :, p % 16].cpu(), li.v_new[t, b])
            np.testing.assert_allclose(layer.key_norms[b, :, p].cpu().numpy(),
                                       np.linalg.norm(H.to64(li.k_new[t, b]), axis=1), rtol=H.NORM_RTOL)


def _select_inputs(cfg, li, layer, L):
    """Oracle float64 logits and lse over C, rounded to fp32 as the CUDA
    Selector receives them from the dense kernel."""
    kp, vp, pt = H.to64(li.k_pool), H.to64(li.v_pool), li.page_table.numpy()
    qh = H.to64(li.q[0])
    G = cfg.G
    lo, hi = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
    z = np.zeros((cfg.B, cfg.Hq, L))
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            K, V = H.group_kv(kp, vp, pt, b, g, L)
            z[b, g * G:(g + 1) * G] = O.dense_attention(qh[b, g * G:(g + 1) * G], K, V)[3]
    z32 = z.astype(np.float32)
    zz = z32.astype(np.float64)
    m = zz[:, :, lo:hi].max(axis=2, keepdims=True)
    lsec = (m[..., 0] + np.log(np.exp(zz[:, :, lo:hi] - m).sum(axis=2))).astype(np.float32)
    return z32, lsec


SEL_SHAPES = [
    (1, 4, 2, 64, 1025, dict(k_fixed=128)),
    (2, 8, 2, 128, 6000, dict(budget_frac=0.15)),
    (1, 32, 2, 128, 3000, dict(budget_frac=0.2, outlier_frac=0.005, query_mode="clusters")),
    (2, 4, 4, 64, 2500, dict(budget_frac=0.2)),     # G = 1
    # Selector settings of the ablation sweep
    (1, 16, 4, 128, 4000, dict(budget_frac=0.2, lam=0.0)),                       # evidence only
    (1, 16, 4, 128, 4000, dict(budget_frac=0.2, lam=1.0, lam_clip=1.0)),         # prior only
    (1, 16, 4, 128, 4000, dict(budget_frac=0.2, lam=0.8, lam_clip=0.5)),         # clip active
    (1, 16, 4, 128, 4000, dict(budget_frac=0.2, alpha_soft=0.0, alpha_cross=0.0)),
    (1, 16, 4, 128, 4000, dict(budget_frac=0.2, nms_window=8, alpha_soft=1.0, alpha_cross=0.25)),
]


@pytest.mark.parametrize("B,Hq,Hkv,D,L,kw", SEL_SHAPES)
def test_selector_scores_topk_and_compaction(B, Hq, Hkv, D, L, kw):
    cfg = _cfg(B, Hq, Hkv, D, L, **kw)
    li, layer, ws = _setup(cfg)
    shape, params = shape_of(cfg), params_of(cfg)
    G = cfg.G
    z32, lsec = _select_inputs(cfg, li, layer, L)
    lo, hi = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
    nC = hi - lo
    logits = torch.from_numpy(z32).to(DEV).contiguous()
    lse_c = torch.from_numpy(lsec).to(DEV)
    scores = torch.empty(B, Hq, nC, device=DEV)
    S.sfi_select_scores(shape, params, layer.kv, L, logits, L, lse_c, scores, ws)
    K = S.sfi_budget(params, L)
    sel = torch.empty(B, Hq, K + 3, dtype=torch.int32, device=DEV)
    tws = torch.zeros(S.sfi_topk_workspace_size(B * Hq, nC), dtype=torch.uint8, device=DEV)
    S.sfi_topk(B * Hq, nC, scores, nC, K, lo, sel, K + 3, tws)
    sel2 = torch.empty_like(sel)
    assert S.sfi_select(shape, params, layer.kv, L, logits, L, lse_c, sel2, K + 3, ws) == K
    S.sfi_compact(shape, params, layer.kv, L, sel2, K + 3, K, layer.packed, ws)
    torch.cuda.synchronize()
    assert S.sfi_poll_error(layer.kv) == 0
    sc = scores.cpu().numpy()
    sel_g = sel.cpu().numpy()[:, :, :K]
    assert np.array_equal(sel_g, sel2.cpu().numpy()[:, :, :K])
    norms = layer.key_norms.cpu().numpy().astype(np.float64)
    kp, vp, pt = li.k_pool, li.v_pool, li.page_table.numpy()
    for b in range(B):
        for g in range(Hkv):
            rows = slice(g * G, (g + 1) * G)
            # top-K on the GPU's own scores: bit-exact against the oracle's top-K
            ref_top = O.topk(sc[b, rows].astype(np.float64), K) + lo
            np.testing.assert_array_equal(sel_g[b, rows], ref_top)
            # scores and sets against the oracle Selector fed the same fp32
            # logits and norms: every score inside its interval, the sets as
            # check_selection requires
            bnd, _ = H.kernel_selection_bounds(z32[b, rows], norms[b, g], L, cfg)
            H.check_selection(sel_g[b, rows], bnd, K, lo, f"b{b} g{g}", gpu_scores=sc[b, rows])
            # compaction: rows, order, masks, copies (bit-exact)
            pos_ref, hm_ref = O.compact(sel_g[b, rows] , cfg.n_sink)
            n = int(layer.n_rows[b, g])
            assert n == len(pos_ref)
            np.testing.assert_array_equal(layer.pos[b, g, :n].cpu().numpy(), pos_ref)
            np.testing.assert_array_equal(layer.headmask[b, g, :n].cpu().numpy().astype(np.uint32), hm_ref)
            pidx = torch.from_numpy(pos_ref)
            pages = li.page_table[b][pidx // 16].long()
            assert torch.equal(layer.pk[b, g, :n].cpu(), kp[pages, g, pidx % 16])
            assert torch.equal(layer.pv[b, g, :n].cpu(), vp[pages, g, pidx % 16])
            pad = (n + 15) // 16 * 16
            assert torch.all(layer.pk[b, g, n:pad] == 0) and torch.all(layer.headmask[b, g, n:pad] == 0)


@pytest.mark.parametrize("B,Hq,Hkv,D,L,kw", [
    (1, 4, 2, 64, 1025, dict(k_fixed=128)),
    (2, 32, 8, 128, 4000, dict(budget_frac=0.15, n_recent=256)),
    (1, 32, 2, 128, 3000, dict(budget_frac=0.2)),
    (2, 8, 8, 128, 700, dict(budget_frac=0.3)),
])
def test_fast_attention_parity(B, Hq, Hkv, D, L, kw):
    """Random per-head selections -> compaction -> fast attention three steps
    later (after three appends), against the oracle's sparse attention."""
    cfg = _cfg(B, Hq, Hkv, D, L, **kw)
    li, layer, ws = _setup(cfg)
    shape, params = shape_of(cfg), params_of(cfg)
    G = cfg.G
    lo, hi = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
    K = S.sfi_budget(params, L)
    rng = np.random.default_rng(L)
    sel = np.zeros((B, Hq, K), np.int32)
    for b in range(B):
        for g in range(Hkv):
            common = rng.choice(np.arange(lo, hi), size=K // 2, replace=False)
            for h in range(G):
                rest = np.setdiff1d(np.arange(lo, hi), common)
                own = rng.choice(rest, size=K - K // 2, replace=False)
                sel[b, g * G + h] = np.sort(np.concatenate([common, own]))
    sel_t = torch.from_numpy(sel).to(DEV)
    S.sfi_compact(shape, params, layer.kv, L, sel_t, K, K, layer.packed, ws)
    Lt = L
    for t in range(3):
        Lt = L + t + 1
        S.sfi_append_kv(shape, layer.kv, Lt, li.k_new[t].to(DEV), li.v_new[t].to(DEV))
    q = li.q[3].to(DEV)
    out = torch.empty(B, Hq, D, device=DEV)
    lse = torch.empty(B, Hq, device=DEV)
    S.sfi_fast_attn(shape, params, layer.kv, Lt, q, layer.packed, out, ws, lse)
    torch.cuda.synchronize()
    assert S.sfi_poll_error(layer.kv) == 0
    kp, vp = H.to64(layer.k_pool), H.to64(layer.v_pool)
    pt = li.page_table.numpy()
    qh = H.to64(li.q[3])
    for b in range(B):
        for g in range(Hkv):
            Kc, Vc = H.group_kv(kp, vp, pt, b, g, Lt)
            sets = O.sparse_sets(Lt, cfg.n_sink, cfg.n_recent, [sel[b, g * G + h] for h in range(G)])
            o = O.sparse_attention(qh[b, g * G:(g + 1) * G], Kc, Vc, sets)
            H.assert_attn_close(out[b, g * G:(g + 1) * G].cpu().numpy(), o, f"fast b{b} g{g}")
            for h in range(G):
                z = Kc[sets[h]] @ qh[b, g * G + h] / np.sqrt(D)
                m = z.max()
                np.testing.assert_allclose(float(lse[b, g * G + h]), m + np.log(np.exp(z - m).sum()),
                                           atol=H.PROB_ATOL)


def test_fast_attention_full_coverage_equals_dense():
    """K = |C| at the slow step: at that same L the fast step sees every
    position, so it must reproduce dense attention."""
    cfg = _cfg(1, 16, 4, 128, 1500, k_fixed=100_000, n_recent=128)
    li, layer, ws = _setup(cfg)
    shape, params = shape_of(cfg), params_of(cfg)
    L = cfg.context
    lo, hi = O.candidate_range(L, cfg.n_sink, cfg.n_recent)
    K = S.sfi_budget(params, L)
    assert K == hi - lo
    sel = torch.arange(lo, hi, dtype=torch.int32, device=DEV).repeat(1, 16, 1).contiguous()
    S.sfi_compact(shape, params, layer.kv, L, sel, K, K, layer.packed, ws)
    q = li.q[0].to(DEV)
    o_fast = torch.empty(1, 16, 128, device=DEV)
    o_dense = torch.empty_like(o_fast)
    S.sfi_fast_attn(shape, params, layer.kv, L, q, layer.packed, o_fast, ws)
    S.sfi_dense_attn(shape, layer.kv, L, q, o_dense, ws)
    torch.cuda.synchronize()
    H.assert_attn_close(o_fast.cpu().numpy(), o_dense.cpu().numpy().astype(np.float64))
