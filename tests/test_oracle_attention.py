"""Pins of the oracle's attention, paged-cache and key-norm functions.

Each check ties the oracle to something other than itself: torch's
scaled_dot_product_attention in float64 (a library routine), closed forms,
special cases and the full-coverage invariant.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

from oracle import sfi_oracle as O


def _sdpa(q, K, V, mask=None):
    qt = torch.from_numpy(np.asarray(q, np.float64))[None, :, None, :]   # [1,G,1,D]
    Kt = torch.from_numpy(np.asarray(K, np.float64))[None, None].expand(1, q.shape[0], -1, -1)
    Vt = torch.from_numpy(np.asarray(V, np.float64))[None, None].expand(1, q.shape[0], -1, -1)
    m = None if mask is None else torch.from_numpy(mask)[None, :, None, :]
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=m)[0, :, 0].numpy()


@pytest.mark.parametrize("G,L,D", [(1, 7, 8), (4, 50, 16), (16, 33, 64)])
def test_dense_matches_library_sdpa(G, L, D):
    rng = np.random.default_rng(G * 1000 + L)
    q, K, V = rng.normal(size=(G, D)), rng.normal(size=(L, D)), rng.normal(size=(L, D))
    o, f, lse, z = O.dense_attention(q, K, V)
    np.testing.assert_allclose(o, _sdpa(q, K, V), rtol=1e-12, atol=1e-12)
    # f is attention with V = identity: each output row is the distribution
    np.testing.assert_allclose(f, _sdpa(q, K, np.eye(L)), rtol=1e-12, atol=1e-14)


def test_dense_closed_forms():
    rng = np.random.default_rng(1)
    L, D = 21, 4
    V = rng.normal(size=(L, D))
    # q = 0: uniform distribution, lse = log L, o = mean of V
    o, f, lse, _ = O.dense_attention(np.zeros((2, D)), rng.normal(size=(L, D)), V)
    np.testing.assert_allclose(f, 1.0 / L, rtol=1e-14)
    np.testing.assert_allclose(lse, math.log(L), rtol=1e-14)
    np.testing.assert_allclose(o, np.broadcast_to(V.mean(axis=0), o.shape), rtol=1e-12)
    # scale 1/sqrt(D): with q = 2 e0 and k_j = a_j e0, z_j = 2 a_j / 2 = a_j
    a = rng.normal(size=L)
    K = np.zeros((L, D))
    K[:, 0] = a
    q = np.zeros((1, D))
    q[0, 0] = 2.0
    _, f, lse, z = O.dense_attention(q, K, V)
    np.testing.assert_allclose(z[0], a, rtol=1e-14)
    np.testing.assert_allclose(lse[0], scipy.special.logsumexp(a), rtol=1e-14)
    np.testing.assert_allclose(f[0], scipy.special.softmax(a), rtol=1e-12)


def test_dense_permutation_equivariance():
    rng = np.random.default_rng(2)
    q, K, V = rng.normal(size=(3, 8)), rng.normal(size=(40, 8)), rng.normal(size=(40, 8))
    perm = rng.permutation(40)
    o1, f1, l1, _ = O.dense_attention(q, K, V)
    o2, f2, l2, _ = O.dense_attention(q, K[perm], V[perm])
    np.testing.assert_allclose(o1, o2, rtol=1e-12)
    np.testing.assert_allclose(f1[:, perm], f2, rtol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=1e-14)


def test_sparse_matches_masked_sdpa():
    rng = np.random.default_rng(3)
    G, L, D = 4, 60, 16
    q, K, V = rng.normal(size=(G, D)), rng.normal(size=(L, D)), rng.normal(size=(L, D))
    sets = [np.sort(rng.choice(L, size=s, replace=False)) for s in (1, 5, 30, 60)]
    mask = np.zeros((G, L), bool)
    for h, S in enumerate(sets):
        mask[h, S] = True
    got = O.sparse_attention(q, K, V, sets)
    np.testing.assert_allclose(got, _sdpa(q, K, V, mask), rtol=1e-12, atol=1e-12)


def test_sparse_equals_dense_under_full_coverage():
    rng = np.random.default_rng(4)
    G, L, D = 2, 100, 32
    q, K, V = rng.normal(size=(G, D)), rng.normal(size=(L, D)), rng.normal(size=(L, D))
    n_sink, n_recent = 4, 10
    lo, hi = O.candidate_range(L, n_sink, n_recent)
    sel = [np.arange(lo, hi)] * G
    sets = O.sparse_sets(L, n_sink, n_recent, sel)
    for S in sets:
        np.testing.assert_array_equal(S, np.arange(L))
    np.testing.assert_allclose(O.sparse_attention(q, K, V, sets),
                               O.dense_attention(q, K, V)[0], rtol=1e-12)


def test_sparse_sets_structure():
    sets = O.sparse_sets(50, 4, 8, [np.array([10, 20]), np.array([5])])
    np.testing.assert_array_equal(sets[0], [0, 1, 2, 3, 10, 20] + list(range(42, 50)))
    np.testing.assert_array_equal(sets[1], [0, 1, 2, 3, 5] + list(range(42, 50)))


def test_gather_cache_follows_page_table():
    rng = np.random.default_rng(5)
    B, H, D, npb = 2, 3, 8, 4
    logical = rng.normal(size=(B, H, npb * 16, D))
    perm = rng.permutation(B * npb)
    pt = perm.reshape(B, npb)
    pool = np.zeros((B * npb, H, 16, D))
    for b in range(B):
        for i in range(npb):
            pool[pt[b, i]] = logical[b, :, i * 16:(i + 1) * 16]
    for b in range(B):
        for h in range(H):
            got = O.gather_cache(pool, pt, b, h, 53)
            np.testing.assert_array_equal(got, logical[b, h, :53])


def test_key_norms_library():
    rng = np.random.default_rng(6)
    K = rng.normal(size=(30, 64)) * rng.lognormal(size=(30, 1))
    np.testing.assert_allclose(O.key_norms(K), np.linalg.norm(K, axis=1), rtol=1e-14)
    assert O.key_norms(np.zeros((1, 4)))[0] == 0.0


def test_workload_pool_matches_logical_rows():
    """The generator's paged pool read back through the oracle's page-table
    walk gives the same rows as the generator's own logical layout."""
    from slow_sparse_kv_sfi_b200 import workload as W
    cfg = W.CONFIGS[0].replace(context=100, steps=8, B=2)
    li = W.make_layer(cfg, 0, "cpu")
    pool = li.k_pool.float().numpy()
    pt = li.page_table.numpy()
    # rows at or beyond the context start as zeros
    for b in range(cfg.B):
        K = O.gather_cache(pool, pt, b, 1, cfg.capacity)
        assert np.all(K[cfg.context:] == 0)
        assert np.all(np.abs(K[:cfg.context]).sum(axis=1) > 0)
    # the queries point at their planted keys: those keys rank near the top
    q = li.q.float().numpy()
    for b in range(cfg.B):
        for h in range(cfg.Hq):
            K = O.gather_cache(pool, pt, b, h // cfg.G, cfg.context)
            z = K @ q[0, b, h] / np.linalg.norm(K, axis=1)
            top = set(np.argsort(-z)[:10].tolist())
            assert set(li.planted[0, b, h].tolist()) <= top
