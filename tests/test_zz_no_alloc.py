"""sfi_dense_attn_noalloc: dense attention for callers that cannot allocate
device memory at the call (runtimes that hand the library only input and
output tensors, hosts without access to the CUDA allocator).  Its scratch is a static device array inside the
library.  Checked through the C ABI against sfi_dense_attn, which takes a
caller-allocated workspace, on two calls in a row (the static area keeps the
previous call's contents), and for the clear rejection of a shape whose
scratch would not fit.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from slow_sparse_kv_sfi_b200 import sfi as S
from slow_sparse_kv_sfi_b200 import workload as W
from slow_sparse_kv_sfi_b200.state import alloc_layer, params_of, shape_of

import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(B, Hq, Hkv, D, L, seed):
    cfg = W.SFIConfig("noalloc", B=B, Hq=Hq, Hkv=Hkv, D=D, context=L, steps=4, n_recent=64,
                      boundary_mode="none", seed=seed)
    li = W.make_layer(cfg, 0, "cpu")
    layer = alloc_layer(cfg, li, DEV)
    return cfg, li, layer


@pytest.mark.parametrize("B,Hq,Hkv,D,L", [(2, 32, 8, 128, 3001), (1, 4, 2, 64, 1025)])
def test_noalloc_matches_workspace_entry_point_twice(B, Hq, Hkv, D, L):
    shape = None
    outs = []
    for call, seed in enumerate((21, 22)):          # two calls in a row, different inputs
        cfg, li, layer = _case(B, Hq, Hkv, D, L, seed)
        shape = shape_of(cfg)
        ws = torch.zeros(S.sfi_workspace_size(shape, params_of(cfg)), dtype=torch.uint8, device=DEV)
        q = li.q[0].to(DEV)
        ref = torch.empty(B, Hq, D, device=DEV)
        ref_lse = torch.empty(B, Hq, device=DEV)
        S.sfi_dense_attn(shape, layer.kv, L, q, ref, ws,
                         S.DenseExtras(ref_lse.data_ptr(), None, None, 0, None, 0, 0))
        got = torch.full((B, Hq, D), float("nan"), device=DEV)
        got_lse = torch.full((B, Hq), float("nan"), device=DEV)
        S.sfi_dense_attn_noalloc(shape, layer.kv, L, q, got,
                                 S.DenseExtras(got_lse.data_ptr(), None, None, 0, None, 0, 0))
        torch.cuda.synchronize()
        assert S.sfi_poll_error(layer.kv) == 0
        H.assert_attn_close(got.cpu().numpy(), ref.cpu().numpy().astype(np.float64), f"call {call}")
        np.testing.assert_allclose(got_lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=H.PROB_ATOL, rtol=0)
        outs.append(got.cpu())
    assert not torch.equal(outs[0], outs[1])        # the second call really recomputed


def test_noalloc_rejects_scratch_beyond_its_maximum():
    """G = 16, 64 (sequence, KV head) pairs at L = 8192 need ~34 MB of
    partials, more than the static area holds: refused, nothing launched."""
    cfg = W.SFIConfig("noalloc-big", B=16, Hq=64, Hkv=4, D=128, context=8192, steps=16, n_recent=64,
                      boundary_mode="none", seed=3)
    shape = shape_of(cfg)
    k_pool = torch.zeros(cfg.num_pages, cfg.Hkv, 16, cfg.D, dtype=torch.bfloat16, device=DEV)
    v_pool = torch.zeros_like(k_pool)
    pt = torch.arange(cfg.num_pages, dtype=torch.int32, device=DEV).view(cfg.B, cfg.pages_per_seq)
    kv = S.make_kv(k_pool, v_pool, pt)
    q = torch.zeros(cfg.B, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=DEV)
    out = torch.full((cfg.B, cfg.Hq, cfg.D), 7.0, device=DEV)
    with pytest.raises(S.SFIError) as e:
        S.sfi_dense_attn_noalloc(shape, kv, 8192, q, out)
    assert e.value.status == 7   # SFI_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
