"""Failure detection of the device-side waits, without a GPU fault: the
library's bounded mbarrier wait, run on a barrier that nothing completes,
expires at its limit, latches SFI_ERR_TIMEOUT with its site, and lets the
kernel return; the host reads it through sfi_poll_error and the context stays
usable.  The attention kernels take their wait limit from sfi_set_wait_limit
at every launch."""
import time

import pytest
import torch

from slow_sparse_kv_sfi_b200 import sfi as S
from slow_sparse_kv_sfi_b200 import workload as W
from slow_sparse_kv_sfi_b200.state import alloc_layer, params_of, shape_of

import helpers as H
from oracle import sfi_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
SFI_ERR_TIMEOUT = 6
SITE_SELFTEST = 11


def test_bounded_wait_expires_and_is_reported():
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    kv = S.PagedKV(None, None, None, None, err.data_ptr())
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    S.sfi_selftest_wait(kv, 50_000)          # 50 us
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert elapsed < 1.0, f"the wait did not return at its limit ({elapsed:.3f} s)"
    code = S.sfi_poll_error(kv)
    assert code & 0xFF == SFI_ERR_TIMEOUT and code >> 8 == SITE_SELFTEST, hex(code)
    assert S.sfi_poll_error(kv) == 0           # read and cleared


def test_wait_limit_is_a_launch_argument_and_work_goes_on():
    old = S.sfi_get_wait_limit()
    assert old == 2_000_000_000
    cfg = W.SFIConfig("wait", B=1, Hq=8, Hkv=2, D=128, context=4096, steps=2, n_recent=64, seed=21)
    li = W.make_layer(cfg, 0, "cpu")
    layer = alloc_layer(cfg, li, DEV)
    ws = torch.zeros(S.sfi_workspace_size(shape_of(cfg), params_of(cfg)), dtype=torch.uint8, device=DEV)
    q = li.q[0].to(DEV)
    out = torch.empty(cfg.B, cfg.Hq, cfg.D, device=DEV)
    try:
        S.sfi_set_wait_limit(100_000_000)      # 100 ms: far above any legitimate wait here
        assert S.sfi_get_wait_limit() == 100_000_000
        # an expired self-test leaves the context usable for real work
        S.sfi_selftest_wait(layer.kv, 20_000)
        torch.cuda.synchronize()
        assert S.sfi_poll_error(layer.kv) & 0xFF == SFI_ERR_TIMEOUT
        S.sfi_dense_attn(shape_of(cfg), layer.kv, cfg.context, q, out, ws)
        torch.cuda.synchronize()
        assert S.sfi_poll_error(layer.kv) == 0
    finally:
        S.sfi_set_wait_limit(old)
    K, V = H.group_kv(H.to64(li.k_pool), H.to64(li.v_pool), li.page_table.numpy(), 0, 0, cfg.context)
    o = O.dense_attention(H.to64(li.q[0, 0, :4]), K, V)[0]
    H.assert_attn_close(out[0, :4].cpu().numpy(), o, "dense after an expired wait")
