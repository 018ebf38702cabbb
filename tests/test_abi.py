"""The C-ABI library loads and exports every entry point include/sfi.h
declares; host-side argument checks answer without touching a GPU."""
import ctypes as C
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "sfi.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sfi_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def S():
    from slow_sparse_kv_sfi_b200 import build, sfi
    build.build()
    return sfi


def test_every_declared_symbol_is_exported(S):
    lib = S.lib()
    names = _declared()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(S.EXPORTED)


def test_version_and_status_strings(S):
    assert "sm_100a" in S.sfi_version()
    lib = S.lib()
    for code in range(8):
        assert lib.sfi_status_str(code)
    assert lib.sfi_status_str(99) == b"unknown status"


def test_budget_rule_host(S):
    p = S.make_params(4, 64, 128, 0.2, 0.2, 0.5, 0.5, 0.5, 32, 8)
    assert S.sfi_budget(p, 1025) == 128
    p = S.make_params(4, 128, 0, 0.2, 0.2, 0.5, 0.5, 0.5, 32, 32)
    assert S.sfi_budget(p, 8193) == int(0.2 * 8193)
    assert S.sfi_budget(p, 200) == 40
    p = S.make_params(4, 128, 0, 0.9, 0.2, 0.5, 0.5, 0.5, 32, 32)
    assert S.sfi_budget(p, 200) == 200 - 128 - 4          # clamped to |C|
    with pytest.raises(S.SFIError):
        S.sfi_budget(p, 132)          # |C| = 0


def test_packed_rows_capacity(S):
    from slow_sparse_kv_sfi_b200.state import shape_of, params_of
    from slow_sparse_kv_sfi_b200 import workload as W
    cfg = W.CONFIGS[0]
    rows = S.sfi_packed_rows(shape_of(cfg), params_of(cfg))
    nC = cfg.capacity - cfg.n_recent - cfg.n_sink
    assert rows % 64 == 0
    assert rows >= cfg.n_sink + min(cfg.G * 128, nC)
    assert rows - 64 < cfg.n_sink + min(cfg.G * 128, nC)


@pytest.mark.parametrize("field,value,code", [
    ("D", 96, 3), ("Hkv", 3, 2), ("page_size", 32, 3), ("B", 0, 2), ("Hq", 64, 3)])
def test_shape_validation(S, field, value, code):
    sh = S.make_shape(1, 4, 2, 64, 10, 10)
    setattr(sh, field, value)
    p = S.make_params(4, 64, 128, 0.2, 0.2, 0.5, 0.5, 0.5, 32, 8)
    n = C.c_size_t()
    assert S.lib().sfi_workspace_size(C.byref(sh), C.byref(p), C.byref(n)) == code


def test_null_pointers_rejected_before_any_launch(S):
    sh = S.make_shape(1, 4, 2, 64, 10, 10)
    p = S.make_params(4, 64, 128, 0.2, 0.2, 0.5, 0.5, 0.5, 32, 8)
    kv = S.PagedKV(None, None, None, None, None)
    lib = S.lib()
    assert lib.sfi_dense_attn(C.byref(sh), C.byref(kv), 100, None, None, None, None, 0, None) == 1
    assert lib.sfi_append_kv(C.byref(sh), C.byref(kv), 100, None, None, None) == 1
    assert lib.sfi_topk(4, 10, None, 10, 3, 0, None, 3, None, 0, None) == 1
    # misaligned pool pointer
    kv = S.PagedKV(8, 16, 16, 16, None)
    assert lib.sfi_key_norms(C.byref(sh), C.byref(kv), 0, 10, None) == 1
    # context longer than the cache
    kv = S.PagedKV(16, 16, 16, 16, None)
    assert lib.sfi_append_kv(C.byref(sh), C.byref(kv), 161, 16, 16, None) == 2
    assert lib.sfi_topk(4, 10, 16, 10, 11, 0, 16, 11, 16, 1 << 20, None) == 2   # K > n
    # the top-K keeps its state on chip: it reports no scratch
    need = C.c_size_t(1)
    assert lib.sfi_topk_workspace_size(4, 10, C.byref(need)) == 0 and need.value == 0
    assert lib.sfi_topk(70000, 10, 16, 10, 3, 0, 16, 3, None, 0, None) == 3
    assert lib.sfi_ctx_set_workspace(None, None, 0) == 1
    # wait limits outside their range, a self-test without an error word
    assert lib.sfi_set_wait_limit(10) == 1 and lib.sfi_set_wait_limit(10 ** 12) == 1
    got = C.c_int64(0)
    assert lib.sfi_get_wait_limit(C.byref(got)) == 0 and got.value == 2_000_000_000
    assert lib.sfi_selftest_wait(C.byref(S.PagedKV(None, None, None, None, None)), 50_000, None) == 1


def test_context_rejects_bad_calls(S):
    sh = S.make_shape(1, 4, 2, 64, 10, 10)
    p = S.make_params(4, 64, 128, 0.2, 0.2, 0.5, 0.5, 0.5, 32, 8)
    h = C.c_void_p()
    st = S.lib().sfi_ctx_create(C.byref(sh), C.byref(p), 0, 1, C.byref(h))
    assert st == 1
    # kernel timing: no context, a negative stride or first layer
    lib = S.lib()
    assert lib.sfi_ctx_set_timing(None, 1) == 1
    assert lib.sfi_ctx_set_timing_layers(None, 0, 1) == 1


@pytest.mark.parametrize("window,code", [(0, 0), (1, 0), (4, 0), (33, 1), (65, 1), (-1, 1)])
def test_evidence_window_validation(S, window, code):
    """W in [0, 32] (0 and 1: the slow step's query alone) and W <= n_recent."""
    sh = S.make_shape(1, 4, 2, 64, 10, 10)
    p = S.make_params(4, 64, 128, 0.2, 0.2, 0.5, 0.5, 0.5, 32, 8, window)
    n = C.c_size_t()
    assert S.lib().sfi_workspace_size(C.byref(sh), C.byref(p), C.byref(n)) == code


def test_new_entry_points_reject_bad_arguments(S):
    sh = S.make_shape(1, 4, 2, 64, 10, 10)
    p = S.make_params(4, 64, 128, 0.2, 0.2, 0.5, 0.5, 0.5, 32, 8)
    kv = S.PagedKV(16, 16, 16, 16, None)
    lib = S.lib()
    # incremental compaction: no packed buffer / no selection
    assert lib.sfi_compact_incremental(C.byref(sh), C.byref(p), C.byref(kv), 100, None, 3, 3, None, 0, None, 0,
                                       None) == 1
    pk = S.Packed(16, 16, 16, 16, 16, 64)
    assert lib.sfi_compact_incremental(C.byref(sh), C.byref(p), C.byref(kv), 100, None, 3, 3, C.byref(pk), 0,
                                       None, 0, None) == 1
    # a packed buffer below the row capacity is refused (the refresh keeps slots up to it)
    cap = S.sfi_packed_rows(sh, p)
    if cap > 64:
        assert lib.sfi_compact_incremental(C.byref(sh), C.byref(p), C.byref(kv), 100, 16, 3, 3, C.byref(pk), 0,
                                           None, 0, None) == 2
    # the driver's per-sequence step and compaction switch without a context
    assert lib.sfi_decode_step_rows(None, 0, 0, None, 100, None, None, None, None, None, None, None, None) == 7
    assert lib.sfi_ctx_set_compaction(None, 1) == 1


def test_noalloc_rejects_bad_arguments_like_the_workspace_call(S):
    """sfi_dense_attn_noalloc shares sfi_dense_attn's argument checks: every
    refusal below happens on the host, before the scratch address is looked up
    or anything is launched, with the status sfi_dense_attn returns."""
    lib = S.lib()
    f = lib.sfi_dense_attn_noalloc
    sh = S.make_shape(1, 4, 2, 64, 10, 10)
    kv = S.PagedKV(16, 16, 16, None, None)
    cases = [
        (None, kv, 100, 16, 16, None, 1),                          # no shape
        (sh, None, 100, 16, 16, None, 1),                          # no cache
        (sh, kv, 100, None, 16, None, 1),                          # no query
        (sh, kv, 100, 16, None, None, 1),                          # no output
        (sh, kv, 100, 24, 16, None, 1),                            # query not 16-byte aligned
        (sh, S.PagedKV(8, 16, 16, None, None), 100, 16, 16, None, 1),   # pool not aligned
        (sh, kv, 161, 16, 16, None, 2),                            # longer than the cache
        (S.make_shape(1, 34, 1, 64, 10, 10), kv, 100, 16, 16, None, 2),  # G > 32
        (S.make_shape(1, 32, 1, 64, 10, 10), kv, 100, 16, 16, None, 3),  # G = 32 > 16
        (S.make_shape(1, 4, 2, 96, 10, 10), kv, 100, 16, 16, None, 3),   # D not 64 / 128
        (sh, kv, 100, 16, 16, S.DenseExtras(None, 16, None, 50, None, 0, 0), 2),          # ld < L
        (sh, kv, 100, 16, 16, S.DenseExtras(None, None, None, 0, 16, 60, 40), 2),         # empty candidate range
        (sh, kv, 100, 16, 16, S.DenseExtras(None, None, 16, 100, None, 0, 0), 1),         # probs without lse
    ]
    for shape, kvv, L, q, out, extras, code in cases:
        args = [None if shape is None else C.byref(shape), None if kvv is None else C.byref(kvv), L, q, out,
                None if extras is None else C.byref(extras), None]
        assert f(*args) == code, (shape, L, q, out, code)
        wsargs = args[:6] + [16, 1 << 20, None]
        assert lib.sfi_dense_attn(*wsargs) == code
