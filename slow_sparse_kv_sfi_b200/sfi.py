"""ctypes binding of libsfi.so, the C ABI declared in include/sfi.h.

Argument marshalling only: every function passes device pointers, sizes and
a CUDA stream to the entry point of the same name and turns a non-zero
sfi_status into SFIError.  PyTorch tensors serve as device memory; nothing
here computes.  The library must be built (``python -m
slow_sparse_kv_sfi_b200.build``); loading fails loudly otherwise.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsfi.so")
_lib = None


class SFIError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().sfi_status_str(status).decode() if _lib is not None else str(status)
        super().__init__(f"{where}: {msg} (status {status})")


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libsfi.so is not built ({_LIB_PATH}); run "
                               "`python -m slow_sparse_kv_sfi_b200.build`")
        _lib = C.CDLL(_LIB_PATH)
        _declare(_lib)
    return _lib


class Shape(C.Structure):
    _fields_ = [("B", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32), ("D", C.c_int32),
                ("page_size", C.c_int32), ("max_pages", C.c_int32), ("num_pages", C.c_int32)]


class Params(C.Structure):
    _fields_ = [("n_sink", C.c_int32), ("n_recent", C.c_int32), ("k_fixed", C.c_int32),
                ("budget_frac", C.c_double), ("lam", C.c_float), ("lambda_clip", C.c_float),
                ("alpha_soft", C.c_float), ("alpha_cross", C.c_float),
                ("nms_window", C.c_int32), ("refresh_budget", C.c_int32),
                ("evidence_window", C.c_int32)]


class PagedKV(C.Structure):
    _fields_ = [("k_pool", C.c_void_p), ("v_pool", C.c_void_p), ("page_table", C.c_void_p),
                ("key_norms", C.c_void_p), ("err", C.c_void_p)]


class Packed(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("pos", C.c_void_p),
                ("headmask", C.c_void_p), ("n_rows", C.c_void_p), ("p_max", C.c_int32)]


class DenseExtras(C.Structure):
    _fields_ = [("lse", C.c_void_p), ("logits", C.c_void_p), ("probs", C.c_void_p),
                ("ld", C.c_int64), ("lse_cand", C.c_void_p), ("cand_lo", C.c_int32),
                ("cand_hi", C.c_int32)]


def _declare(L):
    P, I32, I64, SZ = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
    sig = {
        "sfi_status_str": (C.c_char_p, [C.c_int]),
        "sfi_version": (C.c_char_p, []),
        "sfi_workspace_size": (C.c_int, [P, P, C.POINTER(SZ)]),
        "sfi_packed_rows": (C.c_int, [P, P, C.POINTER(I32)]),
        "sfi_budget": (C.c_int, [P, I32, C.POINTER(I32)]),
        "sfi_append_kv": (C.c_int, [P, P, I32, P, P, P]),
        "sfi_key_norms": (C.c_int, [P, P, I32, I32, P]),
        "sfi_dense_attn": (C.c_int, [P, P, I32, P, P, P, P, SZ, P]),
        "sfi_dense_attn_append": (C.c_int, [P, P, I32, P, P, P, P, P, P, SZ, P]),
        "sfi_dense_attn_noalloc": (C.c_int, [P, P, I32, P, P, P, P]),
        "sfi_attn_probs": (C.c_int, [P, I32, P, I64, P, P, P]),
        "sfi_fast_attn": (C.c_int, [P, P, P, I32, P, P, P, P, P, SZ, P]),
        "sfi_fast_attn_append": (C.c_int, [P, P, P, I32, P, P, P, P, P, P, P, SZ, P]),
        "sfi_select_scores": (C.c_int, [P, P, P, I32, P, I64, P, P, P, SZ, P]),
        "sfi_topk_workspace_size": (C.c_int, [I32, I32, C.POINTER(SZ)]),
        "sfi_topk": (C.c_int, [I32, I32, P, I64, I32, I32, P, I64, P, SZ, P]),
        "sfi_select": (C.c_int, [P, P, P, I32, P, I64, P, P, I32, C.POINTER(I32), P, SZ, P]),
        "sfi_compact": (C.c_int, [P, P, P, I32, P, I32, I32, P, P, SZ, P]),
        "sfi_compact_incremental": (C.c_int, [P, P, P, I32, P, I32, I32, P, I32, P, SZ, P]),
        "sfi_poll_error": (C.c_int, [P, C.POINTER(I32)]),
        "sfi_set_wait_limit": (C.c_int, [C.c_int64]),
        "sfi_get_wait_limit": (C.c_int, [C.POINTER(C.c_int64)]),
        "sfi_selftest_wait": (C.c_int, [P, C.c_int64, P]),
        "sfi_ctx_create": (C.c_int, [P, P, I32, I32, C.POINTER(P)]),
        "sfi_ctx_destroy": (C.c_int, [P]),
        "sfi_ctx_workspace_size": (C.c_int, [P, C.POINTER(SZ)]),
        "sfi_ctx_set_workspace": (C.c_int, [P, P, SZ]),
        "sfi_decode_step": (C.c_int, [P, I32, I32, I32, I32, P, P, P, P, P, P, P, C.POINTER(I32)]),
        "sfi_decode_step_rows": (C.c_int, [P, I32, I32, P, I32, P, P, P, P, P, P, P, P]),
        "sfi_ctx_join": (C.c_int, [P, P]),
        "sfi_ctx_set_timing": (C.c_int, [P, I32]),
        "sfi_ctx_set_timing_layers": (C.c_int, [P, I32, I32]),
        "sfi_ctx_set_compaction": (C.c_int, [P, I32]),
        "sfi_ctx_timing": (C.c_int, [P, I32, C.POINTER(C.c_double), C.POINTER(I64), I32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args


EXPORTED = ["sfi_status_str", "sfi_version", "sfi_workspace_size", "sfi_packed_rows", "sfi_budget",
            "sfi_append_kv", "sfi_key_norms", "sfi_dense_attn", "sfi_dense_attn_append",
            "sfi_dense_attn_noalloc", "sfi_attn_probs", "sfi_fast_attn", "sfi_fast_attn_append",
            "sfi_select_scores", "sfi_topk_workspace_size", "sfi_topk", "sfi_select", "sfi_compact",
            "sfi_compact_incremental", "sfi_poll_error", "sfi_set_wait_limit", "sfi_get_wait_limit",
            "sfi_selftest_wait",
            "sfi_ctx_create", "sfi_ctx_destroy", "sfi_ctx_workspace_size", "sfi_ctx_set_workspace",
            "sfi_decode_step", "sfi_decode_step_rows", "sfi_ctx_join", "sfi_ctx_set_timing", "sfi_ctx_set_timing_layers", "sfi_ctx_set_compaction",
            "sfi_ctx_timing"]


def _check(st: int, where: str):
    if st != 0:
        raise SFIError(st, where)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _ref(x):
    return C.byref(x) if x is not None else None


# ---------------------------------------------------------------- structs from tensors
def make_shape(B, Hq, Hkv, D, max_pages, num_pages) -> Shape:
    return Shape(B, Hq, Hkv, D, 16, max_pages, num_pages)


def make_params(n_sink, n_recent, k_fixed, budget_frac, lam, lam_clip, alpha_soft, alpha_cross,
                nms_window, refresh_budget, evidence_window=1) -> Params:
    return Params(n_sink, n_recent, k_fixed, budget_frac, lam, lam_clip, alpha_soft, alpha_cross,
                  nms_window, refresh_budget, evidence_window)


def make_kv(k_pool, v_pool, page_table, key_norms=None, err=None) -> PagedKV:
    return PagedKV(k_pool.data_ptr(), v_pool.data_ptr(), page_table.data_ptr(),
                   None if key_norms is None else key_norms.data_ptr(),
                   None if err is None else err.data_ptr())


def make_packed(k, v, pos, headmask, n_rows) -> Packed:
    return Packed(k.data_ptr(), v.data_ptr(), pos.data_ptr(), headmask.data_ptr(),
                  n_rows.data_ptr(), k.shape[2])


# ---------------------------------------------------------------- entry points
def sfi_version() -> str:
    return lib().sfi_version().decode()


def sfi_workspace_size(shape: Shape, params: Params) -> int:
    n = C.c_size_t(0)
    _check(lib().sfi_workspace_size(C.byref(shape), C.byref(params), C.byref(n)), "sfi_workspace_size")
    return n.value


def sfi_packed_rows(shape: Shape, params: Params) -> int:
    n = C.c_int32(0)
    _check(lib().sfi_packed_rows(C.byref(shape), C.byref(params), C.byref(n)), "sfi_packed_rows")
    return n.value


def sfi_budget(params: Params, L: int) -> int:
    k = C.c_int32(0)
    _check(lib().sfi_budget(C.byref(params), L, C.byref(k)), "sfi_budget")
    return k.value


def sfi_append_kv(shape, kv, L, k_new, v_new, stream=None):
    _check(lib().sfi_append_kv(C.byref(shape), C.byref(kv), L, _p(k_new), _p(v_new), _stream(stream)),
           "sfi_append_kv")


def sfi_key_norms(shape, kv, pos_lo, pos_hi, stream=None):
    _check(lib().sfi_key_norms(C.byref(shape), C.byref(kv), pos_lo, pos_hi, _stream(stream)),
           "sfi_key_norms")


def sfi_dense_attn(shape, kv, L, q, out, ws, extras: Optional[DenseExtras] = None, stream=None):
    _check(lib().sfi_dense_attn(C.byref(shape), C.byref(kv), L, _p(q), _p(out), _ref(extras),
                                _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "sfi_dense_attn")


def sfi_dense_attn_append(shape, kv, L, k_new, v_new, q, out, ws, extras: Optional[DenseExtras] = None,
                          stream=None):
    """sfi_append_kv + sfi_dense_attn in one launch."""
    _check(lib().sfi_dense_attn_append(C.byref(shape), C.byref(kv), L, _p(k_new), _p(v_new), _p(q), _p(out),
                                       _ref(extras), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "sfi_dense_attn_append")


def sfi_dense_attn_noalloc(shape, kv, L, q, out, extras: Optional[DenseExtras] = None, stream=None):
    """sfi_dense_attn with its scratch in the library's static device array
    (no workspace, nothing allocated)."""
    _check(lib().sfi_dense_attn_noalloc(C.byref(shape), C.byref(kv), L, _p(q), _p(out), _ref(extras),
                                        _stream(stream)), "sfi_dense_attn_noalloc")


def sfi_attn_probs(shape, L, logits, ld, lse, probs, stream=None):
    _check(lib().sfi_attn_probs(C.byref(shape), L, _p(logits), ld, _p(lse), _p(probs), _stream(stream)),
           "sfi_attn_probs")


def sfi_fast_attn(shape, params, kv, L, q, packed, out, ws, lse=None, stream=None):
    _check(lib().sfi_fast_attn(C.byref(shape), C.byref(params), C.byref(kv), L, _p(q), C.byref(packed),
                               _p(out), _p(lse), _p(ws), ws.numel() * ws.element_size(),
                               _stream(stream)), "sfi_fast_attn")


def sfi_fast_attn_append(shape, params, kv, L, k_new, v_new, q, packed, out, ws, lse=None, stream=None):
    """sfi_append_kv + sfi_fast_attn in one launch."""
    _check(lib().sfi_fast_attn_append(C.byref(shape), C.byref(params), C.byref(kv), L, _p(k_new), _p(v_new),
                                      _p(q), C.byref(packed), _p(out), _p(lse), _p(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)), "sfi_fast_attn_append")


def sfi_select_scores(shape, params, kv, L, logits, ld, lse_cand, scores, ws, stream=None):
    _check(lib().sfi_select_scores(C.byref(shape), C.byref(params), C.byref(kv), L, _p(logits), ld,
                                   _p(lse_cand), _p(scores), _p(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)), "sfi_select_scores")


def sfi_topk_workspace_size(rows, n) -> int:
    v = C.c_size_t(0)
    _check(lib().sfi_topk_workspace_size(rows, n, C.byref(v)), "sfi_topk_workspace_size")
    return v.value


def sfi_topk(rows, n, scores, ld_s, K, offset, idx, ld_i, ws, stream=None):
    """ws: scratch of sfi_topk_workspace_size(rows, n) bytes (0: none needed; ws may be None)."""
    _check(lib().sfi_topk(rows, n, _p(scores), ld_s, K, offset, _p(idx), ld_i, _p(ws),
                          0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)), "sfi_topk")


def sfi_select(shape, params, kv, L, logits, ld, lse_cand, sel_idx, sel_ld, ws, stream=None) -> int:
    k = C.c_int32(0)
    _check(lib().sfi_select(C.byref(shape), C.byref(params), C.byref(kv), L, _p(logits), ld,
                            _p(lse_cand), _p(sel_idx), sel_ld, C.byref(k), _p(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "sfi_select")
    return k.value


def sfi_compact(shape, params, kv, L, sel_idx, sel_ld, K, packed, ws, stream=None):
    _check(lib().sfi_compact(C.byref(shape), C.byref(params), C.byref(kv), L, _p(sel_idx), sel_ld, K,
                             C.byref(packed), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "sfi_compact")


def sfi_compact_incremental(shape, params, kv, L, sel_idx, sel_ld, K, packed, fresh, ws, stream=None):
    _check(lib().sfi_compact_incremental(C.byref(shape), C.byref(params), C.byref(kv), L, _p(sel_idx), sel_ld, K,
                                         C.byref(packed), int(fresh), _p(ws), ws.numel() * ws.element_size(),
                                         _stream(stream)), "sfi_compact_incremental")


def sfi_poll_error(kv) -> int:
    code = C.c_int32(0)
    _check(lib().sfi_poll_error(C.byref(kv), C.byref(code)), "sfi_poll_error")
    return code.value


def sfi_set_wait_limit(ns: int):
    _check(lib().sfi_set_wait_limit(int(ns)), "sfi_set_wait_limit")


def sfi_get_wait_limit() -> int:
    v = C.c_int64(0)
    _check(lib().sfi_get_wait_limit(C.byref(v)), "sfi_get_wait_limit")
    return v.value


def sfi_selftest_wait(kv, limit_ns: int, stream=None):
    _check(lib().sfi_selftest_wait(C.byref(kv), int(limit_ns), _stream(stream)), "sfi_selftest_wait")


class Context:
    """Owns an sfi_ctx (side stream, per-layer events) and its workspace tensor."""

    def __init__(self, shape: Shape, params: Params, n_layers: int, overlap: bool = True,
                 device=None, incremental: bool = True):
        self.shape, self.params = shape, params
        h = C.c_void_p()
        _check(lib().sfi_ctx_create(C.byref(shape), C.byref(params), n_layers, int(overlap),
                                    C.byref(h)), "sfi_ctx_create")
        self.h = h
        n = C.c_size_t(0)
        _check(lib().sfi_ctx_workspace_size(h, C.byref(n)), "sfi_ctx_workspace_size")
        self.ws = torch.empty(n.value, dtype=torch.uint8, device=device or "cuda")
        _check(lib().sfi_ctx_set_workspace(h, _p(self.ws), n.value), "sfi_ctx_set_workspace")
        _check(lib().sfi_ctx_set_compaction(h, int(incremental)), "sfi_ctx_set_compaction")
        self._slow = C.c_int32(0)

    def decode_step(self, layer, step, boundary_prev, L, kv, packed, q, k_new, v_new, out,
                    stream=None) -> bool:
        slow = C.c_int32(0)
        _check(lib().sfi_decode_step(self.h, layer, step, int(boundary_prev), L, C.byref(kv),
                                     C.byref(packed), _p(q), _p(k_new), _p(v_new), _p(out),
                                     _stream(stream), C.byref(slow)), "sfi_decode_step")
        return bool(slow.value)

    def decode_step_rows(self, layer, step, boundary_prev, L, kv, packed, q, k_new, v_new, out,
                         stream=None):
        """One layer-step with a trigger per sequence; boundary_prev: B flags
        (or None).  Returns the per-sequence slow decisions."""
        B = self.shape.B
        bnd = None
        if boundary_prev is not None:
            bnd = (C.c_int32 * B)(*[int(x) for x in boundary_prev])
        slow = (C.c_int32 * B)()
        _check(lib().sfi_decode_step_rows(self.h, layer, step, bnd, L, C.byref(kv), C.byref(packed), _p(q),
                                          _p(k_new), _p(v_new), _p(out), _stream(stream), slow),
               "sfi_decode_step_rows")
        return [bool(x) for x in slow]

    def decode_step_ptr(self, layer, step, boundary_prev, L, kv_ref, packed_ref, q, k_new, v_new, out,
                        stream) -> bool:
        """decode_step with raw device addresses (ints), C.byref(...) of the
        cache and packed structs and a raw stream handle: no tensor
        marshalling, for drivers that issue many layer-steps."""
        st = lib().sfi_decode_step(self.h, layer, step, boundary_prev, L, kv_ref, packed_ref, q, k_new, v_new, out,
                                   stream, C.byref(self._slow))
        if st != 0:
            raise SFIError(st, "sfi_decode_step")
        return bool(self._slow.value)

    def join(self, stream=None):
        _check(lib().sfi_ctx_join(self.h, _stream(stream)), "sfi_ctx_join")

    def set_timing(self, layer_stride: int, first_layer: int = 0):
        """Time the attention launches of layers first, first + n, ... (n = layer_stride; 0 = off)."""
        _check(lib().sfi_ctx_set_timing_layers(self.h, int(first_layer), int(layer_stride)),
               "sfi_ctx_set_timing_layers")

    def timing(self, kind: int, reset: bool = True):
        ms = C.c_double(0)
        n = C.c_int64(0)
        _check(lib().sfi_ctx_timing(self.h, kind, C.byref(ms), C.byref(n), int(reset)), "sfi_ctx_timing")
        return ms.value, n.value

    def close(self):
        if getattr(self, "h", None):
            lib().sfi_ctx_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
