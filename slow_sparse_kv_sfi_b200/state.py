"""Device-side state of one attention layer for the SFI decode path.

Plumbing only: allocates the paged cache, page table, key-norm cache, packed
buffer and error word as torch tensors and wraps them in the C structs of
include/sfi.h.  The kernels do all of the work.
"""
from __future__ import annotations

import dataclasses

import torch

from . import sfi as S
from .workload import SFIConfig, LayerInputs


def shape_of(cfg: SFIConfig) -> S.Shape:
    return S.make_shape(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.pages_per_seq, cfg.num_pages)


def params_of(cfg: SFIConfig) -> S.Params:
    return S.make_params(cfg.n_sink, cfg.n_recent, cfg.k_fixed, cfg.budget_frac, cfg.lam,
                         cfg.lam_clip, cfg.alpha_soft, cfg.alpha_cross, cfg.nms_window,
                         cfg.refresh_budget, cfg.evidence_window)


@dataclasses.dataclass
class DeviceLayer:
    cfg: SFIConfig
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    page_table: torch.Tensor
    key_norms: torch.Tensor
    err: torch.Tensor
    pk: torch.Tensor
    pv: torch.Tensor
    pos: torch.Tensor
    headmask: torch.Tensor
    n_rows: torch.Tensor
    kv: S.PagedKV = None
    packed: S.Packed = None

    def __post_init__(self):
        self.kv = S.make_kv(self.k_pool, self.v_pool, self.page_table, self.key_norms, self.err)
        self.packed = S.make_packed(self.pk, self.pv, self.pos, self.headmask, self.n_rows)


def alloc_layer(cfg: SFIConfig, inputs: LayerInputs, device="cuda", p_max: int = None,
                with_norms: bool = True) -> DeviceLayer:
    """Copies one layer's cache to the device, allocates its packed buffer and
    fills the key-norm cache of the prefilled positions (sfi_key_norms)."""
    dev = torch.device(device)
    shape, params = shape_of(cfg), params_of(cfg)
    if p_max is None:
        p_max = S.sfi_packed_rows(shape, params)
    kp = inputs.k_pool.to(dev).contiguous()
    vp = inputs.v_pool.to(dev).contiguous()
    pt = inputs.page_table.to(dev, torch.int32).contiguous()
    norms = torch.zeros(cfg.B, cfg.Hkv, cfg.capacity, dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pk = torch.zeros(cfg.B, cfg.Hkv, p_max, cfg.D, dtype=torch.bfloat16, device=dev)
    pv = torch.zeros_like(pk)
    pos = torch.full((cfg.B, cfg.Hkv, p_max), -1, dtype=torch.int32, device=dev)
    hm = torch.zeros(cfg.B, cfg.Hkv, p_max, dtype=torch.int32, device=dev)
    nr = torch.zeros(cfg.B, cfg.Hkv, dtype=torch.int32, device=dev)
    layer = DeviceLayer(cfg, kp, vp, pt, norms, err, pk, pv, pos, hm, nr)
    if with_norms:
        S.sfi_key_norms(shape, layer.kv, 0, cfg.context)
    return layer
