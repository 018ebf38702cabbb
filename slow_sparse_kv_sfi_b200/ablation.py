"""Selector ablation sweep on the synthetic workloads.

    python -m slow_sparse_kv_sfi_b200.ablation [--config NAME] [--steps T] [--settings I,J,...]

The pages' ablations vary the fusion weight λ, its clamp λ_clip and the
soft-NMS / cross-head refinements (Slow-Fast Inference, gist.science/zh,
§4 Results; the quality benchmarks they report are out of scope here).  This
driver measures, for each setting, what the Selector's choices do to the
attention itself, with the decode path's own kernels:

* support recall: at every fast step, the share of the dense attention
  distribution over the whole context (the slow-step kernel's f at that
  step's L) that falls on the head's sparse set S_h = sink ∪ selected ∪ recent
  (1.0 means the fast step attends exactly what dense attention would), also
  relative to the mass a selection at the last slow step could reach at all
  (tokens that left the recent window since then are in no set);
* selection stability: at every slow step after the first, the share of each
  head's K selected positions that the previous slow step had selected too.

Every number comes from the library (`sfi_decode_step` for the decode,
`sfi_dense_attn` + probabilities for f); torch only gathers and sums them.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
from typing import Dict, List

import torch

from . import sfi as S
from . import workload as W
from .state import alloc_layer, params_of, shape_of

# (name, overrides of the workload's Selector settings)
SETTINGS = [
    ("default (lambda 0.2)", {}),
    ("evidence only (lambda 0)", {"lam": 0.0}),
    ("lambda 0.5", {"lam": 0.5, "lam_clip": 1.0}),
    ("prior only (lambda 1)", {"lam": 1.0, "lam_clip": 1.0}),
    ("lambda 0.8 clipped at 0.5", {"lam": 0.8, "lam_clip": 0.5}),
    ("no soft-NMS", {"alpha_soft": 0.0}),
    ("no cross-head exclusivity", {"alpha_cross": 0.0}),
    ("no refinements", {"alpha_soft": 0.0, "alpha_cross": 0.0}),
]


def _sets_mask(layer, cfg: W.SFIConfig, L: int) -> torch.Tensor:
    """bool [B, Hq, L]: S_h of every head from the packed buffer plus sink and recent."""
    B, Hq, Hkv, G = cfg.B, cfg.Hq, cfg.Hkv, cfg.G
    mask = torch.zeros(B, Hq, L, dtype=torch.bool, device=layer.pos.device)
    mask[:, :, : cfg.n_sink] = True
    mask[:, :, max(L - cfg.n_recent, 0):] = True
    n = layer.n_rows.long()
    for b in range(B):
        for g in range(Hkv):
            rows = int(n[b, g])
            pos = layer.pos[b, g, :rows].long()
            hm = layer.headmask[b, g, :rows].long() & 0xFFFFFFFF
            for h in range(G):
                sel = pos[((hm >> h) & 1) == 1]
                mask[b, g * G + h, sel] = True
    return mask


def _selected(layer, cfg: W.SFIConfig) -> List[set]:
    """Per (b, head): the selected candidate positions (sinks removed)."""
    out = []
    n = layer.n_rows.cpu()
    pos = layer.pos.cpu()
    hm = layer.headmask.cpu().long() & 0xFFFFFFFF
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            rows = int(n[b, g])
            p = pos[b, g, :rows]
            m = hm[b, g, :rows]
            for h in range(cfg.G):
                sel = p[((m >> h) & 1) == 1]
                out.append(set(int(x) for x in sel if int(x) >= cfg.n_sink))
    return out


def run_setting(cfg: W.SFIConfig, device, detail: bool = False) -> Dict[str, float]:
    """Decodes one layer of cfg and returns the sweep's measurements; with
    detail, also every fast step's recall per (sequence, query head) and every
    slow step's stability per (sequence, query head), keyed by step."""
    shape, params = shape_of(cfg), params_of(cfg)
    li = W.make_layer(cfg, 0, device)
    layer = alloc_layer(cfg, li, device)
    ctx = S.Context(shape, params, 1, overlap=False, device=device)
    ws = torch.zeros(S.sfi_workspace_size(shape, params), dtype=torch.uint8, device=device)
    boundary = W.boundary_stream(cfg)
    out = torch.empty(cfg.B, cfg.Hq, cfg.D, device=device)
    dense_out = torch.empty_like(out)
    ld = cfg.capacity
    probs = torch.empty(cfg.B, cfg.Hq, ld, device=device)
    lse = torch.empty(cfg.B, cfg.Hq, device=device)
    recalls, reach, overlaps = [], [], []
    per_step_recall, per_step_stability = {}, {}
    prev = None
    n_slow = 0
    L_slow = cfg.seq_len(0)
    for t in range(cfg.steps):
        L = cfg.seq_len(t)
        slow = ctx.decode_step(0, t, int(boundary[t - 1]) if t > 0 else 0, L, layer.kv, layer.packed,
                               li.q[t], li.k_new[t], li.v_new[t], out)
        ctx.join()
        if slow:
            n_slow += 1
            L_slow = L
            cur = _selected(layer, cfg)
            if prev is not None:
                st = [len(a & b) / max(len(a), 1) for a, b in zip(cur, prev)]
                overlaps.extend(st)
                per_step_stability[t] = st
            prev = cur
            continue
        ex = S.DenseExtras(lse.data_ptr(), None, probs.data_ptr(), ld, None, 0, 0)
        S.sfi_dense_attn(shape, layer.kv, L, li.q[t], dense_out, ws, ex)
        mask = _sets_mask(layer, cfg, L)
        f = probs[:, :, :L]
        r = (f * mask).sum(dim=2)                        # [B, Hq]
        # what any selection made at the last slow step could reach: sink,
        # that step's candidates, this step's recent window
        cover = torch.zeros(L, dtype=torch.bool, device=device)
        cover[: max(L_slow - cfg.n_recent, 0)] = True
        cover[max(L - cfg.n_recent, 0):] = True
        recalls.append(r.flatten())
        if detail:
            per_step_recall[t] = r.flatten().cpu().tolist()
        reach.append((r / (f * cover).sum(dim=2)).flatten())
    torch.cuda.synchronize()
    assert S.sfi_poll_error(layer.kv) == 0
    ctx.close()
    rec = torch.cat(recalls) if recalls else torch.zeros(1, device=device)
    rea = torch.cat(reach) if reach else torch.zeros(1, device=device)
    res = {
        "fast_steps": len(recalls), "slow_steps": n_slow,
        "recall_mean": float(rec.mean()), "recall_p10": float(rec.quantile(0.10)), "recall_min": float(rec.min()),
        "recall_of_reachable_mean": float(rea.mean()), "recall_of_reachable_min": float(rea.min()),
        "stability_mean": float(sum(overlaps) / len(overlaps)) if overlaps else float("nan"),
    }
    if detail:
        res["recall_steps"] = per_step_recall
        res["stability_steps"] = per_step_stability
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="qwen3-0.6b-8k")
    ap.add_argument("--steps", type=int, default=96)
    ap.add_argument("--settings", default="all", help="comma-separated indices into SETTINGS, or all")
    args = ap.parse_args()
    base = W.CONFIG_BY_NAME[args.config].replace(n_layers=1, steps=args.steps)
    idx = range(len(SETTINGS)) if args.settings == "all" else [int(i) for i in args.settings.split(",")]
    dev = torch.device("cuda")
    for i in idx:
        name, over = SETTINGS[i]
        cfg = dataclasses.replace(base, **over)
        res = run_setting(cfg, dev)
        print(json.dumps({"workload": base.name, "setting": name, **over, "lambda": cfg.lam,
                          "lambda_clip": cfg.lam_clip, "alpha_soft": cfg.alpha_soft,
                          "alpha_cross": cfg.alpha_cross, **res}), flush=True)


if __name__ == "__main__":
    main()
