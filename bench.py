"""Benchmark of the SFI decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl sfi|reference]

One bench *step* is one complete decode run of the workload: every decode
step of the configured trigger schedule (slow and fast) through every layer,
i.e. all rows of the hot path (append + key norm, trigger, dense slow-step
attention with logits, Selector scoring and top-K, compaction, fast
attention over packed + recent, side-stream overlap).  The default workload is
the 128K-context, 36-layer Qwen3-4B-shaped configuration: B=2, 32 query / 8
KV heads, D=128, 131072 cached tokens, 256 decode steps, budget 15 %, sink 4,
recent 256, Bernoulli(1/16) boundary trigger with refresh budget 32.

value = decode tok/s per attention layer = B * decode_steps * layers / time,
inputs resident in HBM (the 38.7 GB cache is far larger than L2, so no L2
flush is needed).  Also reported: the same run through host buffers (e2e),
the in-house dense full-KV decode on the same cache, the roofline of the
dominant kernel, and the CPU oracle on a bounded sample.

--impl reference times the CPU oracle on the same workload (the reference
arm of this repository).  With N > 1 GPUs (torchrun) every rank runs an
independent replica; the decode path has no cross-GPU exchange.
"""
from __future__ import annotations

import argparse
import ctypes as C
import hashlib
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from slow_sparse_kv_sfi_b200 import sfi as S                      # noqa: E402
from slow_sparse_kv_sfi_b200 import workload as W                 # noqa: E402
from slow_sparse_kv_sfi_b200.state import alloc_layer, params_of, shape_of   # noqa: E402

METRIC = "decode tok/s per attn layer (fast/slow mix) vs dense full-KV; % of HBM roofline"
UNIT = "tok/s per attn layer"
DEFAULT_CONFIG = "qwen3-4b-128k-36l"
# The attention launches of one layer in the middle of the stack are bracketed
# by CUDA events in the timed region.  An event between two launches stops the
# second from overlapping the first, so one layer per step is sampled.  Layer
# 0 is not: it follows the step's own event, and its launch gap after two
# events would be counted as kernel time.
def timed_layer(n_layers):
    return n_layers // 2


# With a single layer the sampled layer is every launch; there only every
# TIMED_STEP_STRIDE-th step is sampled, so that the events slow the run little.
TIMED_STEP_STRIDE = 8


def timed_step_stride(n_layers):
    return 1 if n_layers > 1 else TIMED_STEP_STRIDE


# ---------------------------------------------------------------- helpers
def peaks():
    """HBM peak in GB/s: the measured copy bandwidth of MEASURED_PEAKS.json,
    else the fallback 6650 GB/s (also when the file cannot be read)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            v = float(json.load(fh)["hbm_gbs"])
        if v > 0:
            return v, "measured"
    except (OSError, ValueError, KeyError, TypeError):
        pass
    return 6650.0, "fallback"


def kernel_traffic(kind: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the counters were taken or the summary was
    taken on another workload."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh)
    if d.get("workload") != workload:
        return None
    src = open(os.path.join(ROOT, "slow_sparse_kv_sfi_b200", "csrc", "attn.cu"), "rb").read()
    if d.get("attn_cu_sha256") != hashlib.sha256(src).hexdigest():
        return None
    e = d.get(kind)
    return None if e is None else float(e)


class Clocks:
    """nvidia-smi sampler for the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None
        self.fh = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix=f"sfi_clocks_rank{self.index}_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            if self.fh is not None:
                self.fh.close()
            if self.path:
                os.unlink(self.path)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as fh:
            lines = fh.readlines()
        os.unlink(self.path)
        return clock_summary(lines)


def clock_summary(lines):
    """Median SM clock under load, the maximum clock and the throttle reasons
    seen, from nvidia-smi samples (csv, no header, no units) of the query in
    `Clocks.Q`."""
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in lines:
        f = [x.strip() for x in line.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            smax.append(float(f[2]))
        except ValueError:
            continue
        for n, v in zip(names, f[5:9]):
            if v.lower().startswith("active"):
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    busy = [x for x in sm if x > 0.5 * max(sm)] or sm
    return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
            "samples": len(sm)}


# ---------------------------------------------------------------- the workload on the device
class Bench:
    def __init__(self, cfg: W.SFIConfig, device):
        self.cfg = cfg
        self.dev = device
        self.shape, self.params = shape_of(cfg), params_of(cfg)
        self.boundary = W.boundary_stream(cfg)
        self.layers, self.inputs = [], []
        for l in range(cfg.n_layers):
            li = W.make_layer(cfg, l, device, boundary=self.boundary)
            self.layers.append(alloc_layer(cfg, li, device))
            self.inputs.append(li)
        # per-step inputs stacked by step: [T, layers, ...]
        self.q = torch.stack([li.q for li in self.inputs], dim=1).contiguous()
        self.kn = torch.stack([li.k_new for li in self.inputs], dim=1).contiguous()
        self.vn = torch.stack([li.v_new for li in self.inputs], dim=1).contiguous()
        for li in self.inputs:
            li.q = li.k_new = li.v_new = None
        self.out = torch.empty(cfg.n_layers, cfg.B, cfg.Hq, cfg.D, device=device)
        self.ctx = S.Context(self.shape, self.params, cfg.n_layers, overlap=True, device=device)
        self.ws = torch.zeros(S.sfi_workspace_size(self.shape, self.params), dtype=torch.uint8, device=device)
        torch.cuda.synchronize()

    def run_sfi(self, step_events=None, probe=None, q=None, kn=None, vn=None, out=None, timing=False):
        """One decode run.  timing: the attention launches of the sampled layer
        are event-timed on the sampled steps (`timed_layer`, `timed_step_stride`)."""
        cfg = self.cfg
        q = self.q if q is None else q
        kn = self.kn if kn is None else kn
        vn = self.vn if vn is None else vn
        out = self.out if out is None else out
        slows = []
        # raw addresses of every (step, layer) slice: [T, layers, ...] contiguous
        NL = len(self.layers)
        qb, qs = q.data_ptr(), q[0, 0].numel() * q.element_size()
        kb, ks = kn.data_ptr(), kn[0, 0].numel() * kn.element_size()
        vb, vs = vn.data_ptr(), vn[0, 0].numel() * vn.element_size()
        ob, os_ = out.data_ptr(), out[0].numel() * out.element_size()
        refs = [(C.byref(layer.kv), C.byref(layer.packed)) for layer in self.layers]
        stream = torch.cuda.current_stream().cuda_stream
        step_fn = self.ctx.decode_step_ptr
        every = timed_step_stride(NL)
        for t in range(cfg.steps):
            L = cfg.seq_len(t)
            bprev = int(self.boundary[t - 1]) if t > 0 else 0
            slow = False
            if timing and every > 1:
                self.ctx.set_timing(NL if t % every == 0 else 0, first_layer=timed_layer(NL))
            for l in range(NL):
                i = t * NL + l
                slow = step_fn(l, t, bprev, L, refs[l][0], refs[l][1], qb + i * qs, kb + i * ks, vb + i * vs,
                               ob + l * os_, stream)
            slows.append(slow)
            if step_events is not None:
                step_events[t].record()
            if probe is not None and slow:
                self.ctx.join()
                probe[t] = [layer.n_rows.clone() for layer in self.layers]
        self.ctx.join()
        return slows

    def run_dense(self):
        cfg = self.cfg
        for t in range(cfg.steps):
            L = cfg.seq_len(t)
            for l, layer in enumerate(self.layers):
                S.sfi_dense_attn_append(self.shape, layer.kv, L, self.kn[t, l], self.vn[t, l], self.q[t, l],
                                        self.out[l], self.ws)

    def run_e2e(self, host_in, host_out, dq, dk, dv, din, dout, copy_stream, evs):
        """Every decode step copies that step's inputs (q, k and v of all
        layers, packed in one pinned host row per step) from host memory and
        reads all layers' outputs back.  The copies run on a second stream
        into two device buffers: step t + 1's inputs arrive and step t's
        outputs leave while the next step computes."""
        cfg = self.cfg
        NL = len(self.layers)
        T = cfg.steps
        qs, ks, vs = (dq[0, 0].numel() * dq.element_size(), dk[0, 0].numel() * dk.element_size(),
                      dv[0, 0].numel() * dv.element_size())
        os_ = dout[0, 0].numel() * dout.element_size()
        refs = [(C.byref(layer.kv), C.byref(layer.packed)) for layer in self.layers]
        main = torch.cuda.current_stream()
        stream = main.cuda_stream
        step_fn = self.ctx.decode_step_ptr
        ev_in, ev_done, ev_read = evs

        def fetch(t, b):   # on the copy stream: one copy per step
            din[b].copy_(host_in[t], non_blocking=True)
            ev_in[b].record(copy_stream)

        copy_stream.wait_stream(main)
        with torch.cuda.stream(copy_stream):
            fetch(0, 0)
        for t in range(T):
            b = t % 2
            if t + 1 < T:
                with torch.cuda.stream(copy_stream):
                    if t >= 1:
                        copy_stream.wait_event(ev_done[1 - b])   # step t - 1 is done with buffer 1 - b
                    fetch(t + 1, 1 - b)
            main.wait_event(ev_in[b])
            if t >= 2:
                main.wait_event(ev_read[b])   # step t - 2's outputs have left buffer b
            L = cfg.seq_len(t)
            bprev = int(self.boundary[t - 1]) if t > 0 else 0
            qb, kb, vb, ob = dq[b].data_ptr(), dk[b].data_ptr(), dv[b].data_ptr(), dout[b].data_ptr()
            for l in range(NL):
                step_fn(l, t, bprev, L, refs[l][0], refs[l][1], qb + l * qs, kb + l * ks, vb + l * vs,
                        ob + l * os_, stream)
            ev_done[b].record(main)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(ev_done[b])
                host_out[t].copy_(dout[b], non_blocking=True)
                ev_read[b].record(copy_stream)
        main.wait_stream(copy_stream)   # every output is on the host before the region ends
        self.ctx.join()


def _sync_barrier(dist_on):
    """Device idle on every rank, then all ranks meet."""
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    if dist_on:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def _max_over_ranks(x, dist_on):
    """The largest x over all ranks (the slowest rank's time)."""
    if not dist_on:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world, units_per_rank_run, runs, seconds):
    """Whole-job throughput: every rank (replica) processed units_per_rank_run
    per run, `runs` runs took `seconds` on the slowest rank."""
    return world * units_per_rank_run * runs / seconds


def _timed(fn, K, dist_on):
    _sync_barrier(dist_on)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K):
        fn()
    e1.record()
    _sync_barrier(dist_on)
    return _max_over_ranks(e0.elapsed_time(e1) / 1000.0, dist_on)


# ---------------------------------------------------------------- CPU oracle sample
def _group_rows(layer_or_li, b, g, L, device_tensors=True):
    pool_k, pool_v, pt = layer_or_li.k_pool, layer_or_li.v_pool, layer_or_li.page_table
    pages = pt[b, : (L + 15) // 16].long()
    sub_k = pool_k[pages][:, g:g + 1].float().cpu().numpy()
    sub_v = pool_v[pages][:, g:g + 1].float().cpu().numpy()
    sub_pt = np.arange(len(pages), dtype=np.int64)[None, :]
    return sub_k, sub_v, sub_pt


def host_cores():
    """CPU threads this process may run on (its affinity), and the machine's count."""
    try:
        aff = len(os.sched_getaffinity(0))
    except AttributeError:
        aff = os.cpu_count() or 1
    return aff, os.cpu_count() or aff


FAST_SAMPLE = 8     # fast layer-steps per sampled group


def oracle_sample(cfg, layer, q_t, slow_frac, budget_s=20.0):
    """Times the CPU oracle, as it stands, on one slow layer-step (dense
    attention + Selector) and FAST_SAMPLE fast layer-steps (sparse attention
    over the slow step's sets) of layer 0, group by group until about
    budget_s seconds are spent, and scales to all (sequence, KV head) groups.
    Returns tok/s per attention layer for the run's slow/fast mix, the
    seconds spent, the groups sampled, the groups in all, and the seconds per
    slow and per fast layer-step."""
    from oracle import sfi_oracle as O
    G = cfg.G
    L = cfg.seq_len(0)
    groups = [(b, g) for b in range(cfg.B) for g in range(cfg.Hkv)]
    qh = q_t.float().cpu().numpy().astype(np.float64)
    t_slow = t_fast = 0.0
    done = 0
    for (b, g) in groups:
        sk, sv, spt = _group_rows(layer, b, g, L)
        qg = qh[b, g * G:(g + 1) * G]
        t0 = time.perf_counter()
        K = O.gather_cache(sk, spt, 0, 0, L)
        V = O.gather_cache(sv, spt, 0, 0, L)
        _, f, _, _ = O.dense_attention(qg, K, V)
        sel = O.select(f, O.key_norms(K), L, cfg.n_sink, cfg.n_recent, cfg.k_fixed, cfg.budget_frac, cfg.lam,
                       cfg.lam_clip, cfg.alpha_soft, cfg.alpha_cross, cfg.nms_window)
        t1 = time.perf_counter()
        for _ in range(FAST_SAMPLE):
            K = O.gather_cache(sk, spt, 0, 0, L)
            V = O.gather_cache(sv, spt, 0, 0, L)
            O.sparse_attention(qg, K, V, O.sparse_sets(L, cfg.n_sink, cfg.n_recent, list(sel)))
        t2 = time.perf_counter()
        t_slow += t1 - t0
        t_fast += (t2 - t1) / FAST_SAMPLE
        done += 1
        if t_slow + FAST_SAMPLE * t_fast >= budget_s:
            break
    scale = len(groups) / done
    slow_step, fast_step = scale * t_slow, scale * t_fast
    per_layer_step = slow_frac * slow_step + (1 - slow_frac) * fast_step
    spent = t_slow + FAST_SAMPLE * t_fast
    return cfg.B / per_layer_step, spent, done, len(groups), slow_step, fast_step


def cpu_baseline_line(value, spent, done, n_groups, slow_step, fast_step, slow_frac):
    cores, nproc = host_cores()
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"layer 0: one slow and {FAST_SAMPLE} fast layer-steps of {done} of the {n_groups} "
                      f"(sequence, KV head) groups ({spent:.1f} s), scaled to all groups: "
                      f"{slow_step:.1f} s per slow and {fast_step:.2f} s per fast layer-step, weighted by the "
                      f"run's slow fraction {slow_frac:.3f}; {cores} of {nproc} host threads available",
            "nproc": nproc}


def config_dict(cfg, n_slow, world):
    """The workload description both arms print."""
    D = cfg.D
    cache = cfg.n_layers * 2 * cfg.num_pages * cfg.Hkv * 16 * D * 2
    if cfg.boundary_mode == "bernoulli":
        trig = f"bernoulli({cfg.boundary_p:g}), M={cfg.refresh_budget}"
    elif cfg.boundary_mode == "slow_prefix":
        trig = f"slow steps 0..{cfg.slow_prefix - 1}, then fast"
    else:
        trig = f"every {cfg.refresh_budget} steps"
    return {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "D": D,
            "context": cfg.context, "layers": cfg.n_layers, "decode_steps": cfg.steps,
            "budget": cfg.budget_frac if cfg.k_fixed <= 0 else f"K={cfg.k_fixed}",
            "sink": cfg.n_sink, "recent": cfg.n_recent, "trigger": trig, "slow_steps": int(n_slow),
            "evidence_window": cfg.evidence_window,
            "parallelism": "replicas" if world > 1 else "single",
            "l2": ("inputs larger than L2 (KV cache %.1f GB)" if cache > 126e6 else
                   "inputs fit in L2, no flush (KV cache %.3f GB)") % (cache / 1e9)}


# ---------------------------------------------------------------- arms
def run_reference(args, cfg, rank, world):
    if rank != 0:
        return
    from oracle import sfi_oracle as O
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    li = W.make_layer(cfg.replace(n_layers=1), 0, dev)
    slow = O.trigger(W.boundary_stream(cfg), cfg.refresh_budget)
    slow_frac = float(np.mean(slow))
    vals, secs = [], []
    last = None
    for i in range(args.warmup + args.steps):
        last = oracle_sample(cfg, li, li.q[0], slow_frac, budget_s=args.cpu_budget)
        if i >= args.warmup:
            vals.append(last[0])
            secs.append(last[1])
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * float(np.mean(secs)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_dict(cfg, int(slow.sum()), world),
        "cpu_baseline": cpu_baseline_line(value, *last[1:], slow_frac),
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, the nominal figure


def step_bytes(cfg, L, packed_rows, slow, moved_rows=None):
    """Algorithmic bytes of one layer-step (what the method must move).
    Fast: the packed and recent rows of every (sequence, KV head), the
    queries and the outputs.  Slow: the whole cache, the logits written and
    read once by the Selector, the candidates' key norms, and the packed rows
    the refresh copies (read and written; all of them when the buffer is
    built, moved_rows when it is refreshed in place)."""
    B, Hq, Hkv, D, R = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.n_recent
    row = 4 * D
    qo = B * Hq * D * (2 + 4)
    if not slow:
        return float((packed_rows.astype(np.float64) + R).sum()) * row + qo
    nC = L - R - cfg.n_sink
    copied = float(packed_rows.sum()) if moved_rows is None else float(moved_rows)
    return (B * Hkv * L * row + B * Hq * L * 4 + B * Hq * nC * 4 + B * Hkv * nC * 4 + 2 * copied * row + qo)


def frac_entry(bytes_, seconds, peak):
    gbs = bytes_ / seconds / 1e9 if seconds > 0 else 0.0
    return {"GBps": gbs, "frac_measured": gbs / peak, "frac_nominal": gbs / NOMINAL_HBM_GBS}


def run_sfi(args, cfg, rank, world, dist_on):
    dev = torch.device("cuda", torch.cuda.current_device())
    bench = Bench(cfg, dev)
    T, NL, B = cfg.steps, cfg.n_layers, cfg.B
    tokens = B * T * NL
    # warm-up, then a probe run recording the packed row counts of every slow step
    for _ in range(args.warmup):
        bench.run_sfi()
    probe = {}
    slows = bench.run_sfi(probe=probe)
    torch.cuda.synchronize()
    n_slow = sum(slows)
    D = cfg.D
    R = cfg.n_recent
    # algorithmic bytes: of the attention launches whose durations are sampled
    # (one layer), and of every layer-step of the run
    sampled = [timed_layer(NL)]
    every = timed_step_stride(NL)
    fast_bytes = 0.0
    run_fast_bytes = run_slow_bytes = 0.0
    union_rows = []
    cur = None
    first = True
    for t in range(T):
        L = cfg.seq_len(t)
        if slows[t]:
            cur = [x.cpu().numpy() for x in probe[t]]
            union_rows.extend([float(x.mean()) for x in cur])
            # the refresh after the first slow step copies few rows (not
            # counted: the incremental refresh moves well under 1 % of them)
            for l in range(NL):
                run_slow_bytes += step_bytes(cfg, L, cur[l], True, None if first else 0)
            first = False
        else:
            for l in range(NL):
                b_ = step_bytes(cfg, L, cur[l], False)
                run_fast_bytes += b_
                if l in sampled and t % every == 0:
                    fast_bytes += b_
    dense_bytes_slow = sum(float(B * cfg.Hkv * cfg.seq_len(t) * 4 * D + B * cfg.Hq * cfg.seq_len(t) * 4)
                           for t in range(T) if slows[t] and t % every == 0) * len(sampled)
    # timed region: SFI mixed decode, with kernel and step events
    clocks = Clocks(torch.cuda.current_device())
    bench.ctx.set_timing(NL, first_layer=timed_layer(NL))
    bench.ctx.timing(0, reset=True)
    bench.ctx.timing(1, reset=True)
    step_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(T)] for _ in range(args.steps)]
    start_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks.start()
    _sync_barrier(dist_on)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for k in range(args.steps):
        start_ev[k].record()
        bench.run_sfi(step_events=step_ev[k], timing=True)
    e1.record()
    _sync_barrier(dist_on)
    clk_sfi = clocks.stop()
    t_sfi = _max_over_ranks(e0.elapsed_time(e1) / 1000.0, dist_on)
    fast_ms, fast_n = bench.ctx.timing(0, reset=True)
    dense_ms, dense_n = bench.ctx.timing(1, reset=True)
    bench.ctx.set_timing(0)
    # step-type breakdown from main-stream step events
    st_fast, st_slow = [], []
    for k in range(args.steps):
        prev = start_ev[k]
        for t in range(T):
            ms = prev.elapsed_time(step_ev[k][t])
            (st_slow if slows[t] else st_fast).append(ms)
            prev = step_ev[k][t]
    # dense full-KV baseline on the same cache
    bench.run_dense()
    clocks = Clocks(torch.cuda.current_device())
    clocks.start()
    t_dense = _timed(bench.run_dense, args.steps, dist_on)
    clk_dense = clocks.stop()
    # end to end through host buffers
    hq, hk, hv = bench.q.cpu(), bench.kn.cpu(), bench.vn.cpu()
    hout = torch.empty((T,) + tuple(bench.out.shape), dtype=torch.float32).pin_memory()
    # each step's q, k and v side by side in one pinned row, one device row per buffer
    nq, nk, nv = hq[0].numel(), hk[0].numel(), hv[0].numel()
    hin = torch.cat([hq.reshape(T, nq), hk.reshape(T, nk), hv.reshape(T, nv)], dim=1).pin_memory()
    din = torch.empty((2, nq + nk + nv), dtype=bench.q.dtype, device=dev)
    dq = din[:, :nq].view((2,) + tuple(bench.q[0].shape))
    dk = din[:, nq:nq + nk].view((2,) + tuple(bench.kn[0].shape))
    dv = din[:, nq + nk:].view((2,) + tuple(bench.vn[0].shape))
    dout = torch.empty((2,) + tuple(bench.out.shape), dtype=bench.out.dtype, device=dev)
    copy_stream = torch.cuda.Stream(device=dev)
    evs = tuple([torch.cuda.Event(), torch.cuda.Event()] for _ in range(3))
    e2e_args = (hin, hout, dq, dk, dv, din, dout, copy_stream, evs)
    bench.run_e2e(*e2e_args)
    clocks = Clocks(torch.cuda.current_device())
    clocks.start()
    t_e2e = _timed(lambda: bench.run_e2e(*e2e_args), args.steps, dist_on)
    clk_e2e = clocks.stop()
    h2d = (hq[0].numel() * 2 + hk[0].numel() * 2 + hv[0].numel() * 2) * T
    d2h = hout[0].numel() * 4 * T
    # roofline of the dominant kernel, with launches measured in the timed region
    peak, peak_kind = peaks()
    k = args.steps
    ach_fast = (fast_bytes * k / 1e9) / (fast_ms / 1e3) if fast_ms > 0 else 0.0
    ach_dense = (dense_bytes_slow * k / 1e9) / (dense_ms / 1e3) if dense_ms > 0 else 0.0
    dominant = "fast" if fast_ms >= dense_ms else "dense"
    if dominant == "fast":
        roof = {"kernel": f"attn_kernel<{D},*,kFast> (fast step)", "bound": "hbm", "achieved": ach_fast,
                "peak": peak, "unit": "GB/s", "frac": ach_fast / peak,
                "traffic": kernel_traffic("fast_attn_bytes_per_launch", cfg.name),
                "algorithmic_bytes_per_launch": fast_bytes / max(fast_n / k, 1),
                "launches": fast_n, "avg_launch_us": 1000 * fast_ms / max(fast_n, 1),
                "peak_source": f"{peak_kind} hbm_gbs"}
    else:
        roof = {"kernel": f"attn_kernel<{D},*,kDenseExtras> (slow step)", "bound": "hbm", "achieved": ach_dense,
                "peak": peak, "unit": "GB/s", "frac": ach_dense / peak,
                "traffic": kernel_traffic("dense_attn_bytes_per_launch", cfg.name),
                "algorithmic_bytes_per_launch": dense_bytes_slow / max(dense_n / k, 1),
                "launches": dense_n, "avg_launch_us": 1000 * dense_ms / max(dense_n, 1),
                "peak_source": f"{peak_kind} hbm_gbs"}
    roof["frac_nominal"] = roof["achieved"] / NOMINAL_HBM_GBS
    # every step type as a fraction of the HBM roofline: algorithmic bytes of
    # the run's fast (slow) layer-steps over the main stream's fast (slow)
    # step time, the whole run's bytes over the whole run's time, and the
    # dense baseline's cache bytes over its time
    n_fast = T - n_slow
    dense_run_bytes = sum(float(B * cfg.Hkv * cfg.seq_len(t) * 4 * D + B * cfg.Hq * D * 6) for t in range(T)) * NL
    roof["steps"] = {
        "fast": frac_entry(run_fast_bytes / max(n_fast, 1), statistics.mean(st_fast) / 1e3, peak) if st_fast else None,
        "slow": frac_entry(run_slow_bytes / max(n_slow, 1), statistics.mean(st_slow) / 1e3, peak) if st_slow else None,
        "mix": frac_entry(run_fast_bytes + run_slow_bytes, t_sfi / args.steps, peak),
        "dense_baseline": frac_entry(dense_run_bytes, t_dense / args.steps, peak),
        "bytes": "fast: (packed + recent rows) x 4D + q, o; slow: cache + logits written and read once + "
                 "candidate norms + rows copied by the refresh (all at the first slow step); per layer-step",
    }
    value = aggregate_rate(world, tokens, args.steps, t_sfi)
    # fast layer-step: attention (with the append) + combine; slow: the same
    # two, 3 statistics, scores and the top-K, then the compaction: 3 kernels
    # when step 0 builds the packed buffers, 1 (the incremental refresh) when
    # a later slow step refreshes them (side stream)
    n_fresh = 1 if slows and slows[0] else 0
    launches_per_run = NL * (n_fresh * 10 + (n_slow - n_fresh) * 8 + (T - n_slow) * 2)
    legs = {"sfi": clk_sfi, "dense": clk_dense, "e2e": clk_e2e}
    mhz = [v["sm_mhz"] for v in legs.values() if v.get("sm_mhz")]
    clk = {"sm_mhz": statistics.median(mhz) if mhz else None,
           "sm_max_mhz": max([v["sm_max_mhz"] for v in legs.values() if v.get("sm_max_mhz")] or [0]) or None,
           "reasons": sorted(set(r for v in legs.values() for r in v.get("reasons", []))),
           "legs": legs}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000 * t_sfi / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(cfg, n_slow, world),
        "roofline": roof,
        "e2e": {"value": aggregate_rate(world, tokens, args.steps, t_e2e), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_run * args.steps,
        "clocks": clk,
        "breakdown": {
            "dense_full_kv_tok_s": aggregate_rate(world, tokens, args.steps, t_dense),
            "speedup_vs_dense": t_dense / t_sfi,
            "fast_step_tok_s": B * NL / (statistics.mean(st_fast) / 1e3) if st_fast else None,
            "slow_step_tok_s": B * NL / (statistics.mean(st_slow) / 1e3) if st_slow else None,
            "slow_layer_step_us": 1000 * statistics.mean(st_slow) / NL if st_slow else None,
            "fast_layer_step_us": 1000 * statistics.mean(st_fast) / NL if st_fast else None,
            "fast_attn_GBps": ach_fast, "dense_attn_GBps": ach_dense,
            "timed_layers": f"layer {timed_layer(NL)} (1 of {NL}), every {timed_step_stride(NL)} step(s)",
            "fast_attn_ms_sampled": fast_ms, "dense_attn_ms_sampled": dense_ms,
            "mean_packed_rows": float(np.mean(union_rows)) if union_rows else None,
            "fast_frac_of_dense_bytes": None if not union_rows else
            (float(np.mean(union_rows)) + R) / cfg.seq_len(T // 2),
        },
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        slow_frac = n_slow / T
        res = oracle_sample(cfg, bench.layers[0], bench.q[0, 0], slow_frac, budget_s=args.cpu_budget)
        line["cpu_baseline"] = cpu_baseline_line(*res, slow_frac)
    if rank == 0:
        print(json.dumps(line), flush=True)
    bench.ctx.close()


def run_layer_probe(args, cfg):
    """A few launches of every hot-path kernel on one layer of the workload
    (for profiler captures): per repetition a slow layer-step that builds the
    packed buffer (dense attention with logits, Selector, full compaction), a
    fast layer-step, and after 15 more fast steps a slow layer-step that
    refreshes the buffer incrementally, as the decode loop's later slow steps
    do."""
    cfg1 = cfg.replace(n_layers=1)
    dev = torch.device("cuda", torch.cuda.current_device())
    li = W.make_layer(cfg1, 0, dev)
    layer = alloc_layer(cfg1, li, dev)
    ctx = S.Context(shape_of(cfg1), params_of(cfg1), 1, overlap=False, device=dev)
    out = torch.empty(cfg1.B, cfg1.Hq, cfg1.D, device=dev)
    torch.cuda.synchronize()
    for r in range(args.layer_probe):
        for t in range(18):   # steps 0 and 16 slow (a boundary at step 15), the rest fast
            ctx.decode_step(0, t, int(t == 16), cfg1.seq_len(t), layer.kv, layer.packed, li.q[t], li.k_new[t],
                            li.v_new[t], out)
        ctx.join()
    torch.cuda.synchronize()
    assert S.sfi_poll_error(layer.kv) == 0
    ctx.close()
    print(json.dumps({"layer_probe": cfg1.name, "repetitions": args.layer_probe}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="sfi", choices=["sfi", "reference"])
    ap.add_argument("--decode-steps", type=int, default=0, help="override the workload's decode steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0,
                    help="seconds of oracle work per CPU-baseline sample")
    ap.add_argument("--layer-probe", type=int, default=0,
                    help="only run this many slow+fast layer-steps of one layer (profiler captures)")
    ap.add_argument("--evidence-window", type=int, default=0,
                    help="average the Selector's evidence over this many queries (default: the workload's)")
    args = ap.parse_args()
    cfg = W.CONFIG_BY_NAME[args.config]
    if args.decode_steps:
        cfg = cfg.replace(steps=args.decode_steps)
    if args.evidence_window:
        cfg = cfg.replace(evidence_window=args.evidence_window)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        # the CPU oracle runs on rank 0 alone; the other ranks exit at once
        if rank == 0:
            run_reference(args, cfg, rank, world)
        return
    dist_on = world > 1
    if dist_on:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    if args.layer_probe:
        run_layer_probe(args, cfg)
    else:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py --impl sfi needs a CUDA device")
        S.lib()
        run_sfi(args, cfg, rank, world, dist_on)
    if dist_on:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
