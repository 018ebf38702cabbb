// Decode-step driver: the slow/fast trigger and the asynchronous two-stream
// pipeline of Slow-Fast Inference ([ES] "2. Metodología", Pasos Lentos;
// "3. Optimización del Sistema", item 1; [FR] "C. Optimisations Système",
// Pipeline Asynchrone; [ZH] "2.3" 异步流水线).
//
// On a slow step the main stream runs dense attention for layer i (also
// writing the logits and the candidate log-sum-exp into one of a ring of
// buffers) and moves on to layer i+1; the Selector and the compaction of
// layer i run on the context's side stream after an event.  The next step of
// layer i waits for that refresh before it touches the layer's cache or
// packed buffer.  A logits buffer is rewritten only after the side stream has
// finished reading it.  The side stream has the lowest priority: a layer's
// Selector is needed only at the layer's next step, so its kernels fill the
// SMs the main stream leaves (the tails of the attention launches) instead
// of holding the next layer's dense attention back.  The dense launches let
// the next kernel be scheduled only when their CTAs run out of work.
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "internal.h"

// Logits buffers the slow steps of consecutive layers rotate through: layer
// i's dense launch waits until the Selector of layer i - kLogitBufs has read
// its buffer, so a Selector may lag that many layers behind the attention.
constexpr int kLogitBufs = 4;

struct sfi_ctx {
  sfi_shape s;
  sfi_params p;
  int n_layers;
  int overlap;
  int device;
  int p_max_ws;
  cudaStream_t side = nullptr;
  std::vector<cudaEvent_t> ev_pre, ev_dense, ev_sel;
  std::vector<uint8_t> pending;
  cudaEvent_t ev_buf_free[kLogitBufs] = {};
  int cur_step = -1;
  // per-sequence trigger state: the last slow step of every sequence and the
  // decision of the current step (layer 0 decides, the other layers reuse it)
  std::vector<int> last_slow;
  std::vector<uint8_t> row_slow;
  int n_slow = 0;
  sfi::RowMap slow_rows, fast_rows;   // lists of a mixed step
  // evidence window of W queries: per layer a ring of the last W steps'
  // queries (slot = step mod W) and the step each slot holds (-1: none)
  int win = 1;
  char* ring = nullptr;
  size_t ring_layer_bytes = 0;
  float* wout = nullptr;
  std::vector<int> slot_step;   // [n_layers][win]
  // workspace carving
  char* ws = nullptr;
  size_t ws_bytes = 0;
  float* part = nullptr;
  size_t part_bytes = 0;
  float* logits[kLogitBufs] = {};
  float* lse_cand[kLogitBufs] = {};
  int64_t ld = 0;
  void* stats = nullptr;
  float* scores = nullptr;
  uint32_t* bits = nullptr;
  int64_t bits_ld = 0;
  sfi::CompactScratch cmp;
  // compaction: incremental (rows that stay selected keep their slots) once
  // a layer's packed buffer holds this context's previous result
  int incremental = 1;
  std::vector<const void*> packed_seen;   // per layer: pos pointer of the last refresh
  std::vector<sfi::AttnMapCache> maps;   // per layer
  // timing of the attention kernels (kind 0 fast, 1 dense) of every
  // timing-th layer (0: off)
  int timing = 0;         // layer stride of the timed attention launches (0: off)
  int timing_first = 0;   // first timed layer
  std::vector<cudaEvent_t> tev[2];
  size_t tused[2] = {0, 0};
};

namespace sfi {
namespace {

struct CtxLayout {
  size_t part_off, part_bytes, logit_off, logit_bytes, lsec_off, lsec_bytes, stat_off, stat_bytes, score_off,
      score_bytes, bits_off, bits_bytes, tc_off, tc_bytes, ring_off, ring_layer_bytes,
      wout_off, total;
  int64_t bits_ld;
};

// The slow step's dense-attention shape: with an evidence window of W
// queries, the group's last W queries are Hkv * W * G heads of one launch.
sfi_shape window_shape(const sfi_shape& s, const sfi_params& p) {
  sfi_shape w = s;
  w.Hq = s.Hkv * evidence_window(p) * (s.Hq / s.Hkv);
  return w;
}

CtxLayout ctx_layout(const sfi_shape& s, const sfi_params& p, int n_layers) {
  const WsLayout w = ws_layout(s, p);
  const sfi_shape sw = window_shape(s, p);
  const int W = evidence_window(p);
  CtxLayout c{};
  const int Lmax = s.max_pages * kPage;
  size_t off = 256;
  c.part_off = off;
  c.part_bytes = W > 1 ? std::max(w.part_bytes, ws_layout(sw, p).part_bytes) : w.part_bytes;
  off += c.part_bytes;
  c.logit_off = off;
  c.logit_bytes = align_up((size_t)s.B * sw.Hq * Lmax * sizeof(float), 256);
  off += kLogitBufs * c.logit_bytes;
  c.lsec_off = off;
  c.lsec_bytes = align_up((size_t)s.B * sw.Hq * sizeof(float), 256);
  off += kLogitBufs * c.lsec_bytes;
  c.stat_off = off;
  c.stat_bytes = w.stat_bytes;
  off += c.stat_bytes;
  c.score_off = off;
  c.score_bytes = w.sel_bytes;
  off += c.score_bytes;
  c.bits_off = off;
  c.bits_bytes = w.bits_bytes;
  c.bits_ld = w.bits_ld;
  off += c.bits_bytes;
  c.tc_off = off;
  c.tc_bytes = w.cmp_bytes;
  off += c.tc_bytes;
  // evidence window: every layer's last W queries, [B][Hkv][W][G][D] bf16,
  // and the window launch's outputs [B][Hkv * W * G][D] fp32
  c.ring_off = off;
  c.ring_layer_bytes = W > 1 ? align_up((size_t)s.B * sw.Hq * s.D * 2, 256) : 0;
  off += (size_t)n_layers * c.ring_layer_bytes;
  c.wout_off = off;
  off += W > 1 ? align_up((size_t)s.B * sw.Hq * s.D * sizeof(float), 256) : 0;
  c.total = off;
  return c;
}

#define SFI_TRY(x)               \
  do {                           \
    sfi_status _r = (x);         \
    if (_r != SFI_OK) return _r; \
  } while (0)

sfi_status cu(cudaError_t e) { return e == cudaSuccess ? SFI_OK : SFI_ERR_CUDA; }

// Event pair for one timed launch, or nulls when timing is off.
void timing_events(sfi_ctx* c, int kind, int layer, cudaEvent_t* b, cudaEvent_t* e) {
  *b = *e = nullptr;
  if (c->timing <= 0 || layer < c->timing_first || (layer - c->timing_first) % c->timing != 0) return;
  auto& v = c->tev[kind];
  if (c->tused[kind] + 2 > v.size()) {
    for (int i = 0; i < 256; ++i) {
      cudaEvent_t ev;
      if (cudaEventCreate(&ev) != cudaSuccess) return;
      v.push_back(ev);
    }
  }
  *b = v[c->tused[kind]];
  *e = v[c->tused[kind] + 1];
  c->tused[kind] += 2;
}

}  // namespace
}  // namespace sfi

namespace sfi {
namespace {

sfi_status check_step(const sfi_ctx* c, int layer, int step, int L, const sfi_paged_kv* kv,
                      const sfi_packed* packed, const sfi_bf16* q, const sfi_bf16* k_new, const sfi_bf16* v_new,
                      const float* out) {
  if (!c || !c->ws) return SFI_ERR_WORKSPACE;
  if (layer < 0 || layer >= c->n_layers || step < 0) return SFI_ERR_INVALID_ARG;
  if (!kv || !packed || !q || !k_new || !v_new || !out || !kv->key_norms) return SFI_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & 15u) != 0)
    return SFI_ERR_INVALID_ARG;
  if (L < c->p.n_sink + c->p.n_recent + 1 || L > c->s.max_pages * kPage) return SFI_ERR_SHAPE;
  if (packed->p_max < packed_rows_capacity(c->s, c->p)) return SFI_ERR_SHAPE;
  return SFI_OK;
}

// Trigger of every sequence for the step (layer 0): slow at step 0, after a
// boundary token of that sequence, or when its refresh budget runs out.
// boundary(b) gives the sequence's previous-step boundary flag.
template <class F>
sfi_status decide(sfi_ctx* c, int step, F boundary) {
  const int B = c->s.B;
  int n = 0;
  for (int b = 0; b < B; ++b) {
    const bool slow = step == 0 || boundary(b) || (step - c->last_slow[b]) >= c->p.refresh_budget;
    if (slow) c->last_slow[b] = step;
    c->row_slow[b] = slow ? 1 : 0;
    n += slow ? 1 : 0;
  }
  c->cur_step = step;
  c->n_slow = n;
  if (n > 0 && n < B) {   // a mixed step: the two lists
    if (B > kMaxRowMap) return SFI_ERR_UNSUPPORTED;
    c->slow_rows.n = c->fast_rows.n = 0;
    for (int b = 0; b < B; ++b) {
      RowMap& m = c->row_slow[b] ? c->slow_rows : c->fast_rows;
      m.b[m.n++] = (int16_t)b;
    }
  }
  return SFI_OK;
}

// One layer of the current step: the slow path (dense attention, then the
// Selector and compaction on the side stream) on the slow sequences, the
// fast path on the others.
sfi_status run_layer(sfi_ctx* c, int layer, int step, int L, const sfi_paged_kv* kv, sfi_packed* packed,
                     const sfi_bf16* q, const sfi_bf16* k_new, const sfi_bf16* v_new, float* out,
                     cudaStream_t main) {
  const sfi_shape& s = c->s;
  const sfi_params& p = c->p;
  const int B = s.B;
  const RowMap all{};
  const RowMap& slow_map = c->n_slow == B ? all : c->slow_rows;
  const RowMap& fast_map = c->n_slow == 0 ? all : c->fast_rows;

  // this layer's previous refresh must land before its cache or packed buffer is touched
  if (c->pending[layer]) {
    SFI_TRY(cu(cudaStreamWaitEvent(main, c->ev_sel[layer], 0)));
    c->pending[layer] = 0;
  }
  // the attention launches append the step's token themselves
  const StepToken tok{k_new, v_new};
  const int W = c->win, G = s.Hq / s.Hkv;
  char* ring = c->ring + (size_t)layer * c->ring_layer_bytes;
  uint32_t wmask = 1u;
  if (W > 1) {
    // the step's queries into the layer's ring (after the wait above: the
    // last refresh of this layer has read the slot this overwrites)
    int* ss = &c->slot_step[(size_t)layer * W];
    if (step == 0) std::fill(ss, ss + W, -1);
    const int slot = step % W;
    const size_t row = (size_t)G * s.D * sizeof(sfi_bf16);
    SFI_TRY(cu(cudaMemcpy2DAsync(ring + slot * row, W * row, q, row, row, (size_t)s.B * s.Hkv,
                                 cudaMemcpyDeviceToDevice, main)));
    ss[slot] = step;
    wmask = 0u;
    for (int i = 0; i < W; ++i)
      if (ss[i] >= 0 && ss[i] > step - W) wmask |= 1u << i;
  }
  if (c->n_slow > 0) {
    const int buf = layer % kLogitBufs;
    SFI_TRY(cu(cudaStreamWaitEvent(main, c->ev_buf_free[buf], 0)));
    // the prior's statistics read key norms only (the step's appended token
    // is in the recent window, never a candidate): on the side stream, beside
    // this layer's attention
    SFI_TRY(cu(cudaEventRecord(c->ev_pre[layer], main)));
    SFI_TRY(cu(cudaStreamWaitEvent(c->side, c->ev_pre[layer], 0)));
    SFI_TRY(run_select_stats(s, p, *kv, L, c->stats, c->side, slow_map));
    sfi_dense_extras ex{};
    ex.logits = c->logits[buf];
    ex.ld = c->ld;
    ex.lse_cand = c->lse_cand[buf];
    ex.cand_lo = p.n_sink;
    ex.cand_hi = L - p.n_recent;
    {
      cudaEvent_t b, e;
      timing_events(c, 1, layer, &b, &e);
      if (W == 1) {
        SFI_TRY(run_dense_attn(s, *kv, L, q, out, &ex, reinterpret_cast<int*>(c->ws), c->part, c->part_bytes,
                               main, b, e, &tok, &c->maps[layer], slow_map, c->overlap != 0));
      } else {
        // one pass over the cache for the group's last W queries (Hkv * W * G
        // heads); the outputs of the step's own queries are copied out
        const sfi_shape sw = window_shape(s, p);
        SFI_TRY(run_dense_attn(sw, *kv, L, reinterpret_cast<const sfi_bf16*>(ring), c->wout, &ex,
                               reinterpret_cast<int*>(c->ws), c->part, c->part_bytes, main, b, e, &tok,
                               &c->maps[layer], slow_map, c->overlap != 0));
        const size_t orow = (size_t)G * s.D * sizeof(float);
        SFI_TRY(cu(cudaMemcpy2DAsync(out, orow, reinterpret_cast<const char*>(c->wout) + (step % W) * orow, W * orow,
                                     orow, (size_t)s.B * s.Hkv, cudaMemcpyDeviceToDevice, main)));
      }
    }
    SFI_TRY(cu(cudaEventRecord(c->ev_dense[layer], main)));
    cudaStream_t side = c->side;
    SFI_TRY(cu(cudaStreamWaitEvent(side, c->ev_dense[layer], 0)));
    const int nC = L - p.n_recent - p.n_sink;
    const int K = budget_k(p, L);
    if (K < 1) return SFI_ERR_SHAPE;
    const int ld_s = (nC + 3) / 4 * 4;
    if (nC > topk_max_n()) return SFI_ERR_UNSUPPORTED;
    const int rows = slow_map.count(B) * s.Hq;   // logical rows of the Selector
    SFI_TRY(run_select_scores(s, p, *kv, L, c->logits[buf], c->ld, c->lse_cand[buf], c->scores, ld_s,
                              c->stats, side, slow_map, wmask, false, true));
    SFI_TRY(cu(cudaEventRecord(c->ev_buf_free[buf], side)));
    SFI_TRY(run_topk(rows, nC, c->scores, ld_s, K, p.n_sink, nullptr, 0, c->bits, c->bits_ld, side,
                     select_row_range(s, p, L, c->stats)));
    if (c->incremental && packed->p_max >= c->cmp.cap) {
      // step 0 starts a new decode: cache rows copied before may have changed
      const bool fresh = step == 0 || c->packed_seen[layer] != packed->pos;
      SFI_TRY(run_compact_inc(s, p, *kv, c->bits, c->bits_ld, *packed, c->cmp, L, fresh, side, slow_map));
      c->packed_seen[layer] = packed->pos;
    } else {
      SFI_TRY(run_compact_bits(s, p, *kv, c->bits, c->bits_ld, *packed, c->cmp, L, side, slow_map));
      c->packed_seen[layer] = nullptr;
    }
    SFI_TRY(cu(cudaEventRecord(c->ev_sel[layer], side)));
  }
  if (c->n_slow < B) {
    cudaEvent_t b, e;
    timing_events(c, 0, layer, &b, &e);
    SFI_TRY(run_fast_attn(s, p, *kv, L, q, *packed, out, nullptr, reinterpret_cast<int*>(c->ws), c->part,
                          c->part_bytes, main, b, e, &tok, &c->maps[layer], fast_map));
  }
  if (c->n_slow > 0) {
    if (c->overlap) c->pending[layer] = 1;
    else SFI_TRY(cu(cudaStreamWaitEvent(main, c->ev_sel[layer], 0)));
  }
  return SFI_OK;
}

}  // namespace
}  // namespace sfi

using namespace sfi;

extern "C" {

sfi_status sfi_ctx_create(const sfi_shape* shape, const sfi_params* params, int32_t n_layers,
                          int32_t overlap, sfi_ctx** out) {
  if (!out) return SFI_ERR_INVALID_ARG;
  *out = nullptr;
  size_t probe = 0;
  SFI_TRY(sfi_workspace_size(shape, params, &probe));
  if (n_layers < 1) return SFI_ERR_INVALID_ARG;
  // the window's queries are the heads of one dense launch: at most 16 per group
  if (evidence_window(*params) * (shape->Hq / shape->Hkv) > 16) return SFI_ERR_UNSUPPORTED;
  auto* c = new sfi_ctx();
  c->s = *shape;
  c->p = *params;
  c->n_layers = n_layers;
  c->overlap = overlap ? 1 : 0;
  cudaGetDevice(&c->device);
  // the side stream gets the lowest priority: the Selector kernels run where
  // the main stream's attention leaves SMs free (measured on the 128K
  // workload: slow layer-step 269 us with the highest priority, 262 us with
  // the lowest)
  int least = 0, greatest = 0;
  bool ok = cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess &&
            cudaStreamCreateWithPriority(&c->side, cudaStreamNonBlocking, least) == cudaSuccess;
  c->ev_pre.resize(n_layers, nullptr);
  c->ev_dense.resize(n_layers, nullptr);
  c->ev_sel.resize(n_layers, nullptr);
  c->pending.assign(n_layers, 0);
  c->maps.resize(n_layers);
  c->packed_seen.assign(n_layers, nullptr);
  c->last_slow.assign(shape->B, 0);
  c->row_slow.assign(shape->B, 0);
  c->win = evidence_window(*params);
  c->slot_step.assign((size_t)n_layers * c->win, -1);
  for (int i = 0; i < n_layers && ok; ++i)
    ok = cudaEventCreateWithFlags(&c->ev_pre[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->ev_dense[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->ev_sel[i], cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; i < kLogitBufs && ok; ++i)
    ok = cudaEventCreateWithFlags(&c->ev_buf_free[i], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    sfi_ctx_destroy(c);
    return SFI_ERR_CUDA;
  }
  *out = c;
  return SFI_OK;
}

sfi_status sfi_ctx_destroy(sfi_ctx* c) {
  if (!c) return SFI_OK;
  if (c->side) cudaStreamSynchronize(c->side);
  for (auto e : c->ev_pre) if (e) cudaEventDestroy(e);
  for (auto e : c->ev_dense) if (e) cudaEventDestroy(e);
  for (auto e : c->ev_sel) if (e) cudaEventDestroy(e);
  for (auto e : c->ev_buf_free) if (e) cudaEventDestroy(e);
  for (int k = 0; k < 2; ++k)
    for (auto e : c->tev[k]) cudaEventDestroy(e);
  if (c->side) cudaStreamDestroy(c->side);
  delete c;
  return SFI_OK;
}

sfi_status sfi_ctx_workspace_size(const sfi_ctx* c, size_t* bytes) {
  if (!c || !bytes) return SFI_ERR_INVALID_ARG;
  *bytes = ctx_layout(c->s, c->p, c->n_layers).total;
  return SFI_OK;
}

sfi_status sfi_ctx_set_workspace(sfi_ctx* c, void* ws, size_t bytes) {
  if (!c || !ws) return SFI_ERR_INVALID_ARG;
  const CtxLayout l = ctx_layout(c->s, c->p, c->n_layers);
  if (bytes < l.total) return SFI_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  // the counters in the workspace (attention work counter, combine and top-K
  // arrival counters, histograms) start at zero; every step leaves them so
  if (cudaMemset(w, 0, l.total) != cudaSuccess) return SFI_ERR_CUDA;
  c->ws = w;
  c->ws_bytes = bytes;
  c->part = reinterpret_cast<float*>(w + l.part_off);
  c->part_bytes = l.part_bytes;
  c->ld = (int64_t)c->s.max_pages * kPage;
  for (int i = 0; i < kLogitBufs; ++i) {
    c->logits[i] = reinterpret_cast<float*>(w + l.logit_off + i * l.logit_bytes);
    c->lse_cand[i] = reinterpret_cast<float*>(w + l.lsec_off + i * l.lsec_bytes);
  }
  c->ring = w + l.ring_off;
  c->ring_layer_bytes = l.ring_layer_bytes;
  c->wout = reinterpret_cast<float*>(w + l.wout_off);
  c->stats = w + l.stat_off;
  c->scores = reinterpret_cast<float*>(w + l.score_off);
  c->bits = reinterpret_cast<uint32_t*>(w + l.bits_off);
  c->bits_ld = l.bits_ld;
  c->cmp = compact_scratch(w + l.tc_off, c->s, c->p);
  // a new workspace holds no previous-selection state and no queries
  std::fill(c->packed_seen.begin(), c->packed_seen.end(), nullptr);
  std::fill(c->slot_step.begin(), c->slot_step.end(), -1);
  return SFI_OK;
}


sfi_status sfi_decode_step(sfi_ctx* c, int32_t layer, int32_t step, int32_t boundary_prev,
                           int32_t L, const sfi_paged_kv* kv, sfi_packed* packed,
                           const sfi_bf16* q, const sfi_bf16* k_new, const sfi_bf16* v_new,
                           float* out, sfi_stream stream, int32_t* was_slow) {
  SFI_TRY(check_step(c, layer, step, L, kv, packed, q, k_new, v_new, out));
  if (layer == 0) SFI_TRY(decide(c, step, [&](int) { return boundary_prev != 0; }));
  else if (step != c->cur_step) return SFI_ERR_INVALID_ARG;   // layer 0 decides the step
  if (was_slow) *was_slow = c->n_slow > 0 ? 1 : 0;
  return run_layer(c, layer, step, L, kv, packed, q, k_new, v_new, out, (cudaStream_t)stream);
}

sfi_status sfi_decode_step_rows(sfi_ctx* c, int32_t layer, int32_t step, const int32_t* boundary_prev,
                                int32_t L, const sfi_paged_kv* kv, sfi_packed* packed,
                                const sfi_bf16* q, const sfi_bf16* k_new, const sfi_bf16* v_new,
                                float* out, sfi_stream stream, int32_t* slow_rows) {
  SFI_TRY(check_step(c, layer, step, L, kv, packed, q, k_new, v_new, out));
  if (c->s.B > kMaxRowMap) return SFI_ERR_UNSUPPORTED;
  if (layer == 0) SFI_TRY(decide(c, step, [&](int b) { return boundary_prev && boundary_prev[b] != 0; }));
  else if (step != c->cur_step) return SFI_ERR_INVALID_ARG;
  if (slow_rows)
    for (int b = 0; b < c->s.B; ++b) slow_rows[b] = c->row_slow[b];
  return run_layer(c, layer, step, L, kv, packed, q, k_new, v_new, out, (cudaStream_t)stream);
}

sfi_status sfi_ctx_set_compaction(sfi_ctx* c, int32_t incremental) {
  if (!c) return SFI_ERR_INVALID_ARG;
  c->incremental = incremental ? 1 : 0;
  std::fill(c->packed_seen.begin(), c->packed_seen.end(), nullptr);
  return SFI_OK;
}

sfi_status sfi_ctx_join(sfi_ctx* c, sfi_stream stream) {
  if (!c) return SFI_ERR_INVALID_ARG;
  for (int i = 0; i < c->n_layers; ++i) {
    if (c->pending[i]) {
      SFI_TRY(cu(cudaStreamWaitEvent((cudaStream_t)stream, c->ev_sel[i], 0)));
      c->pending[i] = 0;
    }
  }
  return SFI_OK;
}

sfi_status sfi_ctx_set_timing(sfi_ctx* c, int32_t layer_stride) {
  return sfi_ctx_set_timing_layers(c, 0, layer_stride);
}

sfi_status sfi_ctx_set_timing_layers(sfi_ctx* c, int32_t first_layer, int32_t layer_stride) {
  if (!c || layer_stride < 0 || first_layer < 0) return SFI_ERR_INVALID_ARG;
  c->timing = layer_stride;
  c->timing_first = first_layer;
  return SFI_OK;
}

sfi_status sfi_ctx_timing(sfi_ctx* c, int32_t kind, double* total_ms, int64_t* launches,
                          int32_t reset) {
  if (!c || kind < 0 || kind > 1 || !total_ms || !launches) return SFI_ERR_INVALID_ARG;
  double tot = 0.0;
  const size_t n = c->tused[kind] / 2;
  for (size_t i = 0; i < n; ++i) {
    cudaEvent_t b = c->tev[kind][2 * i], e = c->tev[kind][2 * i + 1];
    if (cudaEventSynchronize(e) != cudaSuccess) return SFI_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, b, e) != cudaSuccess) return SFI_ERR_CUDA;
    tot += ms;
  }
  *total_ms = tot;
  *launches = (int64_t)n;
  if (reset) c->tused[kind] = 0;
  return SFI_OK;
}

}  // extern "C"
