// C-ABI entry points: argument validation, workspace carving and dispatch.
// Nothing here computes; every step of the path runs in the kernels of
// attn.cu, select.cu, compact.cu and kv.cu.
#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace sfi {

int num_sms() {
  static int cache[64] = {0};
  int d = 0;
  cudaGetDevice(&d);
  d &= 63;
  if (cache[d] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    cache[d] = n;
  }
  return cache[d];
}

int budget_k(const sfi_params& p, int L) {
  const int nC = L - p.n_recent - p.n_sink;
  if (nC < 1) return -1;
  long k = p.k_fixed > 0 ? p.k_fixed : (long)std::floor(p.budget_frac * (double)L);
  if (k > nC) k = nC;
  return k < 1 ? -1 : (int)k;
}

int packed_rows_capacity(const sfi_shape& s, const sfi_params& p) {
  const int G = s.Hq / s.Hkv;
  const int Lmax = s.max_pages * kPage;
  const int nC = Lmax - p.n_recent - p.n_sink;
  long k = p.k_fixed > 0 ? p.k_fixed : (long)std::floor(p.budget_frac * (double)Lmax);
  if (k > nC) k = nC;
  if (k < 0) k = 0;
  long u = std::min<long>((long)G * k, std::max(nC, 0));
  long rows = p.n_sink + u;
  return (int)((rows + 63) / 64 * 64);
}

WsLayout ws_layout(const sfi_shape& s, const sfi_params& p) {
  WsLayout w{};
  const int G = s.Hq / s.Hkv;
  const long bh = (long)s.B * s.Hkv;
  const int Lmax = s.max_pages * kPage;
  const long dense_chunks = dense_chunks_bound(s);
  const int kmax = std::max(budget_k(p, Lmax), 0);
  // the fast step's chunk count grows with the expected selection size, which
  // is largest at L_max
  const long fast_items = bh * fast_chunks(s, packed_rows_capacity(s, p), p.n_recent, kmax + p.n_sink);
  const long items = std::max(bh * dense_chunks, fast_items);
  size_t off = 256;   // first 256 bytes reserved
  w.part_off = off;
  w.part_bytes = align_up(attn_part_bytes((int)items, G, s.D), 256);
  off += w.part_bytes;
  const long nC = std::max<long>(Lmax - p.n_recent - p.n_sink, 1);
  w.stat_off = off;
  // the rows' score ranges for the top-K, per-chunk partial sums and the
  // position factors (fp64), kappa * pi of every candidate and lambda / Z of
  // every row (fp32)
  const size_t kp_ld = (size_t)((nC + 1) / 2 * 2);
  w.stat_bytes = align_up((size_t)s.B * s.Hq * 2 * sizeof(uint32_t) +
                              (size_t)bh * stat_chunks((int)nC) * 2 * sizeof(double) + kp_ld * sizeof(double) +
                              (size_t)bh * kp_ld * sizeof(float) + (size_t)bh * sizeof(float), 256);
  off += w.stat_bytes;
  w.sel_off = off;
  w.sel_bytes = align_up((size_t)s.B * s.Hq * ((nC + 3) / 4 * 4) * sizeof(float), 256);
  off += w.sel_bytes;
  w.cmp_off = off;
  w.cmp_bytes = align_up(compact_scratch_bytes(s, p), 256);
  off += w.cmp_bytes;
  w.bits_ld = (nC + 31) / 32;
  w.bits_off = off;
  w.bits_bytes = align_up((size_t)s.B * s.Hq * w.bits_ld * sizeof(uint32_t), 256);
  off += w.bits_bytes;
  w.total = off;
  return w;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sfi_status check_shape(const sfi_shape* s) {
  if (!s) return SFI_ERR_INVALID_ARG;
  if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->Hq % s->Hkv != 0) return SFI_ERR_SHAPE;
  const int G = s->Hq / s->Hkv;
  if (G > 32) return SFI_ERR_SHAPE;
  if (G > 16) return SFI_ERR_UNSUPPORTED;
  if (s->D != 64 && s->D != 128) return SFI_ERR_UNSUPPORTED;
  if (s->page_size != kPage) return SFI_ERR_UNSUPPORTED;
  if (s->max_pages < 1 || s->num_pages < 1) return SFI_ERR_SHAPE;
  if ((long long)s->num_pages * s->Hkv * kPage >= (1LL << 31)) return SFI_ERR_SHAPE;
  if ((long long)s->max_pages * kPage >= (1LL << 30)) return SFI_ERR_SHAPE;
  return SFI_OK;
}

sfi_status check_params(const sfi_params* p) {
  if (!p) return SFI_ERR_INVALID_ARG;
  if (p->n_sink < 0 || p->n_recent < 1 || p->k_fixed < 0 || p->nms_window < 0) return SFI_ERR_INVALID_ARG;
  if (!(p->budget_frac >= 0.0 && p->budget_frac <= 1.0)) return SFI_ERR_INVALID_ARG;
  if (!(p->lambda_clip >= 0.f) || !std::isfinite(p->lambda) || !(p->alpha_soft >= 0.f) ||
      !(p->alpha_cross >= 0.f) || !std::isfinite(p->alpha_soft) || !std::isfinite(p->alpha_cross))
    return SFI_ERR_INVALID_ARG;
  if (p->refresh_budget < 1) return SFI_ERR_INVALID_ARG;
  if (p->evidence_window < 0 || p->evidence_window > 32 || p->evidence_window > p->n_recent)
    return SFI_ERR_INVALID_ARG;
  return SFI_OK;
}

sfi_status check_kv(const sfi_paged_kv* kv) {
  if (!kv || !kv->k_pool || !kv->v_pool || !kv->page_table) return SFI_ERR_INVALID_ARG;
  if (!aligned16(kv->k_pool) || !aligned16(kv->v_pool)) return SFI_ERR_INVALID_ARG;
  return SFI_OK;
}

sfi_status check_L(const sfi_shape* s, int L) {
  if (L < 1 || L > s->max_pages * kPage) return SFI_ERR_SHAPE;
  return SFI_OK;
}

sfi_status check_sparse_L(const sfi_shape* s, const sfi_params* p, int L) {
  sfi_status r = check_L(s, L);
  if (r != SFI_OK) return r;
  if (L < p->n_sink + p->n_recent + 1) return SFI_ERR_SHAPE;
  return SFI_OK;
}

sfi_status check_packed(const sfi_shape* s, const sfi_params* p, const sfi_packed* pk) {
  if (!pk || !pk->k || !pk->v || !pk->pos || !pk->headmask || !pk->n_rows) return SFI_ERR_INVALID_ARG;
  if (!aligned16(pk->k) || !aligned16(pk->v)) return SFI_ERR_INVALID_ARG;
  if (pk->p_max < 64 || pk->p_max % 64 != 0) return SFI_ERR_SHAPE;
  if ((long long)s->B * s->Hkv * pk->p_max >= (1LL << 31)) return SFI_ERR_SHAPE;
  if (pk->p_max < p->n_sink) return SFI_ERR_SHAPE;
  return SFI_OK;
}

#define SFI_TRY(x)                     \
  do {                                 \
    sfi_status _r = (x);               \
    if (_r != SFI_OK) return _r;       \
  } while (0)

}  // namespace

// Arguments of a dense-attention call (all but the scratch): shared by the
// workspace and the allocation-free entry points.
sfi_status check_dense_call(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L, const sfi_bf16* q,
                            const float* out, const sfi_dense_extras* extras) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_kv(kv));
  SFI_TRY(check_L(shape, L));
  if (!q || !out) return SFI_ERR_INVALID_ARG;
  if (extras) {
    if ((extras->logits || extras->probs) && extras->ld < L) return SFI_ERR_SHAPE;
    if (extras->probs && !extras->lse) return SFI_ERR_INVALID_ARG;
    if (extras->lse_cand && (extras->cand_lo < 0 || extras->cand_hi > L || extras->cand_lo >= extras->cand_hi))
      return SFI_ERR_SHAPE;
  }
  if (!aligned16(q)) return SFI_ERR_INVALID_ARG;
  return SFI_OK;
}

namespace {

// Shared bodies of the attention entry points with and without the fused
// append of the step's token (tok == nullptr: none).
sfi_status dense_attn_impl(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L, const StepToken* tok,
                           const sfi_bf16* q, float* out, const sfi_dense_extras* extras, void* ws,
                           size_t ws_bytes, sfi_stream stream) {
  SFI_TRY(check_dense_call(shape, kv, L, q, out, extras));
  if (!ws || !aligned16(ws)) return SFI_ERR_WORKSPACE;
  const size_t part_bytes = ws_bytes > 256 ? ws_bytes - 256 : 0;
  return run_dense_attn(*shape, *kv, L, q, out, extras, static_cast<int*>(ws),
                        reinterpret_cast<float*>(static_cast<char*>(ws) + 256), part_bytes,
                        (cudaStream_t)stream, nullptr, nullptr, tok);
}

sfi_status fast_attn_impl(const sfi_shape* shape, const sfi_params* params, const sfi_paged_kv* kv, int32_t L,
                          const StepToken* tok, const sfi_bf16* q, const sfi_packed* packed, float* out,
                          float* lse, void* ws, size_t ws_bytes, sfi_stream stream) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_params(params));
  SFI_TRY(check_kv(kv));
  SFI_TRY(check_sparse_L(shape, params, L));
  SFI_TRY(check_packed(shape, params, packed));
  if (!q || !out) return SFI_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws)) return SFI_ERR_WORKSPACE;
  if (!aligned16(q)) return SFI_ERR_INVALID_ARG;
  const size_t part_bytes = ws_bytes > 256 ? ws_bytes - 256 : 0;
  return run_fast_attn(*shape, *params, *kv, L, q, *packed, out, lse, static_cast<int*>(ws),
                       reinterpret_cast<float*>(static_cast<char*>(ws) + 256), part_bytes,
                       (cudaStream_t)stream, nullptr, nullptr, tok);
}

}  // namespace
}  // namespace sfi

using namespace sfi;

extern "C" {

const char* sfi_status_str(sfi_status s) {
  switch (s) {
    case SFI_OK: return "ok";
    case SFI_ERR_INVALID_ARG: return "invalid argument";
    case SFI_ERR_SHAPE: return "invalid shape";
    case SFI_ERR_UNSUPPORTED: return "unsupported configuration";
    case SFI_ERR_CUDA: return "CUDA runtime error";
    case SFI_ERR_DEVICE_CHECK: return "device-side bounds check failed";
    case SFI_ERR_TIMEOUT: return "device-side wait timed out";
    case SFI_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* sfi_version(void) { return "sfi-b200 0.1 (sm_100a)"; }

sfi_status sfi_workspace_size(const sfi_shape* shape, const sfi_params* params, size_t* bytes) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_params(params));
  if (!bytes) return SFI_ERR_INVALID_ARG;
  *bytes = ws_layout(*shape, *params).total;
  return SFI_OK;
}

sfi_status sfi_packed_rows(const sfi_shape* shape, const sfi_params* params, int32_t* p_max) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_params(params));
  if (!p_max) return SFI_ERR_INVALID_ARG;
  *p_max = packed_rows_capacity(*shape, *params);
  return SFI_OK;
}

sfi_status sfi_budget(const sfi_params* params, int32_t L, int32_t* K) {
  SFI_TRY(check_params(params));
  if (!K) return SFI_ERR_INVALID_ARG;
  const int k = budget_k(*params, L);
  if (k < 1) return SFI_ERR_SHAPE;
  *K = k;
  return SFI_OK;
}

sfi_status sfi_append_kv(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L,
                         const sfi_bf16* k_new, const sfi_bf16* v_new, sfi_stream stream) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_kv(kv));
  SFI_TRY(check_L(shape, L));
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return SFI_ERR_INVALID_ARG;
  return run_append(*shape, *kv, L, k_new, v_new, (cudaStream_t)stream);
}

sfi_status sfi_key_norms(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t pos_lo,
                         int32_t pos_hi, sfi_stream stream) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_kv(kv));
  if (!kv->key_norms) return SFI_ERR_INVALID_ARG;
  if (pos_lo < 0 || pos_hi < pos_lo || pos_hi > shape->max_pages * kPage) return SFI_ERR_SHAPE;
  return run_key_norms(*shape, *kv, pos_lo, pos_hi, (cudaStream_t)stream);
}

sfi_status sfi_dense_attn(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L,
                          const sfi_bf16* q, float* out, const sfi_dense_extras* extras,
                          void* ws, size_t ws_bytes, sfi_stream stream) {
  return dense_attn_impl(shape, kv, L, nullptr, q, out, extras, ws, ws_bytes, stream);
}

sfi_status sfi_dense_attn_append(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L,
                                 const sfi_bf16* k_new, const sfi_bf16* v_new, const sfi_bf16* q,
                                 float* out, const sfi_dense_extras* extras, void* ws, size_t ws_bytes,
                                 sfi_stream stream) {
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return SFI_ERR_INVALID_ARG;
  const StepToken tok{k_new, v_new};
  return dense_attn_impl(shape, kv, L, &tok, q, out, extras, ws, ws_bytes, stream);
}

sfi_status sfi_attn_probs(const sfi_shape* shape, int32_t L, const float* logits, int64_t ld,
                          const float* lse, float* probs, sfi_stream stream) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_L(shape, L));
  if (!logits || !lse || !probs) return SFI_ERR_INVALID_ARG;
  if (ld < L) return SFI_ERR_SHAPE;
  return run_attn_probs(*shape, L, logits, ld, lse, probs, (cudaStream_t)stream);
}

sfi_status sfi_fast_attn(const sfi_shape* shape, const sfi_params* params,
                         const sfi_paged_kv* kv, int32_t L, const sfi_bf16* q,
                         const sfi_packed* packed, float* out, float* lse, void* ws,
                         size_t ws_bytes, sfi_stream stream) {
  return fast_attn_impl(shape, params, kv, L, nullptr, q, packed, out, lse, ws, ws_bytes, stream);
}

sfi_status sfi_fast_attn_append(const sfi_shape* shape, const sfi_params* params,
                                const sfi_paged_kv* kv, int32_t L, const sfi_bf16* k_new,
                                const sfi_bf16* v_new, const sfi_bf16* q, const sfi_packed* packed,
                                float* out, float* lse, void* ws, size_t ws_bytes, sfi_stream stream) {
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return SFI_ERR_INVALID_ARG;
  const StepToken tok{k_new, v_new};
  return fast_attn_impl(shape, params, kv, L, &tok, q, packed, out, lse, ws, ws_bytes, stream);
}

sfi_status sfi_select_scores(const sfi_shape* shape, const sfi_params* params,
                             const sfi_paged_kv* kv, int32_t L, const float* logits, int64_t ld,
                             const float* lse_cand, float* scores, void* ws, size_t ws_bytes,
                             sfi_stream stream) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_params(params));
  SFI_TRY(check_sparse_L(shape, params, L));
  if (!kv || !kv->key_norms || !logits || !lse_cand || !scores) return SFI_ERR_INVALID_ARG;
  if (ld < L) return SFI_ERR_SHAPE;
  const WsLayout w = ws_layout(*shape, *params);
  if (!ws || ws_bytes < w.total) return SFI_ERR_WORKSPACE;
  const int nC = L - params->n_recent - params->n_sink;
  return run_select_scores(*shape, *params, *kv, L, logits, ld, lse_cand, scores, nC,
                           static_cast<char*>(ws) + w.stat_off, (cudaStream_t)stream);
}

sfi_status sfi_topk_workspace_size(int32_t rows, int32_t n, size_t* bytes) {
  if (!bytes) return SFI_ERR_INVALID_ARG;
  if (rows < 0 || n < 1) return SFI_ERR_SHAPE;
  if (n > topk_max_n()) return SFI_ERR_UNSUPPORTED;
  *bytes = 0;   // the top-K keeps its state on chip
  return SFI_OK;
}

sfi_status sfi_topk(int32_t rows, int32_t n, const float* scores, int64_t ld_s, int32_t K,
                    int32_t offset, int32_t* idx, int64_t ld_i, void* ws, size_t ws_bytes,
                    sfi_stream stream) {
  if (!scores || !idx) return SFI_ERR_INVALID_ARG;
  if (rows < 0 || n < 1 || K < 1 || K > n || ld_s < n || ld_i < K) return SFI_ERR_SHAPE;
  if (n > topk_max_n()) return SFI_ERR_UNSUPPORTED;
  (void)ws;
  (void)ws_bytes;
  return run_topk(rows, n, scores, ld_s, K, offset, idx, ld_i, nullptr, 0, (cudaStream_t)stream);
}

sfi_status sfi_select(const sfi_shape* shape, const sfi_params* params, const sfi_paged_kv* kv,
                      int32_t L, const float* logits, int64_t ld, const float* lse_cand,
                      int32_t* sel_idx, int32_t sel_ld, int32_t* K_out, void* ws,
                      size_t ws_bytes, sfi_stream stream) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_params(params));
  SFI_TRY(check_sparse_L(shape, params, L));
  if (!kv || !kv->key_norms || !logits || !lse_cand || !sel_idx) return SFI_ERR_INVALID_ARG;
  if (ld < L) return SFI_ERR_SHAPE;
  const int K = budget_k(*params, L);
  if (K < 1) return SFI_ERR_SHAPE;
  if (sel_ld < K) return SFI_ERR_SHAPE;
  const WsLayout w = ws_layout(*shape, *params);
  if (!ws || ws_bytes < w.total) return SFI_ERR_WORKSPACE;
  const int nC = L - params->n_recent - params->n_sink;
  float* scores = reinterpret_cast<float*>(static_cast<char*>(ws) + w.sel_off);
  const int ld_s = (nC + 3) / 4 * 4;
  cudaStream_t st = (cudaStream_t)stream;
  if (nC > topk_max_n()) return SFI_ERR_UNSUPPORTED;
  void* stat_ws = static_cast<char*>(ws) + w.stat_off;
  SFI_TRY(run_select_scores(*shape, *params, *kv, L, logits, ld, lse_cand, scores, ld_s, stat_ws, st, RowMap(),
                            0xffffffffu, true, true));
  const int rows = shape->B * shape->Hq;
  SFI_TRY(run_topk(rows, nC, scores, ld_s, K, params->n_sink, sel_idx, sel_ld, nullptr, 0, st,
                   select_row_range(*shape, *params, L, stat_ws)));
  if (K_out) *K_out = K;
  return SFI_OK;
}

sfi_status sfi_compact(const sfi_shape* shape, const sfi_params* params, const sfi_paged_kv* kv,
                       int32_t L, const int32_t* sel_idx, int32_t sel_ld, int32_t K,
                       sfi_packed* packed, void* ws, size_t ws_bytes, sfi_stream stream) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_params(params));
  SFI_TRY(check_kv(kv));
  SFI_TRY(check_sparse_L(shape, params, L));
  SFI_TRY(check_packed(shape, params, packed));
  if (!sel_idx) return SFI_ERR_INVALID_ARG;
  const int nC = L - params->n_recent - params->n_sink;
  if (K < 1 || K > nC || sel_ld < K) return SFI_ERR_SHAPE;
  const WsLayout w = ws_layout(*shape, *params);
  if (!ws || ws_bytes < w.total) return SFI_ERR_WORKSPACE;
  uint32_t* bits = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + w.bits_off);
  cudaStream_t st = (cudaStream_t)stream;
  SFI_TRY(run_idx_to_bits(*shape, *params, *kv, L, sel_idx, sel_ld, K, bits, w.bits_ld, st));
  return run_compact_bits(*shape, *params, *kv, bits, w.bits_ld, *packed,
                          compact_scratch(static_cast<char*>(ws) + w.cmp_off, *shape, *params), L, st);
}

sfi_status sfi_compact_incremental(const sfi_shape* shape, const sfi_params* params, const sfi_paged_kv* kv,
                                   int32_t L, const int32_t* sel_idx, int32_t sel_ld, int32_t K,
                                   sfi_packed* packed, int32_t fresh, void* ws, size_t ws_bytes,
                                   sfi_stream stream) {
  SFI_TRY(check_shape(shape));
  SFI_TRY(check_params(params));
  SFI_TRY(check_kv(kv));
  SFI_TRY(check_sparse_L(shape, params, L));
  SFI_TRY(check_packed(shape, params, packed));
  if (!sel_idx) return SFI_ERR_INVALID_ARG;
  const int nC = L - params->n_recent - params->n_sink;
  if (K < 1 || K > nC || sel_ld < K) return SFI_ERR_SHAPE;
  if (packed->p_max < packed_rows_capacity(*shape, *params)) return SFI_ERR_SHAPE;
  const WsLayout w = ws_layout(*shape, *params);
  if (!ws || ws_bytes < w.total) return SFI_ERR_WORKSPACE;
  uint32_t* bits = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + w.bits_off);
  cudaStream_t st = (cudaStream_t)stream;
  SFI_TRY(run_idx_to_bits(*shape, *params, *kv, L, sel_idx, sel_ld, K, bits, w.bits_ld, st));
  return run_compact_inc(*shape, *params, *kv, bits, w.bits_ld, *packed,
                         compact_scratch(static_cast<char*>(ws) + w.cmp_off, *shape, *params), L, fresh != 0, st);
}

sfi_status sfi_poll_error(const sfi_paged_kv* kv, int32_t* code) {
  if (!kv || !code) return SFI_ERR_INVALID_ARG;
  *code = 0;
  if (!kv->err) return SFI_OK;
  if (cudaMemcpy(code, kv->err, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess) return SFI_ERR_CUDA;
  if (*code != 0 && cudaMemset(kv->err, 0, sizeof(int32_t)) != cudaSuccess) return SFI_ERR_CUDA;
  return SFI_OK;
}

}  // extern "C"
