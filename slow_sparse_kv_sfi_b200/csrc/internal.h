// Internal host-side interfaces shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <utility>
#include <cstddef>
#include <cstdint>

#include "../../include/sfi.h"

namespace sfi {

// Streaming-multiprocessor count of the current device (cached per device).
int num_sms();

// Limit of every device-side pipeline wait, in nanoseconds (sfi_set_wait_limit;
// default 2 s), passed to each launch.
unsigned long long wait_limit_ns();

// Per-device one-time flag (up to 64 devices).
struct DeviceOnce {
  std::atomic<uint64_t> bits{0};
  bool done() const {
    int d = 0;
    cudaGetDevice(&d);
    return (bits.load() >> (d & 63)) & 1u;
  }
  bool mark(cudaError_t e) {
    if (e != cudaSuccess) return false;
    int d = 0;
    cudaGetDevice(&d);
    bits.fetch_or(uint64_t(1) << (d & 63));
    return true;
  }
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launches a kernel of the library with programmatic stream serialization:
// its launch and prologue overlap the tail of the previous kernel on `st`.
// Every kernel of the library waits for that kernel (grid_dep_wait) before
// touching global memory, so stream order is kept.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Workspace carving: the per-op calls take one caller-provided buffer.
struct WsLayout {
  size_t part_off, part_bytes;      // attention split-K partials
  size_t sel_off, sel_bytes;        // Selector: per-(b,kv) stats + scores
  size_t stat_off, stat_bytes;
  size_t cmp_off, cmp_bytes;        // compaction tile counts
  size_t bits_off, bits_bytes;      // selection bitmaps [B*Hq][bits_ld]
  int64_t bits_ld;
  size_t total;
};
WsLayout ws_layout(const sfi_shape& s, const sfi_params& p);

int dense_chunk_tiles(const sfi_shape& s, int L);
int dense_chunks_bound(const sfi_shape& s);
int fast_chunks(const sfi_shape& s, int p_max, int n_recent, int k_est);
size_t attn_part_bytes(int n_items, int G, int D);
int packed_rows_capacity(const sfi_shape& s, const sfi_params& p);
int budget_k(const sfi_params& p, int L);   // -1 if |C| < 1
// queries whose attention distributions the Selector's evidence averages
inline int evidence_window(const sfi_params& p) { return p.evidence_window > 1 ? p.evidence_window : 1; }

// Tensor maps of one layer's paged cache and packed buffer, kept by the
// decode-step driver so that a launch does not encode them again (a host
// cost paid on every call otherwise).  Valid while the pointers and sizes
// they were built from are unchanged; the attention calls check that.
struct AttnMapCache {
  const void* k_pool = nullptr;
  const void* v_pool = nullptr;
  const void* pk = nullptr;
  const void* pv = nullptr;
  uint64_t rows = 0, prows = 0;
  int D = 0;
  bool paged = false, packed = false;
  alignas(128) unsigned char maps[6 * 128];   // the kernel's tensor maps (k, v, pk, pv, pk8, pv8)
};

// Sequences of one launch (per-sequence triggers: a step whose sequences are
// partly slow and partly fast runs the slow path on some, the fast path on
// the others).  Logical row i indexes what the launch owns — work items,
// split-K partials, Selector statistics, scores, top-K rows, selection
// bitmaps, compaction scratch — and stands for sequence b[i], which indexes
// what persists — cache pages, key norms, logits, packed buffers, outputs.
// n == 0: every sequence, in order.  Passed by value into the kernels, so a
// launch queued on the side stream never sees a later step's rows.
constexpr int kMaxRowMap = 256;
struct RowMap {
  int32_t n = 0;
  int16_t b[kMaxRowMap];
  __host__ __device__ __forceinline__ int count(int B) const { return n ? n : B; }
  __host__ __device__ __forceinline__ int phys(int i) const { return n ? (int)b[i] : i; }
};

// The decode step's new token (bf16 [B, Hkv, D] each), appended at L - 1 by
// the attention launch itself.
struct StepToken {
  const sfi_bf16* k_new;
  const sfi_bf16* v_new;
};

// Validation of a dense-attention call's shape, cache, length, query, output
// and extras (api.cu); SFI_OK or the status the entry points return.
sfi_status check_dense_call(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L, const sfi_bf16* q,
                            const float* out, const sfi_dense_extras* extras);

sfi_status run_dense_attn(const sfi_shape& s, const sfi_paged_kv& kv, int L, const sfi_bf16* q,
                          float* out, const sfi_dense_extras* ex, int* ctr, float* part,
                          size_t part_bytes, cudaStream_t st, cudaEvent_t ev_begin, cudaEvent_t ev_end,
                          const StepToken* tok = nullptr, AttnMapCache* maps = nullptr,
                          const RowMap& rows = RowMap(), bool late_trigger = false);
sfi_status run_fast_attn(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv, int L,
                         const sfi_bf16* q, const sfi_packed& pk, float* out, float* lse, int* ctr,
                         float* part, size_t part_bytes, cudaStream_t st, cudaEvent_t ev_begin,
                         cudaEvent_t ev_end, const StepToken* tok = nullptr, AttnMapCache* maps = nullptr,
                         const RowMap& rows = RowMap());
sfi_status run_attn_probs(const sfi_shape& s, int L, const float* logits, int64_t ld,
                          const float* lse, float* probs, cudaStream_t st);

sfi_status run_append(const sfi_shape& s, const sfi_paged_kv& kv, int L, const sfi_bf16* k_new,
                      const sfi_bf16* v_new, cudaStream_t st);
sfi_status run_key_norms(const sfi_shape& s, const sfi_paged_kv& kv, int lo, int hi,
                         cudaStream_t st);

// The prior's statistics of a slow step at context L (key norms only: they
// may run before the step's attention, whose appended token is never a
// candidate) into stat_ws; then the scores, which read them.  with_stats:
// run_select_scores launches the statistics itself first.
sfi_status run_select_stats(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv, int L,
                            void* stat_ws, cudaStream_t st, const RowMap& rows = RowMap());
sfi_status run_select_scores(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv,
                             int L, const float* logits, int64_t ld, const float* lse_cand,
                             float* scores, int64_t ld_s, void* stat_ws,
                             cudaStream_t st, const RowMap& rows = RowMap(),
                             uint32_t window_mask = 0xffffffffu, bool with_stats = true,
                             bool row_range = false);
// row_range: the score kernel also records every row's largest key and key
// complement (the order the top-K uses) at select_row_range(...), [B*Hq][2]
// uint32 at the start of the statistics area, which must be zero before the
// scores and which the top-K given it zeroes again.
uint32_t* select_row_range(const sfi_shape& s, const sfi_params& p, int L, void* stat_ws);
// K largest of every row (ties to the lower index): bitmap bits[rows][ld_b]
// and / or ascending positions idx[rows][ld_i] (+ offset).  No scratch: the
// cluster kernel of topk.cu keeps its state on chip.
// minmax: [rows][2] the largest key and largest key complement of every row
// (see run_select_scores), zeroed again by the top-K; null: found by it.
sfi_status run_topk(int rows, int n, const float* scores, int64_t ld_s, int K, int offset, int32_t* idx,
                    int64_t ld_i, uint32_t* bits, int64_t ld_b, cudaStream_t st, uint32_t* minmax = nullptr);
int topk_max_n();
// Compaction scratch (inside the workspace): per-tile counts of the full
// compaction, and the incremental refresh's mover and hole lists.
struct CompactScratch {
  int32_t* wcounts = nullptr;   // [BH][n_tiles][2]
  size_t wcount_bytes = 0;
  int32_t* mover_pos = nullptr; // [BH][cap]
  int32_t* hole_slot = nullptr; // [BH][cap]
  int cap = 0;                  // packed_rows_capacity
};
size_t compact_scratch_bytes(const sfi_shape& s, const sfi_params& p);
CompactScratch compact_scratch(void* base, const sfi_shape& s, const sfi_params& p);
sfi_status run_compact_bits(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv,
                            const uint32_t* bits, int64_t ld_b, const sfi_packed& pk,
                            const CompactScratch& cs, int L_slow, cudaStream_t st,
                            const RowMap& rows = RowMap());
// fresh: build from scratch (sinks + union ascending) whatever the buffer holds
sfi_status run_compact_inc(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv,
                           const uint32_t* bits, int64_t ld_b, const sfi_packed& pk, const CompactScratch& cs,
                           int L_slow, bool fresh, cudaStream_t st, const RowMap& rows = RowMap());
sfi_status run_idx_to_bits(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv, int L_slow,
                           const int32_t* sel_idx, int sel_ld, int K, uint32_t* bits, int64_t ld_b,
                           cudaStream_t st);
int compact_tiles(int nC);
int score_tile(int G);
int stat_chunks(int nC);

}  // namespace sfi
