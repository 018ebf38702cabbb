// Decode attention for Slow-Fast Inference on sm_100a.
//
// One persistent kernel serves both steps of the method:
//  * slow step ([ES] "2. Metodología", Pasos Lentos; [FR] "A. Le Paradigme
//    Lente-Rapide"; [ZH] "2.1"): dense attention over every page of the
//    context; optionally also writes the logits z and the candidate-range
//    log-sum-exp the Selector needs;
//  * fast step ([ES] Pasos Rápidos; [NL] Methodologie; [ZH] "2.3"
//    显存合并的内核): attention over the contiguous packed buffer (sinks +
//    selected rows, per-head bitmask) followed by the recent window read
//    straight from the pages.
//
// Work: the token range of every (sequence, KV head) is cut into chunks; a
// work item is one chunk.  Grid = one CTA per SM, items round-robin.  Warp 4
// is the producer: it walks the items' 16-row tiles and issues TMA loads (a
// 16x64 bf16 box per 128-byte column block, 128B-swizzled) for K and V into a
// ring of shared-memory stages of 4 tiles, with mbarrier completion.  Warps
// 0-3 each take one tile of a stage and run the group's contraction on the
// tensor cores with tokens as the M dimension:
//    S^T[16 tok x 8 heads] = K_tile[16 x D] . Q^T[D x 8]     (mma m16n8k16)
//    O^T[D x 8 heads]     += V_tile^T[D x 16] . P^T[16 x 8]
// P^T comes from the S^T accumulator through movmatrix (an 8x8 transpose in
// registers); P is split into bf16 hi + lo parts so the PV product keeps
// ~16 bits of P.  Online softmax per head; at the end of an item the four
// warps merge through shared memory and write one partial (m, l, l_cand,
// O) per query head; attn_combine merges the partials of every chunk.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace sfi {

constexpr int kConsumerWarps = 4;   // consumer warps of one head group: one per tile of a stage
constexpr int kBoxBytes = 16 * 128;   // 16 rows x 128 bytes: one column block of a tile
constexpr long kDenseItemsPerSm = 8;  // dense step: work items per SM
constexpr long kFastItemTiles = 64;   // fast step: target tiles per work item
// A fast launch with two CTAs per SM leaves this many CTA slots empty.  In a
// decode loop the next layer's CTAs enter them while this launch's last items
// finish, instead of waiting for its last CTAs to leave (128K workload: fast
// layer-step 30.4 -> 26.8 us).
constexpr int kFastFreeSlots = 32;

enum AttnMode : int { kDense = 0, kDenseExtras = 1, kFast = 2 };

struct AttnArgs {
  int B, Hq, Hkv, G, L;
  int num_pages, max_pages;
  const int32_t* page_table;
  const __nv_bfloat16* q;
  float* part;          // [n_items][G][D + 4]
  int* ctr;             // work counter (zero on entry; the combine kernel re-zeroes it)
  int n_chunks;         // chunks per (b, kv head)
  int chunk_tiles;      // dense: tiles per chunk (a multiple of the stage, <= kMaxChunkTiles)
  int n_items;
  float scale_log2;     // log2(e) / sqrt(D)
  float scale;          // 1 / sqrt(D)
  // dense extras
  float* logits;
  int64_t ld;
  int cand_lo, cand_hi;
  // fast
  const int32_t* n_rows;
  const uint32_t* headmask;
  int p_max;
  int rec_lo;           // L - n_recent
  int* err;
  unsigned long long wait_ns;   // limit of every pipeline wait
  // 1: let the dependent launches be scheduled only once this CTA has no
  // work item left (a persistent grid that signals at its start has the next
  // kernel's CTAs take every SM it frees, ahead of other streams' kernels)
  int late_trigger;
  // the step's token, appended at L - 1 by the item holding the last tile
  // (k_new == nullptr: already in the cache)
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_pool;
  __nv_bfloat16* v_pool;
  float* norms;
  int64_t norm_ld;
  RowMap rows;          // the sequences of this launch
};

constexpr int kMaxChunkTiles = 256;
constexpr int kMaxBH = 512;

// Shared-memory plan.  A tile is 16 rows of K (or V): one TMA box of
// [D/64 column blocks][16 rows][128 B], 128B-swizzled.  Each consumer warp
// takes TT tiles of every stage, so a stage holds 4 * TT tiles of K and V.
// NT head groups of 8: the consumer warps come in NT sets of four, set s
// taking heads 8s .. 8s + 7 of every tile (the sets read the same tiles).
// kCps CTAs share an SM; together they keep about 192 KB of copies in flight.
template <int D, int NT>
struct Plan {
  static constexpr int kCW = kConsumerWarps * NT;        // consumer warps
  static constexpr int kThreads = (kCW + 1) * 32;        // + the producer warp
  static constexpr int kCps = (NT == 1) ? 2 : 1;
  static constexpr int TT = (NT == 1 && kCps == 1) ? 2 : 1;
  static constexpr int kTPS = 4 * TT;
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kHalves * kBoxBytes;
  static constexpr int kKBytes = kTPS * kTileBytes;
  static constexpr int kStageBytes = 2 * kKBytes;
  static constexpr int kStages = (192 * 1024 / kCps) / kStageBytes;
  static constexpr int kHeads = NT * 8;
  // Registers per thread: with two CTAs per SM at most 152 (19 x 256 per
  // warp), which leaves 16 K registers per SM for the merge kernel that runs
  // beside them after a fast step.
  static constexpr int kMaxRegs = kCps == 2 ? 152 : 168;
  static constexpr int kQBytes = kHeads * D * 2;
};

struct StageMeta {
  int item;        // work item, or -1: no more work
  int b, g;
  int flags;       // bit 0: first stage of the item, bit 1: last stage of the item
  int ntiles;      // tiles in this stage
  int kinds;       // 2 bits per tile: 0 page, 1 packed, 2 skipped (bad page-table entry)
  int pos0[8];     // page tiles: cache position of row 0; packed: packed row
  int pad[2];
};
static_assert(sizeof(StageMeta) == 64, "meta size");

template <int D, int NT>
struct Smem {
  using P = Plan<D, NT>;
  static constexpr int kStages = P::kStages;
  static constexpr int kMaskOff = kStages * P::kStageBytes;
  static constexpr int kMaskBytes = kStages * P::kTPS * 16 * 4;
  static constexpr int kQOff = kMaskOff + kMaskBytes;
  static constexpr int kMetaOff = kQOff + kStages * P::kQBytes;
  static constexpr int kPtOff = kMetaOff + kStages * (int)sizeof(StageMeta);
  static constexpr int kNrOff = kPtOff + kMaxChunkTiles * 4;
  static constexpr int kBarOff = kNrOff + kMaxBH * 4;
  static constexpr int kTotal = kBarOff + 2 * kStages * 8 + 64 + 1024;   // + alignment slack
  static_assert(kTotal * P::kCps + 1024 * P::kCps <= 228 * 1024, "shared memory budget");
};

// Tile range and page range of one work item.
struct Item {
  int bg, b, g;
  int t_begin, t_end;     // tiles of the item
  int t_total;            // tiles of the whole (b, kv head); the last one holds position L - 1
  int n_packed_tiles;     // tiles before this index are packed-buffer tiles
  int first_page;         // page number of tile n_packed_tiles (fast) or tile 0 (dense)
};

template <int MODE, int TPS>
__device__ __forceinline__ Item decode_item(const AttnArgs& a, int item, const int* nrows_s) {
  Item it;
  const int bgl = item / a.n_chunks;   // logical (row of the launch, kv head)
  const int c = item - bgl * a.n_chunks;
  const int bl = bgl / a.Hkv;
  it.g = bgl - bl * a.Hkv;
  it.b = a.rows.phys(bl);
  it.bg = it.b * a.Hkv + it.g;
  if (MODE != kFast) {
    const int T = (a.L + kPage - 1) / kPage;
    it.t_total = T;
    it.t_begin = min(T, c * a.chunk_tiles);
    it.t_end = min(T, it.t_begin + a.chunk_tiles);
    it.n_packed_tiles = 0;
    it.first_page = 0;
  } else {
    int nr = nrows_s[it.bg];
    if (nr < 0 || nr > a.p_max) nr = nr < 0 ? 0 : a.p_max;   // reported by the combine kernel
    it.n_packed_tiles = (nr + kPage - 1) / kPage;
    it.first_page = a.rec_lo / kPage;
    const int T = it.n_packed_tiles + ((a.L - 1) / kPage - it.first_page + 1);
    it.t_total = T;
    int ct = (T + a.n_chunks - 1) / a.n_chunks;
    ct = (ct + TPS - 1) / TPS * TPS;
    it.t_begin = min(T, c * ct);
    it.t_end = min(T, it.t_begin + ct);
  }
  return it;
}

// Page number of page tile `t` of the item (t >= n_packed_tiles).
__device__ __forceinline__ int item_page(const Item& it, int t) {
  return it.first_page + (t - it.n_packed_tiles);
}

// Address of 16-byte chunk `ci` (0 .. D/8-1) of row `row` in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t swz(uint32_t tile_base, int row, int ci) {
  return tile_base + (ci >> 3) * kBoxBytes + row * 128 + ((((ci & 7) ^ (row & 7))) << 4);
}

// Tensor maps of one launch.  k, v: the page pools, one box = one 16-row
// tile of one (page, KV head).  pk, pv: the packed buffers, one box = one
// tile; pk8, pv8: the packed buffers viewed as [tiles][column block][16
// rows][64 columns], one box = a whole stage of consecutive tiles.
struct Maps {
  CUtensorMap k, v, pk, pv, pk8, pv8;
};

template <int D, int NT, int MODE>
__global__ void __maxnreg__((Plan<D, NT>::kMaxRegs))
    attn_kernel(const __grid_constant__ Maps maps, const __grid_constant__ AttnArgs a) {
  using S = Smem<D, NT>;
  using P = Plan<D, NT>;
  constexpr int kStages = S::kStages;
  constexpr int TT = P::TT;
  constexpr int kTPS = P::kTPS;
  constexpr int kMT = D / 16;   // 16-wide slices of D

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem + S::kMaskOff);
  uint8_t* sq = smem + S::kQOff;
  StageMeta* smeta = reinterpret_cast<StageMeta*>(smem + S::kMetaOff);
  int* ptbuf = reinterpret_cast<int*>(smem + S::kPtOff);
  int* nrows_s = reinterpret_cast<int*>(smem + S::kNrOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);
  uint64_t* mergebar = empty + kStages + 1;   // the consumer warps' merge at an item's end
  // One head group (NT = 1): the consumer warps merge their states of an
  // item in shared memory and write one partial per item.
  constexpr bool kMerge = NT == 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], P::kCW);
    }
    mbar_init(mergebar, P::kCW);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Ordering with the previous kernels of the stream.  The producer issues
  // its first copies at once: the query, the pages, the page table, the
  // packed buffers and n_rows are written by no kernel of this library that
  // lets its dependents start early (the append and the compaction signal
  // them only at exit), so the copies overlap the previous kernels' tails.
  // The producer waits before it touches the work counter (reset by the
  // previous combine).  The dense consumers wait at once (they write logits
  // from their first tile on).  The fast consumers let the next kernel start
  // at once; they read shared memory only until the end of their first item
  // and wait there, before their first partial (the previous combine may
  // still read the partials).  Every write that a kernel before this one
  // reads or writes (the partials, the counter) thus follows a wait, and the
  // waits chain: the previous combine waited for the previous attention,
  // whose consumers waited for the combine before it.
  if (warp != P::kCW) {
    if (MODE != kFast) grid_dep_wait();
    if (!a.late_trigger) grid_dep_launch();
  }

  // ------------------------------------------------------------ producer warp
  if (warp == P::kCW) {
    bool waited = false;
    auto ensure_wait = [&]() {
      if (!waited) {
        grid_dep_wait();
        if (!a.late_trigger) grid_dep_launch();
        waited = true;
      }
    };

    if (lane == 0) {
      prefetch_tensormap(&maps.k);
      prefetch_tensormap(&maps.v);
      if (MODE == kFast) {
        prefetch_tensormap(&maps.pk);
        prefetch_tensormap(&maps.pv);
        prefetch_tensormap(&maps.pk8);
        prefetch_tensormap(&maps.pv8);
      }
    }
    const int BH = a.B * a.Hkv;
    if (MODE == kFast) {
      for (int i = lane; i < BH; i += 32) nrows_s[i] = __ldg(a.n_rows + i);
      __syncwarp();
    }
    const uint64_t policy = l2_policy_evict_first();
    const int G = a.G;
    // CTA i starts on item i without a round trip to memory (the grid is no
    // larger than the CTAs that fit at once); the later items come from a
    // global counter, offset by the grid.  The next
    // item's index and page table entries are fetched ahead so their latency
    // overlaps the current item's copies.
    int nxt = blockIdx.x;
    int pf[kMaxChunkTiles / 32];
    auto prefetch = [&](int item, int* regs) {
#pragma unroll
      for (int j = 0; j < kMaxChunkTiles / 32; ++j) regs[j] = 0;
      if (item >= a.n_items) return;
      const Item it = decode_item<MODE, kTPS>(a, item, nrows_s);
      const int p_lo = item_page(it, max(it.t_begin, it.n_packed_tiles));
      const int p_hi = item_page(it, max(it.t_end, it.n_packed_tiles));
      const int32_t* row = a.page_table + (size_t)it.b * a.max_pages;
#pragma unroll
      for (int j = 0; j < kMaxChunkTiles / 32; ++j) {
        const int p = p_lo + j * 32 + lane;
        if (p < p_hi) regs[j] = __ldg(row + p);
      }
    };
    prefetch(nxt, pf);
    int slot = 0;
    uint32_t phase = 0;
    int inflight = 0;
    bool ok = true;
    // The next item is drawn late in the current one (two stages before its
    // end, leaving time to fetch its page-table entries): a CTA holds no work
    // it cannot start soon, so CTAs that finish early take what remains.
    bool drawn = false;
    auto draw_next = [&]() {
      ensure_wait();
      int v = 0;
      if (lane == 0) v = atomicAdd(a.ctr, 1) + (int)gridDim.x;
      nxt = __shfl_sync(0xffffffffu, v, 0);
      prefetch(nxt, pf);
      drawn = true;
    };
    while (ok) {
      const int item = nxt;
      // publish this item's page entries
      __syncwarp();
#pragma unroll
      for (int j = 0; j < kMaxChunkTiles / 32; ++j) ptbuf[j * 32 + lane] = pf[j];
      __syncwarp();
      drawn = item >= a.n_items;
      // one stage per kTPS tiles; item == n_items: stop.  A dense item without
      // tiles still sends one (empty) stage so the consumers write its
      // partial; a fast-step chunk past its (b, kv head)'s tiles is skipped
      // (the combine kernel reads only the chunks holding tiles), so its CTA
      // does not take one real item more than the others at the end.
      Item it{};
      int nst = 1;
      int p_lo = 0;
      if (item < a.n_items) {
        it = decode_item<MODE, kTPS>(a, item, nrows_s);
        nst = max(1, (it.t_end - it.t_begin + kTPS - 1) / kTPS);
        p_lo = item_page(it, max(it.t_begin, it.n_packed_tiles));
        // the item holding position L - 1 first appends the step's token
        // there (the whole warp), before any copy of that tile is issued.  A
        // fast step appends without waiting: the kernels that may still run
        // (earlier attention launches and their combines) neither read nor
        // write that row of this cache (the library's ordering rule).
        if (a.k_new && it.t_begin < it.t_end && it.t_end == it.t_total) {
          if (MODE != kFast) ensure_wait();
          const int pos = a.L - 1;
          append_row_warp<D>(lane, it.bg, it.g, pos, ptbuf[pos / kPage - p_lo], a.Hkv, a.num_pages, a.k_pool,
                             a.v_pool, a.k_new, a.v_new, a.norms, a.norm_ld, a.err);
          __syncwarp();
        }
        if (MODE == kFast && it.t_begin >= it.t_end) {
          draw_next();
          continue;
        }
      }
      for (int st = 0; st < nst; ++st) {
        if (!drawn && st >= nst - 2) draw_next();
        bool good = true;
        if (lane == 0) {
          good = !*abort_flag && mbar_wait(&empty[slot], phase ^ 1, a.err, kSiteAttnProducer, a.wait_ns);
          if (good) {
            StageMeta& m = smeta[slot];
            if (item >= a.n_items) {
              m.item = -1;
              m.ntiles = 0;
              mbar_arrive_expect_tx(&full[slot], 0);
            } else {
              uint32_t bytes = 0;
              const int t0 = it.t_begin + st * kTPS;
              const int nt = max(0, min(kTPS, it.t_end - t0));
              int kinds = 0;
              m.item = item;
              m.b = it.b;
              m.g = it.g;
              m.flags = (st == 0 ? 1 : 0) | (st == nst - 1 ? 2 : 0);
              m.ntiles = nt;
              uint8_t* sk = smem + slot * P::kStageBytes;
              uint8_t* sv = sk + P::kKBytes;
              if (st == 0) bytes += G * D * 2;
              int ys[kTPS];
              int n_pk = 0;   // packed tiles lead the stage
              for (int i = 0; i < nt; ++i) {
                const int t = t0 + i;
                int kind, y, pos0;
                if (MODE == kFast && t < it.n_packed_tiles) {
                  kind = 1;
                  pos0 = t * kPage;
                  y = it.bg * a.p_max + pos0;
                  bytes += 2 * P::kTileBytes + 64;
                  ++n_pk;
                } else {
                  const int pg = item_page(it, t);
                  const int page = ptbuf[pg - p_lo];
                  pos0 = pg * kPage;
                  if ((unsigned)page >= (unsigned)a.num_pages) {
                    kind = 2;
                    y = 0;
                    latch_error(a.err, SFI_ERR_DEVICE_CHECK, kSiteAttnPage);
                  } else {
                    kind = 0;
                    y = (page * a.Hkv + it.g) * kPage;
                    bytes += 2 * P::kTileBytes;
                  }
                }
                kinds |= kind << (2 * i);
                m.pos0[i] = pos0;
                ys[i] = y;
              }
              m.kinds = kinds;
              mbar_arrive_expect_tx(&full[slot], bytes);
              if (st == 0)
                bulk_load(sq + slot * P::kQBytes, a.q + ((size_t)it.b * a.Hq + it.g * G) * D, G * D * 2,
                          &full[slot]);
              int i0 = 0;
              if (MODE == kFast && n_pk > 0) {
                // head masks of the stage's packed tiles: one copy
                bulk_load(smask + slot * kTPS * 16, a.headmask + (size_t)it.bg * a.p_max + m.pos0[0],
                          n_pk * 64, &full[slot]);
                if (n_pk == kTPS) {
                  // a whole stage of consecutive packed tiles: one box each for K and V
                  const int tile0 = ys[0] / kPage;
                  tma_load_4d(sk, &maps.pk8, 0, 0, 0, tile0, &full[slot], policy);
                  tma_load_4d(sv, &maps.pv8, 0, 0, 0, tile0, &full[slot], policy);
                  i0 = nt;
                }
              }
              for (int i = i0; i < nt; ++i) {
                const int kind = (kinds >> (2 * i)) & 3;
                if (kind == 2) continue;
                const CUtensorMap* mk = kind == 1 ? &maps.pk : &maps.k;
                const CUtensorMap* mv = kind == 1 ? &maps.pv : &maps.v;
                tma_load_3d(sk + i * P::kTileBytes, mk, 0, ys[i], 0, &full[slot], policy);
                tma_load_3d(sv + i * P::kTileBytes, mv, 0, ys[i], 0, &full[slot], policy);
              }
            }
          } else {
            *abort_flag = 1;
          }
        }
        good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
        if (!good) {
          ok = false;
          break;
        }
        inflight = min(inflight + 1, kStages);
        if (++slot == kStages) {
          slot = 0;
          phase ^= 1;
        }
      }
      if (item >= a.n_items) break;
    }
    if (a.late_trigger) grid_dep_launch();   // no item left for this CTA
    if (!ok && lane == 0) {
      // Drain: wait (bounded) for the copies of stages still in flight so no
      // TMA write lands after this CTA has left the SM.
      for (int k = 0; k < inflight; ++k) {
        if (--slot < 0) {
          slot = kStages - 1;
          phase ^= 1;
        }
        mbar_wait(&full[slot], phase, nullptr, 0);   // own copies: the fixed 2 s limit, whatever wait_ns is
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int r0 = lane >> 2;              // accumulator rows r0, r0 + 8
  const int cq = (lane & 3) * 2;         // accumulator columns cq, cq + 1
  const int rowA = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int chA = lane >> 4;
  const int rowV = (lane & 7) + ((lane >> 4) & 1) * 8;
  const int chV = (lane >> 3) & 1;
  const float NEG_INF = -INFINITY;

  // this warp: tile warp % 4 (+ 4 * tt) of every stage, heads hbase .. hbase + 7
  const int twarp = warp % kConsumerWarps;
  const int hbase = (warp / kConsumerWarps) * 8;
  int slot = 0;
  uint32_t phase = 0;
  uint32_t qb[1][kMT][2];
  float o[1][kMT][4];
  float mrun[1][2], lrun[1][2], lcand[1][2];
  int cur_b = 0, cur_g = 0;
  bool waited = MODE != kFast;   // the dense consumers waited at their start
  uint32_t mphase = 0;           // parity of the next merge barrier phase
  // every consumer warp at the merge barrier (bounded; false: the wait gave up)
  auto merge_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(mergebar);
    const bool ok = mbar_wait(mergebar, mphase, a.err, kSiteAttnConsumer, a.wait_ns);
    mphase ^= 1u;
    return ok;
  };
  for (;;) {
    if (*abort_flag || !mbar_wait(&full[slot], phase, a.err, kSiteAttnConsumer, a.wait_ns)) {
      *abort_flag = 1;
      if (!waited) grid_dep_wait();
      if (a.late_trigger) grid_dep_launch();
      break;
    }
    const StageMeta& m = smeta[slot];
    const int item = m.item;
    if (item < 0) {
      if (!waited) grid_dep_wait();
      if (a.late_trigger) grid_dep_launch();
      break;
    }
    const int flags = m.flags;
    if (flags & 1) {
      // first stage of an item: the group's queries (B operand of S^T) and a fresh state
      cur_b = m.b;
      cur_g = m.g;
      const uint32_t* q32 = reinterpret_cast<const uint32_t*>(sq + slot * P::kQBytes);
#pragma unroll
      for (int nt = 0; nt < 1; ++nt) {
        const int hh = hbase + nt * 8 + r0;
        const bool hv = hh < a.G;
#pragma unroll
        for (int ks = 0; ks < kMT; ++ks) {
          qb[nt][ks][0] = hv ? q32[(hh * D + ks * 16 + cq) / 2] : 0u;
          qb[nt][ks][1] = hv ? q32[(hh * D + ks * 16 + 8 + cq) / 2] : 0u;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          mrun[nt][j] = NEG_INF;
          lrun[nt][j] = 0.f;
          lcand[nt][j] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) o[nt][mt][i] = 0.f;
      }
    }
    // this warp's tiles: warp + 4 * tt
    bool act[TT];
    int kind_[TT], pos0_[TT];
    uint32_t kb_[TT], vb_[TT];
    uint32_t rmask[TT][2];
    bool any = false;
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      const int ti = twarp + 4 * tt;
      kind_[tt] = (m.kinds >> (2 * ti)) & 3;
      act[tt] = ti < m.ntiles && kind_[tt] != 2;
      any |= act[tt];
      pos0_[tt] = m.pos0[ti];
      uint8_t* sk = smem + slot * P::kStageBytes + ti * P::kTileBytes;
      uint8_t* sv = sk + P::kKBytes;
      kb_[tt] = smem_u32(sk);
      vb_[tt] = smem_u32(sv);
      rmask[tt][0] = rmask[tt][1] = 0u;
      if (!act[tt]) continue;
      if (kind_[tt] == 0) {
        const int lo = (MODE == kFast) ? a.rec_lo : 0;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int pos = pos0_[tt] + r0 + 8 * j;
          rmask[tt][j] = (pos < a.L && pos >= lo) ? 0xffffffffu : 0u;
        }
        if (pos0_[tt] + kPage > a.L) {
          // Rows at or beyond L may hold anything: zero their V rows so
          // 0 * garbage cannot poison the PV product.
          const int first_bad = a.L - pos0_[tt];
          const int nchunks = (kPage - first_bad) * (D / 8);
          for (int c = lane; c < nchunks; c += 32) {
            const int row = first_bad + c / (D / 8);
            const int ci = c % (D / 8);
            *reinterpret_cast<uint4*>(sv + (ci >> 3) * kBoxBytes + row * 128 + (ci & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
      } else {
        const uint32_t* mk = smask + (slot * kTPS + ti) * 16;
        rmask[tt][0] = mk[r0];
        rmask[tt][1] = mk[r0 + 8];
      }
    }

    if (any) {
      // S^T = K . Q^T per tile, two independent accumulator chains over D
      float s[TT][1][4];
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        float s2[1][4];
#pragma unroll
        for (int nt = 0; nt < 1; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) s[tt][nt][i] = s2[nt][i] = 0.f;
        if (act[tt]) {
#pragma unroll
          for (int ks = 0; ks < kMT; ks += 2) {
            uint32_t af[4], ag[4];
            ldmatrix_x4(af, swz(kb_[tt], rowA, ks * 2 + chA));
            ldmatrix_x4(ag, swz(kb_[tt], rowA, (ks + 1) * 2 + chA));
#pragma unroll
            for (int nt = 0; nt < 1; ++nt) {
              mma_bf16_16816(s[tt][nt], af, qb[nt][ks][0], qb[nt][ks][1]);
              mma_bf16_16816(s2[nt], ag, qb[nt][ks + 1][0], qb[nt][ks + 1][1]);
            }
          }
        }
#pragma unroll
        for (int nt = 0; nt < 1; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) s[tt][nt][i] += s2[nt][i];
      }

      // mask, scale, online softmax over the warp's TT tiles at once
      uint32_t pb_hi[TT][1][2], pb_lo[TT][1][2];
#pragma unroll
      for (int nt = 0; nt < 1; ++nt) {
        float x[TT][4];
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int hh = hbase + nt * 8 + cq + (i & 1);
            const bool v = (rmask[tt][i >> 1] >> hh) & 1u;
            x[tt][i] = (v && hh < a.G) ? s[tt][nt][i] * a.scale_log2 : NEG_INF;
          }
        if (MODE == kDenseExtras && a.logits) {
#pragma unroll
          for (int tt = 0; tt < TT; ++tt) {
            if (!act[tt] || kind_[tt] != 0) continue;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int hh = hbase + nt * 8 + cq + (i & 1);
              const int pos = pos0_[tt] + r0 + 8 * (i >> 1);
              if (hh < a.G && pos < a.L)
                a.logits[((size_t)cur_b * a.Hq + cur_g * a.G + hh) * a.ld + pos] = s[tt][nt][i] * a.scale;
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float tm = NEG_INF;
#pragma unroll
          for (int tt = 0; tt < TT; ++tt) tm = fmaxf(tm, fmaxf(x[tt][j], x[tt][j + 2]));
          tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
          tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
          tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
          const float mnew = fmaxf(mrun[nt][j], tm);
          const float mref = (mnew == NEG_INF) ? 0.f : mnew;
          const float alpha = fast_exp2(mrun[nt][j] - mref);
          mrun[nt][j] = mnew;
          lrun[nt][j] *= alpha;
          if (MODE == kDenseExtras) lcand[nt][j] *= alpha;
#pragma unroll
          for (int mt = 0; mt < kMT; ++mt) {
            o[nt][mt][j] *= alpha;
            o[nt][mt][j + 2] *= alpha;
          }
#pragma unroll
          for (int tt = 0; tt < TT; ++tt) {
            x[tt][j] = fast_exp2(x[tt][j] - mref);
            x[tt][j + 2] = fast_exp2(x[tt][j + 2] - mref);
            lrun[nt][j] += x[tt][j] + x[tt][j + 2];
            if (MODE == kDenseExtras && kind_[tt] == 0) {
              const int p0 = pos0_[tt] + r0, p1 = p0 + 8;
              if (p0 >= a.cand_lo && p0 < a.cand_hi) lcand[nt][j] += x[tt][j];
              if (p1 >= a.cand_lo && p1 < a.cand_hi) lcand[nt][j] += x[tt][j + 2];
            }
          }
        }
        // P -> bf16 hi + lo, then transpose to the B operand of PV.
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float p0 = x[tt][2 * j], p1 = x[tt][2 * j + 1];
            const uint32_t hi = pack_bf16x2(p0, p1);
            const float2 hf = unpack_bf16x2(hi);
            const uint32_t lo = pack_bf16x2(p0 - hf.x, p1 - hf.y);
            pb_hi[tt][nt][j] = movmatrix_trans(hi);
            pb_lo[tt][nt][j] = movmatrix_trans(lo);
          }
      }

      // O^T += V^T . P^T
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        if (!act[tt]) continue;
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
          uint32_t vf[4];
          ldmatrix_x4_trans(vf, swz(vb_[tt], rowV, mt * 2 + chV));
#pragma unroll
          for (int nt = 0; nt < 1; ++nt) {
            mma_bf16_16816(o[nt][mt], vf, pb_hi[tt][nt][0], pb_hi[tt][nt][1]);
            mma_bf16_16816(o[nt][mt], vf, pb_lo[tt][nt][0], pb_lo[tt][nt][1]);
          }
        }
      }
    }
    __syncwarp();
    const bool item_end = (flags & 2) != 0;
    const int done_slot = slot;   // with kMerge the item's last stage is released after the merge
    if (!(kMerge && item_end) && lane == 0) mbar_arrive(&empty[slot]);
    if (++slot == kStages) {
      slot = 0;
      phase ^= 1;
    }
    if (!item_end) continue;

    // ---- last stage of the item: this warp's partial softmax state (m, l,
    // l_cand and the unnormalised O of each query head) goes to global memory
    // as it is, or (kMerge) first through the merge of the CTA's consumer
    // warps; the combine kernel merges the partials of every item.
#pragma unroll
    for (int nt = 0; nt < 1; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int sh = 4; sh <= 16; sh <<= 1) {
          lrun[nt][j] += __shfl_xor_sync(0xffffffffu, lrun[nt][j], sh);
          if (MODE == kDenseExtras) lcand[nt][j] += __shfl_xor_sync(0xffffffffu, lcand[nt][j], sh);
        }
    if (!waited) {
      grid_dep_wait();
      waited = true;
    }
    if constexpr (kMerge) {
      // This warp's state into its own tiles of the stage just consumed (K
      // tile: O of its 8 head slots, [head][D] with the column rotated by 8 *
      // head against bank conflicts; V tile: m, l, l_cand per head), then,
      // after every consumer warp's, thread t of the 4 warps merges column
      // t % D of heads t / D, t / D + 128 / D, ...: one partial per item.
      uint8_t* stage = smem + done_slot * P::kStageBytes;
      float* so = reinterpret_cast<float*>(stage + twarp * P::kTileBytes);
      float* sml = reinterpret_cast<float*>(stage + P::kKBytes + twarp * P::kTileBytes);
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int hh = cq + (i & 1);
          const int d = mt * 16 + r0 + (i >> 1) * 8;
          so[hh * D + ((d + 8 * hh) & (D - 1))] = o[0][mt][i];
        }
      if (lane < 4) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          sml[(cq + j) * 3] = mrun[0][j];
          sml[(cq + j) * 3 + 1] = lrun[0][j];
          sml[(cq + j) * 3 + 2] = lcand[0][j];
        }
      }
      const bool ok = merge_sync();   // every warp's state is in the stage
      if (ok) {
        float* part = a.part + (size_t)item * a.G * (D + 4);
        const int t = twarp * 32 + lane;
        const int d = t % D;
        for (int hh = t / D; hh < a.G; hh += (kConsumerWarps * 32) / D) {
          float mw[kConsumerWarps];
          float M = NEG_INF;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            mw[w] = reinterpret_cast<const float*>(stage + P::kKBytes + w * P::kTileBytes)[hh * 3];
            M = fmaxf(M, mw[w]);
          }
          const float mref = (M == NEG_INF) ? 0.f : M;
          float ov = 0.f, lv = 0.f, lcv = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            const float sc = fast_exp2(mw[w] - mref);
            const float* ml = reinterpret_cast<const float*>(stage + P::kKBytes + w * P::kTileBytes) + hh * 3;
            ov += sc * reinterpret_cast<const float*>(stage + w * P::kTileBytes)[hh * D + ((d + 8 * hh) & (D - 1))];
            lv += sc * ml[1];
            if (MODE == kDenseExtras) lcv += sc * ml[2];
          }
          part[hh * (D + 4) + d] = ov;
          if (d == 0) {
            part[hh * (D + 4) + D] = M;
            part[hh * (D + 4) + D + 1] = lv;
            part[hh * (D + 4) + D + 2] = lcv;
          }
        }
      }
      if (!ok) *abort_flag = 1;
      // The stage goes back to the producer once every consumer warp has
      // arrived on its empty barrier, each after its own reads above.
      fence_proxy_async_smem();   // the generic writes above before the stage's next copies
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[done_slot]);
    } else {
      float* part = a.part + ((size_t)item * kConsumerWarps + twarp) * a.G * (D + 4);
#pragma unroll
      for (int nt = 0; nt < 1; ++nt) {
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int hh = hbase + nt * 8 + cq + (i & 1);
            const int d = mt * 16 + r0 + (i >> 1) * 8;
            if (hh < a.G) part[hh * (D + 4) + d] = o[nt][mt][i];
          }
        if (lane < 4) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int hh = hbase + nt * 8 + cq + j;
            if (hh < a.G) {
              part[hh * (D + 4) + D] = mrun[nt][j];
              part[hh * (D + 4) + D + 1] = lrun[nt][j];
              part[hh * (D + 4) + D + 2] = lcand[nt][j];
            }
          }
        }
      }
    }
  }
}

// Merge the partials of every (b, query head): one CTA of NW warps each, one
// pass.  Warp w folds partials w, w + NW, ... (IN loads in flight per lane,
// each partial's m, l, l_C and a 4-column slice of O per lane) into a running
// (m, l, l_C, O) with online rescaling; the warps' states meet in shared
// memory, where thread d merges column d.
//  - After a dense step: 24 warps, eight loads in flight (the merge is on the
//    path to the Selector).
//  - After a fast step whose attention runs one CTA per SM (G > 8;
//    attn_combine_fast_kernel): 7 warps of at most 64 registers and 4 KB of
//    shared memory, which fit on an SM beside that CTA.
//  - After a fast step with two attention CTAs per SM (G <= 8), whose CTAs
//    wrote one merged partial per item (attn_combine_merged_kernel): 4 warps
//    of at most 96 registers, ten partials in flight per warp, which fit
//    beside the two CTAs.
//  After a fast step the merge lets the next launch start at once, so it
//  runs while the attention finishes and the next layer's attention starts,
//  instead of holding an SM.
//  ppi: partials per work item (one per consumer warp, or 1 when merged).
constexpr int kCombWarps = 24;
constexpr int kCombWarpsFast = 7;
constexpr int kCombWarpsMerged = 4;

template <int D, int NW, int KIN>
__device__ __forceinline__ void combine_body(const float* __restrict__ part, int n_chunks, int B, int Hq, int Hkv,
                                             int G, float* __restrict__ out, float* __restrict__ lse,
                                             float* __restrict__ lse_cand, const int32_t* n_rows, int p_max,
                                             int rec_tiles, int tps, int* err, int* ctr, int early, int ppi,
                                             const RowMap& rows) {
  // After a fast step the next launch may start before this one has waited:
  // it is the next layer's attention, whose consumers wait before their
  // first partial and whose producer waits before it touches the counter.
  if (early) {
    grid_dep_launch();
    grid_dep_wait();
  } else {
    grid_dep_enter();
  }
  constexpr int kPer = D / 32;     // columns of O per lane
  static_assert(kPer == 4 || kPer == 2, "head dim");
  __shared__ float red[NW][D + 4];
  if (blockIdx.x == 0 && threadIdx.x == 0) ctr[0] = 0;   // the attention kernel is done with it
  const int bl = blockIdx.x / Hq, hq = blockIdx.x - bl * Hq;   // logical row of the launch, query head
  const int b = rows.phys(bl);
  const int row = b * Hq + hq;
  const int g = hq / G, hh = hq - g * G;
  const int bg = b * Hkv + g;            // the sequence's (b, kv head)
  const int bgl = bl * Hkv + g;          // its partials
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (n_rows && threadIdx.x == 0 && hh == 0) {
    const int nr = n_rows[bg];
    if (nr < 0 || nr > p_max) latch_error(err, SFI_ERR_DEVICE_CHECK, kSiteAttnRows);
  }
  const size_t stride = (size_t)G * (D + 4);
  // one partial per consumer warp and work item; the fast step's chunks past
  // the (b, kv head)'s tiles were skipped
  int chunks = n_chunks;
  if (n_rows) {
    int nr = n_rows[bg];
    if (nr < 0 || nr > p_max) nr = nr < 0 ? 0 : p_max;
    const int T = (nr + kPage - 1) / kPage + rec_tiles;
    int ct = (T + n_chunks - 1) / n_chunks;
    ct = (ct + tps - 1) / tps * tps;
    chunks = (T + ct - 1) / ct;
  }
  const int n = chunks * ppi;
  constexpr int kIn = KIN;   // partials in flight per warp
  const float* base = part + (size_t)bgl * n_chunks * ppi * stride + (size_t)hh * (D + 4);
  float m = -INFINITY, l = 0.f, lc = 0.f;
  float acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
  for (int c0 = warp; c0 < n; c0 += kIn * NW) {
    float st[kIn][3];
    float ov[kIn][kPer];
#pragma unroll
    for (int u = 0; u < kIn; ++u) {
      const int c = c0 + u * NW;
      if (c < n) {
        const float* pc = base + c * stride;
        st[u][0] = __ldg(pc + D);
        st[u][1] = __ldg(pc + D + 1);
        st[u][2] = __ldg(pc + D + 2);
        if constexpr (kPer == 4) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(pc + lane * 4));
          ov[u][0] = v.x;
          ov[u][1] = v.y;
          ov[u][2] = v.z;
          ov[u][3] = v.w;
        } else {
          const float2 v = __ldg(reinterpret_cast<const float2*>(pc + lane * 2));
          ov[u][0] = v.x;
          ov[u][1] = v.y;
        }
      } else {
        st[u][0] = -INFINITY;
        st[u][1] = st[u][2] = 0.f;
#pragma unroll
        for (int k = 0; k < kPer; ++k) ov[u][k] = 0.f;
      }
    }
    float mb = m;
#pragma unroll
    for (int u = 0; u < kIn; ++u) mb = fmaxf(mb, st[u][0]);
    const float mref = (mb == -INFINITY) ? 0.f : mb;
    const float a = fast_exp2(m - mref);
    l *= a;
    lc *= a;
#pragma unroll
    for (int k = 0; k < kPer; ++k) acc[k] *= a;
#pragma unroll
    for (int u = 0; u < kIn; ++u) {
      const float w = fast_exp2(st[u][0] - mref);
      l += w * st[u][1];
      lc += w * st[u][2];
#pragma unroll
      for (int k = 0; k < kPer; ++k) acc[k] += w * ov[u][k];
    }
    m = mb;
  }
#pragma unroll
  for (int k = 0; k < kPer; ++k) red[warp][lane * kPer + k] = acc[k];
  if (lane == 0) {
    red[warp][D] = m;
    red[warp][D + 1] = l;
    red[warp][D + 2] = lc;
  }
  __syncthreads();
  if (threadIdx.x < D) {
    float M = -INFINITY;
#pragma unroll 8
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red[w][D]);
    const float mref = (M == -INFINITY) ? 0.f : M;
    float lt = 0.f, lct = 0.f, o = 0.f;
#pragma unroll 8
    for (int w = 0; w < NW; ++w) {
      const float wt = fast_exp2(red[w][D] - mref);
      lt += wt * red[w][D + 1];
      lct += wt * red[w][D + 2];
      o += wt * red[w][threadIdx.x];
    }
    out[(size_t)row * D + threadIdx.x] = o / lt;
    if (threadIdx.x == 0) {
      if (lse) lse[row] = (M + log2f(lt)) * kLn2;
      if (lse_cand) lse_cand[row] = lct > 0.f ? (M + log2f(lct)) * kLn2 : -INFINITY;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kCombWarps * 32)
    attn_combine_kernel(const float* __restrict__ part, int n_chunks, int B, int Hq, int Hkv, int G,
                        float* __restrict__ out, float* __restrict__ lse, float* __restrict__ lse_cand,
                        const int32_t* n_rows, int p_max, int rec_tiles, int tps, int* err, int* ctr,
                        int early, int ppi, const __grid_constant__ RowMap rows) {
  combine_body<D, kCombWarps, 8>(part, n_chunks, B, Hq, Hkv, G, out, lse, lse_cand, n_rows, p_max, rec_tiles, tps,
                                 err, ctr, early, ppi, rows);
}

template <int D>
__global__ void __maxnreg__(64)
    attn_combine_fast_kernel(const float* __restrict__ part, int n_chunks, int B, int Hq, int Hkv, int G,
                             float* __restrict__ out, float* __restrict__ lse, float* __restrict__ lse_cand,
                             const int32_t* n_rows, int p_max, int rec_tiles, int tps, int* err, int* ctr,
                             int early, int ppi, const __grid_constant__ RowMap rows) {
  combine_body<D, kCombWarpsFast, 6>(part, n_chunks, B, Hq, Hkv, G, out, lse, lse_cand, n_rows, p_max, rec_tiles,
                                     tps, err, ctr, early, ppi, rows);
}

template <int D>
__global__ void __maxnreg__(96)
    attn_combine_merged_kernel(const float* __restrict__ part, int n_chunks, int B, int Hq, int Hkv, int G,
                               float* __restrict__ out, float* __restrict__ lse, float* __restrict__ lse_cand,
                               const int32_t* n_rows, int p_max, int rec_tiles, int tps, int* err, int* ctr,
                               int early, int ppi, const __grid_constant__ RowMap rows) {
  combine_body<D, kCombWarpsMerged, 10>(part, n_chunks, B, Hq, Hkv, G, out, lse, lse_cand, n_rows, p_max,
                                        rec_tiles, tps, err, ctr, early, ppi, rows);
}

__global__ void probs_kernel(int L, int Hq, const float* __restrict__ logits, int64_t ld,
                             const float* __restrict__ lse, float* __restrict__ probs) {
  grid_dep_enter();
  const int row = blockIdx.y;
  const float m = lse[row];
  const float* z = logits + (size_t)row * ld;
  float* f = probs + (size_t)row * ld;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < L; j += gridDim.x * blockDim.x)
    f[j] = expf(z[j] - m);
}

// ---------------------------------------------------------------- host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// rows x D bf16 matrix viewed as [D/64 column blocks][rows][64 columns]: one
// box is a whole 16-row tile, landing as [block][16 rows][128 B] with the
// 128-byte swizzle (4 KB per load at D = 128).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(D / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, 128};
  cuuint32_t box[3] = {64, 16, (cuuint32_t)(D / 64)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// rows (a multiple of 16) x D bf16 matrix viewed as [tiles][D/64][16][64]:
// one box = `nt` consecutive 16-row tiles, landing exactly as `nt`
// single-tile boxes would, one after another.
bool make_map_tiles(CUtensorMap* m, const void* base, uint64_t rows, int D, int nt) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, 16, (cuuint64_t)(D / 64), (cuuint64_t)(rows / 16)};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, 128, (cuuint64_t)16 * D * 2};
  cuuint32_t box[4] = {64, 16, (cuuint32_t)(D / 64), (cuuint32_t)nt};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static_assert(sizeof(Maps) == sizeof(AttnMapCache::maps), "tensor-map cache size");

// The launch's tensor maps: from the cache when it was built from the same
// pointers and sizes, else encoded (and kept in the cache, if there is one).
bool paged_maps(Maps* m, const sfi_paged_kv& kv, uint64_t rows, int D, AttnMapCache* c) {
  if (c && c->paged && c->k_pool == kv.k_pool && c->v_pool == kv.v_pool && c->rows == rows && c->D == D) {
    const Maps* cm = reinterpret_cast<const Maps*>(c->maps);
    m->k = cm->k;
    m->v = cm->v;
    return true;
  }
  if (!make_map(&m->k, kv.k_pool, rows, D) || !make_map(&m->v, kv.v_pool, rows, D)) return false;
  if (c) {
    Maps* cm = reinterpret_cast<Maps*>(c->maps);
    cm->k = m->k;
    cm->v = m->v;
    c->k_pool = kv.k_pool;
    c->v_pool = kv.v_pool;
    c->rows = rows;
    c->D = D;
    c->paged = true;
    c->packed = false;   // the packed maps are checked against the same D
  }
  return true;
}

bool packed_maps(Maps* m, const sfi_packed& pk, uint64_t prows, int D, int nts, AttnMapCache* c) {
  if (c && c->packed && c->pk == pk.k && c->pv == pk.v && c->prows == prows && c->D == D) {
    const Maps* cm = reinterpret_cast<const Maps*>(c->maps);
    m->pk = cm->pk;
    m->pv = cm->pv;
    m->pk8 = cm->pk8;
    m->pv8 = cm->pv8;
    return true;
  }
  if (!make_map(&m->pk, pk.k, prows, D) || !make_map(&m->pv, pk.v, prows, D) ||
      !make_map_tiles(&m->pk8, pk.k, prows, D, nts) || !make_map_tiles(&m->pv8, pk.v, prows, D, nts))
    return false;
  if (c && c->paged && c->D == D) {
    Maps* cm = reinterpret_cast<Maps*>(c->maps);
    cm->pk = m->pk;
    cm->pv = m->pv;
    cm->pk8 = m->pk8;
    cm->pv8 = m->pv8;
    c->pk = pk.k;
    c->pv = pk.v;
    c->prows = prows;
    c->packed = true;
  }
  return true;
}

// CTAs of one fast attention launch, and the tiles of one stage.
struct AttnGrid {
  long ctas;
  int tps;
};

template <int D, int NT>
AttnGrid grid_of() {
  const long slots = (long)num_sms() * Plan<D, NT>::kCps;
  const long free_slots = (Plan<D, NT>::kCps == 2 && slots > 4 * kFastFreeSlots) ? kFastFreeSlots : 0;
  return AttnGrid{slots - free_slots, Plan<D, NT>::kTPS};
}

template <int D, int NT, int MODE>
sfi_status launch_attn_t(const Maps& maps, const AttnArgs& a, cudaStream_t st) {
  using S = Smem<D, NT>;
  auto kern = attn_kernel<D, NT, MODE>;
  static DeviceOnce attr;   // per instantiation and device
  if (!attr.done()) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (!attr.mark(e)) return SFI_ERR_CUDA;
  }
  // a dense launch fills every slot; a fast one takes the grid its items were cut for
  const int grid = std::min(a.n_items, MODE == kFast ? (int)grid_of<D, NT>().ctas : num_sms() * Plan<D, NT>::kCps);
  launch_k(kern, dim3(grid), dim3(Plan<D, NT>::kThreads), S::kTotal, st, maps, a);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

template <int MODE>
sfi_status launch_attn(int D, int G, const Maps& maps, const AttnArgs& a, cudaStream_t st) {
  if (D == 128) {
    if (G <= 8) return launch_attn_t<128, 1, MODE>(maps, a, st);
    return launch_attn_t<128, 2, MODE>(maps, a, st);
  }
  if (G <= 8) return launch_attn_t<64, 1, MODE>(maps, a, st);
  return launch_attn_t<64, 2, MODE>(maps, a, st);
}

// Which merge follows an attention launch: after a dense step, after a fast
// step whose CTAs wrote one partial per consumer warp (G > 8), or one per item
// (G <= 8; a dense step's CTAs also write one per item then).
enum CombKind { kCombDense = 0, kCombFast = 1, kCombMerged = 2 };

sfi_status launch_combine(int D, const float* part, int n_chunks, const sfi_shape& s, float* out,
                          float* lse, float* lse_cand, const int32_t* n_rows, int p_max, int rec_tiles, int tps,
                          int* err, int* ctr, cudaStream_t st, const RowMap& rows, CombKind kind) {
  const int G = s.Hq / s.Hkv;
  const int grid = rows.count(s.B) * s.Hq;
  const int early = kind == kCombDense ? 0 : 1;
  // one partial per item where the attention's consumer warps merged (G <= 8)
  const int ppi = G <= 8 ? 1 : kConsumerWarps;
  auto go = [&](auto kern, int nw) {
    launch_k(kern, dim3(grid), dim3(nw * 32), 0, st, part, n_chunks, s.B, s.Hq, s.Hkv, G, out, lse, lse_cand, n_rows,
             p_max, rec_tiles, tps, err, ctr, early, ppi, rows);
  };
  // The merges after a fast step share SMs with attention CTAs: the same
  // shared-memory carveout, so an SM that takes a merge CTA first stays able
  // to take attention CTAs.
  static DeviceOnce carve;
  if (kind != kCombDense && !carve.done()) {
    cudaError_t e = cudaFuncSetAttribute(attn_combine_merged_kernel<128>,
                                         cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_combine_merged_kernel<64>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_combine_fast_kernel<128>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_combine_fast_kernel<64>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (!carve.mark(e)) return SFI_ERR_CUDA;
  }
  if (kind == kCombMerged) {
    if (D == 128) go(attn_combine_merged_kernel<128>, kCombWarpsMerged);
    else go(attn_combine_merged_kernel<64>, kCombWarpsMerged);
  } else if (kind == kCombFast) {
    if (D == 128) go(attn_combine_fast_kernel<128>, kCombWarpsFast);
    else go(attn_combine_fast_kernel<64>, kCombWarpsFast);
  } else {
    if (D == 128) go(attn_combine_kernel<128>, kCombWarps);
    else go(attn_combine_kernel<64>, kCombWarps);
  }
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace

namespace {

AttnGrid attn_grid(int D, int G) {
  if (D == 128) return G <= 8 ? grid_of<128, 1>() : grid_of<128, 2>();
  return G <= 8 ? grid_of<64, 1>() : grid_of<64, 2>();
}

}  // namespace

// Tiles of 16 rows per chunk for the dense step: about kDenseItemsPerSm items
// per SM, at least 8 tiles and at most kMaxChunkTiles, a multiple of the stage.
int dense_chunk_tiles(const sfi_shape& s, int L) {
  const AttnGrid g = attn_grid(s.D, s.Hq / s.Hkv);
  const long T = (L + kPage - 1) / kPage;
  const long bh = (long)s.B * s.Hkv;
  const long n = kDenseItemsPerSm * num_sms();
  long ct = (T * bh + n - 1) / n;
  ct = std::max(ct, 8L);
  ct = (ct + g.tps - 1) / g.tps * g.tps;
  return (int)std::min<long>(ct, kMaxChunkTiles);
}

// Upper bound of the dense chunks per (b, kv head) at any L <= max_pages * 16.
int dense_chunks_bound(const sfi_shape& s) {
  const long T = (long)s.max_pages;
  const long bh = (long)s.B * s.Hkv;
  const long a = (kDenseItemsPerSm * num_sms() + bh - 1) / bh + 1;
  const long b = (T + kMaxChunkTiles - 1) / kMaxChunkTiles;
  return (int)std::min<long>((T + 7) / 8, std::max(a, b));
}

// Chunks per (b, kv head) for the fast step.  The expected tiles (n_sink + K
// packed rows plus the recent window) are cut so that no CTA of the launch
// gets more than the same whole number of items of at most about
// kFastItemTiles tiles (the chunk count is rounded down: one more item for a
// few CTAs would add a whole item to the launch's time); an item never
// exceeds kMaxChunkTiles tiles, even with a full packed buffer.  The result
// never decreases as k_est grows.
int fast_chunks(const sfi_shape& s, int p_max, int n_recent, int k_est) {
  const AttnGrid g = attn_grid(s.D, s.Hq / s.Hkv);
  const long bh = (long)s.B * s.Hkv;
  const long t_rec = n_recent / kPage + 2;
  const long t_max = (p_max + kPage - 1) / kPage + t_rec;
  const long t_est = std::min<long>((k_est + kPage - 1) / kPage + 1, (p_max + kPage - 1) / kPage) + t_rec;
  const long per_cta = std::max<long>(1, (bh * t_est + g.ctas * kFastItemTiles - 1) / (g.ctas * kFastItemTiles));
  long nc = std::min<long>(std::max<long>(per_cta * g.ctas / bh, 1), t_est);
  nc = std::max<long>(nc, (t_max + kMaxChunkTiles - 1) / kMaxChunkTiles);
  return (int)std::max(nc, 1L);
}

size_t attn_part_bytes(int n_items, int G, int D) {
  return (size_t)n_items * kConsumerWarps * G * (D + 4) * sizeof(float);
}

namespace {

void set_token(AttnArgs& a, const sfi_shape& s, const sfi_paged_kv& kv, const StepToken* tok) {
  if (!tok) return;
  a.k_new = reinterpret_cast<const __nv_bfloat16*>(tok->k_new);
  a.v_new = reinterpret_cast<const __nv_bfloat16*>(tok->v_new);
  a.k_pool = reinterpret_cast<__nv_bfloat16*>(kv.k_pool);
  a.v_pool = reinterpret_cast<__nv_bfloat16*>(kv.v_pool);
  a.norms = kv.key_norms;
  a.norm_ld = (int64_t)s.max_pages * kPage;
}

}  // namespace

sfi_status run_dense_attn(const sfi_shape& s, const sfi_paged_kv& kv, int L, const sfi_bf16* q,
                          float* out, const sfi_dense_extras* ex, int* ctr, float* part,
                          size_t part_bytes, cudaStream_t st, cudaEvent_t ev_begin, cudaEvent_t ev_end,
                          const StepToken* tok, AttnMapCache* cache, const RowMap& rmap, bool late_trigger) {
  const int G = s.Hq / s.Hkv;
  if (rmap.count(s.B) < 1 || rmap.count(s.B) > s.B) return SFI_ERR_SHAPE;
  Maps maps;
  const uint64_t rows = (uint64_t)s.num_pages * s.Hkv * kPage;
  if (!paged_maps(&maps, kv, rows, s.D, cache)) return SFI_ERR_CUDA;
  maps.pk = maps.pk8 = maps.k;
  maps.pv = maps.pv8 = maps.v;
  AttnArgs a{};
  a.B = s.B; a.Hq = s.Hq; a.Hkv = s.Hkv; a.G = G; a.L = L;
  a.num_pages = s.num_pages; a.max_pages = s.max_pages;
  a.page_table = kv.page_table;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.ctr = ctr;
  a.chunk_tiles = dense_chunk_tiles(s, L);
  const int T = (L + kPage - 1) / kPage;
  a.n_chunks = (T + a.chunk_tiles - 1) / a.chunk_tiles;
  // chunking of the whole batch also for a subset: the partials fit the workspace
  a.rows = rmap;
  a.n_items = rmap.count(s.B) * s.Hkv * a.n_chunks;
  if (attn_part_bytes(a.n_items, G, s.D) > part_bytes) return SFI_ERR_WORKSPACE;
  a.part = part;
  a.scale = 1.0f / sqrtf((float)s.D);
  a.scale_log2 = kLog2e * a.scale;
  a.err = kv.err;
  a.wait_ns = wait_limit_ns();
  a.late_trigger = late_trigger ? 1 : 0;
  set_token(a, s, kv, tok);
  const bool extras = ex && (ex->logits || ex->probs || ex->lse_cand);
  float* zbuf = nullptr;
  if (extras) {
    zbuf = ex->logits ? ex->logits : ex->probs;
    a.logits = zbuf;
    a.ld = ex->ld;
    a.cand_lo = ex->lse_cand ? ex->cand_lo : 0;
    a.cand_hi = ex->lse_cand ? ex->cand_hi : 0;
  }
  if (ev_begin) cudaEventRecord(ev_begin, st);
  sfi_status r;
  if (extras) r = launch_attn<kDenseExtras>(s.D, G, maps, a, st);
  else r = launch_attn<kDense>(s.D, G, maps, a, st);
  if (ev_end) cudaEventRecord(ev_end, st);
  if (r != SFI_OK) return r;
  float* lse_tmp = ex ? ex->lse : nullptr;
  r = launch_combine(s.D, part, a.n_chunks, s, out, lse_tmp, ex ? ex->lse_cand : nullptr, nullptr, 0, 0, 1,
                     kv.err, ctr, st, rmap, kCombDense);
  if (r != SFI_OK) return r;
  if (ex && ex->probs) {
    if (rmap.n) return SFI_ERR_UNSUPPORTED;   // probabilities of the whole batch only
    dim3 grid((L + 1023) / 1024 < 64 ? (L + 1023) / 1024 : 64, s.B * s.Hq);
    launch_k(probs_kernel, dim3(grid), dim3(256), 0, st, L, s.Hq, zbuf, ex->ld, lse_tmp, ex->probs);
    if (cudaPeekAtLastError() != cudaSuccess) return SFI_ERR_CUDA;
  }
  return SFI_OK;
}

sfi_status run_fast_attn(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv, int L,
                         const sfi_bf16* q, const sfi_packed& pk, float* out, float* lse, int* ctr,
                         float* part, size_t part_bytes, cudaStream_t st, cudaEvent_t ev_begin,
                         cudaEvent_t ev_end, const StepToken* tok, AttnMapCache* cache, const RowMap& rmap) {
  const int G = s.Hq / s.Hkv;
  if (rmap.count(s.B) < 1 || rmap.count(s.B) > s.B) return SFI_ERR_SHAPE;
  if ((long)s.B * s.Hkv > kMaxBH) return SFI_ERR_UNSUPPORTED;
  Maps maps;
  const uint64_t rows = (uint64_t)s.num_pages * s.Hkv * kPage;
  const uint64_t prows = (uint64_t)s.B * s.Hkv * pk.p_max;
  const int nts = attn_grid(s.D, G).tps;
  if (!paged_maps(&maps, kv, rows, s.D, cache) || !packed_maps(&maps, pk, prows, s.D, nts, cache))
    return SFI_ERR_CUDA;
  AttnArgs a{};
  a.B = s.B; a.Hq = s.Hq; a.Hkv = s.Hkv; a.G = G; a.L = L;
  a.num_pages = s.num_pages; a.max_pages = s.max_pages;
  a.page_table = kv.page_table;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.ctr = ctr;
  a.n_chunks = fast_chunks(s, pk.p_max, p.n_recent, std::max(budget_k(p, L), 0) * 1 + p.n_sink);
  a.rows = rmap;
  a.n_items = rmap.count(s.B) * s.Hkv * a.n_chunks;
  if (attn_part_bytes(a.n_items, G, s.D) > part_bytes) return SFI_ERR_WORKSPACE;
  a.part = part;
  a.scale = 1.0f / sqrtf((float)s.D);
  a.scale_log2 = kLog2e * a.scale;
  a.n_rows = pk.n_rows;
  a.headmask = pk.headmask;
  a.p_max = pk.p_max;
  a.rec_lo = std::max(L - p.n_recent, 0);
  a.err = kv.err;
  a.wait_ns = wait_limit_ns();
  set_token(a, s, kv, tok);
  if (ev_begin) cudaEventRecord(ev_begin, st);
  sfi_status r = launch_attn<kFast>(s.D, G, maps, a, st);
  if (ev_end) cudaEventRecord(ev_end, st);
  if (r != SFI_OK) return r;
  const int rec_tiles = (L - 1) / kPage - a.rec_lo / kPage + 1;
  // G <= 8: the attention's CTAs merged their warps' states (one partial per
  // item); G > 8: one partial per consumer warp and item.
  const CombKind kind = G <= 8 ? kCombMerged : kCombFast;
  return launch_combine(s.D, part, a.n_chunks, s, out, lse, nullptr, pk.n_rows, pk.p_max, rec_tiles, nts, kv.err,
                        ctr, st, rmap, kind);
}

sfi_status run_attn_probs(const sfi_shape& s, int L, const float* logits, int64_t ld, const float* lse,
                          float* probs, cudaStream_t st) {
  dim3 grid((L + 1023) / 1024 < 64 ? (L + 1023) / 1024 : 64, s.B * s.Hq);
  launch_k(probs_kernel, dim3(grid), dim3(256), 0, st, L, s.Hq, logits, ld, lse, probs);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace sfi
