// Compaction of the selected tokens into the contiguous packed buffer
// ([ES] "3. Optimización del Sistema", item 2; [FR] "C. Optimisations
// Système", réorganisation; [NL] "Systeemontwerp", Memory-Coalesced Kernel;
// [ZH] "2.3" 两段式布局).
//
// Per (sequence, KV head): rows = sink tokens [0, n_sink), then the union of
// the group's per-head selections in ascending position order, each with a
// bitmask of the query heads that chose it (sinks: all heads), then zero rows
// up to the next multiple of 16.  Selections arrive as one bitmap per query
// head over the candidate range (bit c = position n_sink + c), as the top-K
// kernel writes them.  A tile is 256 bitmap words (8192 positions); each
// thread owns one word: the OR of the group's words is the union, its
// popcount the row count.  compact_count writes the per-tile counts;
// compact_gather scans them and writes positions, head masks and n_rows;
// compact_copy then copies the K and V rows, one warp per row, eight rows in
// flight per warp, over fixed 128-row blocks (the selection is far from
// uniform over positions, so per-tile copying would be imbalanced).
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace sfi {

constexpr int kCWords = 256;
constexpr int kCThreads = 256;

struct CompactArgs {
  int Hkv, G, Hq, D, n_sink, lo, nC, nw, n_tiles;
  int max_pages, num_pages, p_max;
  const uint32_t* bits;   // [B*Hq][ld_b]
  int64_t ld_b;
  const int32_t* pt;
  const uint4* kpool;
  const uint4* vpool;
  uint4* pk;
  uint4* pv;
  int32_t* pos;
  uint32_t* headmask;
  int32_t* n_rows;
  int32_t* tile_counts;   // [B*Hkv][n_tiles]
  int* err;
  RowMap rows;            // bits and scratch: logical rows; everything else: the sequences
};

template <int GM>
__device__ __forceinline__ uint32_t union_word(const CompactArgs& a, int b, int g, int w, uint32_t (&hw)[GM]) {
  uint32_t u = 0u;
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    hw[h] = (h < a.G && w < a.nw) ? __ldg(a.bits + ((size_t)b * a.Hq + g * a.G + h) * a.ld_b + w) : 0u;
    u |= hw[h];
  }
  return u;
}

template <int GM>
__global__ void __launch_bounds__(kCThreads) compact_count_kernel(const __grid_constant__ CompactArgs a) {
  grid_dep_enter_writer();
  __shared__ int wsum[kCThreads / 32];
  const int bg = blockIdx.y;
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  uint32_t hw[GM];
  const uint32_t u = union_word<GM>(a, b, g, blockIdx.x * kCWords + threadIdx.x, hw);
  int c = __popc(u);
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) c += __shfl_xor_sync(0xffffffffu, c, sh);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < kCThreads / 32; ++w) t += wsum[w];
    a.tile_counts[(size_t)bg * a.n_tiles + blockIdx.x] = t;
  }
}

template <int GM>
__global__ void __launch_bounds__(kCThreads) compact_gather_kernel(const __grid_constant__ CompactArgs a) {
  grid_dep_enter_writer();
  __shared__ int wtot[kCThreads / 32 + 1];
  __shared__ int base_s, total_s;
  const int bg = blockIdx.y;                    // logical (row, kv head)
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int bp = a.rows.phys(b);                  // the sequence
  const int bgp = bp * a.Hkv + g;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kCThreads / 32;
  const int w = blockIdx.x * kCWords + threadIdx.x;
  uint32_t hw[GM];
  const uint32_t u = union_word<GM>(a, b, g, w, hw);
  // rows before this tile
  if (warp == 0) {
    int s = 0;
    for (int t = lane; t < blockIdx.x; t += 32) s += a.tile_counts[(size_t)bg * a.n_tiles + t];
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) s += __shfl_xor_sync(0xffffffffu, s, sh);
    if (lane == 0) base_s = a.n_sink + s;
  }
  // rank of this word's rows inside the tile
  const int cnt = __popc(u);
  int x = cnt;
#pragma unroll
  for (int sh = 1; sh < 32; sh <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, sh);
    if (lane >= sh) x += y;
  }
  if (lane == 31) wtot[warp] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int i = 0; i < kWarps; ++i) {
      const int t = wtot[i];
      wtot[i] = s;
      s += t;
    }
    total_s = s;
  }
  __syncthreads();
  const int base = base_s;
  const int total = min(total_s, max(a.p_max - base, 0));
  if (total < total_s && threadIdx.x == 0) latch_error(a.err, SFI_ERR_DEVICE_CHECK, kSiteCompactRows);
  int32_t* pos = a.pos + (size_t)bgp * a.p_max;
  uint32_t* hm = a.headmask + (size_t)bgp * a.p_max;
  int r = x - cnt + wtot[warp];
  uint32_t t = u;
  while (t) {
    const int bit = __ffs(t) - 1;
    t &= t - 1u;
    if (r < total) {
      const int p = a.lo + w * 32 + bit;
      uint32_t m = 0u;
#pragma unroll
      for (int h = 0; h < GM; ++h) m |= ((hw[h] >> bit) & 1u) << h;
      pos[base + r] = p;
      hm[base + r] = m;
    }
    ++r;
  }
  // sinks (first tile) and the tail (last tile); rows are copied by compact_copy
  const uint32_t all = a.G >= 32 ? 0xffffffffu : ((1u << a.G) - 1u);
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < min(a.n_sink, a.p_max); i += kCThreads) {
      pos[i] = i;
      hm[i] = all;
    }
  }
  if (blockIdx.x == gridDim.x - 1) {
    const int n = min(base + total_s, a.p_max);
    if (threadIdx.x == 0) a.n_rows[bgp] = n;
    const int pad_end = min((n + kPage - 1) / kPage * kPage, a.p_max);
    for (int rr = n + threadIdx.x; rr < pad_end; rr += kCThreads) {
      pos[rr] = -1;
      hm[rr] = 0u;
    }
  }
}

// Copy the K and V rows of the packed buffer from the pages (rows past
// n_rows up to the next multiple of 16: zeros).  Grid: 128-row blocks of
// every (b, KV head); blocks past the rows in use return at once, so the
// copy work is spread evenly whatever the selection looks like.  A warp moves
// whole rows: for D = 128 lanes 0-15 carry the K row and lanes 16-31 the V
// row (16 bytes each), for D = 64 one warp pass moves two rows; eight passes
// are in flight per warp.
constexpr int kCopyRows = 128;
constexpr int kCopyWarps = 8;

template <int D>
__global__ void __launch_bounds__(kCopyWarps * 32) compact_copy_kernel(const __grid_constant__ CompactArgs a) {
  grid_dep_enter_writer();
  constexpr int kUnits = D / 8;                 // 16-byte units of one K (or V) row
  constexpr int kRowUnits = 2 * kUnits;         // K then V
  constexpr int kRowsPerPass = 32 / kRowUnits;  // rows one warp moves per pass
  constexpr int kRowsPerWarp = kCopyRows / kCopyWarps;
  constexpr int kIn = 8;                        // passes in flight
  static_assert(kRowsPerWarp % (kIn * kRowsPerPass) == 0 || kRowsPerWarp == kIn * kRowsPerPass, "copy plan");
  __shared__ long long src[kCopyRows];          // unit offset of the row in the pools, -1: zero row
  const int bg = blockIdx.y;                    // logical (row, kv head)
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int bp = a.rows.phys(b);                  // the sequence
  const int bgp = bp * a.Hkv + g;
  const int n = min(max(a.n_rows[bgp], 0), a.p_max);
  const int pad_end = min((n + kPage - 1) / kPage * kPage, a.p_max);
  const int r0 = blockIdx.x * kCopyRows;
  if (r0 >= pad_end) return;
  const int nr = min(kCopyRows, pad_end - r0);
  const int32_t* pos = a.pos + (size_t)bgp * a.p_max;
  if (threadIdx.x < kCopyRows) {
    const int r = r0 + threadIdx.x;
    long long off = -1;
    if (threadIdx.x < nr && r < n) {
      const int p = pos[r];
      const int pi = p / kPage;
      int page = -1;
      if (p >= 0 && pi < a.max_pages) page = __ldg(a.pt + (size_t)bp * a.max_pages + pi);
      if ((unsigned)page >= (unsigned)a.num_pages) latch_error(a.err, SFI_ERR_DEVICE_CHECK, kSiteCompactPage);
      else off = ((long long)(page * a.Hkv + g) * kPage + p % kPage) * kUnits;
    }
    src[threadIdx.x] = off;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / kRowUnits;             // row of the pass
  const int u = lane % kRowUnits;
  const bool isv = u >= kUnits;
  const int cu = isv ? u - kUnits : u;
  const uint4* from = isv ? a.vpool : a.kpool;
  uint4* to = isv ? a.pv : a.pk;
  const size_t dst0 = ((size_t)bgp * a.p_max + r0) * kUnits + cu;
#pragma unroll
  for (int i0 = 0; i0 < kRowsPerWarp; i0 += kIn * kRowsPerPass) {
    uint4 v[kIn];
#pragma unroll
    for (int k = 0; k < kIn; ++k) {
      const int r = warp * kRowsPerWarp + i0 + k * kRowsPerPass + sub;
      const long long off = (r < nr) ? src[r] : -1;
      v[k] = off >= 0 ? __ldg(from + off + cu) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < kIn; ++k) {
      const int r = warp * kRowsPerWarp + i0 + k * kRowsPerPass + sub;
      if (r < nr) to[dst0 + (size_t)r * kUnits] = v[k];
    }
  }
}

__global__ void __launch_bounds__(256) idx_to_bits_kernel(const int32_t* __restrict__ sel, int sel_ld, int K,
                                                          int lo, int nC, uint32_t* bits, int64_t ld_b,
                                                          int* err) {
  grid_dep_enter();
  const int row = blockIdx.x;
  const int nw = (nC + 31) / 32;
  uint32_t* brow = bits + (size_t)row * ld_b;
  for (int i = threadIdx.x; i < nw; i += blockDim.x) brow[i] = 0u;
  __syncthreads();
  const int32_t* s = sel + (size_t)row * sel_ld;
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    const int c = s[i] - lo;
    if ((unsigned)c < (unsigned)nC) atomicOr(&brow[c >> 5], 1u << (c & 31));
    else latch_error(err, SFI_ERR_DEVICE_CHECK, kSiteCompactIdx);
  }
}

int compact_tiles(int nC) { return ((nC + 31) / 32 + kCWords - 1) / kCWords; }

// ------------------------------------------------------------ incremental
// Incremental compaction (the support of consecutive slow steps changes
// little — "Slow-Fast Inference", within-sentence support stability — so most
// packed rows can stay where they are).  Layout rule, per (sequence, KV
// head), given the previous buffer (rows [0, n_old)) and the new union U of
// the group's selections, n_new = n_sink + |U|:
//   * a previous row whose position is in U keeps its slot (its head mask is
//     rewritten); the others leave;
//   * holes = slots in [n_sink, n_new) not kept, in slot order;
//   * movers = positions of U not in the previous buffer, ascending, then the
//     kept rows at slots >= n_new, in slot order;
//   * the i-th mover is copied from the pages into the i-th hole.
// Only movers are copied: with a stable support that is a few percent of the
// rows.  A fresh buffer (no previous rows) gets sinks and U in ascending
// order: the full compaction above.
//
// One launch: a cluster of kIncCluster CTAs per (sequence, KV head).  Each CTA
// marks the positions of its share of the previous rows in a bitmap over the
// candidates in its own shared memory (local atomics), so no global state
// has to be cleared between calls.  The phases, each ended by a cluster
// barrier:
//   1. previous rows (split over the CTAs): head mask rewritten (0: the row
//      leaves), position marked in the CTA's bitmap;
//   2. each CTA's slice of bitmap words: the previous positions (the OR of
//      every CTA's bitmap, read through distributed shared memory), |U| and
//      the entering positions U & ~old;
//   3. each CTA's slots of [n_sink, max(n_old, n_new)): kept, hole, moved
//      (kept rows at or past n_new);
//   4. the mover and hole lists, in the order of the rule (cluster-wide
//      exclusive counts from the phases above);
//   5. the copy: the i-th mover into the i-th hole, zero rows from n_new to
//      the next multiple of 16, n_rows.
constexpr int kIncThreads = 512;
constexpr int kIncCluster = 8;
constexpr int kIncMaxWords = 8192;       // candidate bitmap words (|C| <= 262144)
constexpr int kIncMaxSlotWords = 2048;   // slot words per CTA (packed capacity <= 524288)

struct IncArgs {
  CompactArgs c;        // bitmaps, pages, packed buffer, error word
  int cap;              // packed rows any selection can need (multiple of 16)
  int32_t* mover_pos;   // [BH][cap]
  int32_t* hole_slot;   // [BH][cap]
};

template <int GM>
__device__ __forceinline__ uint32_t head_bits_at(const CompactArgs& a, int b, int g, int c) {
  uint32_t m = 0u;
#pragma unroll
  for (int h = 0; h < GM; ++h)
    if (h < a.G) m |= ((__ldg(a.bits + ((size_t)b * a.Hq + g * a.G + h) * a.ld_b + (c >> 5)) >> (c & 31)) & 1u) << h;
  return m;
}

// Exclusive prefix sum over the CTA of one value per thread; *total: the sum.
__device__ __forceinline__ int inc_block_excl(int v, int* ws, int* total) {
  constexpr int kW = kIncThreads / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int sh = 1; sh < 32; sh <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, sh);
    if (lane >= sh) x += y;
  }
  __syncthreads();
  if (lane == 31) ws[w] = x;
  __syncthreads();
  if (w == 0) {
    const int t = lane < kW ? ws[lane] : 0;
    int s = t;
#pragma unroll
    for (int sh = 1; sh < 32; sh <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, sh);
      if (lane >= sh) s += y;
    }
    ws[lane] = s - t;
    if (lane == 31) ws[32] = s;
  }
  __syncthreads();
  const int r = x - v + ws[w];
  *total = ws[32];
  return r;
}

// Bits i of a 32-slot word starting at slot s0 with s0 + i < x.
__device__ __forceinline__ uint32_t below(int s0, int x) {
  if (x <= s0) return 0u;
  if (x >= s0 + 32) return 0xffffffffu;
  return (1u << (x - s0)) - 1u;
}

template <int D, int GM>
__global__ void __launch_bounds__(kIncThreads) inc_refresh_kernel(const __grid_constant__ IncArgs a) {
  grid_dep_enter_writer();
  cg::cluster_group cl = cg::this_cluster();
  constexpr int cs = kIncCluster;               // the launch's cluster size
  const int rank = (int)cl.block_rank();
  const CompactArgs& c = a.c;
  constexpr int T = kIncThreads;
  const int bg = blockIdx.y;                    // logical (row, kv head)
  const int b = bg / c.Hkv, g = bg - b * c.Hkv;
  const int bp = c.rows.phys(b);                // the sequence
  const int bgp = bp * c.Hkv + g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ uint32_t oldw[kIncMaxWords];       // positions of this CTA's share of the previous rows
  __shared__ uint32_t entw[kIncMaxWords / kIncCluster];   // entering positions of its word slice
  __shared__ uint32_t keptw[kIncMaxSlotWords];  // its slots holding a kept row
  __shared__ int pub[4];                        // published: |U|, entering, holes, moved
  __shared__ int ws[33];
  __shared__ int tot[8];
  int32_t* pos = c.pos + (size_t)bgp * c.p_max;
  uint32_t* hm = c.headmask + (size_t)bgp * c.p_max;
  const int nw = c.nw;
  const int Wc = (nw + cs - 1) / cs;
  const int w0 = min(nw, rank * Wc), w1 = min(nw, w0 + Wc);
  for (int i = tid; i < nw; i += T) oldw[i] = 0u;
  // previous rows; a count outside [n_sink, cap] means no usable buffer: the
  // sinks are written again and every selected row enters
  const int n_raw = c.n_rows[bgp];
  const bool valid = n_raw >= c.n_sink && n_raw <= a.cap;
  const int n_old = valid ? n_raw : c.n_sink;
  __syncthreads();

  // ---- 1. previous rows
  {
    const int n1 = n_old - c.n_sink;
    const int per1 = (n1 + cs - 1) / cs;
    const int lo1 = c.n_sink + rank * per1, hi1 = min(n_old, lo1 + per1);
    for (int s = lo1 + tid; s < hi1; s += T) {
      const int ci = pos[s] - c.lo;
      uint32_t m = 0u;
      if ((unsigned)ci < (unsigned)c.nC) {
        m = head_bits_at<GM>(c, b, g, ci);
        atomicOr(&oldw[ci >> 5], 1u << (ci & 31));
      }
      hm[s] = m;   // 0: the row leaves
    }
  }
  cl.sync();

  // ---- 2. this CTA's bitmap words
  {
    int cu = 0, ce = 0;
    for (int w = w0 + tid; w < w1; w += T) {
      uint32_t hw[GM];
      const uint32_t u = union_word<GM>(c, b, g, w, hw);
      uint32_t ow[cs];   // the cluster's loads issued together
#pragma unroll
      for (int r = 0; r < cs; ++r) ow[r] = cl.map_shared_rank(oldw, r)[w];
      uint32_t old = 0u;
#pragma unroll
      for (int r = 0; r < cs; ++r) old |= ow[r];
      const uint32_t e = u & ~old;
      entw[w - w0] = e;
      cu += __popc(u);
      ce += __popc(e);
    }
    int tu, te;
    inc_block_excl(cu, ws, &tu);
    inc_block_excl(ce, ws, &te);
    if (tid == 0) {
      pub[0] = tu;
      pub[1] = te;
    }
  }
  cl.sync();
  if (warp == 0) {   // lane r reads CTA r's totals
    int pu = 0, pe = 0;
    if (lane < cs) {
      const int* pr = cl.map_shared_rank(pub, lane);
      pu = pr[0];
      pe = pr[1];
    }
    int peb = lane < rank ? pe : 0;
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) {
      pu += __shfl_xor_sync(0xffffffffu, pu, sh);
      pe += __shfl_xor_sync(0xffffffffu, pe, sh);
      peb += __shfl_xor_sync(0xffffffffu, peb, sh);
    }
    if (lane == 0) {
      tot[0] = pu;
      tot[1] = pe;
      tot[2] = peb;
    }
  }
  __syncthreads();
  const int n_want = c.n_sink + tot[0];
  const int n_new = min(n_want, a.cap);
  const int E_tot = tot[1], E_before = tot[2];

  // ---- 3. this CTA's slots: kept rows (one ballot per 32 slots), holes, moved
  const int hi3 = max(n_old, n_new);
  const int per3 = ((hi3 - c.n_sink + cs - 1) / cs + 31) / 32 * 32;
  const int lo3 = c.n_sink + rank * per3, up3 = min(hi3, lo3 + per3);
  const int nsw = up3 > lo3 ? (up3 - lo3 + 31) / 32 : 0;
  for (int k = warp; k < nsw; k += T / 32) {
    const int s = lo3 + k * 32 + lane;
    const bool kept = s < up3 && s < n_old && hm[s] != 0u;
    const uint32_t bw = __ballot_sync(0xffffffffu, kept);
    if (lane == 0) keptw[k] = bw;
  }
  __syncthreads();
  const int cw = (nsw + T - 1) / T;   // slot words per thread, contiguous
  const int k0 = min(nsw, tid * cw), k1 = min(nsw, k0 + cw);
  int hc = 0, mc = 0;
  for (int k = k0; k < k1; ++k) {
    const int s0 = lo3 + k * 32;
    const uint32_t in = below(s0, up3), lt = below(s0, n_new), kw = keptw[k];
    hc += __popc(in & lt & ~kw);
    mc += __popc(in & ~lt & kw);
  }
  int th, tm;
  const int h_local = inc_block_excl(hc, ws, &th);
  const int m_local = inc_block_excl(mc, ws, &tm);
  if (tid == 0) {
    pub[2] = th;
    pub[3] = tm;
  }
  cl.sync();
  if (warp == 0) {   // lane r reads CTA r's counts
    int ph = 0, pm = 0;
    if (lane < cs) {
      const int* pr = cl.map_shared_rank(pub, lane);
      ph = pr[2];
      pm = pr[3];
    }
    int phb = lane < rank ? ph : 0, pmb = lane < rank ? pm : 0;
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) {
      ph += __shfl_xor_sync(0xffffffffu, ph, sh);
      pm += __shfl_xor_sync(0xffffffffu, pm, sh);
      phb += __shfl_xor_sync(0xffffffffu, phb, sh);
      pmb += __shfl_xor_sync(0xffffffffu, pmb, sh);
    }
    if (lane == 0) {
      tot[3] = ph;
      tot[4] = phb;
      tot[5] = pm;
      tot[6] = pmb;
    }
  }
  __syncthreads();
  const int H_tot = tot[3], M_tot = E_tot + tot[5];

  // ---- 4. the lists
  int32_t* mv = a.mover_pos + (size_t)bg * a.cap;
  int32_t* hs = a.hole_slot + (size_t)bg * a.cap;
  {
    int hr = tot[4] + h_local, mr = E_tot + tot[6] + m_local;
    for (int k = k0; k < k1; ++k) {
      const int s0 = lo3 + k * 32;
      const uint32_t in = below(s0, up3), lt = below(s0, n_new), kw = keptw[k];
      uint32_t hole = in & lt & ~kw, moved = in & ~lt & kw;
      while (hole) {
        const int i = __ffs(hole) - 1;
        hole &= hole - 1u;
        if (hr < a.cap) hs[hr] = s0 + i;
        ++hr;
      }
      while (moved) {
        const int i = __ffs(moved) - 1;
        moved &= moved - 1u;
        if (mr < a.cap) mv[mr] = pos[s0 + i];
        ++mr;
      }
    }
    // entering positions of this CTA's bitmap words, ascending
    const int nwc = w1 - w0;
    const int cwe = (nwc + T - 1) / T;
    const int e0 = min(nwc, tid * cwe), e1 = min(nwc, e0 + cwe);
    int ec = 0;
    for (int k = e0; k < e1; ++k) ec += __popc(entw[k]);
    int te;
    int er = E_before + inc_block_excl(ec, ws, &te);
    for (int k = e0; k < e1; ++k) {
      uint32_t e = entw[k];
      while (e) {
        const int i = __ffs(e) - 1;
        e &= e - 1u;
        if (er < a.cap) mv[er] = c.lo + (w0 + k) * 32 + i;
        ++er;
      }
    }
  }
  cl.sync();   // every list entry written

  // ---- 5. the copy
  if (rank == 0 && tid == 0) {
    c.n_rows[bgp] = n_new;
    if (n_want > a.cap || M_tot != H_tot) latch_error(c.err, SFI_ERR_DEVICE_CHECK, kSiteCompactRows);
  }
  const int n_hole = min(H_tot, a.cap);
  const int n_mov = min(M_tot, a.cap);
  const int pad_end = min((n_new + kPage - 1) / kPage * kPage, a.cap);
  const int n_pad = pad_end - n_new;
  const int n_sf = valid ? 0 : c.n_sink;
  const int items = n_hole + n_pad + n_sf;
  const int per5 = (items + cs - 1) / cs;
  const int i_lo = rank * per5, i_hi = min(items, i_lo + per5);
  constexpr int kUnits = D / 8;                 // 16-byte units of one K (or V) row
  constexpr int kRowUnits = 2 * kUnits;         // K then V
  constexpr int kRowsPerPass = 32 / kRowUnits;  // rows one warp moves per pass
  constexpr int kIn = 4;                        // passes in flight
  const int sub = lane / kRowUnits;
  const int u = lane % kRowUnits;
  const bool isv = u >= kUnits;
  const int cu = isv ? u - kUnits : u;
  const uint4* from = isv ? c.vpool : c.kpool;
  uint4* to = isv ? c.pv : c.pk;
  const size_t base = (size_t)bgp * c.p_max * kUnits + cu;
  const uint32_t all = c.G >= 32 ? 0xffffffffu : ((1u << c.G) - 1u);
  for (int i0 = i_lo + warp * kIn * kRowsPerPass; i0 < i_hi; i0 += (T / 32) * kIn * kRowsPerPass) {
    uint4 v[kIn];
    int slot[kIn];
#pragma unroll
    for (int k = 0; k < kIn; ++k) {
      const int i = i0 + k * kRowsPerPass + sub;
      slot[k] = -1;
      v[k] = make_uint4(0, 0, 0, 0);
      if (i >= i_hi) continue;
      int p = -1;
      uint32_t m = 0u;
      if (i < n_hole) {
        slot[k] = hs[i];
        if (i < n_mov) {
          p = mv[i];
          m = head_bits_at<GM>(c, b, g, p - c.lo);
        }
      } else if (i < n_hole + n_pad) {
        slot[k] = n_new + (i - n_hole);
      } else {
        slot[k] = i - n_hole - n_pad;
        p = slot[k];
        m = all;
      }
      if (u == 0) {
        pos[slot[k]] = p;
        hm[slot[k]] = m;
      }
      if (p >= 0) {
        const int pi = p / kPage;
        int page = -1;
        if (pi < c.max_pages) page = __ldg(c.pt + (size_t)bp * c.max_pages + pi);
        if ((unsigned)page >= (unsigned)c.num_pages) {
          if (u == 0) latch_error(c.err, SFI_ERR_DEVICE_CHECK, kSiteCompactPage);
        } else {
          v[k] = __ldg(from + ((long long)(page * c.Hkv + g) * kPage + p % kPage) * kUnits + cu);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kIn; ++k)
      if (slot[k] >= 0) to[base + (size_t)slot[k] * kUnits] = v[k];
  }
  cl.sync();   // no CTA leaves while another may still read its shared memory
}

size_t compact_scratch_bytes(const sfi_shape& s, const sfi_params& p) {
  const long bh = (long)s.B * s.Hkv;
  const int Lmax = s.max_pages * kPage;
  const int nC = std::max(Lmax - p.n_recent - p.n_sink, 1);
  const int cap = packed_rows_capacity(s, p);
  return align_up((size_t)bh * compact_tiles(nC) * 2 * sizeof(int32_t), 256) +
         2 * align_up((size_t)bh * cap * sizeof(int32_t), 256);
}

CompactScratch compact_scratch(void* base, const sfi_shape& s, const sfi_params& p) {
  const long bh = (long)s.B * s.Hkv;
  const int Lmax = s.max_pages * kPage;
  const int nC = std::max(Lmax - p.n_recent - p.n_sink, 1);
  const int cap = packed_rows_capacity(s, p);
  char* w = static_cast<char*>(base);
  CompactScratch c{};
  c.cap = cap;
  c.wcounts = reinterpret_cast<int32_t*>(w);
  c.wcount_bytes = align_up((size_t)bh * compact_tiles(nC) * 2 * sizeof(int32_t), 256);
  w += c.wcount_bytes;
  c.mover_pos = reinterpret_cast<int32_t*>(w);
  w += align_up((size_t)bh * cap * sizeof(int32_t), 256);
  c.hole_slot = reinterpret_cast<int32_t*>(w);
  return c;
}

template <int D, int GM>
sfi_status launch_inc_t(const IncArgs& a, int BH, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kIncCluster, BH);
  cfg.blockDim = dim3(kIncThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kIncCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, inc_refresh_kernel<D, GM>, a) == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

template <int GM>
sfi_status launch_inc(const IncArgs& a, int BH, cudaStream_t st) {
  return a.c.D == 128 ? launch_inc_t<128, GM>(a, BH, st) : launch_inc_t<64, GM>(a, BH, st);
}

template <int GM>
sfi_status launch_compact(const CompactArgs& a, int BH, cudaStream_t st) {
  dim3 grid(a.n_tiles, BH);
  launch_k(compact_count_kernel<GM>, dim3(grid), dim3(kCThreads), 0, st, a);
  launch_k(compact_gather_kernel<GM>, dim3(grid), dim3(kCThreads), 0, st, a);
  dim3 cgrid((a.p_max + kCopyRows - 1) / kCopyRows, BH);
  if (a.D == 128) launch_k(compact_copy_kernel<128>, cgrid, dim3(kCopyWarps * 32), 0, st, a);
  else launch_k(compact_copy_kernel<64>, cgrid, dim3(kCopyWarps * 32), 0, st, a);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

namespace {

CompactArgs compact_args(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv, const uint32_t* bits,
                         int64_t ld_b, const sfi_packed& pk, int L_slow) {
  CompactArgs a{};
  a.Hkv = s.Hkv; a.G = s.Hq / s.Hkv; a.Hq = s.Hq; a.D = s.D;
  a.n_sink = p.n_sink;
  a.lo = p.n_sink;
  a.nC = L_slow - p.n_recent - p.n_sink;
  a.nw = (a.nC + 31) / 32;
  a.n_tiles = compact_tiles(a.nC);
  a.max_pages = s.max_pages; a.num_pages = s.num_pages; a.p_max = pk.p_max;
  a.bits = bits; a.ld_b = ld_b;
  a.pt = kv.page_table;
  a.kpool = reinterpret_cast<const uint4*>(kv.k_pool);
  a.vpool = reinterpret_cast<const uint4*>(kv.v_pool);
  a.pk = reinterpret_cast<uint4*>(pk.k);
  a.pv = reinterpret_cast<uint4*>(pk.v);
  a.pos = pk.pos; a.headmask = pk.headmask; a.n_rows = pk.n_rows;
  a.err = kv.err;
  return a;
}

}  // namespace

sfi_status run_compact_bits(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv,
                            const uint32_t* bits, int64_t ld_b, const sfi_packed& pk,
                            const CompactScratch& cs, int L_slow, cudaStream_t st, const RowMap& rows) {
  const int nb = rows.count(s.B);
  if (nb < 1 || nb > s.B) return SFI_ERR_SHAPE;
  CompactArgs a = compact_args(s, p, kv, bits, ld_b, pk, L_slow);
  a.rows = rows;
  if ((size_t)nb * s.Hkv * a.n_tiles * sizeof(int32_t) > cs.wcount_bytes) return SFI_ERR_WORKSPACE;
  a.tile_counts = cs.wcounts;
  const int BH = nb * s.Hkv;
  if (a.G <= 1) return launch_compact<1>(a, BH, st);
  if (a.G <= 2) return launch_compact<2>(a, BH, st);
  if (a.G <= 4) return launch_compact<4>(a, BH, st);
  if (a.G <= 8) return launch_compact<8>(a, BH, st);
  return launch_compact<16>(a, BH, st);
}

sfi_status run_compact_inc(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv,
                           const uint32_t* bits, int64_t ld_b, const sfi_packed& pk, const CompactScratch& cs,
                           int L_slow, bool fresh, cudaStream_t st, const RowMap& rows) {
  const int nb = rows.count(s.B);
  if (nb < 1 || nb > s.B) return SFI_ERR_SHAPE;
  if (fresh)   // sinks and the union in ascending order: the full compaction
    return run_compact_bits(s, p, kv, bits, ld_b, pk, cs, L_slow, st, rows);
  IncArgs a{};
  a.c = compact_args(s, p, kv, bits, ld_b, pk, L_slow);
  a.c.rows = rows;
  a.cap = cs.cap;
  if (a.cap % kPage != 0 || pk.p_max < a.cap) return SFI_ERR_SHAPE;
  if (a.c.nw > kIncMaxWords || a.cap > kIncCluster * kIncMaxSlotWords * 32) return SFI_ERR_UNSUPPORTED;
  a.mover_pos = cs.mover_pos;
  a.hole_slot = cs.hole_slot;
  const int BH = nb * s.Hkv;
  if (a.c.G <= 1) return launch_inc<1>(a, BH, st);
  if (a.c.G <= 2) return launch_inc<2>(a, BH, st);
  if (a.c.G <= 4) return launch_inc<4>(a, BH, st);
  if (a.c.G <= 8) return launch_inc<8>(a, BH, st);
  return launch_inc<16>(a, BH, st);
}

sfi_status run_idx_to_bits(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv, int L_slow,
                           const int32_t* sel_idx, int sel_ld, int K, uint32_t* bits, int64_t ld_b,
                           cudaStream_t st) {
  const int nC = L_slow - p.n_recent - p.n_sink;
  launch_k(idx_to_bits_kernel, dim3(s.B * s.Hq), dim3(256), 0, st, sel_idx, sel_ld, K, p.n_sink, nC, bits, ld_b,
           kv.err);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace sfi
