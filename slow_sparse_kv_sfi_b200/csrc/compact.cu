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
#include "common.cuh"
#include "internal.h"

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
  grid_dep_enter();
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
  grid_dep_enter();
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
  grid_dep_enter();
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
// order, the layout of the full compaction.  Five launches per slow step:
//   inc_old    previous rows: mark their positions, keep or drop them;
//   inc_count  per bitmap tile: |U| and the entering count;
//   inc_slots  per slot tile: holes and kept rows past n_new;
//   inc_list   the mover list (entering positions, then moved rows) and the
//              hole list; clears the previous-position bitmap again;
//   inc_copy   the movers' rows into the holes, zero rows up to the next
//              multiple of 16, sinks of a fresh buffer, n_rows.
constexpr int kSTile = 1024;        // slots per slot tile (4 per thread)

int inc_slot_tiles(int cap) { return (cap + kSTile - 1) / kSTile; }

struct IncArgs {
  CompactArgs c;        // bitmaps, pages, packed buffer, error word
  int cap;              // packed rows any selection can need (multiple of 16)
  int n_stiles;
  int fresh;            // 1: ignore the previous rows
  int32_t* wcounts;     // [BH][n_tiles][2]  |U|, entering
  int32_t* scounts;     // [BH][n_stiles][2] holes, moved
  uint32_t* oldbits;    // [BH][nw] positions of the previous rows (zero between calls)
  int32_t* mover_pos;   // [BH][cap]
  int32_t* hole_slot;   // [BH][cap]
  int32_t* info;        // [BH][4] previous rows taken into account, n_new, holes, movers
};

template <int GM>
__device__ __forceinline__ uint32_t head_bits_at(const CompactArgs& a, int b, int g, int c) {
  uint32_t m = 0u;
#pragma unroll
  for (int h = 0; h < GM; ++h)
    if (h < a.G) m |= ((__ldg(a.bits + ((size_t)b * a.Hq + g * a.G + h) * a.ld_b + (c >> 5)) >> (c & 31)) & 1u) << h;
  return m;
}

// Exclusive block prefix of two counts packed as lo + (hi << 16) (each at
// most blockDim.x per call); returns the prefix, *total the block sum.
__device__ __forceinline__ int block_scan2(int x, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int v = x;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, d);
    if (lane >= d) v += y;
  }
  __syncthreads();
  if (lane == 31) sh[warp] = v;
  __syncthreads();
  int before = 0, all = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    const int t = sh[w];
    if (w < warp) before += t;
    all += t;
  }
  *total = all;
  return before + v - x;
}

__device__ __forceinline__ int n_old_of(const IncArgs& a, int bgp) {
  if (a.fresh) return 0;
  const int n = a.c.n_rows[bgp];
  return (n < a.c.n_sink || n > a.cap) ? 0 : n;
}

template <int GM>
__global__ void __launch_bounds__(kCThreads) inc_old_kernel(const __grid_constant__ IncArgs a) {
  grid_dep_enter();
  const int bg = blockIdx.y;                    // logical (row, kv head)
  const int b = bg / a.c.Hkv, g = bg - b * a.c.Hkv;
  const int bp = a.c.rows.phys(b);                // the sequence
  const int bgp = bp * a.c.Hkv + g;
  const int n_old = n_old_of(a, bgp);
  if (blockIdx.x == 0 && threadIdx.x == 0) a.info[bg * 4] = n_old;
  const int32_t* pos = a.c.pos + (size_t)bgp * a.c.p_max;
  uint32_t* hm = a.c.headmask + (size_t)bgp * a.c.p_max;
  uint32_t* ob = a.oldbits + (size_t)bg * a.c.nw;
  constexpr int kPer = kSTile / kCThreads;
  int c[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {   // all position loads first
    const int s = blockIdx.x * kSTile + i * kCThreads + threadIdx.x;
    c[i] = (s >= a.c.n_sink && s < n_old) ? pos[s] - a.c.lo : -1;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int s = blockIdx.x * kSTile + i * kCThreads + threadIdx.x;
    if (s < a.c.n_sink || s >= n_old) continue;
    uint32_t m = 0u;
    if (c[i] >= 0 && c[i] < a.c.nC) {
      atomicOr(ob + (c[i] >> 5), 1u << (c[i] & 31));
      m = head_bits_at<GM>(a.c, b, g, c[i]);
    }
    hm[s] = m;   // 0: the row leaves
  }
}

template <int GM>
__global__ void __launch_bounds__(kCThreads) inc_count_kernel(const __grid_constant__ IncArgs a) {
  grid_dep_enter();
  __shared__ int sh[kCThreads / 32];
  const int bg = blockIdx.y;
  const int b = bg / a.c.Hkv, g = bg - b * a.c.Hkv;
  const int w = blockIdx.x * kCWords + threadIdx.x;
  uint32_t hw[GM];
  const uint32_t u = union_word<GM>(a.c, b, g, w, hw);
  const uint32_t o = w < a.c.nw ? a.oldbits[(size_t)bg * a.c.nw + w] : 0u;
  int total;
  block_scan2(__popc(u) + (__popc(u & ~o) << 16), sh, &total);
  if (threadIdx.x == 0) {
    int32_t* wc = a.wcounts + ((size_t)bg * a.c.n_tiles + blockIdx.x) * 2;
    wc[0] = total & 0xffff;
    wc[1] = total >> 16;
  }
}

// Totals over the tiles before `upto` (and over all of them) of one count.
__device__ __forceinline__ void tile_prefix(const int32_t* cnt, int n, int upto, int which, int* before,
                                            int* all) {
  int s0 = 0, s1 = 0;
  for (int t = threadIdx.x & 31; t < n; t += 32) {
    const int v = cnt[t * 2 + which];
    s1 += v;
    if (t < upto) s0 += v;
  }
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) {
    s0 += __shfl_xor_sync(0xffffffffu, s0, sh);
    s1 += __shfl_xor_sync(0xffffffffu, s1, sh);
  }
  *before = s0;
  *all = s1;
}

__device__ __forceinline__ int n_new_of(const IncArgs& a, int bg) {
  int before, all;
  tile_prefix(a.wcounts + (size_t)bg * a.c.n_tiles * 2, a.c.n_tiles, 0, 0, &before, &all);
  return a.c.n_sink + all;
}

__global__ void __launch_bounds__(kCThreads) inc_slots_kernel(const __grid_constant__ IncArgs a) {
  grid_dep_enter();
  __shared__ int sh[kCThreads / 32];
  const int bg = blockIdx.y;                    // logical (row, kv head)
  const int bgp = a.c.rows.phys(bg / a.c.Hkv) * a.c.Hkv + bg % a.c.Hkv;
  const int n_old = a.info[bg * 4];
  const int n_new = min(n_new_of(a, bg), a.cap);
  const uint32_t* hm = a.c.headmask + (size_t)bgp * a.c.p_max;
  int x = 0;
#pragma unroll
  for (int i = 0; i < kSTile / kCThreads; ++i) {
    const int s = blockIdx.x * kSTile + i * kCThreads + threadIdx.x;
    const bool kept = s >= a.c.n_sink && s < n_old && hm[s] != 0u;
    x += (s >= a.c.n_sink && s < n_new && !kept) ? 1 : 0;
    x += (s >= n_new && kept) ? (1 << 16) : 0;
  }
  int total;
  block_scan2(x, sh, &total);
  if (threadIdx.x == 0) {
    int32_t* sc = a.scounts + ((size_t)bg * a.n_stiles + blockIdx.x) * 2;
    sc[0] = total & 0xffff;
    sc[1] = total >> 16;
  }
}

template <int GM>
__global__ void __launch_bounds__(kCThreads) inc_list_kernel(const __grid_constant__ IncArgs a) {
  grid_dep_enter();
  __shared__ int sh[kCThreads / 32];
  const int bg = blockIdx.y;                    // logical (row, kv head)
  const int b = bg / a.c.Hkv, g = bg - b * a.c.Hkv;
  const int bp = a.c.rows.phys(b);                // the sequence
  const int bgp = bp * a.c.Hkv + g;
  int32_t* mv = a.mover_pos + (size_t)bg * a.cap;
  const int32_t* wc = a.wcounts + (size_t)bg * a.c.n_tiles * 2;
  if ((int)blockIdx.x < a.c.n_tiles) {
    // entering positions of this bitmap tile, ascending
    const int w = blockIdx.x * kCWords + threadIdx.x;
    uint32_t hw[GM];
    const uint32_t u = union_word<GM>(a.c, b, g, w, hw);
    uint32_t* ob = a.oldbits + (size_t)bg * a.c.nw;
    const uint32_t o = w < a.c.nw ? ob[w] : 0u;
    if (w < a.c.nw && o) ob[w] = 0u;          // back to the zero state
    int before, all, total;
    tile_prefix(wc, a.c.n_tiles, blockIdx.x, 1, &before, &all);
    uint32_t e = u & ~o;
    int r = before + block_scan2(__popc(e), sh, &total);
    while (e) {
      const int bit = __ffs(e) - 1;
      e &= e - 1u;
      if (r < a.cap) mv[r] = a.c.lo + w * 32 + bit;
      ++r;
    }
    return;
  }
  // moved rows and holes of this slot tile, in slot order
  const int t = blockIdx.x - a.c.n_tiles;
  const int n_old = a.info[bg * 4];
  int e_before, e_all, h_before, h_all, m_before, m_all;
  tile_prefix(wc, a.c.n_tiles, 0, 1, &e_before, &e_all);
  const int n_want = n_new_of(a, bg);
  const int n_new = min(n_want, a.cap);
  const int32_t* sc = a.scounts + (size_t)bg * a.n_stiles * 2;
  tile_prefix(sc, a.n_stiles, t, 0, &h_before, &h_all);
  tile_prefix(sc, a.n_stiles, t, 1, &m_before, &m_all);
  if (t == 0 && threadIdx.x == 0) {
    // totals for the copy; n_new > cap is reported there
    a.info[bg * 4 + 1] = n_want;
    a.info[bg * 4 + 2] = h_all;
    a.info[bg * 4 + 3] = e_all + m_all;
  }
  const int32_t* pos = a.c.pos + (size_t)bgp * a.c.p_max;
  const uint32_t* hm = a.c.headmask + (size_t)bgp * a.c.p_max;
  int32_t* hs = a.hole_slot + (size_t)bg * a.cap;
  int hr = h_before, mr = e_all + m_before;
#pragma unroll 1
  for (int i = 0; i < kSTile / kCThreads; ++i) {
    const int s = t * kSTile + i * kCThreads + threadIdx.x;
    const bool kept = s >= a.c.n_sink && s < n_old && hm[s] != 0u;
    const bool hole = s >= a.c.n_sink && s < n_new && !kept;
    const bool moved = s >= n_new && kept;
    int total;
    const int pre = block_scan2((hole ? 1 : 0) + (moved ? 1 << 16 : 0), sh, &total);
    if (hole && hr + (pre & 0xffff) < a.cap) hs[hr + (pre & 0xffff)] = s;
    if (moved && mr + (pre >> 16) < a.cap) mv[mr + (pre >> 16)] = pos[s];
    hr += total & 0xffff;
    mr += total >> 16;
  }
}

template <int D, int GM>
__global__ void __launch_bounds__(kCopyWarps * 32) inc_copy_kernel(const __grid_constant__ IncArgs a) {
  grid_dep_enter();
  constexpr int kUnits = D / 8;
  constexpr int kRowUnits = 2 * kUnits;
  constexpr int kRowsPerPass = 32 / kRowUnits;
  constexpr int kRowsPerWarp = kCopyRows / kCopyWarps;
  constexpr int kIn = 8;
  __shared__ long long src[kCopyRows];
  __shared__ int dst[kCopyRows];
  const int bg = blockIdx.y;                    // logical (row, kv head)
  const int b = bg / a.c.Hkv, g = bg - b * a.c.Hkv;
  const int bp = a.c.rows.phys(b);                // the sequence
  const int bgp = bp * a.c.Hkv + g;
  const int4 inf = *reinterpret_cast<const int4*>(a.info + bg * 4);
  const int n_want = inf.y;
  const int n_new = min(n_want, a.cap);
  const int n_holes = inf.z, n_mov = inf.w;
  const bool fresh = inf.x == 0;
  const int pad_end = min((n_new + kPage - 1) / kPage * kPage, a.cap);
  const int n_pad = pad_end - n_new;
  const int n_sf = fresh ? a.c.n_sink : 0;
  const int items = n_holes + n_pad + n_sf;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    a.c.n_rows[bgp] = n_new;
    if (n_want > a.cap || n_mov < n_holes) latch_error(a.c.err, SFI_ERR_DEVICE_CHECK, kSiteCompactRows);
  }
  int32_t* pos = a.c.pos + (size_t)bgp * a.c.p_max;
  uint32_t* hm = a.c.headmask + (size_t)bgp * a.c.p_max;
  // 128-item chunks, strided over the blocks of this (b, KV head)
  for (int i0 = blockIdx.x * kCopyRows; i0 < items; i0 += gridDim.x * kCopyRows) {
    const int nr = min(kCopyRows, items - i0);
    __syncthreads();   // src/dst of the previous chunk consumed
    if (threadIdx.x < kCopyRows) {
      const int i = i0 + threadIdx.x;
      long long off = -1;
      int slot = -1;
      if (threadIdx.x < nr) {
        int p = -1;
        uint32_t m = 0u;
        if (i < n_holes) {
          slot = a.hole_slot[(size_t)bg * a.cap + i];
          if (i < n_mov) {
            p = a.mover_pos[(size_t)bg * a.cap + i];
            m = head_bits_at<GM>(a.c, b, g, p - a.c.lo);
          }
        } else if (i < n_holes + n_pad) {
          slot = n_new + (i - n_holes);
        } else {
          slot = i - n_holes - n_pad;
          p = slot;
          m = a.c.G >= 32 ? 0xffffffffu : ((1u << a.c.G) - 1u);
        }
        pos[slot] = p;
        hm[slot] = m;
        if (p >= 0) {
          const int pi = p / kPage;
          int page = -1;
          if (pi < a.c.max_pages) page = __ldg(a.c.pt + (size_t)bp * a.c.max_pages + pi);
          if ((unsigned)page >= (unsigned)a.c.num_pages) latch_error(a.c.err, SFI_ERR_DEVICE_CHECK, kSiteCompactPage);
          else off = ((long long)(page * a.c.Hkv + g) * kPage + p % kPage) * kUnits;
        }
      }
      src[threadIdx.x] = off;
      dst[threadIdx.x] = slot;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane / kRowUnits;
    const int u = lane % kRowUnits;
    const bool isv = u >= kUnits;
    const int cu = isv ? u - kUnits : u;
    const uint4* from = isv ? a.c.vpool : a.c.kpool;
    uint4* to = isv ? a.c.pv : a.c.pk;
    const size_t base = (size_t)bgp * a.c.p_max * kUnits + cu;
#pragma unroll
    for (int i0r = 0; i0r < kRowsPerWarp; i0r += kIn * kRowsPerPass) {
      uint4 v[kIn];
#pragma unroll
      for (int k = 0; k < kIn; ++k) {
        const int r = warp * kRowsPerWarp + i0r + k * kRowsPerPass + sub;
        const long long off = (r < nr) ? src[r] : -1;
        v[k] = off >= 0 ? __ldg(from + off + cu) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < kIn; ++k) {
        const int r = warp * kRowsPerWarp + i0r + k * kRowsPerPass + sub;
        if (r < nr) to[base + (size_t)dst[r] * kUnits] = v[k];
      }
    }
  }
}

// Blocks of inc_copy per (b, KV head): enough for a large move to reach the
// copy bandwidth, few enough that a small one is not a launch of idle blocks.
int inc_copy_blocks(int cap, int n_sink, int BH, int sms) {
  const int chunks = (cap + kPage + n_sink + kCopyRows - 1) / kCopyRows;
  return std::max(1, std::min(chunks, (4 * sms + BH - 1) / BH));
}

size_t compact_scratch_bytes(const sfi_shape& s, const sfi_params& p) {
  const long bh = (long)s.B * s.Hkv;
  const int Lmax = s.max_pages * kPage;
  const int nC = std::max(Lmax - p.n_recent - p.n_sink, 1);
  const int cap = packed_rows_capacity(s, p);
  return align_up((size_t)bh * compact_tiles(nC) * 2 * sizeof(int32_t), 256) +
         align_up((size_t)bh * inc_slot_tiles(cap) * 2 * sizeof(int32_t), 256) +
         align_up((size_t)bh * ((nC + 31) / 32) * sizeof(uint32_t), 256) +
         2 * align_up((size_t)bh * cap * sizeof(int32_t), 256) + align_up((size_t)bh * 4 * sizeof(int32_t), 256);
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
  c.scounts = reinterpret_cast<int32_t*>(w);
  w += align_up((size_t)bh * inc_slot_tiles(cap) * 2 * sizeof(int32_t), 256);
  c.oldbits = reinterpret_cast<uint32_t*>(w);
  w += align_up((size_t)bh * ((nC + 31) / 32) * sizeof(uint32_t), 256);
  c.mover_pos = reinterpret_cast<int32_t*>(w);
  w += align_up((size_t)bh * cap * sizeof(int32_t), 256);
  c.hole_slot = reinterpret_cast<int32_t*>(w);
  w += align_up((size_t)bh * cap * sizeof(int32_t), 256);
  c.info = reinterpret_cast<int32_t*>(w);
  return c;
}

template <int GM>
sfi_status launch_inc(const IncArgs& a, int BH, cudaStream_t st) {
  const dim3 sgrid(a.n_stiles, BH), wgrid(a.c.n_tiles, BH);
  launch_k(inc_old_kernel<GM>, sgrid, dim3(kCThreads), 0, st, a);
  launch_k(inc_count_kernel<GM>, wgrid, dim3(kCThreads), 0, st, a);
  launch_k(inc_slots_kernel, sgrid, dim3(kCThreads), 0, st, a);
  launch_k(inc_list_kernel<GM>, dim3(a.c.n_tiles + a.n_stiles, BH), dim3(kCThreads), 0, st, a);
  const dim3 cgrid(inc_copy_blocks(a.cap, a.c.n_sink, BH, num_sms()), BH);
  if (a.c.D == 128) launch_k(inc_copy_kernel<128, GM>, cgrid, dim3(kCopyWarps * 32), 0, st, a);
  else launch_k(inc_copy_kernel<64, GM>, cgrid, dim3(kCopyWarps * 32), 0, st, a);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
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
  IncArgs a{};
  a.c = compact_args(s, p, kv, bits, ld_b, pk, L_slow);
  a.c.rows = rows;
  a.cap = cs.cap;
  if (a.cap % kPage != 0 || pk.p_max < a.cap) return SFI_ERR_SHAPE;
  a.n_stiles = inc_slot_tiles(a.cap);
  if (fresh)   // same layout as the full compaction, which copies faster
    return run_compact_bits(s, p, kv, bits, ld_b, pk, cs, L_slow, st, rows);
  a.fresh = 0;
  a.wcounts = cs.wcounts; a.scounts = cs.scounts; a.oldbits = cs.oldbits;
  a.mover_pos = cs.mover_pos; a.hole_slot = cs.hole_slot; a.info = cs.info;
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
