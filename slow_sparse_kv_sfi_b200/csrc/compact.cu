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
__global__ void __launch_bounds__(kCThreads) compact_count_kernel(const CompactArgs a) {
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
__global__ void __launch_bounds__(kCThreads) compact_gather_kernel(const CompactArgs a) {
  grid_dep_enter();
  __shared__ int wtot[kCThreads / 32 + 1];
  __shared__ int base_s, total_s;
  const int bg = blockIdx.y;
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
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
  int32_t* pos = a.pos + (size_t)bg * a.p_max;
  uint32_t* hm = a.headmask + (size_t)bg * a.p_max;
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
    if (threadIdx.x == 0) a.n_rows[bg] = n;
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
__global__ void __launch_bounds__(kCopyWarps * 32) compact_copy_kernel(const CompactArgs a) {
  grid_dep_enter();
  constexpr int kUnits = D / 8;                 // 16-byte units of one K (or V) row
  constexpr int kRowUnits = 2 * kUnits;         // K then V
  constexpr int kRowsPerPass = 32 / kRowUnits;  // rows one warp moves per pass
  constexpr int kRowsPerWarp = kCopyRows / kCopyWarps;
  constexpr int kIn = 8;                        // passes in flight
  static_assert(kRowsPerWarp % (kIn * kRowsPerPass) == 0 || kRowsPerWarp == kIn * kRowsPerPass, "copy plan");
  __shared__ long long src[kCopyRows];          // unit offset of the row in the pools, -1: zero row
  const int bg = blockIdx.y;
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int n = min(max(a.n_rows[bg], 0), a.p_max);
  const int pad_end = min((n + kPage - 1) / kPage * kPage, a.p_max);
  const int r0 = blockIdx.x * kCopyRows;
  if (r0 >= pad_end) return;
  const int nr = min(kCopyRows, pad_end - r0);
  const int32_t* pos = a.pos + (size_t)bg * a.p_max;
  if (threadIdx.x < kCopyRows) {
    const int r = r0 + threadIdx.x;
    long long off = -1;
    if (threadIdx.x < nr && r < n) {
      const int p = pos[r];
      const int pi = p / kPage;
      int page = -1;
      if (p >= 0 && pi < a.max_pages) page = __ldg(a.pt + (size_t)b * a.max_pages + pi);
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
  const size_t dst0 = ((size_t)bg * a.p_max + r0) * kUnits + cu;
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

sfi_status run_compact_bits(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv,
                            const uint32_t* bits, int64_t ld_b, const sfi_packed& pk,
                            int32_t* tile_counts, size_t tc_bytes, int L_slow, cudaStream_t st) {
  CompactArgs a{};
  a.Hkv = s.Hkv; a.G = s.Hq / s.Hkv; a.Hq = s.Hq; a.D = s.D;
  a.n_sink = p.n_sink;
  a.lo = p.n_sink;
  a.nC = L_slow - p.n_recent - p.n_sink;
  a.nw = (a.nC + 31) / 32;
  a.n_tiles = compact_tiles(a.nC);
  if ((size_t)s.B * s.Hkv * a.n_tiles * sizeof(int32_t) > tc_bytes) return SFI_ERR_WORKSPACE;
  a.max_pages = s.max_pages; a.num_pages = s.num_pages; a.p_max = pk.p_max;
  a.bits = bits; a.ld_b = ld_b;
  a.pt = kv.page_table;
  a.kpool = reinterpret_cast<const uint4*>(kv.k_pool);
  a.vpool = reinterpret_cast<const uint4*>(kv.v_pool);
  a.pk = reinterpret_cast<uint4*>(pk.k);
  a.pv = reinterpret_cast<uint4*>(pk.v);
  a.pos = pk.pos; a.headmask = pk.headmask; a.n_rows = pk.n_rows;
  a.tile_counts = tile_counts; a.err = kv.err;
  const int BH = s.B * s.Hkv;
  if (a.G <= 1) return launch_compact<1>(a, BH, st);
  if (a.G <= 2) return launch_compact<2>(a, BH, st);
  if (a.G <= 4) return launch_compact<4>(a, BH, st);
  if (a.G <= 8) return launch_compact<8>(a, BH, st);
  return launch_compact<16>(a, BH, st);
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
