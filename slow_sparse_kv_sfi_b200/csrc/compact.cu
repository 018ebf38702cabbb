// Compaction of the selected tokens into the contiguous packed buffer
// ([ES] "3. Optimización del Sistema", item 2; [FR] "C. Optimisations
// Système", réorganisation; [NL] "Systeemontwerp", Memory-Coalesced Kernel;
// [ZH] "2.3" 两段式布局).
//
// Per (sequence, KV head): rows = sink tokens [0, n_sink), then the union of
// the group's per-head selections in ascending position order, each with a
// bitmask of the query heads that chose it (sinks: all heads), then zero rows
// up to the next multiple of 16.  The candidate range is cut into tiles of
// kCTile positions.  compact_count: per tile, rebuild the union bitmask in
// shared memory from the sorted selections (binary search per head) and count
// the rows.  compact_gather: the same bitmask, an ordered block scan, the page
// of every row in one round of independent loads, then the K and V rows are
// copied in 16-byte units with eight loads in flight per lane.
#include "common.cuh"
#include "internal.h"

namespace sfi {

constexpr int kCTile = 2048;
constexpr int kCThreads = 256;

struct CompactArgs {
  int Hkv, G, Hq, D, n_sink, lo, nC, K, sel_ld, n_tiles;
  int max_pages, num_pages, p_max;
  const int32_t* sel;
  const int32_t* pt;
  const uint4* kpool;
  const uint4* vpool;
  uint4* pk;
  uint4* pv;
  int32_t* pos;
  uint32_t* headmask;
  int32_t* n_rows;
  int32_t* tile_counts;   // [B*Hkv, n_tiles]
  int* err;
};

__device__ int lower_bound_i(const int32_t* a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < v) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Bitmask of the tile's candidate positions in shared memory.
__device__ void build_tile_mask(const CompactArgs& a, int b, int g, int t_lo, int t_n,
                                uint32_t* mask, int* ranges) {
  for (int i = threadIdx.x; i < kCTile; i += blockDim.x) mask[i] = 0u;
  if (threadIdx.x < a.G) {
    const int32_t* sh = a.sel + ((size_t)b * a.Hq + g * a.G + threadIdx.x) * a.sel_ld;
    ranges[2 * threadIdx.x] = lower_bound_i(sh, a.K, t_lo);
    ranges[2 * threadIdx.x + 1] = lower_bound_i(sh, a.K, t_lo + t_n);
  }
  __syncthreads();
  for (int h = 0; h < a.G; ++h) {
    const int32_t* sh = a.sel + ((size_t)b * a.Hq + g * a.G + h) * a.sel_ld;
    const int r0 = ranges[2 * h], r1 = ranges[2 * h + 1];
    for (int i = r0 + threadIdx.x; i < r1; i += blockDim.x) {
      const int p = sh[i] - t_lo;
      if ((unsigned)p < (unsigned)t_n) atomicOr(&mask[p], 1u << h);
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kCThreads) compact_count_kernel(const CompactArgs a) {
  __shared__ uint32_t mask[kCTile];
  __shared__ int ranges[64];
  __shared__ int wsum[kCThreads / 32];
  const int bg = blockIdx.y;
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int t_lo = a.lo + blockIdx.x * kCTile;
  const int t_n = min(kCTile, a.lo + a.nC - t_lo);
  // selections must lie in the candidate range: count the ones that do not
  if (blockIdx.x == 0 && threadIdx.x < a.G) {
    const int32_t* sh = a.sel + ((size_t)b * a.Hq + g * a.G + threadIdx.x) * a.sel_ld;
    if (a.K > 0 && (sh[0] < a.lo || sh[a.K - 1] >= a.lo + a.nC))
      latch_error(a.err, SFI_ERR_DEVICE_CHECK, kSiteCompactIdx);
  }
  build_tile_mask(a, b, g, t_lo, t_n, mask, ranges);
  int c = 0;
  for (int i = threadIdx.x; i < t_n; i += blockDim.x) c += mask[i] != 0u;
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

__global__ void __launch_bounds__(kCThreads) compact_gather_kernel(const CompactArgs a) {
  __shared__ uint32_t mask[kCTile];
  __shared__ int32_t rows[kCTile];
  __shared__ int32_t pgs[kCTile];
  __shared__ int ranges[64];
  __shared__ int wtot[64];
  __shared__ int base_s, total_s;
  const int bg = blockIdx.y;
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kCThreads / 32;
  const int t_lo = a.lo + blockIdx.x * kCTile;
  const int t_n = min(kCTile, a.lo + a.nC - t_lo);
  build_tile_mask(a, b, g, t_lo, t_n, mask, ranges);
  // rows before this tile
  if (warp == 0) {
    int s = 0;
    for (int t = lane; t < blockIdx.x; t += 32) s += a.tile_counts[(size_t)bg * a.n_tiles + t];
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) s += __shfl_xor_sync(0xffffffffu, s, sh);
    if (lane == 0) base_s = a.n_sink + s;
  }
  // ordered compaction of the tile: each thread owns kCTile / kCThreads consecutive slots
  constexpr int kPer = kCTile / kCThreads;
  const int j0 = threadIdx.x * kPer;
  int cnt = 0;
#pragma unroll
  for (int u = 0; u < kPer; ++u) cnt += (j0 + u < t_n) && mask[j0 + u] != 0u;
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
    for (int w = 0; w < kWarps; ++w) {
      const int t = wtot[w];
      wtot[32 + w] = s;
      s += t;
    }
    total_s = s;
  }
  __syncthreads();
  int off = x - cnt + wtot[32 + warp];
#pragma unroll
  for (int u = 0; u < kPer; ++u)
    if (j0 + u < t_n && mask[j0 + u] != 0u) rows[off++] = j0 + u;
  __syncthreads();
  const int base = base_s;
  const int total = min(total_s, max(a.p_max - base, 0));
  if (total < total_s && threadIdx.x == 0) latch_error(a.err, SFI_ERR_DEVICE_CHECK, kSiteCompactRows);
  // page of every row (independent loads), positions and head masks
  int32_t* pos = a.pos + (size_t)bg * a.p_max;
  uint32_t* hm = a.headmask + (size_t)bg * a.p_max;
  for (int i = threadIdx.x; i < total; i += kCThreads) {
    const int p = t_lo + rows[i];
    int page = a.pt[(size_t)b * a.max_pages + p / kPage];
    if ((unsigned)page >= (unsigned)a.num_pages) {
      latch_error(a.err, SFI_ERR_DEVICE_CHECK, kSiteCompactPage);
      page = -1;
    }
    pgs[i] = page;
    pos[base + i] = p;
    hm[base + i] = mask[rows[i]];
  }
  __syncthreads();
  // copy K and V rows: 16-byte units, eight in flight per lane
  const int chunks = a.D / 8;
  const int upr = 2 * chunks;
  const int nunits = total * upr;
  const size_t dst0 = ((size_t)bg * a.p_max + base) * chunks;
  for (int u0 = warp * 256; u0 < nunits; u0 += kWarps * 256) {
    uint4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int u = u0 + k * 32 + lane;
      v[k] = make_uint4(0, 0, 0, 0);
      if (u < nunits) {
        const int i = u / upr, c = u - i * upr;
        const int page = pgs[i];
        if (page >= 0) {
          const int p = t_lo + rows[i];
          const size_t src = ((size_t)(page * a.Hkv + g) * kPage + p % kPage) * chunks;
          v[k] = (c < chunks) ? __ldg(a.kpool + src + c) : __ldg(a.vpool + src + c - chunks);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int u = u0 + k * 32 + lane;
      if (u < nunits) {
        const int i = u / upr, c = u - i * upr;
        if (c < chunks) a.pk[dst0 + (size_t)i * chunks + c] = v[k];
        else a.pv[dst0 + (size_t)i * chunks + c - chunks] = v[k];
      }
    }
  }
  // sinks (first tile) and the zero tail (last tile)
  const uint32_t all = a.G >= 32 ? 0xffffffffu : ((1u << a.G) - 1u);
  if (blockIdx.x == 0) {
    const int ns = min(a.n_sink, a.p_max);
    for (int u = threadIdx.x; u < ns * upr; u += kCThreads) {
      const int i = u / upr, c = u - i * upr;
      const int page = a.pt[(size_t)b * a.max_pages + i / kPage];
      uint4 v = make_uint4(0, 0, 0, 0);
      if ((unsigned)page < (unsigned)a.num_pages) {
        const size_t src = ((size_t)(page * a.Hkv + g) * kPage + i % kPage) * chunks;
        v = (c < chunks) ? __ldg(a.kpool + src + c) : __ldg(a.vpool + src + c - chunks);
      } else if (c == 0) {
        latch_error(a.err, SFI_ERR_DEVICE_CHECK, kSiteCompactPage);
      }
      const size_t dst = ((size_t)bg * a.p_max + i) * chunks;
      if (c < chunks) a.pk[dst + c] = v;
      else a.pv[dst + c - chunks] = v;
      if (c == 0) {
        pos[i] = i;
        hm[i] = all;
      }
    }
  }
  if (blockIdx.x == gridDim.x - 1) {
    const int n = min(base + total_s, a.p_max);
    if (threadIdx.x == 0) a.n_rows[bg] = n;
    const int pad_end = min((n + kPage - 1) / kPage * kPage, a.p_max);
    for (int u = threadIdx.x; u < (pad_end - n) * upr; u += kCThreads) {
      const int r = n + u / upr, c = u % upr;
      const size_t dst = ((size_t)bg * a.p_max + r) * chunks;
      if (c < chunks) a.pk[dst + c] = make_uint4(0, 0, 0, 0);
      else a.pv[dst + c - chunks] = make_uint4(0, 0, 0, 0);
      if (c == 0) {
        pos[r] = -1;
        hm[r] = 0u;
      }
    }
  }
}

int compact_tiles(int nC) { return (nC + kCTile - 1) / kCTile; }

sfi_status run_compact(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv,
                       const int32_t* sel_idx, int sel_ld, int K, const sfi_packed& pk,
                       int32_t* tile_counts, size_t tc_bytes, int L_slow, cudaStream_t st) {
  CompactArgs a{};
  a.Hkv = s.Hkv; a.G = s.Hq / s.Hkv; a.Hq = s.Hq; a.D = s.D;
  a.n_sink = p.n_sink;
  a.lo = p.n_sink;
  a.nC = L_slow - p.n_recent - p.n_sink;
  a.K = K; a.sel_ld = sel_ld;
  a.n_tiles = compact_tiles(a.nC);
  if ((size_t)s.B * s.Hkv * a.n_tiles * sizeof(int32_t) > tc_bytes) return SFI_ERR_WORKSPACE;
  a.max_pages = s.max_pages; a.num_pages = s.num_pages; a.p_max = pk.p_max;
  a.sel = sel_idx; a.pt = kv.page_table;
  a.kpool = reinterpret_cast<const uint4*>(kv.k_pool);
  a.vpool = reinterpret_cast<const uint4*>(kv.v_pool);
  a.pk = reinterpret_cast<uint4*>(pk.k);
  a.pv = reinterpret_cast<uint4*>(pk.v);
  a.pos = pk.pos; a.headmask = pk.headmask; a.n_rows = pk.n_rows;
  a.tile_counts = tile_counts; a.err = kv.err;
  dim3 grid(a.n_tiles, s.B * s.Hkv);
  compact_count_kernel<<<grid, kCThreads, 0, st>>>(a);
  if (cudaPeekAtLastError() != cudaSuccess) return SFI_ERR_CUDA;
  compact_gather_kernel<<<grid, kCThreads, 0, st>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace sfi
