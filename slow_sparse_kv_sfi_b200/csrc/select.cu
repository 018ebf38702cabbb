// The training-free Selector of Slow-Fast Inference ([ES] "El Selector";
// [FR] "B. Le Sélecteur"; [NL] "De Selector"; [ZH] "2.2 训练无感的 Selector").
//
// For the candidates C = [n_sink, L - n_recent) of a slow step:
//   evidence   f~_{h,j} = exp(z_{h,j} - lse_C,h)     (f restricted to C, renormalised)
//   prior      r_j = kappa_j pi_j / sum_C kappa pi,
//              kappa_j = min(1, nbar / ||k_j||), pi_j = ln(1 + L - j)
//   fusion     s = (1 - lambda) f~ + lambda r          (the closed form of [NL], [ZH])
//   log-score  l = ln(s + 1e-30)
//   soft-NMS   l' = l - alpha_soft * (1 - (d - 1) / w), d = distance to the
//              nearest dominating neighbour within w (none: no penalty)
//   exclusivity l'' = l' - alpha_cross * [h != argmax_h' l'_{h',j}]
//   top-K      K largest l'' per query head, ties to the lower position.
//
// Kernels: stats_norm / stats_prior (per (b, kv head) and chunk of C: fp64
// partial sums of the norms and of kappa pi; every consumer reduces the
// partials in the same fixed order), select_scores (one CTA per (b, kv group,
// candidate tile) holding all G heads plus a halo of w on each side in shared
// memory, so soft-NMS and the cross-head owner need no second pass over
// memory; it also records each row's min and max), topk_kernel (one CTA per
// row: linear bins over [min, max], boundary-bin candidates resolved exactly
// by MSB radix select on order-preserving uint32 keys, ties by position; a
// selection bitmap and / or ascending positions out).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sfi {

constexpr int kStatThreads = 256;
constexpr int kStatChunk = 4096;

__device__ __forceinline__ double block_sum_d(double v, double* red) {
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) v += __shfl_xor_sync(0xffffffffu, v, sh);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x < 32) {
    t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) t += __shfl_xor_sync(0xffffffffu, t, sh);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}

// Sum of the per-chunk partials part[k * 2 + which], k < nch, by warp 0 in a
// fixed order (every CTA that needs it gets the bit-identical value).
__device__ __forceinline__ double reduce_parts(const double* part, int nch, int which, double* bcast) {
  if (threadIdx.x < 32) {
    double t = 0.0;
    for (int k = threadIdx.x; k < nch; k += 32) t += part[k * 2 + which];
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) t += __shfl_xor_sync(0xffffffffu, t, sh);
    if (threadIdx.x == 0) *bcast = t;
  }
  __syncthreads();
  const double r = *bcast;
  __syncthreads();
  return r;
}

__device__ __forceinline__ float kappa_of(float nbar, float n) {
  return n > 0.f ? fminf(1.f, nbar / n) : 1.f;
}

__device__ __forceinline__ float pi_of(int L, int j) { return logf((float)(1 + L - j)); }

__device__ __forceinline__ float nbar_of(double sum_norms, int nC) { return (float)(sum_norms / (double)nC); }

// part[bg][chunk][0] = sum of key norms over the chunk of C
__global__ void __launch_bounds__(kStatThreads) stats_norm_kernel(int lo, int nC, const float* __restrict__ norms,
                                                                  int64_t norm_ld, double* part, int nch,
                                                                  uint32_t* rowmm, int G) {
  grid_dep_enter();
  __shared__ double red[32];
  const int bg = blockIdx.y;
  if (rowmm && blockIdx.x == 0 && threadIdx.x < G) {   // the score kernel folds into these
    rowmm[((size_t)bg * G + threadIdx.x) * 2] = 0xffffffffu;
    rowmm[((size_t)bg * G + threadIdx.x) * 2 + 1] = 0u;
  }
  const float* n = norms + (size_t)bg * norm_ld + lo;
  const int c0 = blockIdx.x * kStatChunk, c1 = min(nC, c0 + kStatChunk);
  double sacc = 0.0;
  for (int c = c0 + threadIdx.x; c < c1; c += blockDim.x) sacc += (double)n[c];
  const double t = block_sum_d(sacc, red);
  if (threadIdx.x == 0) part[((size_t)bg * nch + blockIdx.x) * 2] = t;
}

// part[bg][chunk][1] = sum of kappa * pi over the chunk of C
__global__ void __launch_bounds__(kStatThreads) stats_prior_kernel(int L, int lo, int nC,
                                                                   const float* __restrict__ norms,
                                                                   int64_t norm_ld, double* part, int nch) {
  grid_dep_enter();
  __shared__ double red[32];
  __shared__ double bc;
  const int bg = blockIdx.y;
  double* pbg = part + (size_t)bg * nch * 2;
  const float nbar = nbar_of(reduce_parts(pbg, nch, 0, &bc), nC);
  const float* n = norms + (size_t)bg * norm_ld;
  const int c0 = blockIdx.x * kStatChunk, c1 = min(nC, c0 + kStatChunk);
  double z = 0.0;
  for (int c = c0 + threadIdx.x; c < c1; c += blockDim.x) {
    const int j = lo + c;
    z += (double)(kappa_of(nbar, n[j]) * pi_of(L, j));
  }
  const double t = block_sum_d(z, red);
  if (threadIdx.x == 0) pbg[blockIdx.x * 2 + 1] = t;
}

struct ScoreArgs {
  int L, lo, nC, Hq, Hkv, G, w, tile;
  float lam, alpha_soft, alpha_cross;
  const float* logits;
  int64_t ld;
  const float* lse_cand;
  const float* norms;
  int64_t norm_ld;
  const double* stat_part;   // [B*Hkv][nch][2]
  int nch;
  float* scores;
  int64_t ld_s;
  uint32_t* rowmm;           // [B*Hq][2]: min / max order key of each score row
};

// One CTA per (b, KV group, tile of candidates).  Phase 1 writes the log-score
// of every head of the group over the tile plus a halo of w on each side to
// shared memory (NaN outside C: a NaN never dominates).  Phase 2: the thread
// of a position applies soft-NMS to every head in registers, picks the owner
// and writes l''; it also folds the order keys into per-row min / max.
template <int GM>
__global__ void __launch_bounds__(256) select_scores_kernel(const ScoreArgs a) {
  grid_dep_enter();
  extern __shared__ float sm[];
  const int W = a.tile + 2 * a.w;     // haloed width
  float* ell = sm;                    // [G][W]
  const int bg = blockIdx.y;
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int c0 = blockIdx.x * a.tile;
  const int tile_n = min(a.tile, a.nC - c0);
  const int G = a.G;
  __shared__ double bc;
  const double* pbg = a.stat_part + (size_t)bg * a.nch * 2;
  const float nbar = nbar_of(reduce_parts(pbg, a.nch, 0, &bc), a.nC);
  const float inv_z = (float)(1.0 / reduce_parts(pbg, a.nch, 1, &bc));
  const float* nrm = a.norms + (size_t)bg * a.norm_ld;
  const float lam = a.lam;
  const size_t row0 = (size_t)b * a.Hq + (size_t)g * G;
  const float* z0 = a.logits + row0 * a.ld + a.lo;
  const float nan = __int_as_float(0x7fc00000);
  for (int k = threadIdx.x; k < W; k += blockDim.x) {
    const int c = c0 - a.w + k;
    if (c >= 0 && c < a.nC) {
      const int j = a.lo + c;
      const float r = kappa_of(nbar, nrm[j]) * pi_of(a.L, j) * inv_z;
      float zv[GM];
#pragma unroll
      for (int h = 0; h < GM; ++h) zv[h] = (h < G) ? z0[(size_t)h * a.ld + c] : 0.f;
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        if (h < G) {
          const float ft = expf(zv[h] - a.lse_cand[row0 + h]);
          const float s = (1.f - lam) * ft + lam * r;
          ell[h * W + k] = logf(s + 1e-30f);
        }
      }
    } else {
#pragma unroll
      for (int h = 0; h < GM; ++h)
        if (h < G) ell[h * W + k] = nan;
    }
  }
  __syncthreads();
  const float inv_w = 1.f / (float)a.w;
  uint32_t kmin[GM], kmax[GM];
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    kmin[h] = 0xffffffffu;
    kmax[h] = 0u;
  }
  for (int k = threadIdx.x; k < tile_n; k += blockDim.x) {
    float l1[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      l1[h] = -INFINITY;
      if (h < G) {
        const float* row = ell + h * W + a.w + k;
        const float e = row[0];
        float pen = 0.f;
        for (int d = 1; d <= a.w; ++d) {
          if (row[-d] >= e || row[d] > e) {   // NaN (outside C) compares false
            pen = 1.f - (float)(d - 1) * inv_w;
            break;
          }
        }
        l1[h] = e - a.alpha_soft * pen;
      }
    }
    int owner = 0;
    float best = l1[0];
#pragma unroll
    for (int h = 1; h < GM; ++h)
      if (h < G && l1[h] > best) {
        best = l1[h];
        owner = h;
      }
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      if (h < G) {
        const float v = l1[h] - (h != owner ? a.alpha_cross : 0.f);
        a.scores[(row0 + h) * a.ld_s + c0 + k] = v;
        const uint32_t key = float_key(v);
        kmin[h] = min(kmin[h], key);
        kmax[h] = max(kmax[h], key);
      }
    }
  }
  if (a.rowmm) {
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      if (h >= G) continue;
      uint32_t mn = kmin[h], mx = kmax[h];
#pragma unroll
      for (int sh = 16; sh >= 1; sh >>= 1) {
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, sh));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, sh));
      }
      if ((threadIdx.x & 31) == 0) {
        atomicMin(&a.rowmm[(row0 + h) * 2], mn);
        atomicMax(&a.rowmm[(row0 + h) * 2 + 1], mx);
      }
    }
  }
}

// ---------------------------------------------------------------- top-K
constexpr int kTopkThreads = 1024;
constexpr int kBins = 4096;       // first digit: linear bins over [min, max] of the row
constexpr int kRBins = 2048;      // exact radix digits (11 bits)
constexpr int kCap = 4096;        // boundary-bin candidates resolved in shared memory
constexpr int kTopkMaxWords = 8192;

// Reverse (suffix) inclusive scan of one value per thread across the block.
__device__ __forceinline__ int block_suffix_incl(int v, int* wtot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int sh = 1; sh < 32; sh <<= 1) {
    const int y = __shfl_down_sync(0xffffffffu, x, sh);
    if (lane + sh < 32) x += y;
  }
  if (lane == 0) wtot[w] = x;   // total of this warp
  __syncthreads();
  if (w == 0) {
    const int nwarps = blockDim.x >> 5;
    int t = lane < nwarps ? wtot[lane] : 0;
    int s = t;
#pragma unroll
    for (int sh = 1; sh < 32; sh <<= 1) {
      const int y = __shfl_down_sync(0xffffffffu, s, sh);
      if (lane + sh < 32) s += y;
    }
    wtot[32 + lane] = s - t;      // sum of warps after this one
  }
  __syncthreads();
  const int r = x + wtot[32 + w];
  __syncthreads();
  return r;
}

// Exclusive prefix scan of one value per thread across the block.
__device__ __forceinline__ int block_prefix_excl(int v, int* wtot, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int sh = 1; sh < 32; sh <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, sh);
    if (lane >= sh) x += y;
  }
  if (lane == 31) wtot[w] = x;
  __syncthreads();
  if (w == 0) {
    const int nwarps = blockDim.x >> 5;
    const int t = lane < nwarps ? wtot[lane] : 0;
    int s = t;
#pragma unroll
    for (int sh = 1; sh < 32; sh <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, sh);
      if (lane >= sh) s += y;
    }
    wtot[32 + lane] = s - t;
    if (lane == 31) *total = s;
  }
  __syncthreads();
  const int r = x - v + wtot[32 + w];
  __syncthreads();
  return r;
}

__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Bin b of `hist` (nb bins, held 1024 / nb... by the block) containing the
// k-th largest element counted from the top: sets *bin and *above (elements
// in higher bins).  Each thread owns nb / blockDim consecutive bins.
__device__ __forceinline__ void find_bin(const int* hist, int nb, int k, int* wtot, int* s_bin,
                                         int* s_above) {
  const int per = nb / blockDim.x;
  const int b0 = threadIdx.x * per;
  int mine = 0;
  for (int i = 0; i < per; ++i) mine += hist[b0 + i];
  const int incl = block_suffix_incl(mine, wtot);
  int above = incl - mine;   // bins after this thread's
  for (int i = per - 1; i >= 0; --i) {
    const int h = hist[b0 + i];
    if (above < k && above + h >= k) {
      *s_bin = b0 + i;
      *s_above = above;
    }
    above += h;
  }
  __syncthreads();
}

// One CTA per row: the K largest scores (ties to the lower index) as a
// selection bitmap and / or K ascending positions.
//  1. linear bins over [min, max] of the row (from the score kernel, or one
//     extra pass): histogram, the boundary bin and how many to take from it;
//  2. one pass: elements above the boundary bin are selected (warp ballots
//     become bitmap words), boundary-bin elements are candidates;
//  3. exact MSB radix select of the boundary among the candidates in shared
//     memory (or, if they do not fit, over the row restricted to the bin);
//  4. ties at the threshold key: the lowest positions first;
//  5. bitmap and/or ordered positions out.
template <bool VEC>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(int n, const float* __restrict__ scores,
                                                            int64_t ld_s, int K, int offset,
                                                            int32_t* __restrict__ idx, int64_t ld_i,
                                                            uint32_t* __restrict__ bits, int64_t ld_b,
                                                            const uint32_t* __restrict__ rowmm) {
  grid_dep_enter();
  extern __shared__ uint32_t tsm[];
  const int nw = (n + 31) / 32;
  uint32_t* sel = tsm;                           // [nw]
  uint32_t* tie = sel + nw;                      // [nw]
  int* hist = reinterpret_cast<int*>(tie + nw);  // [kBins]
  uint32_t* ckey = reinterpret_cast<uint32_t*>(hist + kBins);   // [kCap]
  int* cidx = reinterpret_cast<int*>(ckey + kCap);               // [kCap]
  __shared__ int wtot[64];
  __shared__ int s_bin, s_above, s_total, s_nc;
  __shared__ uint32_t s_mn, s_mx;
  const int row_id = blockIdx.x;
  const float* row = scores + (size_t)row_id * ld_s;
  const int tid = threadIdx.x, lane = tid & 31;

  for (int i = tid; i < nw; i += blockDim.x) sel[i] = tie[i] = 0u;
  for (int i = tid; i < kBins; i += blockDim.x) hist[i] = 0;
  if (tid == 0) {
    s_nc = 0;
    s_mn = 0xffffffffu;
    s_mx = 0u;
  }
  __syncthreads();
  // -- 0. key range
  uint32_t mn, mx;
  if (rowmm) {
    mn = rowmm[2 * row_id];
    mx = rowmm[2 * row_id + 1];
  } else {
    uint32_t a = 0xffffffffu, c = 0u;
    for (int j = tid; j < n; j += blockDim.x) {
      const uint32_t k = float_key(__ldg(row + j));
      a = min(a, k);
      c = max(c, k);
    }
    atomicMin(&s_mn, a);
    atomicMax(&s_mx, c);
    __syncthreads();
    mn = s_mn;
    mx = s_mx;
  }
  const float vmin = key_float(mn), vmax = key_float(mx);
  const float scale = (vmax > vmin) ? (float)(kBins - 1) / (vmax - vmin) : 0.f;
  auto bin_of = [&](float v) -> int {
    const int bb = (int)((v - vmin) * scale);
    return min(max(bb, 0), kBins - 1);
  };
  // -- 1. histogram of linear bins
  for (int j = tid; j < n; j += blockDim.x) atomicAdd(&hist[bin_of(__ldg(row + j))], 1);
  __syncthreads();
  find_bin(hist, kBins, K, wtot, &s_bin, &s_above);
  const int b1 = s_bin;
  int k_rem = K - s_above;   // to take from bin b1 (>= 1)
  // -- 2. above the bin: selected; in the bin: candidates
  for (int base = 0; base < n; base += blockDim.x) {
    const int j = base + tid;
    int bb = -1;
    uint32_t key = 0u;
    if (j < n) {
      const float v = __ldg(row + j);
      bb = bin_of(v);
      key = float_key(v);
    }
    const unsigned up = __ballot_sync(0xffffffffu, bb > b1);
    if (lane == 0 && j < n) sel[j >> 5] = up;
    const unsigned cand = __ballot_sync(0xffffffffu, bb == b1);
    if (cand) {
      int slot0 = 0;
      if (lane == 0) slot0 = atomicAdd(&s_nc, __popc(cand));
      slot0 = __shfl_sync(0xffffffffu, slot0, 0);
      if (bb == b1) {
        const int at = slot0 + __popc(cand & ((1u << lane) - 1u));
        if (at < kCap) {
          ckey[at] = key;
          cidx[at] = j;
        }
      }
    }
  }
  __syncthreads();
  const int nc = s_nc;
  const bool fits = nc <= kCap;
  // -- 3. exact threshold key T among the bin's elements: MSB radix, 11/11/10 bits
  uint32_t prefix = 0, pmask = 0;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int sh = shifts[pass];
    const uint32_t dmask = (1u << widths[pass]) - 1u;
    for (int i = tid; i < kRBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    if (fits) {
      for (int c = tid; c < nc; c += blockDim.x) {
        const uint32_t k = ckey[c];
        if ((k & pmask) == prefix) atomicAdd(&hist[(k >> sh) & dmask], 1);
      }
    } else {
      for (int j = tid; j < n; j += blockDim.x) {
        const float v = __ldg(row + j);
        const uint32_t k = float_key(v);
        if (bin_of(v) == b1 && (k & pmask) == prefix) atomicAdd(&hist[(k >> sh) & dmask], 1);
      }
    }
    __syncthreads();
    find_bin(hist, kRBins, k_rem, wtot, &s_bin, &s_above);
    prefix |= (uint32_t)s_bin << sh;
    pmask |= dmask << sh;
    k_rem -= s_above;
  }
  const uint32_t T = prefix;   // take k_rem of the keys equal to T, lowest positions first
  // -- 4. mark the bin's elements above T, and the ties
  if (fits) {
    for (int c = tid; c < nc; c += blockDim.x) {
      const uint32_t k = ckey[c];
      const int j = cidx[c];
      if (k > T) atomicOr(&sel[j >> 5], 1u << (j & 31));
      else if (k == T) atomicOr(&tie[j >> 5], 1u << (j & 31));
    }
  } else {
    for (int j = tid; j < n; j += blockDim.x) {
      const float v = __ldg(row + j);
      const uint32_t k = float_key(v);
      if (bin_of(v) != b1) continue;
      if (k > T) atomicOr(&sel[j >> 5], 1u << (j & 31));
      else if (k == T) atomicOr(&tie[j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();
  // -- 5. the first k_rem ties in position order join the selection
  const int per = (nw + blockDim.x - 1) / blockDim.x;
  const int w0 = tid * per;
  {
    int mine = 0;
    for (int i = 0; i < per; ++i)
      if (w0 + i < nw) mine += __popc(tie[w0 + i]);
    int before = block_prefix_excl(mine, wtot, &s_total);
    for (int i = 0; i < per && before < k_rem; ++i) {
      if (w0 + i >= nw) break;
      uint32_t t = tie[w0 + i];
      uint32_t take = 0u;
      while (t && before < k_rem) {
        const uint32_t lowbit = t & (~t + 1u);
        take |= lowbit;
        t ^= lowbit;
        ++before;
      }
      sel[w0 + i] |= take;
    }
  }
  __syncthreads();
  // -- 6. outputs
  if (bits) {
    uint32_t* brow = bits + (size_t)row_id * ld_b;
    for (int i = tid; i < nw; i += blockDim.x) brow[i] = sel[i];
  }
  if (idx) {
    int32_t* out = idx + (size_t)row_id * ld_i;
    int mine = 0;
    for (int i = 0; i < per; ++i)
      if (w0 + i < nw) mine += __popc(sel[w0 + i]);
    int at = block_prefix_excl(mine, wtot, &s_total);
    for (int i = 0; i < per; ++i) {
      if (w0 + i >= nw) break;
      uint32_t t = sel[w0 + i];
      while (t) {
        const int bpos = __ffs(t) - 1;
        t &= t - 1u;
        if (at < K) out[at] = offset + (w0 + i) * 32 + bpos;
        ++at;
      }
    }
  }
}

// ---------------------------------------------------------------- host
int score_tile(int G) { return std::max(256, 8192 / G); }

size_t score_smem(int G, int tile, int w) { return (size_t)G * (tile + 2 * w) * sizeof(float); }

int stat_chunks(int nC) { return (nC + kStatChunk - 1) / kStatChunk; }

int topk_max_n() { return kTopkMaxWords * 32; }

size_t topk_smem(int n) {
  const size_t nw = (size_t)(n + 31) / 32;
  return (2 * nw + kBins + 2 * kCap) * sizeof(uint32_t);
}

template <int GM>
sfi_status launch_scores(const ScoreArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
  static DeviceOnce attr;
  if (!attr.done() &&
      !attr.mark(cudaFuncSetAttribute(select_scores_kernel<GM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      200 * 1024)))
    return SFI_ERR_CUDA;
  launch_k(select_scores_kernel<GM>, dim3(grid), dim3(256), smem, st, a);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

sfi_status run_select_scores(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv,
                             int L, const float* logits, int64_t ld, const float* lse_cand,
                             float* scores, int64_t ld_s, void* stat_ws, uint32_t* rowmm,
                             cudaStream_t st) {
  const int G = s.Hq / s.Hkv;
  const int lo = p.n_sink, hi = L - p.n_recent;
  const int nC = hi - lo;
  double* part = reinterpret_cast<double*>(stat_ws);
  const int nch = stat_chunks(nC);
  const int64_t norm_ld = (int64_t)s.max_pages * kPage;
  dim3 sgrid(nch, s.B * s.Hkv);
  launch_k(stats_norm_kernel, dim3(sgrid), dim3(kStatThreads), 0, st, lo, nC, kv.key_norms, norm_ld, part, nch, rowmm,
           G);
  launch_k(stats_prior_kernel, dim3(sgrid), dim3(kStatThreads), 0, st, L, lo, nC, kv.key_norms, norm_ld, part, nch);
  if (cudaPeekAtLastError() != cudaSuccess) return SFI_ERR_CUDA;
  ScoreArgs a{};
  a.L = L; a.lo = lo; a.nC = nC; a.Hq = s.Hq; a.Hkv = s.Hkv; a.G = G;
  a.w = std::max(p.nms_window / 2, 1);
  a.tile = score_tile(G);
  const float lam = std::min(std::max(p.lambda, 0.f), p.lambda_clip);
  a.lam = lam;
  a.alpha_soft = p.nms_window / 2 >= 1 ? p.alpha_soft : 0.f;
  a.alpha_cross = p.alpha_cross;
  a.logits = logits; a.ld = ld; a.lse_cand = lse_cand;
  a.norms = kv.key_norms; a.norm_ld = norm_ld;
  a.stat_part = part; a.nch = nch;
  a.scores = scores; a.ld_s = ld_s;
  a.rowmm = rowmm;
  const size_t smem = score_smem(G, a.tile, a.w);
  dim3 grid((nC + a.tile - 1) / a.tile, s.B * s.Hkv);
  if (G <= 1) return launch_scores<1>(a, grid, smem, st);
  if (G <= 2) return launch_scores<2>(a, grid, smem, st);
  if (G <= 4) return launch_scores<4>(a, grid, smem, st);
  if (G <= 8) return launch_scores<8>(a, grid, smem, st);
  return launch_scores<16>(a, grid, smem, st);
}

sfi_status run_topk(int rows, int n, const float* scores, int64_t ld_s, int K, int offset,
                    int32_t* idx, int64_t ld_i, uint32_t* bits, int64_t ld_b, const uint32_t* rowmm,
                    cudaStream_t st) {
  if (rows <= 0) return SFI_OK;
  if (n > topk_max_n()) return SFI_ERR_UNSUPPORTED;
  const size_t smem = topk_smem(n);
  static DeviceOnce attr;
  if (!attr.done() &&
      !attr.mark(cudaFuncSetAttribute(topk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)topk_smem(topk_max_n()))))
    return SFI_ERR_CUDA;
  launch_k(topk_kernel<false>, dim3(rows), dim3(kTopkThreads), smem, st, n, scores, ld_s, K, offset, idx, ld_i, bits,
           ld_b, rowmm);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace sfi
