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
// partials in the same fixed order), select_scores (one CTA per (b, kv group, candidate tile) holding all
// G heads plus a halo of w on each side in shared memory, so soft-NMS and the
// cross-head owner need no second pass over memory), topk_kernel (one CTA
// per row: 3-pass MSB radix select on order-preserving uint32 keys, then one
// ordered pass writing the K positions ascending).
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
                                                                  int64_t norm_ld, double* part, int nch) {
  __shared__ double red[32];
  const int bg = blockIdx.y;
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
};

__global__ void __launch_bounds__(256) select_scores_kernel(const ScoreArgs a) {
  extern __shared__ float sm[];
  const int W = a.tile + 2 * a.w;     // haloed width
  float* ell = sm;                    // [G][W]
  float* ell1 = ell + a.G * W;        // [G][tile]
  float* rr = ell1 + a.G * a.tile;    // [W] prior
  const int bg = blockIdx.y;
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int c0 = blockIdx.x * a.tile;
  const int tile_n = min(a.tile, a.nC - c0);
  __shared__ double bc;
  const double* pbg = a.stat_part + (size_t)bg * a.nch * 2;
  const float nbar = nbar_of(reduce_parts(pbg, a.nch, 0, &bc), a.nC);
  const float inv_z = (float)(1.0 / reduce_parts(pbg, a.nch, 1, &bc));
  const float* nrm = a.norms + (size_t)bg * a.norm_ld;

  // prior over the haloed tile
  for (int k = threadIdx.x; k < W; k += blockDim.x) {
    const int c = c0 - a.w + k;
    float r = 0.f;
    if (c >= 0 && c < a.nC) {
      const int j = a.lo + c;
      r = kappa_of(nbar, nrm[j]) * pi_of(a.L, j) * inv_z;
    }
    rr[k] = r;
  }
  __syncthreads();
  // fused log-score over the haloed tile, all heads of the group
  const float lam = a.lam;
  for (int idx = threadIdx.x; idx < a.G * W; idx += blockDim.x) {
    const int h = idx / W, k = idx - h * W;
    const int c = c0 - a.w + k;
    float e = __int_as_float(0x7fc00000);   // NaN outside C: never a neighbour
    if (c >= 0 && c < a.nC) {
      const int hq = g * a.G + h;
      const float z = a.logits[((size_t)b * a.Hq + hq) * a.ld + a.lo + c];
      const float ft = expf(z - a.lse_cand[(size_t)b * a.Hq + hq]);
      const float s = (1.f - lam) * ft + lam * rr[k];
      e = logf(s + 1e-30f);
    }
    ell[idx] = e;
  }
  __syncthreads();
  // soft-NMS: nearest dominating neighbour within w
  const float inv_w = 1.f / (float)a.w;
  for (int idx = threadIdx.x; idx < a.G * a.tile; idx += blockDim.x) {
    const int h = idx / a.tile, k = idx - h * a.tile;
    if (k >= tile_n) continue;
    const int c = c0 + k;
    const float* row = ell + h * W + a.w + k;
    const float e = row[0];
    float pen = 0.f;
    for (int d = 1; d <= a.w; ++d) {
      const bool left = (c - d >= 0) && (row[-d] >= e);
      const bool right = (c + d < a.nC) && (row[d] > e);
      if (left || right) {
        pen = 1.f - (float)(d - 1) * inv_w;
        break;
      }
    }
    ell1[idx] = e - a.alpha_soft * pen;
  }
  __syncthreads();
  // cross-head exclusivity and output
  for (int k = threadIdx.x; k < tile_n; k += blockDim.x) {
    int owner = 0;
    float best = ell1[k];
    for (int h = 1; h < a.G; ++h) {
      const float v = ell1[h * a.tile + k];
      if (v > best) {
        best = v;
        owner = h;
      }
    }
    for (int h = 0; h < a.G; ++h) {
      const float v = ell1[h * a.tile + k] - (h != owner ? a.alpha_cross : 0.f);
      a.scores[((size_t)b * a.Hq + g * a.G + h) * a.ld_s + c0 + k] = v;
    }
  }
}

// ---------------------------------------------------------------- top-K
constexpr int kTopkThreads = 1024;
constexpr int kBins = 2048;

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
    int t = wtot[lane];
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
    const int t = wtot[lane];
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

// Keys of one block-wide slab of kSlab = 16 * kTopkThreads scores starting at
// `base`: coalesced loads (float4 when the row allows it); element u of a
// thread sits at index slab_index(base, u).  Padding keys are 0, below the
// image of every float but a negative NaN, and are never counted.
constexpr int kPerThread = 16;
constexpr int kSlab = kPerThread * kTopkThreads;

template <bool VEC>
__device__ __forceinline__ int slab_index(int base, int u) {
  return VEC ? base + (u >> 2) * (4 * kTopkThreads) + threadIdx.x * 4 + (u & 3)
             : base + u * kTopkThreads + threadIdx.x;
}

template <bool VEC>
__device__ __forceinline__ void load_slab(const float* row, int n, int base, uint32_t (&k)[kPerThread]) {
  if (VEC) {
#pragma unroll
    for (int v = 0; v < kPerThread / 4; ++v) {
      const int j = base + v * (4 * kTopkThreads) + threadIdx.x * 4;
      if (j + 4 <= n) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(row + j));
        k[4 * v + 0] = float_key(f.x);
        k[4 * v + 1] = float_key(f.y);
        k[4 * v + 2] = float_key(f.z);
        k[4 * v + 3] = float_key(f.w);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) k[4 * v + e] = (j + e < n) ? float_key(__ldg(row + j + e)) : 0u;
      }
    }
  } else {
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int j = base + u * kTopkThreads + threadIdx.x;
      k[u] = (j < n) ? float_key(__ldg(row + j)) : 0u;
    }
  }
}

// One CTA per row.  Keys are order-preserving uint32 images of the scores.
// Three MSB radix passes (11, 11, 10 bits) find the key T of the K-th largest
// and how many keys equal to T to keep (the lowest positions first); one
// ordered pass writes the positions ascending.
template <bool VEC>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(int n, const float* __restrict__ scores,
                                                            int64_t ld_s, int K, int offset,
                                                            int32_t* __restrict__ idx, int64_t ld_i) {
  __shared__ int hist[kBins];
  __shared__ int wtot[64];
  __shared__ int sel_bin, sel_above, total;
  const float* row = scores + (size_t)blockIdx.x * ld_s;
  int32_t* out = idx + (size_t)blockIdx.x * ld_i;
  const int lane = threadIdx.x & 31;

  uint32_t prefix = 0, pmask = 0;
  int k_rem = K;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int sh = shifts[pass];
    const uint32_t dmask = (1u << widths[pass]) - 1u;
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kSlab) {
      uint32_t k[kPerThread];
      load_slab<VEC>(row, n, base, k);
#pragma unroll
      for (int u = 0; u < kPerThread; ++u) {
        const bool in = slab_index<VEC>(base, u) < n && (k[u] & pmask) == prefix;
        const uint32_t bin = (k[u] >> sh) & dmask;
        const unsigned act = __ballot_sync(0xffffffffu, in);
        if (in) {
          const unsigned peers = __match_any_sync(act, bin);
          if ((int)(__ffs(peers) - 1) == lane) atomicAdd(&hist[bin], __popc(peers));
        }
      }
    }
    __syncthreads();
    // the bin holding the k_rem-th largest: suffix sums over bins
    const int b0 = 2 * threadIdx.x, b1 = b0 + 1;
    const int h0 = hist[b0], h1 = hist[b1];
    const int incl = block_suffix_incl(h0 + h1, wtot);
    const int above = incl - h0 - h1;   // bins > b1
    if (above < k_rem && above + h1 >= k_rem) {
      sel_bin = b1;
      sel_above = above;
    } else if (above + h1 < k_rem && above + h1 + h0 >= k_rem) {
      sel_bin = b0;
      sel_above = above + h1;
    }
    __syncthreads();
    prefix |= (uint32_t)sel_bin << sh;
    pmask |= dmask << sh;
    k_rem -= sel_above;
    __syncthreads();
  }
  const uint32_t T = prefix;   // key of the K-th largest; keep k_rem of the ties
  // ordered pass: 4 consecutive elements per thread per round, rounds in order
  int gt_run = 0, eq_run = 0;
  for (int base = 0; base < n; base += 4 * kTopkThreads) {
    const int j0 = base + threadIdx.x * 4;
    uint32_t k[4];
    if (VEC && j0 + 4 <= n) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(row + j0));
      k[0] = float_key(f.x);
      k[1] = float_key(f.y);
      k[2] = float_key(f.z);
      k[3] = float_key(f.w);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) k[e] = (j0 + e < n) ? float_key(__ldg(row + j0 + e)) : 0u;
    }
    int ngt = 0, neq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (j0 + e < n) {
        ngt += k[e] > T;
        neq += k[e] == T;
      }
    }
    const int ex = block_prefix_excl((neq << 16) | ngt, wtot, &total);
    int gt_before = gt_run + (ex & 0xffff);
    int eq_before = eq_run + (ex >> 16);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (j0 + e >= n) break;
      if (k[e] > T) {
        const int at = gt_before + min(eq_before, k_rem);
        if (at < K) out[at] = offset + j0 + e;
        ++gt_before;
      } else if (k[e] == T) {
        const int at = gt_before + eq_before;
        if (eq_before < k_rem && at < K) out[at] = offset + j0 + e;
        ++eq_before;
      }
    }
    gt_run += total & 0xffff;
    eq_run += total >> 16;
    __syncthreads();
  }
}

// ---------------------------------------------------------------- host
int score_tile(int G) { return std::max(256, 8192 / G); }

size_t score_smem(int G, int tile, int w) {
  return ((size_t)G * (tile + 2 * w) + (size_t)G * tile + (tile + 2 * w)) * sizeof(float);
}

int stat_chunks(int nC) { return (nC + kStatChunk - 1) / kStatChunk; }

sfi_status run_select_scores(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv,
                             int L, const float* logits, int64_t ld, const float* lse_cand,
                             float* scores, int64_t ld_s, void* stat_ws, cudaStream_t st) {
  const int G = s.Hq / s.Hkv;
  const int lo = p.n_sink, hi = L - p.n_recent;
  const int nC = hi - lo;
  double* part = reinterpret_cast<double*>(stat_ws);
  const int nch = stat_chunks(nC);
  const int64_t norm_ld = (int64_t)s.max_pages * kPage;
  dim3 sgrid(nch, s.B * s.Hkv);
  stats_norm_kernel<<<sgrid, kStatThreads, 0, st>>>(lo, nC, kv.key_norms, norm_ld, part, nch);
  stats_prior_kernel<<<sgrid, kStatThreads, 0, st>>>(L, lo, nC, kv.key_norms, norm_ld, part, nch);
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
  const size_t smem = score_smem(G, a.tile, a.w);
  static DeviceOnce attr;
  if (!attr.done() &&
      !attr.mark(cudaFuncSetAttribute(select_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      200 * 1024)))
    return SFI_ERR_CUDA;
  dim3 grid((nC + a.tile - 1) / a.tile, s.B * s.Hkv);
  select_scores_kernel<<<grid, 256, smem, st>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

sfi_status run_topk(int rows, int n, const float* scores, int64_t ld_s, int K, int offset,
                    int32_t* idx, int64_t ld_i, cudaStream_t st) {
  if (rows <= 0) return SFI_OK;
  const bool vec = (ld_s % 4 == 0) && ((reinterpret_cast<uintptr_t>(scores) & 15u) == 0);
  if (vec) topk_kernel<true><<<rows, kTopkThreads, 0, st>>>(n, scores, ld_s, K, offset, idx, ld_i);
  else topk_kernel<false><<<rows, kTopkThreads, 0, st>>>(n, scores, ld_s, K, offset, idx, ld_i);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace sfi
