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
//   exclusivity l'' = l' - alpha_cross * [h != owner(j)], owner(j) = the
//              lowest head whose l' is within 1e-3 of the group's largest
//              (near-ties go to the lowest head)
//   top-K      K largest l'' per query head, ties to the lower position.
//
// The soft-NMS dominance follows real arithmetic, not the last bit of a
// rounded sum: l_i vs l_j has the sign of s_i - s_j (ln is monotone), with
// s = (1 - lambda) f~ + lambda r formed by one fp32 FMA from lambda r (fp64
// prior, rounded to fp32): within 1 ulp of s, where the prior dominates
// neighbouring candidates differ in r by ~1e-6 relative, far above that.
// With lambda = 0 the dominance is decided on the log-evidence x = z - lse_C,
// which does not underflow.  l = ln(s) is the accurate logf (1 ulp); the
// owner's tie tolerance (1e-3) is far above the kernel's error on l'.
//
// Kernels: stats_norm / stats_prior (per (b, kv head) and chunk of C: fp64
// partial sums of the norms and of kappa pi; every consumer reduces the
// partials in the same fixed order), select_scores (one CTA per (b, kv group,
// candidate tile) holding all G heads plus a halo of w on each side in shared
// memory, so soft-NMS and the cross-head owner need no second pass over
// memory); the top-K follows in topk.cu.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sfi {

constexpr int kStatThreads = 256;
constexpr float kOwnerTie = 1e-3f;
constexpr double kMaxProductPenalty = 18.0;   // tie tolerance of the cross-head owner (log-score units)
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

// Prior factors in fp64 (the stored norms are fp32): kappa_j = min(1, nbar /
// n_j) (1 for a zero key), pi_j = ln(1 + L - j).  stats_prior and
// select_scores evaluate them with the same code, so the normaliser is the
// sum of exactly the values the scores use.
__device__ __forceinline__ double kappa_of(double nbar, float n) {
  return n > 0.f ? fmin(1.0, nbar / (double)n) : 1.0;
}

__device__ __forceinline__ double pi_of(int L, int j) { return log((double)(1 + L - j)); }

__device__ __forceinline__ double nbar_of(double sum_norms, int nC) { return sum_norms / (double)nC; }

// Key-norm row of the launch's logical (row, kv head) bgl.
__device__ __forceinline__ const float* norm_row(const float* norms, int64_t norm_ld, const RowMap& rows, int Hkv,
                                                 int bgl) {
  const int bl = bgl / Hkv;
  return norms + ((size_t)rows.phys(bl) * Hkv + (bgl - bl * Hkv)) * norm_ld;
}

// part[bgl][chunk][0] = sum of key norms over the chunk of C (bgl: logical
// (row, kv head) of the launch); the CTAs of row 0 also write the position
// factor pi[c] = ln(1 + L - (lo + c)) of their chunk, shared by every row
__global__ void __launch_bounds__(kStatThreads) stats_norm_kernel(int L, int lo, int nC,
                                                                  const float* __restrict__ norms,
                                                                  int64_t norm_ld, double* part, int nch, int Hkv,
                                                                  double* __restrict__ pitab,
                                                                  const __grid_constant__ RowMap rows) {
  grid_dep_enter();
  __shared__ double red[32];
  const int bg = blockIdx.y;
  if (bg == 0) {
    const int c1 = min(nC, (int)(blockIdx.x + 1) * kStatChunk);
    for (int c = blockIdx.x * kStatChunk + threadIdx.x; c < c1; c += blockDim.x) pitab[c] = pi_of(L, lo + c);
  }
  const float* n = norm_row(norms, norm_ld, rows, Hkv, bg) + lo;
  const int c0 = blockIdx.x * kStatChunk, c1 = min(nC, c0 + kStatChunk);
  double sacc = 0.0;
  for (int c = c0 + threadIdx.x; c < c1; c += blockDim.x) sacc += (double)n[c];
  const double t = block_sum_d(sacc, red);
  if (threadIdx.x == 0) part[((size_t)bg * nch + blockIdx.x) * 2] = t;
}

// part[bgl][chunk][1] = sum of kappa * pi over the chunk of C (fp64), and
// kp[bgl][c] = kappa_j pi_j (j = lo + c) rounded once to fp32 for the score
// kernel, which multiplies it by lambda / Z in fp32
__global__ void __launch_bounds__(kStatThreads) stats_prior_kernel(int L, int lo, int nC,
                                                                   const float* __restrict__ norms,
                                                                   int64_t norm_ld, double* part, int nch, int Hkv,
                                                                   const double* __restrict__ pitab,
                                                                   float* __restrict__ kp, int64_t kp_ld,
                                                                   const __grid_constant__ RowMap rows) {
  grid_dep_enter();
  __shared__ double red[32];
  __shared__ double bc;
  const int bg = blockIdx.y;
  double* pbg = part + (size_t)bg * nch * 2;
  const double nbar = nbar_of(reduce_parts(pbg, nch, 0, &bc), nC);
  const float* n = norm_row(norms, norm_ld, rows, Hkv, bg);
  const int c0 = blockIdx.x * kStatChunk, c1 = min(nC, c0 + kStatChunk);
  double z = 0.0;
  float* kpr = kp + (size_t)bg * kp_ld;
  for (int c = c0 + threadIdx.x; c < c1; c += blockDim.x) {
    const int j = lo + c;
    const double v = kappa_of(nbar, n[j]) * pitab[c];
    kpr[c] = (float)v;
    z += v;
  }
  const double t = block_sum_d(z, red);
  if (threadIdx.x == 0) pbg[blockIdx.x * 2 + 1] = t;
}

// lamz[bgl] = lambda / Z rounded once to fp32, Z = sum of kappa pi over C
// (the chunk partials summed in a fixed order): one warp per (row, kv head).
__global__ void __launch_bounds__(32) stats_final_kernel(const double* __restrict__ part, int nch, double lam,
                                                         float* __restrict__ lamz) {
  grid_dep_enter();
  __shared__ double bc;
  const double z = reduce_parts(part + (size_t)blockIdx.x * nch * 2, nch, 1, &bc);
  if (threadIdx.x == 0) lamz[blockIdx.x] = (float)(lam / z);
}

struct ScoreArgs {
  int L, lo, nC, Hq, Hkv, G, w, tile;
  double lam;                   // lambda_eff
  float one_minus_lam;          // 1 - lambda_eff
  float alpha_soft, alpha_cross;
  const float* logits;
  int64_t ld;
  const float* lse_cand;
  const float* lamz;         // [B*Hkv] lambda / Z
  uint32_t* minmax;          // [rows][2] largest key / complement of the row's l'' (atomic max), or null
  const float* kp;           // [B*Hkv][kp_ld] kappa_j pi_j of the candidates (fp32)
  int64_t kp_ld;
  float* scores;         // logical rows of the launch
  int64_t ld_s;
  RowMap rows;
  // evidence window: logits / lse_cand hold nq query slots of G heads per
  // group; the slots in qmask are averaged (weight inv_nq each)
  int nq;
  uint32_t qmask;
  float inv_nq;
};

// How a CTA of the score kernel spreads a group's GM heads: kHPT heads per
// thread, kTPP consecutive lanes per position.
template <int GM>
struct ScoreLanes {
  static constexpr int kHPT = GM < 4 ? GM : 4;
  static constexpr int kTPP = GM / kHPT;
};

// Phase 3 of one position, by its kTPP threads, this one holding heads h0 ..
// h0 + kHPT - 1: l' = ln(s + 1e-30) - alpha_soft * weight(d) of every head
// (s = exp(x) when the key is x), the owner = the lowest head within the tie
// tolerance of the largest l' (both found across the position's threads),
// and l'' = l' - alpha_cross off the owner, written to outp[h * ld_s + k].
// Every lane of the warp calls it (act: the lane holds a position).
template <int GM, bool EXACT>
__device__ __forceinline__ void finish_position(const float (&kv)[ScoreLanes<GM>::kHPT],
                                                const int (&d)[ScoreLanes<GM>::kHPT], int h0, bool act, int G,
                                                bool by_x, float alpha_soft, float alpha_cross, const float* wt,
                                                float* outp, int64_t ld_s, int k,
                                                uint32_t (&kmx)[ScoreLanes<GM>::kHPT],
                                                uint32_t (&knx)[ScoreLanes<GM>::kHPT]) {
  constexpr int H = ScoreLanes<GM>::kHPT, P = ScoreLanes<GM>::kTPP;
  float l1[H];
  float M = -INFINITY;
#pragma unroll
  for (int j = 0; j < H; ++j) {
    l1[j] = -INFINITY;
    if (act && (EXACT || h0 + j < G)) {
      const float sv = by_x ? fast_exp2(kv[j] * kLog2e) : kv[j];
      l1[j] = logf(sv + 1e-30f) - alpha_soft * wt[d[j]];
      M = fmaxf(M, l1[j]);
    }
  }
#pragma unroll
  for (int sh = 1; sh < P; sh <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, sh));
  const float thr = M - kOwnerTie;
  int owner = GM;
#pragma unroll
  for (int j = H - 1; j >= 0; --j)
    if (act && (EXACT || h0 + j < G) && l1[j] >= thr) owner = h0 + j;
#pragma unroll
  for (int sh = 1; sh < P; sh <<= 1) owner = min(owner, __shfl_xor_sync(0xffffffffu, owner, sh));
#pragma unroll
  for (int j = 0; j < H; ++j)
    if (act && (EXACT || h0 + j < G)) {
      const float v = l1[j] - (h0 + j != owner ? alpha_cross : 0.f);
      outp[(size_t)(h0 + j) * ld_s + k] = v;
      const uint32_t key = float_key(v);   // the top-K's order
      kmx[j] = max(kmx[j], key);
      knx[j] = max(knx[j], ~key);
    }
}

// N consecutive keys (16-byte loads for N = 4).
template <int N>
__device__ __forceinline__ void load_keys(const float* p, float (&v)[N]) {
  if constexpr (N == 4) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    v[0] = t.x;
    v[1] = t.y;
    v[2] = t.z;
    v[3] = t.w;
  } else if constexpr (N == 2) {
    const float2 t = *reinterpret_cast<const float2*>(p);
    v[0] = t.x;
    v[1] = t.y;
  } else {
    v[0] = p[0];
  }
}

template <int N>
__device__ __forceinline__ void store_keys(float* p, const float (&v)[N]) {
  if constexpr (N == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  } else if constexpr (N == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else {
    p[0] = v[0];
  }
}

// One CTA per (b, KV group, tile of candidates).  Phase 1 writes, for every
// position of the tile plus a halo of w on each side, the dominance keys of
// the group's heads side by side (s in fp32, or x when lambda = 0; NaN
// outside C and for heads >= G: a NaN never dominates).  Phase 2: the kTPP
// threads of a position find the nearest dominator of their kHPT heads each,
// distances 1..kNear for their heads at once (one vector load per side and
// distance), then the heads still without one alone, to w; phase 3
// (finish_position) applies soft-NMS, picks the owner and writes l''.
// EXACT: G == GM, so every lane's heads exist.
template <int GM, bool EXACT>
__global__ void __launch_bounds__(256, 4) select_scores_kernel(const __grid_constant__ ScoreArgs a) {
  constexpr int H = ScoreLanes<GM>::kHPT, P = ScoreLanes<GM>::kTPP;
  grid_dep_enter();
  extern __shared__ float sm[];
  const int W = a.tile + 2 * a.w;     // haloed width
  float* key = sm;                    // [W][GM] dominance keys
  const int bg = blockIdx.y;                        // logical (row, kv head)
  const int bl = bg / a.Hkv, g = bg - bl * a.Hkv;
  const int b = a.rows.phys(bl);                    // the sequence
  const int c0 = blockIdx.x * a.tile;
  const int tile_n = min(a.tile, a.nC - c0);
  const int G = EXACT ? GM : a.G;
  const float* kpr = a.kp + (size_t)bg * a.kp_ld;
  const bool by_x = a.lam <= 0.0;          // lambda = 0: s = f~, decided on x
  const float lam_r = a.lamz[bg];          // lambda / Z, rounded once
  __shared__ float wt[64];                 // soft-NMS weight of a nearest dominator at distance d
  for (int d = threadIdx.x; d <= a.w && d < 64; d += blockDim.x)
    wt[d] = d > 0 ? 1.f - (float)(d - 1) / (float)a.w : 0.f;
  // this thread's heads and its place among a position's threads
  const int h0 = (int)(threadIdx.x % P) * H;
  const int pstride = blockDim.x / P;      // positions per pass of the block
  // logits rows of the group: nq query slots of G heads (nq = 1: row b * Hq + g * G + h)
  const size_t row0 = ((size_t)b * a.Hkv + g) * (size_t)(a.nq * G);
  const float* z0 = a.logits + row0 * a.ld + a.lo;
  const float nan = __int_as_float(0x7fc00000);
  float lsec[H];
#pragma unroll
  for (int j = 0; j < H; ++j) lsec[j] = (EXACT || h0 + j < G) ? a.lse_cand[row0 + h0 + j] : 0.f;
  if (a.nq > 1) {
    // evidence window: f~ = the mean of the slots' restricted distributions,
    // x = ln f~ = m + ln(mean exp(x_i - m)), m the largest x_i
    for (int k = threadIdx.x / P; k < W; k += pstride) {
      const int c = c0 - a.w + k;
      float kv[H];
#pragma unroll
      for (int j = 0; j < H; ++j) kv[j] = nan;
      if (c >= 0 && c < a.nC) {
        const float r = kpr[c] * lam_r;   // lambda r_j
#pragma unroll
        for (int j = 0; j < H; ++j) {
          const int h = h0 + j;
          if (EXACT || h < G) {
            float m = -INFINITY;
            for (int i = 0; i < a.nq; ++i)
              if ((a.qmask >> i) & 1u) {
                const size_t row = (size_t)i * G + h;
                m = fmaxf(m, z0[row * a.ld + c] - a.lse_cand[row0 + row]);
              }
            float acc = 0.f;
            for (int i = 0; i < a.nq; ++i)
              if ((a.qmask >> i) & 1u) {
                const size_t row = (size_t)i * G + h;
                acc += fast_exp2((z0[row * a.ld + c] - a.lse_cand[row0 + row] - m) * kLog2e);
              }
            const float x = m + logf(acc * a.inv_nq);
            const float ft = fast_exp2(x * kLog2e);
            kv[j] = by_x ? x : fmaf(a.one_minus_lam, ft, r);
          }
        }
      }
      store_keys<H>(key + (size_t)k * GM + h0, kv);
    }
  }
  // kU positions per thread and round: all their loads are issued first
  constexpr int kU = 4;
  for (int k0 = threadIdx.x / P; a.nq == 1 && k0 < W; k0 += kU * pstride) {
    float kp[kU];
    float zv[kU][H];
    bool in[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 - a.w + k0 + u * pstride;
      in[u] = k0 + u * pstride < W && c >= 0 && c < a.nC;
      const int cc = in[u] ? c : 0;
      kp[u] = in[u] ? kpr[cc] : 0.f;
#pragma unroll
      for (int j = 0; j < H; ++j) zv[u][j] = (in[u] && (EXACT || h0 + j < G)) ? z0[(size_t)(h0 + j) * a.ld + cc] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int k = k0 + u * pstride;
      if (k >= W) continue;
      float kv[H];
      const float r = kp[u] * lam_r;   // lambda r_j
#pragma unroll
      for (int j = 0; j < H; ++j) {
        // exp through the hardware's base-2 approximation (relative error
        // ~1e-7, below the error of the logits themselves)
        const float x = zv[u][j] - lsec[j];
        const float ft = fast_exp2(x * kLog2e);
        kv[j] = (in[u] && (EXACT || h0 + j < G)) ? (by_x ? x : fmaf(a.one_minus_lam, ft, r)) : nan;
      }
      store_keys<H>(key + (size_t)k * GM + h0, kv);
    }
  }
  __syncthreads();
  // Phases 2 and 3.  dh = distance of the nearest dominator, 0: none within w.
  constexpr int kNear = 4;
  const int near = min(kNear, a.w);
  float* outp = a.scores + ((size_t)bl * a.Hq + (size_t)g * G) * a.ld_s + c0;
  uint32_t kmx[H], knx[H];
#pragma unroll
  for (int j = 0; j < H; ++j) kmx[j] = knx[j] = 0u;
  for (int base = 0; base < tile_n; base += pstride) {
    const int k = base + (int)threadIdx.x / P;
    const bool act = k < tile_n;
    float e[H];
    int dh[H];
#pragma unroll
    for (int j = 0; j < H; ++j) {
      e[j] = 0.f;
      dh[j] = 0;
    }
    if (act) {
      const float* row = key + (size_t)(a.w + k) * GM + h0;
      load_keys<H>(row, e);
#pragma unroll
      for (int d = kNear; d >= 1; --d) {   // descending: the nearest hit is written last
        if (d > near) continue;
        float lv[H], rv[H];
        load_keys<H>(row - d * GM, lv);
        load_keys<H>(row + d * GM, rv);
#pragma unroll
        for (int j = 0; j < H; ++j)   // a left neighbour dominates on ties; NaN compares false
          if (lv[j] >= e[j] || rv[j] > e[j]) dh[j] = d;
      }
      if (a.w > kNear) {
        // the heads still without a dominator (about 1 % of positions): alone, to w
#pragma unroll
        for (int j = 0; j < H; ++j) {
          if ((EXACT || h0 + j < G) && dh[j] == 0) {
            for (int d = kNear + 1; d <= a.w; ++d) {
              if (row[j - d * GM] >= e[j] || row[j + d * GM] > e[j]) {
                dh[j] = d;
                break;
              }
            }
          }
        }
      }
    }
    finish_position<GM, EXACT>(e, dh, h0, act, G, by_x, a.alpha_soft, a.alpha_cross, wt, outp, a.ld_s, k, kmx,
                               knx);
  }
  if (a.minmax) {
    // the rows' largest key and key complement over the CTA, then one atomic
    // each: the top-K reads them instead of finding the range itself
    __shared__ uint32_t mm[8][GM][2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < H; ++j)
#pragma unroll
      for (int sh = P; sh < 32; sh <<= 1) {
        kmx[j] = max(kmx[j], __shfl_xor_sync(0xffffffffu, kmx[j], sh));
        knx[j] = max(knx[j], __shfl_xor_sync(0xffffffffu, knx[j], sh));
      }
    if (lane < P) {
#pragma unroll
      for (int j = 0; j < H; ++j) {
        mm[warp][h0 + j][0] = kmx[j];
        mm[warp][h0 + j][1] = knx[j];
      }
    }
    __syncthreads();
    if ((int)threadIdx.x < G) {
      const int h = threadIdx.x;
      uint32_t x = 0u, y = 0u;
      for (int w8 = 0; w8 < (int)(blockDim.x >> 5); ++w8) {
        x = max(x, mm[w8][h][0]);
        y = max(y, mm[w8][h][1]);
      }
      uint32_t* mrow = a.minmax + ((size_t)bl * a.Hq + (size_t)g * G + h) * 2;
      atomicMax(mrow, x);
      atomicMax(mrow + 1, y);
    }
  }
}

// ---------------------------------------------------------------- host
int score_tile(int G) { return std::max(512, 4096 / G); }

// dominance keys of the tile with its halo, GM (G rounded up to a power of
// two) per position
size_t score_smem(int G, int tile, int w) {
  int gm = 1;
  while (gm < G) gm *= 2;
  return (size_t)gm * (tile + 2 * w) * sizeof(float);
}

int stat_chunks(int nC) { return (nC + kStatChunk - 1) / kStatChunk; }

template <int GM, bool EXACT>
sfi_status launch_scores_t(const ScoreArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
  static DeviceOnce attr;
  if (!attr.done() &&
      !attr.mark(cudaFuncSetAttribute(select_scores_kernel<GM, EXACT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      200 * 1024)))
    return SFI_ERR_CUDA;
  launch_k(select_scores_kernel<GM, EXACT>, dim3(grid), dim3(256), smem, st, a);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

template <int GM>
sfi_status launch_scores(const ScoreArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
  return a.G == GM ? launch_scores_t<GM, true>(a, grid, smem, st) : launch_scores_t<GM, false>(a, grid, smem, st);
}

namespace {

// The statistics area: partial sums, then the position factors, then
// kappa * pi (fp32) of every candidate of every row.
struct StatLayout {
  int nb, nC, nch;
  int64_t kp_ld;
  uint32_t* minmax;          // [B*Hq][2], at the same place for every row map
  double *part, *pitab;
  float* kp;
  float* lamz;
  StatLayout(const sfi_shape& s, const sfi_params& p, int L, const RowMap& rows, void* ws) {
    nb = rows.count(s.B);
    nC = L - p.n_recent - p.n_sink;
    nch = stat_chunks(nC);
    kp_ld = (nC + 1) / 2 * 2;
    minmax = reinterpret_cast<uint32_t*>(ws);
    part = reinterpret_cast<double*>(minmax + (size_t)s.B * s.Hq * 2);
    pitab = part + (size_t)nb * s.Hkv * nch * 2;
    kp = reinterpret_cast<float*>(pitab + kp_ld);
    lamz = kp + (size_t)nb * s.Hkv * kp_ld;
  }
};

}  // namespace

uint32_t* select_row_range(const sfi_shape& s, const sfi_params& p, int L, void* stat_ws) {
  return StatLayout(s, p, L, RowMap(), stat_ws).minmax;
}

sfi_status run_select_stats(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv, int L,
                            void* stat_ws, cudaStream_t st, const RowMap& rows) {
  const StatLayout sl(s, p, L, rows, stat_ws);
  if (sl.nb < 1 || sl.nb > s.B) return SFI_ERR_SHAPE;
  const int lo = p.n_sink;
  const int64_t norm_ld = (int64_t)s.max_pages * kPage;
  dim3 sgrid(sl.nch, sl.nb * s.Hkv);
  launch_k(stats_norm_kernel, dim3(sgrid), dim3(kStatThreads), 0, st, L, lo, sl.nC, kv.key_norms, norm_ld, sl.part,
           sl.nch, s.Hkv, sl.pitab, rows);
  launch_k(stats_prior_kernel, dim3(sgrid), dim3(kStatThreads), 0, st, L, lo, sl.nC, kv.key_norms, norm_ld, sl.part,
           sl.nch, s.Hkv, sl.pitab, sl.kp, sl.kp_ld, rows);
  const double lam = std::min(std::max((double)p.lambda, 0.0), (double)p.lambda_clip);
  launch_k(stats_final_kernel, dim3(sl.nb * s.Hkv), dim3(32), 0, st, sl.part, sl.nch, lam, sl.lamz);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

sfi_status run_select_scores(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv,
                             int L, const float* logits, int64_t ld, const float* lse_cand,
                             float* scores, int64_t ld_s, void* stat_ws,
                             cudaStream_t st, const RowMap& rows, uint32_t window_mask, bool with_stats,
                             bool row_range) {
  const int G = s.Hq / s.Hkv;
  const int nb = rows.count(s.B);
  if (nb < 1 || nb > s.B) return SFI_ERR_SHAPE;
  const int nq = evidence_window(p);
  const uint32_t qmask = window_mask & (nq >= 32 ? 0xffffffffu : ((1u << nq) - 1u));
  if (qmask == 0u) return SFI_ERR_INVALID_ARG;
  const int lo = p.n_sink;
  const StatLayout sl(s, p, L, rows, stat_ws);
  const int nC = sl.nC;
  if (std::max(p.nms_window / 2, 1) > 63) return SFI_ERR_UNSUPPORTED;   // the weight table
  if (with_stats) {
    const sfi_status r = run_select_stats(s, p, kv, L, stat_ws, st, rows);
    if (r != SFI_OK) return r;
  }
  float* kp = sl.kp;
  const int64_t kp_ld = sl.kp_ld;
  ScoreArgs a{};
  a.L = L; a.lo = lo; a.nC = nC; a.Hq = s.Hq; a.Hkv = s.Hkv; a.G = G;
  a.w = std::max(p.nms_window / 2, 1);
  a.tile = score_tile(G);
  const double lam = std::min(std::max((double)p.lambda, 0.0), (double)p.lambda_clip);
  a.lam = lam;
  a.one_minus_lam = (float)(1.0 - lam);
  a.alpha_soft = p.nms_window / 2 >= 1 ? p.alpha_soft : 0.f;
  a.alpha_cross = p.alpha_cross;
  a.logits = logits; a.ld = ld; a.lse_cand = lse_cand;
  a.lamz = sl.lamz;
  a.minmax = row_range ? sl.minmax : nullptr;
  a.kp = kp; a.kp_ld = kp_ld;
  a.scores = scores; a.ld_s = ld_s;
  a.rows = rows;
  a.nq = nq;
  a.qmask = qmask;
  a.inv_nq = 1.f / (float)__builtin_popcount(qmask);
  const size_t smem = score_smem(G, a.tile, a.w);
  dim3 grid((nC + a.tile - 1) / a.tile, nb * s.Hkv);
  if (G <= 1) return launch_scores<1>(a, grid, smem, st);
  if (G <= 2) return launch_scores<2>(a, grid, smem, st);
  if (G <= 4) return launch_scores<4>(a, grid, smem, st);
  if (G <= 8) return launch_scores<8>(a, grid, smem, st);
  return launch_scores<16>(a, grid, smem, st);
}

}  // namespace sfi
