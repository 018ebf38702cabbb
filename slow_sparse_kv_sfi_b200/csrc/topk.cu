// Per-row top-K of the Selector's refined log-scores ([ES] "El Selector";
// [FR] "B. Le Sélecteur"; [ZH] "2.2 训练无感的 Selector": the K tokens of
// highest score per query head), ties to the lower position.
//
// Exact MSB radix select on the order-preserving uint32 image of every fp32
// score, one thread-block cluster per row.  The row is cut into slices of
// T * 32 scores, one CTA of T threads each (up to 8 CTAs, cluster rank =
// slice), and every thread keeps its 32 keys in registers for the whole
// kernel, so the scores are read once:
//   1. the cluster's smallest and largest key: their common leading bits are
//      every key's, so the digit passes cover only the bits below the highest
//      one where they differ, in as few passes of at most 14 bits as cover
//      them (rows of log-scores share sign and most of the exponent: two);
//   2. per digit pass: each CTA builds the histogram of its keys that match
//      the prefix found so far in shared memory; after a cluster barrier CTA
//      c sums bins [c * per, (c + 1) * per) over every CTA's histogram through
//      distributed shared memory; after a second barrier every CTA reads the
//      range totals and the reduced bins of the range holding the remaining
//      k-th largest key, and extends the prefix by that bin;
//   3. the prefix is now the threshold key T: keys above it are selected,
//      keys equal to it are ties, taken in position order (a cluster-wide
//      exclusive count of the ties in lower slices) until K are chosen.
// Outputs: the selection bitmap (one bit per score) and / or the K positions
// in ascending order.  The prior makes the scores of distant positions
// nearly equal, so the digits (not a binning by value range) split such rows
// exactly.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace sfi {

namespace {

constexpr int kKPT = 32;              // keys per thread: 8 loads of 4
constexpr int kMaxCluster = 8;        // portable cluster size
constexpr int kDigitBits = 14;        // widest digit
constexpr int kDigitBins = 1 << kDigitBits;
constexpr int kMaxN = kMaxCluster * 1024 * kKPT;   // 262144

struct TopkArgs {
  int rows, n, K, offset;
  const float* scores;
  int64_t ld_s;
  bool vec;                  // rows 16-byte aligned: float4 loads
  uint32_t* bits;            // [rows][ld_b] selection bitmap, or null
  int64_t ld_b;
  int32_t* idx;              // [rows][ld_i] ascending positions + offset, or null
  int64_t ld_i;
};

// Element e of load u of thread t: score s0 + (u * T + t) * 4 + e, so every
// warp-wide load reads 512 consecutive bytes.
template <int T>
__device__ __forceinline__ int pos_of(int s0, int u, int e) {
  return s0 + (u * T + (int)threadIdx.x) * 4 + e;
}

// Exclusive prefix sum over the block (T threads) of one value per thread;
// *total = the block's sum.  ws holds 33 ints.
template <int T>
__device__ __forceinline__ int block_excl(int v, int* ws, int* total) {
  constexpr int kW = T / 32;
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

template <int T>
__device__ __forceinline__ uint32_t block_reduce_u32(uint32_t v, bool take_max, uint32_t* ws) {
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) {
    const uint32_t y = __shfl_xor_sync(0xffffffffu, v, sh);
    v = take_max ? max(v, y) : min(v, y);
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) ws[w] = v;
  __syncthreads();
  uint32_t r = ws[0];
  for (int i = 1; i < T / 32; ++i) r = take_max ? max(r, ws[i]) : min(r, ws[i]);
  __syncthreads();
  return r;
}

// Dynamic shared memory of the kernel: the digit histogram, then (clusters of
// more than one CTA) this CTA's range of the cluster-wide histogram.
__host__ __device__ constexpr size_t topk_smem_bytes(int cs) {
  return (size_t)kDigitBins * 4 + (cs > 1 ? (size_t)((kDigitBins + cs - 1) / cs) * 4 : 0);
}

template <int T>
__global__ void __launch_bounds__(T) topk_cluster_kernel(const __grid_constant__ TopkArgs a) {
  grid_dep_enter();
  cg::cluster_group cl = cg::this_cluster();
  const int cs = (int)cl.num_blocks();
  const int rank = (int)cl.block_rank();
  const int row = blockIdx.y;
  const int s0 = rank * T * kKPT;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  extern __shared__ int dyn[];
  int* hist = dyn;                                   // [2^nbits] this CTA's digit counts
  int* red = cs > 1 ? dyn + kDigitBins : dyn;        // this CTA's range, summed over the cluster
  __shared__ uint32_t selw[T], tiew[T];
  __shared__ int ws[33];
  __shared__ uint32_t wsu[32];
  __shared__ int pub[4];            // published to the cluster: range total, ties, selected
  __shared__ int s_pick[3];         // bin, keys above it, k
  __shared__ uint32_t s_mm[2];

  // ---- keys
  const float* srow = a.scores + (size_t)row * a.ld_s;
  uint32_t key[8][4];
  if (a.vec && s0 + T * kKPT <= a.n) {
    float4 f[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) f[u] = __ldg(reinterpret_cast<const float4*>(srow + pos_of<T>(s0, u, 0)));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      key[u][0] = float_key(f[u].x);
      key[u][1] = float_key(f[u].y);
      key[u][2] = float_key(f[u].z);
      key[u][3] = float_key(f[u].w);
    }
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = pos_of<T>(s0, u, e);
        key[u][e] = j < a.n ? float_key(__ldg(srow + j)) : 0u;
      }
  }
  // ---- 1. common leading bits of the whole row
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (pos_of<T>(s0, u, e) < a.n) {
        kmin = min(kmin, key[u][e]);
        kmax = max(kmax, key[u][e]);
      }
  kmin = block_reduce_u32<T>(kmin, false, wsu);
  kmax = block_reduce_u32<T>(kmax, true, wsu);
  if (threadIdx.x == 0) {
    s_mm[0] = kmin;
    s_mm[1] = kmax;
  }
  cl.sync();
  if (threadIdx.x == 0) {
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int c = 0; c < cs; ++c) {
      const uint32_t* r = cl.map_shared_rank(s_mm, c);
      lo = min(lo, r[0]);
      hi = max(hi, r[1]);
    }
    wsu[0] = lo;
    wsu[1] = hi;
  }
  __syncthreads();
  const uint32_t gmin = wsu[0], gmax = wsu[1];
  // hb: highest bit where the row's keys differ (-1: all equal)
  const int hb = gmin == gmax ? -1 : 31 - __clz((int)(gmin ^ gmax));
  uint32_t pmask = hb < 0 ? 0xffffffffu : (hb >= 31 ? 0u : ~((2u << hb) - 1u));
  uint32_t prefix = gmax & pmask;
  int k = a.K;

  // ---- 2. digit passes over bits hb .. 0, as few as cover them, balanced
  const int npass = (hb + 1 + kDigitBits - 1) / kDigitBits;
  const int width = npass > 0 ? (hb + 1 + npass - 1) / npass : 0;
  int done_bits = 0;
  while (done_bits < hb + 1) {
    const int nbits = min(width, hb + 1 - done_bits);
    const int shift = hb + 1 - done_bits - nbits;
    const int nb = 1 << nbits;
    const uint32_t dm = (uint32_t)nb - 1u;
    for (int i = threadIdx.x; i < nb; i += T) hist[i] = 0;
    __syncthreads();
    // the keys still matching the prefix, counted by digit
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t kk = key[u][e];
        if (pos_of<T>(s0, u, e) < a.n && (kk & pmask) == prefix) atomicAdd(&hist[(kk >> shift) & dm], 1);
      }
    cl.sync();   // every histogram of the cluster complete
    // this CTA's bin range, summed over the cluster (one CTA: its own histogram)
    const int per = (nb + cs - 1) / cs;
    const int r0 = rank * per;
    int mine = 0;
    for (int i = threadIdx.x; i < per; i += T) {
      const int bin = r0 + i;
      int s = 0;
      if (cs == 1) {
        s = hist[i];
      } else if (bin < nb) {
        for (int c = 0; c < cs; ++c) s += cl.map_shared_rank(hist, c)[bin];
        red[i] = s;
      }
      mine += s;
    }
    int tot;
    block_excl<T>(mine, ws, &tot);
    if (threadIdx.x == 0) pub[0] = tot;
    cl.sync();   // every range reduced
    // the range holding the k-th largest key (ranges of higher bins first),
    // then the bin inside it: every CTA does this on the same data
    if (threadIdx.x == 0) {
      int above = 0, c = cs - 1;
      for (; c > 0; --c) {
        const int t = cl.map_shared_rank(pub, c)[0];
        if (above + t >= k) break;
        above += t;
      }
      s_pick[0] = c;
      s_pick[1] = above;
    }
    __syncthreads();
    const int cr = s_pick[0];
    const int above_r = s_pick[1];
    const int* rred = cl.map_shared_rank(red, cr);
    const int nr = min(per, nb - cr * per);
    // thread t takes bins [t * bp, (t + 1) * bp) of the range; suffix counts
    const int bp = (nr + T - 1) / T;
    const int b0 = threadIdx.x * bp;
    int part = 0;
    for (int i = 0; i < bp; ++i)
      if (b0 + i < nr) part += rred[b0 + i];
    int sum_all;
    const int before = block_excl<T>(part, ws, &sum_all);   // bins below this thread's
    int above = above_r + (sum_all - before - part);         // keys in higher bins of the range
    for (int i = bp - 1; i >= 0; --i) {
      if (b0 + i >= nr) continue;
      const int h = rred[b0 + i];
      if (above < k && above + h >= k) {
        s_pick[0] = cr * per + b0 + i;
        s_pick[2] = above;
      }
      above += h;
    }
    __syncthreads();
    prefix |= (uint32_t)s_pick[0] << shift;
    pmask |= dm << shift;
    k -= s_pick[2];
    done_bits += nbits;
    __syncthreads();
  }
  // ---- 3. keys above the threshold, ties in position order
  const uint32_t thr = hb < 0 ? gmin : prefix;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int jb = pos_of<T>(s0, u, 0);
    uint32_t up = 0u, eq = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (jb + e < a.n) {
        up |= (key[u][e] > thr ? 1u : 0u) << e;
        eq |= (key[u][e] == thr ? 1u : 0u) << e;
      }
    }
    // the word of lanes 8q .. 8q + 7: nibble (lane & 7) of word q
    uint32_t wu = up << (4 * (lane & 7)), we = eq << (4 * (lane & 7));
#pragma unroll
    for (int sh = 1; sh <= 4; sh <<= 1) {
      wu |= __shfl_xor_sync(0xffffffffu, wu, sh);
      we |= __shfl_xor_sync(0xffffffffu, we, sh);
    }
    if ((lane & 7) == 0) {
      const int wi = (u * T + warp * 32) / 8 + (lane >> 3);
      selw[wi] = wu;
      tiew[wi] = we;
    }
  }
  __syncthreads();
  // thread i owns word i of the slice (words are in position order)
  const int i = threadIdx.x;
  const uint32_t tw = tiew[i];
  int ties_tot;
  const int tie_before_local = block_excl<T>(__popc(tw), ws, &ties_tot);
  if (threadIdx.x == 0) pub[1] = ties_tot;
  cl.sync();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int c = 0; c < rank; ++c) s += cl.map_shared_rank(pub, c)[1];
    s_pick[1] = s;
  }
  __syncthreads();
  int rk = s_pick[1] + tie_before_local;
  uint32_t t = tw, take = 0u;
  while (t && rk < k) {
    const uint32_t lowbit = t & (~t + 1u);
    take |= lowbit;
    t ^= lowbit;
    ++rk;
  }
  const uint32_t sw = selw[i] | take;
  const int word = rank * T + i;
  const int nw = (a.n + 31) / 32;
  if (a.bits && word < nw) a.bits[(size_t)row * a.ld_b + word] = sw;
  if (a.idx) {
    int sel_tot;
    const int sel_before_local = block_excl<T>(__popc(sw), ws, &sel_tot);
    if (threadIdx.x == 0) pub[2] = sel_tot;
    cl.sync();
    if (threadIdx.x == 0) {
      int s = 0;
      for (int c = 0; c < rank; ++c) s += cl.map_shared_rank(pub, c)[2];
      s_pick[1] = s;
    }
    __syncthreads();
    int at = s_pick[1] + sel_before_local;
    int32_t* out = a.idx + (size_t)row * a.ld_i;
    uint32_t x = sw;
    while (x) {
      const int bpos = __ffs(x) - 1;
      x &= x - 1u;
      if (at < a.K) out[at] = a.offset + word * 32 + bpos;
      ++at;
    }
  }
  cl.sync();   // no CTA leaves while another may still read its shared memory
}

template <int T>
sfi_status launch_topk(const TopkArgs& a, int cs, cudaStream_t st) {
  static DeviceOnce smem_attr;
  if (!smem_attr.done() && !smem_attr.mark(cudaFuncSetAttribute(topk_cluster_kernel<T>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      (int)topk_smem_bytes(2))))
    return SFI_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, a.rows);
  cfg.blockDim = dim3(T);
  cfg.dynamicSmemBytes = topk_smem_bytes(cs);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<T>, a);
  return e == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace

int topk_max_n() { return kMaxN; }

sfi_status run_topk(int rows, int n, const float* scores, int64_t ld_s, int K, int offset, int32_t* idx,
                    int64_t ld_i, uint32_t* bits, int64_t ld_b, cudaStream_t st) {
  if (rows <= 0) return SFI_OK;
  if (n > topk_max_n() || n < 1 || K < 1 || K > n) return SFI_ERR_UNSUPPORTED;
  if (rows > 65535) return SFI_ERR_UNSUPPORTED;
  TopkArgs a{};
  a.rows = rows;
  a.n = n;
  a.K = K;
  a.offset = offset;
  a.scores = scores;
  a.ld_s = ld_s;
  a.vec = (ld_s % 4 == 0) && ((reinterpret_cast<uintptr_t>(scores) & 15u) == 0);
  a.bits = bits;
  a.ld_b = ld_b;
  a.idx = idx;
  a.ld_i = ld_i;
  // slices of T * 32 scores: at most 8 per row, the fewest threads that cover it
  const int cs = std::min(kMaxCluster, (n + 256 * kKPT - 1) / (256 * kKPT));
  const int need = (n + cs * kKPT - 1) / (cs * kKPT);   // threads per slice
  if (need <= 256) return launch_topk<256>(a, cs, st);
  if (need <= 512) return launch_topk<512>(a, cs, st);
  return launch_topk<1024>(a, cs, st);
}

}  // namespace sfi
