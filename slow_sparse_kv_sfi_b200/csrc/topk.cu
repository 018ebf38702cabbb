// Per-row top-K of the Selector's refined log-scores ([ES] "El Selector";
// [FR] "B. Le Sélecteur"; [ZH] "2.2 训练无感的 Selector": the K tokens of
// highest score per query head), ties to the lower position.
//
// Exact MSB radix select on the order-preserving uint32 image of every fp32
// score, one thread-block cluster per row.  The row is cut into slices of
// T * 32 * KU / 8 scores, one CTA of T threads each (1, 2, 4 or 8 CTAs,
// cluster rank = slice), and every thread keeps its keys on chip for the
// whole kernel, so the scores are read once: 32 in registers, and with KU =
// 16 another 32 in shared memory (a CTA of 1024 threads fills an SM's
// registers, so the second half halves the CTAs of a row and the waves of a
// launch):
//   1. the cluster's smallest and largest key: the passes work on the offset
//      key - smallest, whose bits above the highest bit of (largest -
//      smallest) are zero, in as few passes of at most 14 bits as cover the
//      rest (a row of log-scores spans about 2^26 keys: two passes, where the
//      keys' own leading bits would need three once the scores straddle a
//      power of two);
//   2. per digit pass: each CTA builds the histogram of its keys that match
//      the prefix found so far in shared memory; after a cluster barrier CTA
//      c sums bins [c * per, (c + 1) * per) over every CTA's histogram through
//      distributed shared memory (the CS loads of a bin issued together);
//      after a second barrier every CTA reads the range totals (one lane per
//      CTA), copies the reduced bins of the range holding the remaining k-th
//      largest key and extends the prefix by that bin;
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

constexpr int kKPT = 32;              // keys per thread in registers: 8 loads of 4
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
  // [rows][2]: the largest key and the largest complement of a key of every
  // row, found by the kernel that wrote the scores (zero between uses; this
  // kernel zeroes them again), or null: the kernel finds them itself
  uint32_t* minmax;
};

// Element e of load u of thread t: score s0 + (u * T + t) * 4 + e, so every
// warp-wide load reads 512 consecutive bytes.  Loads 0 .. 7 stay in
// registers, loads 8 .. 15 (KU = 16) in shared memory.
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

// Dynamic shared memory of the kernel: the digit histogram (after the passes:
// the selection and tie words), then (clusters of more than one CTA) this
// CTA's range of the cluster-wide histogram, then (KU = 16) the keys of loads
// 8 .. 15, [32][T].
__host__ __device__ constexpr size_t topk_red_ints(int cs) { return cs > 1 ? (size_t)((kDigitBins + cs - 1) / cs) : 0; }
__host__ __device__ constexpr size_t topk_smem_bytes(int cs, int t, int ku) {
  return (size_t)kDigitBins * 4 + topk_red_ints(cs) * 4 + (ku > 8 ? (size_t)32 * t * 4 : 0);
}

// Reads one int that every CTA of the cluster published at `pub` (lanes c <
// CS of the calling warp read CTA c's) and returns this lane's value; lanes
// >= CS get 0.
template <int CS>
__device__ __forceinline__ int read_published(cg::cluster_group& cl, int* pub, int lane) {
  if (lane >= CS) return 0;
  if constexpr (CS > 1) return cl.map_shared_rank(pub, lane)[0];
  return pub[0];
}

// Sum of the values published by the CTAs of ranks below `rank` (warp 0).
template <int CS>
__device__ __forceinline__ int published_before(cg::cluster_group& cl, int* pub, int lane, int rank) {
  int v = read_published<CS>(cl, pub, lane);
  v = lane < rank ? v : 0;
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) v += __shfl_xor_sync(0xffffffffu, v, sh);
  return v;
}

// Key of element e of load u: registers for u < 8, shared memory for u >= 8
// (u and e are constants after unrolling).
template <int T>
__device__ __forceinline__ uint32_t& key_at(uint32_t (&key)[8][4], uint32_t* skey, int u, int e) {
  return u < 8 ? key[u & 7][e] : skey[((u - 8) * 4 + e) * T + threadIdx.x];
}

template <int T, int CS, int KU>
__global__ void __launch_bounds__(T) topk_cluster_kernel(const __grid_constant__ TopkArgs a) {
  static_assert(KU == 8 || KU == 16, "loads per thread");
  constexpr int W = KU / 8;         // bitmap words per thread
  grid_dep_enter();
  cg::cluster_group cl = cg::this_cluster();
  const int rank = CS > 1 ? (int)cl.block_rank() : 0;
  const int row = blockIdx.y;
  const int s0 = rank * T * KU * 4;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  extern __shared__ int dyn[];
  int* hist = dyn;                  // [2^nbits] this CTA's digit counts; then a copy of the chosen range
  int* red = dyn + kDigitBins;      // this CTA's range, summed over the cluster (CS > 1)
  uint32_t* skey = reinterpret_cast<uint32_t*>(dyn + kDigitBins + topk_red_ints(CS));   // KU = 16: [32][T]
  // after the passes the histogram holds the selection and tie words of the
  // slice: thread i owns words i, T + i, ... (in position order, word w
  // covering scores s0 + 32 w .. s0 + 32 w + 31)
  uint32_t* selw = reinterpret_cast<uint32_t*>(hist);
  uint32_t* tiew = selw + W * T;
  __shared__ int ws[33];
  __shared__ uint32_t wsu[32];
  __shared__ int pub[3];            // published to the cluster: range total, ties, selected
  __shared__ int s_pick[4];         // range / bin, keys above it, k, keys in the bin
  __shared__ uint32_t s_mm[2];
  auto csync = [&]() {
    if constexpr (CS > 1) cl.sync();
    else __syncthreads();
  };

  // ---- keys (loads 8 .. 15 first, into shared memory)
  const float* srow = a.scores + (size_t)row * a.ld_s;
  uint32_t key[8][4];
  const bool full = a.vec && s0 + T * KU * 4 <= a.n;
  if constexpr (KU > 8) {
    if (full) {
      float4 f[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) f[u] = __ldg(reinterpret_cast<const float4*>(srow + pos_of<T>(s0, 8 + u, 0)));
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        skey[(u * 4 + 0) * T + threadIdx.x] = float_key(f[u].x);
        skey[(u * 4 + 1) * T + threadIdx.x] = float_key(f[u].y);
        skey[(u * 4 + 2) * T + threadIdx.x] = float_key(f[u].z);
        skey[(u * 4 + 3) * T + threadIdx.x] = float_key(f[u].w);
      }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = pos_of<T>(s0, 8 + u, e);
          skey[(u * 4 + e) * T + threadIdx.x] = j < a.n ? float_key(__ldg(srow + j)) : 0u;
        }
    }
  }
  if (full) {
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
  // ---- 1. smallest and largest key of the row (given, or found here)
  if (a.minmax == nullptr) {
    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int u = 0; u < KU; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (pos_of<T>(s0, u, e) < a.n) {
          const uint32_t v = key_at<T>(key, skey, u, e);
          kmin = min(kmin, v);
          kmax = max(kmax, v);
        }
    kmin = block_reduce_u32<T>(kmin, false, wsu);
    kmax = block_reduce_u32<T>(kmax, true, wsu);
    if (threadIdx.x == 0) {
      s_mm[0] = kmin;
      s_mm[1] = kmax;
    }
    csync();
    if (warp == 0) {
      uint32_t lo = 0xffffffffu, hi = 0u;
      if (lane < CS) {
        const uint32_t* r = s_mm;
        if constexpr (CS > 1) r = cl.map_shared_rank(s_mm, lane);
        lo = r[0];
        hi = r[1];
      }
#pragma unroll
      for (int sh = 16; sh >= 1; sh >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, sh));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, sh));
      }
      if (lane == 0) {
        wsu[0] = lo;
        wsu[1] = hi;
      }
    }
    __syncthreads();
  } else if (threadIdx.x == 0) {
    wsu[0] = ~a.minmax[(size_t)row * 2 + 1];
    wsu[1] = a.minmax[(size_t)row * 2];
  }
  if (a.minmax) __syncthreads();
  const uint32_t gmin = wsu[0], gmax = wsu[1];
  // the passes work on off = key - gmin in [0, gmax - gmin]; hb: its highest
  // bit that can be set (-1: all keys equal)
  const uint32_t span = gmax - gmin;
  const int hb = span == 0u ? -1 : 31 - __clz((int)span);
  uint32_t pmask = hb < 0 ? 0xffffffffu : (hb >= 31 ? 0u : ~((2u << hb) - 1u));
  uint32_t prefix = 0u;
  int k = a.K;
#pragma unroll
  for (int u = 0; u < KU; ++u)
#pragma unroll
    for (int e = 0; e < 4; ++e) key_at<T>(key, skey, u, e) -= gmin;

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
    for (int u = 0; u < KU; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t off = key_at<T>(key, skey, u, e);
        if (pos_of<T>(s0, u, e) < a.n && (off & pmask) == prefix) atomicAdd(&hist[(off >> shift) & dm], 1);
      }
    csync();   // every histogram of the cluster complete
    // this CTA's bin range, summed over the cluster: the CS loads of a bin
    // are issued together
    const int per = (nb + CS - 1) / CS;
    int mine = 0;
    if constexpr (CS == 1) {
      for (int i = threadIdx.x; i < nb; i += T) mine += hist[i];
    } else {
      const int* hs[CS];
#pragma unroll
      for (int c = 0; c < CS; ++c) hs[c] = cl.map_shared_rank(hist, c);
      const int r0 = rank * per;
      for (int i = threadIdx.x; i < per; i += T) {
        const int bin = r0 + i;
        int sum = 0;
        if (bin < nb) {
          int v[CS];
#pragma unroll
          for (int c = 0; c < CS; ++c) v[c] = hs[c][bin];
#pragma unroll
          for (int c = 0; c < CS; ++c) sum += v[c];
        }
        red[i] = sum;
        mine += sum;
      }
    }
    int tot;
    block_excl<T>(mine, ws, &tot);
    if (threadIdx.x == 0) pub[0] = tot;
    csync();   // every range reduced and published
    // the range holding the k-th largest key (ranges of higher bins first):
    // the highest rank whose suffix total reaches k
    if (warp == 0) {
      const int t = read_published<CS>(cl, pub, lane);
      int suf = t;
#pragma unroll
      for (int sh = 1; sh < 32; sh <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, suf, sh);
        if (lane + sh < 32) suf += y;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, lane < CS && suf >= k);
      const int c = bal ? 31 - __clz((int)bal) : 0;
      const int above = __shfl_sync(0xffffffffu, suf - t, c);
      if (lane == 0) {
        s_pick[0] = c;
        s_pick[1] = above;
      }
    }
    __syncthreads();
    const int cr = s_pick[0];
    const int above_r = s_pick[1];
    const int nr = CS == 1 ? nb : min(per, nb - cr * per);
    if constexpr (CS > 1) {
      // every CTA is past its reads of this CTA's histogram: the chosen
      // range is copied into it
      const int* src = cl.map_shared_rank(red, cr);
#pragma unroll 4
      for (int i = threadIdx.x; i < nr; i += T) hist[i] = src[i];
      __syncthreads();
    }
    // thread t takes bins [t * bp, (t + 1) * bp) of the range; suffix counts
    const int bp = (nr + T - 1) / T;
    const int b0 = threadIdx.x * bp;
    int part = 0;
    for (int i = 0; i < bp; ++i)
      if (b0 + i < nr) part += hist[b0 + i];
    int sum_all;
    const int before = block_excl<T>(part, ws, &sum_all);   // bins below this thread's
    int above = above_r + (sum_all - before - part);         // keys in higher bins of the range
    for (int i = bp - 1; i >= 0; --i) {
      if (b0 + i >= nr) continue;
      const int h = hist[b0 + i];
      if (above < k && above + h >= k) {
        s_pick[0] = cr * per + b0 + i;
        s_pick[2] = above;
        s_pick[3] = h;
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
  // ---- 3. keys above the threshold, ties in position order (offset keys:
  // the threshold is the prefix; all keys equal: every key is a tie).  The
  // last pass's bin holds exactly the keys equal to the threshold: when all
  // of them are taken no cluster-wide count of ties is needed.
  const uint32_t thr = prefix;
  const bool take_all_ties = (hb < 0 ? a.n : s_pick[3]) == k;
#pragma unroll
  for (int u = 0; u < KU; ++u) {
    const int jb = pos_of<T>(s0, u, 0);
    uint32_t up = 0u, eq = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (jb + e < a.n) {
        const uint32_t off = key_at<T>(key, skey, u, e);
        up |= (off > thr ? 1u : 0u) << e;
        eq |= (off == thr ? 1u : 0u) << e;
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
  // thread i owns words i, T + i, ... of the slice
  const int i = threadIdx.x;
  uint32_t sw[W];
  if (take_all_ties) {
#pragma unroll
    for (int j = 0; j < W; ++j) sw[j] = selw[j * T + i] | tiew[j * T + i];
  } else {   // the same decision in every CTA of the cluster
    int before[W];
    int base = 0;
#pragma unroll
    for (int j = 0; j < W; ++j) {
      int tot;
      before[j] = base + block_excl<T>(__popc(tiew[j * T + i]), ws, &tot);
      base += tot;
    }
    if (threadIdx.x == 0) pub[1] = base;
    csync();
    if (warp == 0) {
      const int sb = published_before<CS>(cl, pub + 1, lane, rank);
      if (lane == 0) s_pick[1] = sb;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < W; ++j) {
      int rk = s_pick[1] + before[j];
      uint32_t t = tiew[j * T + i];
      uint32_t take = 0u;
      while (t && rk < k) {
        const uint32_t lowbit = t & (~t + 1u);
        take |= lowbit;
        t ^= lowbit;
        ++rk;
      }
      sw[j] = selw[j * T + i] | take;
    }
  }
  const int nw = (a.n + 31) / 32;
#pragma unroll
  for (int j = 0; j < W; ++j) {
    const int word = rank * W * T + j * T + i;
    if (a.bits && word < nw) a.bits[(size_t)row * a.ld_b + word] = sw[j];
  }
  if (a.idx) {
    int before[W];
    int base = 0;
#pragma unroll
    for (int j = 0; j < W; ++j) {
      int tot;
      before[j] = base + block_excl<T>(__popc(sw[j]), ws, &tot);
      base += tot;
    }
    if (threadIdx.x == 0) pub[2] = base;
    csync();
    if (warp == 0) {
      const int sb = published_before<CS>(cl, pub + 2, lane, rank);
      if (lane == 0) s_pick[1] = sb;
    }
    __syncthreads();
    int32_t* out = a.idx + (size_t)row * a.ld_i;
#pragma unroll
    for (int j = 0; j < W; ++j) {
      const int word = rank * W * T + j * T + i;
      int at = s_pick[1] + before[j];
      uint32_t x = sw[j];
      while (x) {
        const int bpos = __ffs(x) - 1;
        x &= x - 1u;
        if (at < a.K) out[at] = a.offset + word * 32 + bpos;
        ++at;
      }
    }
  }
  if constexpr (CS > 1) cl.sync();   // no CTA leaves while another may still read its shared memory
  // every CTA of the row has read the given range: zero it for the next use
  if (a.minmax && rank == 0 && threadIdx.x == 0) {
    a.minmax[(size_t)row * 2] = 0u;
    a.minmax[(size_t)row * 2 + 1] = 0u;
  }
}

template <int T, int CS, int KU>
sfi_status launch_topk(const TopkArgs& a, cudaStream_t st) {
  static DeviceOnce smem_attr;
  if (!smem_attr.done() && !smem_attr.mark(cudaFuncSetAttribute(topk_cluster_kernel<T, CS, KU>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      (int)topk_smem_bytes(CS, T, KU))))
    return SFI_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, a.rows);
  cfg.blockDim = dim3(T);
  cfg.dynamicSmemBytes = topk_smem_bytes(CS, T, KU);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<T, CS, KU>, a);
  return e == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

template <int CS>
sfi_status launch_topk_cs(const TopkArgs& a, int threads, cudaStream_t st) {
  if (threads <= 256) return launch_topk<256, CS, 8>(a, st);
  if (threads <= 512) return launch_topk<512, CS, 8>(a, st);
  return launch_topk<1024, CS, 8>(a, st);
}

}  // namespace

int topk_max_n() { return kMaxN; }

sfi_status run_topk(int rows, int n, const float* scores, int64_t ld_s, int K, int offset, int32_t* idx,
                    int64_t ld_i, uint32_t* bits, int64_t ld_b, cudaStream_t st, uint32_t* minmax) {
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
  a.minmax = minmax;
  // slices of T * 32 scores: the fewest CTAs of up to 1024 threads that
  // cover the row, a power of two of them, at most 4 while that suffices.
  // A cluster's CTAs land on distinct SMs of one GPC and a CTA of 1024
  // threads fills an SM's registers, so clusters of 4 run about twice as
  // many at once as clusters of 8 of 512-thread CTAs.
  int cs = 1;
  while (cs < kMaxCluster && cs * 1024 * kKPT < n) cs *= 2;
  // With more CTAs than SMs (one CTA of 1024 threads per SM) the rows run in
  // waves; 32 more keys per thread in shared memory halve the CTAs of a row.
  // Then every CTA has 1024 threads: cs * 1024 * 32 < n made cs, so the half
  // needs more than 512 threads.
  if (cs >= 2 && (long)rows * cs > num_sms()) {
    switch (cs / 2) {
      case 1: return launch_topk<1024, 1, 16>(a, st);
      case 2: return launch_topk<1024, 2, 16>(a, st);
      default: return launch_topk<1024, 4, 16>(a, st);
    }
  }
  const int need = (n + cs * kKPT - 1) / (cs * kKPT);   // threads per slice
  switch (cs) {
    case 1: return launch_topk_cs<1>(a, need, st);
    case 2: return launch_topk_cs<2>(a, need, st);
    case 4: return launch_topk_cs<4>(a, need, st);
    default: return launch_topk_cs<8>(a, need, st);
  }
}

}  // namespace sfi
