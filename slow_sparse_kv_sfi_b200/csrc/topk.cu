// Per-row top-K of the Selector's refined log-scores ([ES] "El Selector";
// [FR] "B. Le Sélecteur"; [ZH] "2.2 训练无感的 Selector": the K tokens of
// highest score per query head), ties to the lower position.
//
// Exact MSB radix select on the order-preserving uint32 image of every fp32
// score.  The rows are long (one score per candidate position) and few (one
// per query head), so every row is cut into slices of kSlice scores with one
// CTA per (slice, row):
//   topk_digit<p>, p = 0, 1, 2: histogram of digit p (key bits 31-20, 19-8,
//                7-0) over the scores whose higher digits equal the prefix
//                found so far, added into the row's global histogram; the
//                last CTA of the row to arrive (arrival counter) extends the
//                prefix by the digit that holds the remaining k-th largest,
//                lowers k by the scores in higher digits and clears the
//                histogram for the next pass.  After pass 2 the prefix is the
//                threshold key T and k the number of scores equal to T taken;
//   topk_mark    scores above T are selected, scores equal to T are ties
//                (both as bitmap words);
//   topk_ties    one CTA per row: the first k ties in position order join the
//                selection; then, if asked, the bitmap becomes K ascending
//                positions.
// The prior makes the scores of distant positions nearly equal (the position
// factor ln(1 + L - j) flattens), so any binning by value range would pile
// most of a row into one bin; the radix digits split such rows exactly.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sfi {

namespace {

constexpr int kSlice = 8192;          // scores per slice (a multiple of 128)
constexpr int kTkThreads = 256;       // digit / mark / ties: 32 scores per thread
constexpr int kDigitBins = 4096;      // largest digit: 12 bits
constexpr int kMaxWords = 8192;       // rows of at most 262144 scores

struct Digit {
  int shift, bits;
};
__host__ __device__ constexpr Digit digit_of(int pass) {
  return pass == 0 ? Digit{20, 12} : (pass == 1 ? Digit{8, 12} : Digit{0, 8});
}

// The 32 scores of this thread in slice [s0, s0 + kSlice) of a row, as keys:
// element e of load u is score s0 + (u * kTkThreads + tid) * 4 + e, so every
// warp-wide load reads 512 consecutive bytes.  All eight loads are issued
// before any is used.  Scores past n read as key 0 and are flagged by the
// callers.
struct SliceKeys {
  uint32_t k[8][4];
};

__device__ __forceinline__ int pos_of(int s0, int u, int e) { return s0 + (u * kTkThreads + threadIdx.x) * 4 + e; }

__device__ __forceinline__ void load_keys(const float* row, int n, int s0, bool vec, SliceKeys& x) {
  if (vec && s0 + kSlice <= n) {
    float4 f[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) f[u] = __ldg(reinterpret_cast<const float4*>(row + pos_of(s0, u, 0)));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      x.k[u][0] = float_key(f[u].x);
      x.k[u][1] = float_key(f[u].y);
      x.k[u][2] = float_key(f[u].z);
      x.k[u][3] = float_key(f[u].w);
    }
  } else {
    float f[8][4];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = pos_of(s0, u, e);
        f[u][e] = j < n ? __ldg(row + j) : 0.f;
      }
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) x.k[u][e] = float_key(f[u][e]);
  }
}

// Reverse (suffix) inclusive scan of one value per thread across the block;
// wtot holds 64 ints.
__device__ __forceinline__ int suffix_incl(int v, int* wtot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int sh = 1; sh < 32; sh <<= 1) {
    const int y = __shfl_down_sync(0xffffffffu, x, sh);
    if (lane + sh < 32) x += y;
  }
  if (lane == 0) wtot[w] = x;
  __syncthreads();
  if (w == 0) {
    const int nwarps = blockDim.x >> 5;
    const int t = lane < nwarps ? wtot[lane] : 0;
    int s = t;
#pragma unroll
    for (int sh = 1; sh < 32; sh <<= 1) {
      const int y = __shfl_down_sync(0xffffffffu, s, sh);
      if (lane + sh < 32) s += y;
    }
    wtot[32 + lane] = s - t;
  }
  __syncthreads();
  const int r = x + wtot[32 + w];
  __syncthreads();
  return r;
}

// Exclusive prefix scan of one value per thread across the block.
__device__ __forceinline__ int prefix_excl(int v, int* wtot) {
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
  }
  __syncthreads();
  const int r = x - v + wtot[32 + w];
  __syncthreads();
  return r;
}

// The bin of `hist` (nb bins, a multiple of the block size) holding the k-th
// largest element counted from the top: *bin, and *above = elements in
// higher bins.
__device__ __forceinline__ void find_bin(const int* hist, int nb, int k, int* wtot, int* s_bin, int* s_above) {
  const int per = nb / blockDim.x;
  const int b0 = threadIdx.x * per;
  int mine = 0;
  for (int i = 0; i < per; ++i) mine += hist[b0 + i];
  int above = suffix_incl(mine, wtot) - mine;
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

struct TopkArgs {
  int rows, n, K, offset;
  const float* scores;
  int64_t ld_s;
  bool vec;                  // rows 16-byte aligned: float4 loads
  int slices;
  TopkScratch w;
  uint32_t* bits;            // [rows][ld_b] selection bitmap (output)
  int64_t ld_b;
  int32_t* idx;              // [rows][ld_i] ascending positions + offset, or null
  int64_t ld_i;
};

// Row state in w.info: [0] prefix of the threshold key, [1] scores still to
// take (k), [2] mask of the digits fixed so far.
template <int PASS>
__global__ void __launch_bounds__(kTkThreads) topk_digit_kernel(const TopkArgs a) {
  grid_dep_enter();
  constexpr Digit dg = digit_of(PASS);
  constexpr int kNb = 1 << dg.bits;
  constexpr uint32_t kDm = (uint32_t)kNb - 1u;
  __shared__ int hist[kNb];
  __shared__ int wtot[64];
  __shared__ int s_last, s_bin, s_above;
  const int row = blockIdx.y, s0 = blockIdx.x * kSlice;
  for (int i = threadIdx.x; i < kNb; i += kTkThreads) hist[i] = 0;
  SliceKeys x;
  load_keys(a.scores + (size_t)row * a.ld_s, a.n, s0, a.vec, x);
  int* info = a.w.info + (size_t)row * 4;
  const uint32_t prefix = PASS == 0 ? 0u : (uint32_t)info[0];
  const uint32_t pmask = PASS == 0 ? 0u : (uint32_t)info[2];
  const int k = PASS == 0 ? a.K : info[1];
  __syncthreads();
  // Neighbouring scores share digits, and the bins of a row's bulk are few:
  // a lane whose 4 scores share one digit counts them as one, and a run of
  // such lanes with one digit adds once (from its first lane); lanes with
  // mixed digits add their scores one by one.
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    int d[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t key = x.k[u][e];
      d[e] = (pos_of(s0, u, e) < a.n && (key & pmask) == prefix) ? (int)((key >> dg.shift) & kDm) : -1;
    }
    const bool uni = d[0] == d[1] && d[0] == d[2] && d[0] == d[3];
    const int dl = uni ? d[0] : -2;
    const int dprev = __shfl_up_sync(0xffffffffu, dl, 1);
    const bool head = lane == 0 || dprev != dl;
    const unsigned heads = __ballot_sync(0xffffffffu, head);
    if (uni) {
      if (head && dl >= 0) {
        const unsigned later = heads & ~((2u << lane) - 1u);   // run heads after this lane
        const int next = later ? __ffs(later) - 1 : 32;
        atomicAdd(&hist[dl], 4 * (next - lane));
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (d[e] >= 0) atomicAdd(&hist[d[e]], 1);
    }
  }
  __syncthreads();
  int* gh = a.w.ghist + (size_t)row * kDigitBins;
  for (int i = threadIdx.x; i < kNb; i += kTkThreads)
    if (hist[i]) atomicAdd(&gh[i], hist[i]);
  // the last CTA of the row to arrive fixes this digit
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&a.w.done[row], 1) == a.slices - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  {
    // every load in flight before any store (the row's histogram, from L2)
    constexpr int kPer = kNb / kTkThreads;
    int v[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) v[i] = __ldcg(&gh[i * kTkThreads + threadIdx.x]);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      hist[i * kTkThreads + threadIdx.x] = v[i];
      gh[i * kTkThreads + threadIdx.x] = 0;   // cleared for the next pass / call
    }
  }
  __syncthreads();
  find_bin(hist, kNb, k, wtot, &s_bin, &s_above);
  if (threadIdx.x == 0) {
    info[0] = (int)(prefix | ((uint32_t)s_bin << dg.shift));
    info[1] = k - s_above;
    info[2] = (int)(pmask | (kDm << dg.shift));
    a.w.done[row] = 0;
  }
}

// Bitmap words of the slice: scores above T selected, scores equal to T ties.
__global__ void __launch_bounds__(kTkThreads) topk_mark_kernel(const TopkArgs a) {
  grid_dep_enter();
  const int row = blockIdx.y, s0 = blockIdx.x * kSlice;
  const int lane = threadIdx.x & 31;
  SliceKeys x;
  load_keys(a.scores + (size_t)row * a.ld_s, a.n, s0, a.vec, x);
  const uint32_t T = (uint32_t)a.w.info[(size_t)row * 4];
  uint32_t* brow = a.bits + (size_t)row * a.ld_b;
  uint32_t* trow = a.w.ties + (size_t)row * a.w.words_ld;
  const int nw = (a.n + 31) / 32;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    // this warp's 128 scores of load u: lane l holds 4l .. 4l + 3
    const int jb = pos_of(s0, u, 0);
    uint32_t up = 0u, eq = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (jb + e < a.n) {
        up |= (x.k[u][e] > T ? 1u : 0u) << e;
        eq |= (x.k[u][e] == T ? 1u : 0u) << e;
      }
    }
    // bitmap word of lanes 8q .. 8q + 7: nibble (l & 7) of word q
    uint32_t wu = up << (4 * (lane & 7)), we = eq << (4 * (lane & 7));
#pragma unroll
    for (int sh = 1; sh <= 4; sh <<= 1) {
      wu |= __shfl_xor_sync(0xffffffffu, wu, sh);
      we |= __shfl_xor_sync(0xffffffffu, we, sh);
    }
    const int wi = jb >> 5;
    if ((lane & 7) == 0 && wi < nw) {
      brow[wi] = wu;
      trow[wi] = we;
    }
  }
}

// One CTA per row: the first k ties in position order join the selection;
// then the selection as ascending positions, if wanted.  Thread t owns the
// bitmap words [t * per, (t + 1) * per), held in registers.
constexpr int kMaxPer = kMaxWords / kTkThreads;

__global__ void __launch_bounds__(kTkThreads) topk_ties_kernel(const TopkArgs a) {
  grid_dep_enter();
  __shared__ int wtot[64];
  const int row = blockIdx.x, tid = threadIdx.x;
  const int nw = (a.n + 31) / 32;
  const int k = a.w.info[(size_t)row * 4 + 1];
  uint32_t* brow = a.bits + (size_t)row * a.ld_b;
  const uint32_t* trow = a.w.ties + (size_t)row * a.w.words_ld;
  const int per = (nw + kTkThreads - 1) / kTkThreads;
  const int w0 = tid * per;
  uint32_t tw[kMaxPer], sw[kMaxPer];
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    const bool in = i < per && w0 + i < nw;
    tw[i] = in ? trow[w0 + i] : 0u;
    sw[i] = in ? brow[w0 + i] : 0u;
  }
  int mine = 0;
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) mine += __popc(tw[i]);
  int before = prefix_excl(mine, wtot);
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    uint32_t t = tw[i];
    uint32_t take = 0u;
    while (t && before < k) {
      const uint32_t lowbit = t & (~t + 1u);
      take |= lowbit;
      t ^= lowbit;
      ++before;
    }
    if (take) {
      sw[i] |= take;
      brow[w0 + i] = sw[i];   // this thread owns the word
    }
  }
  if (!a.idx) return;
  mine = 0;
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) mine += __popc(sw[i]);
  int at = prefix_excl(mine, wtot);
  int32_t* out = a.idx + (size_t)row * a.ld_i;
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    uint32_t t = sw[i];
    while (t) {
      const int bpos = __ffs(t) - 1;
      t &= t - 1u;
      if (at < a.K) out[at] = a.offset + (w0 + i) * 32 + bpos;
      ++at;
    }
  }
}

}  // namespace

int topk_max_n() { return kMaxWords * 32; }

// Layout: the state that must stay zero between calls (histograms, arrival
// counters) first, at offsets that depend on `rows` only, then the per-call
// arrays.
size_t topk_scratch_bytes(int rows, int n) {
  const size_t nw = (size_t)(n + 31) / 32;
  size_t b = 0;
  b += align_up((size_t)rows * kDigitBins * sizeof(int), 256);   // ghist
  b += align_up((size_t)rows * 5 * sizeof(int), 256);            // done, info
  b += 2 * align_up((size_t)rows * nw * sizeof(uint32_t), 256);  // ties, bitmap
  return b;
}

TopkScratch topk_scratch(void* base, int rows, int n) {
  const size_t nw = (size_t)(n + 31) / 32;
  char* p = static_cast<char*>(base);
  TopkScratch w{};
  w.ghist = reinterpret_cast<int*>(p);
  p += align_up((size_t)rows * kDigitBins * sizeof(int), 256);
  w.done = reinterpret_cast<int*>(p);
  w.info = w.done + rows;
  p += align_up((size_t)rows * 5 * sizeof(int), 256);
  w.ties = reinterpret_cast<uint32_t*>(p);
  p += align_up((size_t)rows * nw * sizeof(uint32_t), 256);
  w.bits = reinterpret_cast<uint32_t*>(p);
  w.words_ld = (int64_t)nw;
  return w;
}

sfi_status run_topk(int rows, int n, const float* scores, int64_t ld_s, int K, int offset, int32_t* idx,
                    int64_t ld_i, uint32_t* bits, int64_t ld_b, const TopkScratch& w, cudaStream_t st) {
  if (rows <= 0) return SFI_OK;
  if (n > topk_max_n() || n < 1 || K < 1 || K > n) return SFI_ERR_UNSUPPORTED;
  TopkArgs a{};
  a.rows = rows;
  a.n = n;
  a.K = K;
  a.offset = offset;
  a.scores = scores;
  a.ld_s = ld_s;
  a.vec = (ld_s % 4 == 0) && ((reinterpret_cast<uintptr_t>(scores) & 15u) == 0);
  a.slices = (n + kSlice - 1) / kSlice;
  a.w = w;
  a.bits = bits ? bits : w.bits;
  a.ld_b = bits ? ld_b : w.words_ld;
  a.idx = idx;
  a.ld_i = ld_i;
  const dim3 sgrid(a.slices, rows);
  launch_k(topk_digit_kernel<0>, sgrid, dim3(kTkThreads), 0, st, a);
  launch_k(topk_digit_kernel<1>, sgrid, dim3(kTkThreads), 0, st, a);
  launch_k(topk_digit_kernel<2>, sgrid, dim3(kTkThreads), 0, st, a);
  launch_k(topk_mark_kernel, sgrid, dim3(kTkThreads), 0, st, a);
  launch_k(topk_ties_kernel, dim3(rows), dim3(kTkThreads), 0, st, a);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace sfi
