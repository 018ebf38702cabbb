// Decode attention for Slow-Fast Inference on sm_100a.
//
// One persistent kernel serves both steps of the method:
//  * slow step ([ES] "2. Metodología", Pasos Lentos; [FR] "A. Le Paradigme
//    Lente-Rapide"; [ZH] "2.1"): dense attention over every page of the
//    context; optionally also writes the logits z and the candidate-range
//    log-sum-exp the Selector needs;
//  * fast step ([ES] Pasos Rápidos; [NL] Methodologie; [ZH] "2.3"
//    显存合并的内核): attention over the contiguous packed buffer (sinks +
//    selected rows, per-head bitmask) followed by the recent window read
//    straight from the pages.
//
// Work: the token range of every (sequence, KV head) is cut into chunks; a
// work item is one chunk.  Grid = one CTA per SM, items round-robin.  Warp 4
// is the producer: it walks the items' 16-row tiles and issues TMA loads (a
// 16x64 bf16 box per 128-byte column block, 128B-swizzled) for K and V into a
// ring of shared-memory stages of 4 tiles, with mbarrier completion.  Warps
// 0-3 each take one tile of a stage and run the group's contraction on the
// tensor cores with tokens as the M dimension:
//    S^T[16 tok x 8 heads] = K_tile[16 x D] . Q^T[D x 8]     (mma m16n8k16)
//    O^T[D x 8 heads]     += V_tile^T[D x 16] . P^T[16 x 8]
// P^T comes from the S^T accumulator through movmatrix (an 8x8 transpose in
// registers); P is split into bf16 hi + lo parts so the PV product keeps
// ~16 bits of P.  Online softmax per head; at the end of an item the four
// warps merge through shared memory and write one partial (m, l, l_cand,
// O) per query head; attn_combine merges the partials of every chunk.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace sfi {

constexpr int kConsumerWarps = 4;
constexpr int kAttnThreads = (kConsumerWarps + 1) * 32;
constexpr int kTilesPerStage = 4;
constexpr int kBoxBytes = 16 * 128;   // one 16-row x 64-col bf16 box

enum AttnMode : int { kDense = 0, kDenseExtras = 1, kFast = 2 };

struct AttnArgs {
  int B, Hq, Hkv, G, L;
  int num_pages, max_pages;
  const int32_t* page_table;
  const __nv_bfloat16* q;
  float* part;          // [n_items][G][D + 4]
  int n_chunks;         // chunks per (b, kv head)
  int chunk_tiles;      // dense: tiles per chunk (multiple of 4)
  int n_items;
  float scale_log2;     // log2(e) / sqrt(D)
  float scale;          // 1 / sqrt(D)
  // dense extras
  float* logits;
  int64_t ld;
  int cand_lo, cand_hi;
  // fast
  const int32_t* n_rows;
  const uint32_t* headmask;
  int p_max;
  int rec_lo;           // L - n_recent
  int* err;
};

template <int D>
struct Layout {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kHalves * kBoxBytes;          // one 16-row tile of K (or V)
  static constexpr int kKBytes = kTilesPerStage * kTileBytes;     // K part of a stage
  static constexpr int kStageBytes = 2 * kKBytes;                 // K + V
};

template <int D, int NT>
struct Smem {
  static constexpr int kStages = (D == 128) ? (NT == 1 ? 5 : 4) : 8;
  static constexpr int kHeads = NT * 8;
  static constexpr int kStageBytes = Layout<D>::kStageBytes;
  static constexpr int kMaskOff = kStages * kStageBytes;
  static constexpr int kMaskBytes = kStages * kTilesPerStage * 16 * 4;
  static constexpr int kBarOff = kMaskOff + kMaskBytes;
  static constexpr int kStatOff = kBarOff + 2 * kStages * 8 + 64;
  static constexpr int kStatBytes = kConsumerWarps * kHeads * 3 * 4;
  static constexpr int kOOff = (kStatOff + kStatBytes + 15) / 16 * 16;
  static constexpr int kOBytes = kConsumerWarps * kHeads * D * 4;
  static constexpr int kTotal = kOOff + kOBytes + 1024;   // + alignment slack
  static_assert(kTotal <= 227 * 1024, "shared memory budget");
};

struct Item {
  int bg, b, g;
  int t_begin, t_end;
  int n_packed_tiles;
  int rec_first_page;
  int n_rows;
};

template <int MODE>
__device__ __forceinline__ Item decode_item(const AttnArgs& a, int item) {
  Item it;
  it.bg = item / a.n_chunks;
  const int c = item - it.bg * a.n_chunks;
  it.b = it.bg / a.Hkv;
  it.g = it.bg - it.b * a.Hkv;
  if (MODE != kFast) {
    const int T = (a.L + kPage - 1) / kPage;
    it.t_begin = min(T, c * a.chunk_tiles);
    it.t_end = min(T, it.t_begin + a.chunk_tiles);
    it.n_packed_tiles = 0;
    it.rec_first_page = 0;
    it.n_rows = 0;
  } else {
    int nr = a.n_rows[it.bg];
    if (nr < 0 || nr > a.p_max) nr = nr < 0 ? 0 : a.p_max;   // reported by the combine check
    it.n_rows = nr;
    it.n_packed_tiles = (nr + kPage - 1) / kPage;
    it.rec_first_page = a.rec_lo / kPage;
    const int rec_last_page = (a.L - 1) / kPage;
    const int T = it.n_packed_tiles + (rec_last_page - it.rec_first_page + 1);
    int ct = (T + a.n_chunks - 1) / a.n_chunks;
    ct = (ct + kTilesPerStage - 1) / kTilesPerStage * kTilesPerStage;
    it.t_begin = min(T, c * ct);
    it.t_end = min(T, it.t_begin + ct);
  }
  return it;
}

struct TileRef {
  int kind;   // 0 page, 1 packed, -1 skip (bad page-table entry)
  int y;      // TMA row coordinate
  int pos0;   // page tiles: cache position of row 0; packed: packed row of row 0
};

template <int MODE>
__device__ __forceinline__ TileRef resolve_tile(const AttnArgs& a, const Item& it, int tile) {
  TileRef r;
  if (MODE == kFast && tile < it.n_packed_tiles) {
    r.kind = 1;
    r.pos0 = tile * kPage;
    r.y = it.bg * a.p_max + r.pos0;
    return r;
  }
  const int page_no = (MODE == kFast) ? it.rec_first_page + (tile - it.n_packed_tiles) : tile;
  const int page = __ldg(a.page_table + (size_t)it.b * a.max_pages + page_no);
  r.pos0 = page_no * kPage;
  if ((unsigned)page >= (unsigned)a.num_pages) {
    r.kind = -1;
    r.y = 0;
  } else {
    r.kind = 0;
    r.y = (page * a.Hkv + it.g) * kPage;
  }
  return r;
}

// Address of 16-byte chunk `ci` (0 .. D/8-1) of row `row` in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t swz(uint32_t tile_base, int row, int ci) {
  return tile_base + (ci >> 3) * kBoxBytes + row * 128 + ((((ci & 7) ^ (row & 7))) << 4);
}

template <int D, int NT, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                const __grid_constant__ CUtensorMap tpk, const __grid_constant__ CUtensorMap tpv,
                const AttnArgs a) {
  using S = Smem<D, NT>;
  using Lay = Layout<D>;
  constexpr int kStages = S::kStages;
  constexpr int kMT = D / 16;   // 16-wide slices of D

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem + S::kMaskOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);
  float* sstat = reinterpret_cast<float*>(smem + S::kStatOff);
  float* so = reinterpret_cast<float*>(smem + S::kOOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // ------------------------------------------------------------ producer
  if (warp == kConsumerWarps) {
    if (lane != 0) return;
    prefetch_tensormap(&tk);
    prefetch_tensormap(&tv);
    if (MODE == kFast) {
      prefetch_tensormap(&tpk);
      prefetch_tensormap(&tpv);
    }
    const uint64_t policy = l2_policy_evict_first();
    int slot = 0;
    uint32_t phase = 0;
    int inflight = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < a.n_items && ok; item += gridDim.x) {
      const Item it = decode_item<MODE>(a, item);
      for (int t0 = it.t_begin; t0 < it.t_end; t0 += kTilesPerStage) {
        if (*abort_flag || !mbar_wait(&empty[slot], phase ^ 1, a.err, kSiteAttnProducer)) {
          ok = false;
          *abort_flag = 1;
          break;
        }
        const int nt = min(kTilesPerStage, it.t_end - t0);
        TileRef refs[kTilesPerStage];
        uint32_t bytes = 0;
        for (int i = 0; i < nt; ++i) {
          refs[i] = resolve_tile<MODE>(a, it, t0 + i);
          if (refs[i].kind >= 0) bytes += 2 * Lay::kTileBytes + (refs[i].kind == 1 ? 64 : 0);
          else latch_error(a.err, SFI_ERR_DEVICE_CHECK, kSiteAttnPage);
        }
        mbar_arrive_expect_tx(&full[slot], bytes);
        uint8_t* sk = smem + slot * S::kStageBytes;
        uint8_t* sv = sk + Lay::kKBytes;
        for (int i = 0; i < nt; ++i) {
          if (refs[i].kind < 0) continue;
          const CUtensorMap* mk = refs[i].kind == 1 ? &tpk : &tk;
          const CUtensorMap* mv = refs[i].kind == 1 ? &tpv : &tv;
#pragma unroll
          for (int h = 0; h < Lay::kHalves; ++h) {
            tma_load_2d(sk + i * Lay::kTileBytes + h * kBoxBytes, mk, h * 64, refs[i].y, &full[slot], policy);
            tma_load_2d(sv + i * Lay::kTileBytes + h * kBoxBytes, mv, h * 64, refs[i].y, &full[slot], policy);
          }
          if (refs[i].kind == 1)
            bulk_load(smask + (slot * kTilesPerStage + i) * 16,
                      a.headmask + (size_t)it.bg * a.p_max + refs[i].pos0, 64, &full[slot]);
        }
        inflight = min(inflight + 1, kStages);
        if (++slot == kStages) {
          slot = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok) {
      // Drain: wait (bounded) for the copies of stages still in flight so no
      // TMA write lands after this CTA has left the SM.
      for (int k = 0; k < inflight; ++k) {
        if (--slot < 0) {
          slot = kStages - 1;
          phase ^= 1;
        }
        mbar_wait(&full[slot], phase, nullptr, 0);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int ctid = threadIdx.x;          // 0..127
  const int r0 = lane >> 2;              // accumulator rows r0, r0 + 8
  const int cq = (lane & 3) * 2;         // accumulator columns cq, cq + 1
  const int rowA = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int chA = lane >> 4;
  const int rowV = (lane & 7) + ((lane >> 4) & 1) * 8;
  const int chV = (lane >> 3) & 1;
  const float NEG_INF = -INFINITY;

  int slot = 0;
  uint32_t phase = 0;
  bool dead = false;   // set once any wait of this CTA failed: keep only the barrier protocol
  for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
    const Item it = decode_item<MODE>(a, item);

    // Q^T fragments (B operand): head nt*8 + r0, dims ks*16 + cq (+8).
    uint32_t qb[NT][kMT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hh = nt * 8 + r0;
      const bool hv = hh < a.G;
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          a.q + ((size_t)it.b * a.Hq + it.g * a.G + (hv ? hh : 0)) * D);
#pragma unroll
      for (int ks = 0; ks < kMT; ++ks) {
        qb[nt][ks][0] = hv ? __ldg(qrow + (ks * 16 + cq) / 2) : 0u;
        qb[nt][ks][1] = hv ? __ldg(qrow + (ks * 16 + 8 + cq) / 2) : 0u;
      }
    }
    float o[NT][kMT][4];
    float mrun[NT][2], lrun[NT][2], lcand[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        mrun[nt][j] = NEG_INF;
        lrun[nt][j] = 0.f;
        lcand[nt][j] = 0.f;
      }
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[nt][mt][i] = 0.f;
    }

    for (int t0 = it.t_begin; t0 < it.t_end; t0 += kTilesPerStage) {
      if (!dead && (*abort_flag || !mbar_wait(&full[slot], phase, a.err, kSiteAttnConsumer))) {
        *abort_flag = 1;
        dead = true;
      }
      const int tile = t0 + warp;
      if (!dead && tile < it.t_end) {
        const TileRef ref = resolve_tile<MODE>(a, it, tile);
        if (ref.kind >= 0) {
          uint8_t* sk = smem + slot * S::kStageBytes + warp * Lay::kTileBytes;
          uint8_t* sv = sk + Lay::kKBytes;
          const uint32_t kb = smem_u32(sk);
          const uint32_t vb = smem_u32(sv);
          // Row validity.  Page tiles: positions in range (and inside the
          // recent window for the fast step).  Packed tiles: per-head mask.
          uint32_t rmask[2];
          if (ref.kind == 0) {
            const int lo = (MODE == kFast) ? a.rec_lo : 0;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int pos = ref.pos0 + r0 + 8 * j;
              rmask[j] = (pos < a.L && pos >= lo) ? 0xffffffffu : 0u;
            }
            if (ref.pos0 + kPage > a.L) {
              // Rows at or beyond L may hold anything: zero their V rows so
              // 0 * garbage cannot poison the PV product.
              const int first_bad = a.L - ref.pos0;
              const int nchunks = (kPage - first_bad) * (D / 8);
              for (int c = lane; c < nchunks; c += 32) {
                const int row = first_bad + c / (D / 8);
                const int ci = c % (D / 8);
                *reinterpret_cast<uint4*>(sv + (ci >> 3) * kBoxBytes + row * 128 + (ci & 7) * 16) =
                    make_uint4(0, 0, 0, 0);
              }
              fence_proxy_async_smem();
              __syncwarp();
            }
          } else {
            const uint32_t* mk = smask + (slot * kTilesPerStage + warp) * 16;
            rmask[0] = mk[r0];
            rmask[1] = mk[r0 + 8];
          }

          // S^T = K . Q^T
          float s[NT][4];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) s[nt][i] = 0.f;
#pragma unroll
          for (int ks = 0; ks < kMT; ++ks) {
            uint32_t af[4];
            ldmatrix_x4(af, swz(kb, rowA, ks * 2 + chA));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[nt], af, qb[nt][ks][0], qb[nt][ks][1]);
          }

          // mask, scale, online softmax
          uint32_t pb_hi[NT][2], pb_lo[NT][2];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            float x[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int hh = nt * 8 + cq + (i & 1);
              const bool v = (rmask[i >> 1] >> hh) & 1u;
              x[i] = (v && hh < a.G) ? s[nt][i] * a.scale_log2 : NEG_INF;
            }
            if (MODE == kDenseExtras && ref.kind == 0 && a.logits) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int hh = nt * 8 + cq + (i & 1);
                const int pos = ref.pos0 + r0 + 8 * (i >> 1);
                if (hh < a.G && pos < a.L)
                  a.logits[((size_t)it.b * a.Hq + it.g * a.G + hh) * a.ld + pos] = s[nt][i] * a.scale;
              }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              float tm = fmaxf(x[j], x[j + 2]);
              tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
              tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
              tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
              const float mnew = fmaxf(mrun[nt][j], tm);
              const float mref = (mnew == NEG_INF) ? 0.f : mnew;
              const float alpha = fast_exp2(mrun[nt][j] - mref);
              mrun[nt][j] = mnew;
              lrun[nt][j] *= alpha;
              if (MODE == kDenseExtras) lcand[nt][j] *= alpha;
#pragma unroll
              for (int mt = 0; mt < kMT; ++mt) {
                o[nt][mt][j] *= alpha;
                o[nt][mt][j + 2] *= alpha;
              }
              x[j] = fast_exp2(x[j] - mref);
              x[j + 2] = fast_exp2(x[j + 2] - mref);
              lrun[nt][j] += x[j] + x[j + 2];
              if (MODE == kDenseExtras && ref.kind == 0) {
                const int p0 = ref.pos0 + r0, p1 = p0 + 8;
                if (p0 >= a.cand_lo && p0 < a.cand_hi) lcand[nt][j] += x[j];
                if (p1 >= a.cand_lo && p1 < a.cand_hi) lcand[nt][j] += x[j + 2];
              }
            }
            // P -> bf16 hi + lo, then transpose to the B operand of PV.
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float p0 = x[2 * j], p1 = x[2 * j + 1];
              const uint32_t hi = pack_bf16x2(p0, p1);
              const float2 hf = unpack_bf16x2(hi);
              const uint32_t lo = pack_bf16x2(p0 - hf.x, p1 - hf.y);
              pb_hi[nt][j] = movmatrix_trans(hi);
              pb_lo[nt][j] = movmatrix_trans(lo);
            }
          }

          // O^T += V^T . P^T
#pragma unroll
          for (int mt = 0; mt < kMT; ++mt) {
            uint32_t vf[4];
            ldmatrix_x4_trans(vf, swz(vb, rowV, mt * 2 + chV));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_bf16_16816(o[nt][mt], vf, pb_hi[nt][0], pb_hi[nt][1]);
              mma_bf16_16816(o[nt][mt], vf, pb_lo[nt][0], pb_lo[nt][1]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0 && !dead) mbar_arrive(&empty[slot]);
      if (++slot == kStages) {
        slot = 0;
        phase ^= 1;
      }
    }

    // ---- merge the four warps' partial softmax states of this item
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int sh = 4; sh <= 16; sh <<= 1) {
          lrun[nt][j] += __shfl_xor_sync(0xffffffffu, lrun[nt][j], sh);
          if (MODE == kDenseExtras) lcand[nt][j] += __shfl_xor_sync(0xffffffffu, lcand[nt][j], sh);
        }
    constexpr int H8 = S::kHeads;
    if (lane < 4) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int hh = nt * 8 + cq + j;
          float* st = sstat + (warp * H8 + hh) * 3;
          st[0] = mrun[nt][j];
          st[1] = lrun[nt][j];
          st[2] = lcand[nt][j];
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int hh = nt * 8 + cq + (i & 1);
          const int d = mt * 16 + r0 + (i >> 1) * 8;
          so[(warp * H8 + hh) * D + d] = o[nt][mt][i];
        }
    named_barrier(1, kConsumerWarps * 32);
    float* part = a.part + (size_t)item * a.G * (D + 4);
    for (int idx = ctid; idx < a.G * D; idx += kConsumerWarps * 32) {
      const int hh = idx / D, d = idx - hh * D;
      float M = NEG_INF;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sstat[(w * H8 + hh) * 3]);
      const float mref = (M == NEG_INF) ? 0.f : M;
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w)
        acc += exp2f(sstat[(w * H8 + hh) * 3] - mref) * so[(w * H8 + hh) * D + d];
      part[hh * (D + 4) + d] = acc;
      if (d == 0) {
        float l = 0.f, lc = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float wt = exp2f(sstat[(w * H8 + hh) * 3] - mref);
          l += wt * sstat[(w * H8 + hh) * 3 + 1];
          lc += wt * sstat[(w * H8 + hh) * 3 + 2];
        }
        part[hh * (D + 4) + D] = M;
        part[hh * (D + 4) + D + 1] = l;
        part[hh * (D + 4) + D + 2] = lc;
      }
    }
    named_barrier(1, kConsumerWarps * 32);
  }
}

// Merge the per-chunk partials of every (b, query head): one warp each.
template <int D>
__global__ void attn_combine_kernel(const float* __restrict__ part, int n_chunks, int B, int Hq,
                                    int Hkv, int G, float* __restrict__ out, float* __restrict__ lse,
                                    float* __restrict__ lse_cand, const int32_t* n_rows, int p_max,
                                    int* err) {
  constexpr int kPer = D / 32;
  const int wid = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= B * Hq) return;
  const int b = wid / Hq, hq = wid - b * Hq;
  const int g = hq / G, hh = hq - g * G;
  const int bg = b * Hkv + g;
  if (n_rows && lane == 0 && hh == 0) {
    const int nr = n_rows[bg];
    if (nr < 0 || nr > p_max) latch_error(err, SFI_ERR_DEVICE_CHECK, kSiteAttnRows);
  }
  const size_t stride = (size_t)G * (D + 4);
  const float* base = part + (size_t)bg * n_chunks * stride + (size_t)hh * (D + 4);
  float M = -INFINITY;
  for (int c = lane; c < n_chunks; c += 32) M = fmaxf(M, base[c * stride + D]);
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, sh));
  const float mref = (M == -INFINITY) ? 0.f : M;
  float acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
  float l = 0.f, lc = 0.f;
  for (int c = 0; c < n_chunks; ++c) {
    const float* pc = base + c * stride;
    const float w = exp2f(pc[D] - mref);
    l += w * pc[D + 1];
    lc += w * pc[D + 2];
#pragma unroll
    for (int k = 0; k < kPer; ++k) acc[k] += w * pc[lane * kPer + k];
  }
  const float inv = 1.f / l;
  float* orow = out + ((size_t)b * Hq + hq) * D + lane * kPer;
#pragma unroll
  for (int k = 0; k < kPer; ++k) orow[k] = acc[k] * inv;
  if (lane == 0) {
    if (lse) lse[(size_t)b * Hq + hq] = (M + log2f(l)) * kLn2;
    if (lse_cand) lse_cand[(size_t)b * Hq + hq] = lc > 0.f ? (M + log2f(lc)) * kLn2 : -INFINITY;
  }
}

__global__ void probs_kernel(int L, int Hq, const float* __restrict__ logits, int64_t ld,
                             const float* __restrict__ lse, float* __restrict__ probs) {
  const int row = blockIdx.y;
  const float m = lse[row];
  const float* z = logits + (size_t)row * ld;
  float* f = probs + (size_t)row * ld;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < L; j += gridDim.x * blockDim.x)
    f[j] = expf(z[j] - m);
}

// ---------------------------------------------------------------- host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// rows x D bf16 matrix, box of 16 rows x 64 columns, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, 16};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int NT, int MODE>
sfi_status launch_attn_t(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tpk,
                         const CUtensorMap& tpv, const AttnArgs& a, cudaStream_t st) {
  using S = Smem<D, NT>;
  auto kern = attn_kernel<D, NT, MODE>;
  static DeviceOnce attr;   // per instantiation and device
  if (!attr.done() &&
      !attr.mark(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal)))
    return SFI_ERR_CUDA;
  const int grid = std::min(a.n_items, num_sms());
  kern<<<grid, kAttnThreads, S::kTotal, st>>>(tk, tv, tpk, tpv, a);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

template <int MODE>
sfi_status launch_attn(int D, int G, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tpk, const CUtensorMap& tpv, const AttnArgs& a,
                       cudaStream_t st) {
  if (D == 128) {
    if (G <= 8) return launch_attn_t<128, 1, MODE>(tk, tv, tpk, tpv, a, st);
    return launch_attn_t<128, 2, MODE>(tk, tv, tpk, tpv, a, st);
  }
  if (G <= 8) return launch_attn_t<64, 1, MODE>(tk, tv, tpk, tpv, a, st);
  return launch_attn_t<64, 2, MODE>(tk, tv, tpk, tpv, a, st);
}

sfi_status launch_combine(int D, const float* part, int n_chunks, const sfi_shape& s, float* out,
                          float* lse, float* lse_cand, const int32_t* n_rows, int p_max, int* err,
                          cudaStream_t st) {
  const int G = s.Hq / s.Hkv;
  const int warps = s.B * s.Hq;
  const int grid = (warps + 3) / 4;
  if (D == 128)
    attn_combine_kernel<128><<<grid, 128, 0, st>>>(part, n_chunks, s.B, s.Hq, s.Hkv, G, out, lse,
                                                   lse_cand, n_rows, p_max, err);
  else
    attn_combine_kernel<64><<<grid, 128, 0, st>>>(part, n_chunks, s.B, s.Hq, s.Hkv, G, out, lse,
                                                  lse_cand, n_rows, p_max, err);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace

// Tiles of 16 rows per chunk for the dense step: about 8 work items per SM,
// at least 8 tiles, a multiple of the 4-tile stage.
int dense_chunk_tiles(const sfi_shape& s, int L) {
  const long T = (L + kPage - 1) / kPage;
  const long bh = (long)s.B * s.Hkv;
  long ct = (T * bh + 8L * num_sms() - 1) / (8L * num_sms());
  ct = std::max(ct, 8L);
  ct = (ct + kTilesPerStage - 1) / kTilesPerStage * kTilesPerStage;
  return (int)ct;
}

int fast_chunks(const sfi_shape& s, int p_max, int n_recent) {
  const long bh = (long)s.B * s.Hkv;
  const long tiles_max = (p_max + kPage - 1) / kPage + n_recent / kPage + 2;
  long nc = (8L * num_sms() + bh - 1) / bh;
  nc = std::min(nc, std::max(1L, tiles_max / 8));
  return (int)std::max(nc, 1L);
}

size_t attn_part_bytes(int n_items, int G, int D) { return (size_t)n_items * G * (D + 4) * sizeof(float); }

sfi_status run_dense_attn(const sfi_shape& s, const sfi_paged_kv& kv, int L, const sfi_bf16* q,
                          float* out, const sfi_dense_extras* ex, float* part, size_t part_bytes,
                          cudaStream_t st, cudaEvent_t ev_begin, cudaEvent_t ev_end) {
  const int G = s.Hq / s.Hkv;
  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)s.num_pages * s.Hkv * kPage;
  if (!make_map(&tk, kv.k_pool, rows, s.D) || !make_map(&tv, kv.v_pool, rows, s.D)) return SFI_ERR_CUDA;
  AttnArgs a{};
  a.B = s.B; a.Hq = s.Hq; a.Hkv = s.Hkv; a.G = G; a.L = L;
  a.num_pages = s.num_pages; a.max_pages = s.max_pages;
  a.page_table = kv.page_table;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.chunk_tiles = dense_chunk_tiles(s, L);
  const int T = (L + kPage - 1) / kPage;
  a.n_chunks = (T + a.chunk_tiles - 1) / a.chunk_tiles;
  a.n_items = s.B * s.Hkv * a.n_chunks;
  if (attn_part_bytes(a.n_items, G, s.D) > part_bytes) return SFI_ERR_WORKSPACE;
  a.part = part;
  a.scale = 1.0f / sqrtf((float)s.D);
  a.scale_log2 = kLog2e * a.scale;
  a.err = kv.err;
  const bool extras = ex && (ex->logits || ex->probs || ex->lse_cand);
  float* zbuf = nullptr;
  if (extras) {
    zbuf = ex->logits ? ex->logits : ex->probs;
    a.logits = zbuf;
    a.ld = ex->ld;
    a.cand_lo = ex->lse_cand ? ex->cand_lo : 0;
    a.cand_hi = ex->lse_cand ? ex->cand_hi : 0;
  }
  if (ev_begin) cudaEventRecord(ev_begin, st);
  sfi_status r;
  if (extras) r = launch_attn<kDenseExtras>(s.D, G, tk, tv, tk, tv, a, st);
  else r = launch_attn<kDense>(s.D, G, tk, tv, tk, tv, a, st);
  if (ev_end) cudaEventRecord(ev_end, st);
  if (r != SFI_OK) return r;
  float* lse_tmp = ex ? ex->lse : nullptr;
  r = launch_combine(s.D, part, a.n_chunks, s, out, lse_tmp, ex ? ex->lse_cand : nullptr, nullptr, 0,
                     kv.err, st);
  if (r != SFI_OK) return r;
  if (ex && ex->probs) {
    dim3 grid((L + 1023) / 1024 < 64 ? (L + 1023) / 1024 : 64, s.B * s.Hq);
    probs_kernel<<<grid, 256, 0, st>>>(L, s.Hq, zbuf, ex->ld, lse_tmp, ex->probs);
    if (cudaPeekAtLastError() != cudaSuccess) return SFI_ERR_CUDA;
  }
  return SFI_OK;
}

sfi_status run_fast_attn(const sfi_shape& s, const sfi_params& p, const sfi_paged_kv& kv, int L,
                         const sfi_bf16* q, const sfi_packed& pk, float* out, float* lse,
                         float* part, size_t part_bytes, cudaStream_t st, cudaEvent_t ev_begin,
                         cudaEvent_t ev_end) {
  const int G = s.Hq / s.Hkv;
  CUtensorMap tk, tv, tpk, tpv;
  const uint64_t rows = (uint64_t)s.num_pages * s.Hkv * kPage;
  const uint64_t prows = (uint64_t)s.B * s.Hkv * pk.p_max;
  if (!make_map(&tk, kv.k_pool, rows, s.D) || !make_map(&tv, kv.v_pool, rows, s.D) ||
      !make_map(&tpk, pk.k, prows, s.D) || !make_map(&tpv, pk.v, prows, s.D))
    return SFI_ERR_CUDA;
  AttnArgs a{};
  a.B = s.B; a.Hq = s.Hq; a.Hkv = s.Hkv; a.G = G; a.L = L;
  a.num_pages = s.num_pages; a.max_pages = s.max_pages;
  a.page_table = kv.page_table;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.n_chunks = fast_chunks(s, pk.p_max, p.n_recent);
  a.n_items = s.B * s.Hkv * a.n_chunks;
  if (attn_part_bytes(a.n_items, G, s.D) > part_bytes) return SFI_ERR_WORKSPACE;
  a.part = part;
  a.scale = 1.0f / sqrtf((float)s.D);
  a.scale_log2 = kLog2e * a.scale;
  a.n_rows = pk.n_rows;
  a.headmask = pk.headmask;
  a.p_max = pk.p_max;
  a.rec_lo = std::max(L - p.n_recent, 0);
  a.err = kv.err;
  if (ev_begin) cudaEventRecord(ev_begin, st);
  sfi_status r = launch_attn<kFast>(s.D, G, tk, tv, tpk, tpv, a, st);
  if (ev_end) cudaEventRecord(ev_end, st);
  if (r != SFI_OK) return r;
  return launch_combine(s.D, part, a.n_chunks, s, out, lse, nullptr, pk.n_rows, pk.p_max, kv.err, st);
}

sfi_status run_attn_probs(const sfi_shape& s, int L, const float* logits, int64_t ld, const float* lse,
                          float* probs, cudaStream_t st) {
  dim3 grid((L + 1023) / 1024 < 64 ? (L + 1023) / 1024 : 64, s.B * s.Hq);
  probs_kernel<<<grid, 256, 0, st>>>(L, s.Hq, logits, ld, lse, probs);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace sfi
