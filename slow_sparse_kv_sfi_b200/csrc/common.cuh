// Shared device helpers for the SFI kernels (sm_100a).
//
// Hand-written PTX wrappers for the pieces the kernels are built from:
// mbarriers, TMA tile loads (cp.async.bulk.tensor) and 1-D bulk copies into
// shared memory, ldmatrix / movmatrix fragment moves and the bf16 mma.sync
// tile used for the GQA-group contractions.  Every wait on an mbarrier is
// bounded in time; on expiry it latches an error code and returns false.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sfi.h"

namespace sfi {

// Programmatic dependent launch.  The library launches its kernels with
// programmatic stream serialization, so a kernel may be scheduled while the
// previous kernel on its stream is still running.  A kernel calls
// grid_dep_wait() before it touches global memory that the previous kernel
// may write or read; it returns once the previous kernel has finished and its
// writes are visible.  grid_dep_launch() lets the next kernel get scheduled
// early; kernels that write the cache or the packed buffers (the append, the
// key norms, the compaction) never call it, because the attention's producer
// reads pages, packed rows and queries before its wait.  Both are no-ops for
// a kernel launched the ordinary way.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_enter() {
  grid_dep_wait();
  grid_dep_launch();
}
// The start of a kernel that writes the cache or the packed buffers: wait,
// and let the next kernel start only when this one has finished.
__device__ __forceinline__ void grid_dep_enter_writer() { grid_dep_wait(); }


constexpr int kPage = 16;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // default limit of one wait: 2 s

// Device error word layout: low byte = sfi_status, next byte = site id.
enum ErrSite : int {
  kSiteAppend = 1, kSiteNorms = 2, kSiteAttnProducer = 3, kSiteAttnConsumer = 4,
  kSiteAttnPage = 5, kSiteAttnRows = 6, kSiteCompactIdx = 7, kSiteCompactPage = 8,
  kSiteSelectPage = 9, kSiteCompactRows = 10, kSiteSelfTest = 11,
};

__device__ __forceinline__ void latch_error(int* err, int status, int site) {
  if (err) atomicCAS(err, 0, status | (site << 8));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's earlier generic-proxy global writes before later
// async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: true when the phase with the given parity completed, false
// (after latching SFI_ERR_TIMEOUT) when limit_ns elapsed first.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err, int site,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0 && global_ns() - t0 > limit_ns) {
      latch_error(err, SFI_ERR_TIMEOUT, site);
      return false;
    }
  }
}

// ---------------------------------------------------------------- TMA / bulk copies
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 2-D tiled tensor load global -> shared, completion counted on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 3-D tiled tensor load global -> shared, completion counted on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 4-D tiled tensor load global -> shared, completion counted on `bar`.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- fragments
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t v) {
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&v);
  return __bfloat1622float2(b);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Named barrier over `nthreads` threads (multiple of 32), id 1..15.
__device__ __forceinline__ void named_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Order-preserving map of fp32 to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Append of one decode token by one warp: row `pos` of (b, kv head h) in the
// paged cache receives k_new / v_new (bf16 [B, Hkv, D] at row bg = b * Hkv + h),
// and norms[bg * norm_ld + pos] (when non-null) the fp32 rounding of the
// fp64-accumulated Euclidean norm of the stored key.  Lane l moves elements
// [l * D / 32, (l + 1) * D / 32).  A page-table entry outside the pool is
// latched as SFI_ERR_DEVICE_CHECK and nothing is written; returns whether the
// row was written.  The writes are fenced for later TMA reads of the row.
template <int D>
__device__ __forceinline__ bool append_row_warp(int lane, int bg, int h, int pos, int page, int Hkv, int num_pages,
                                                __nv_bfloat16* kpool, __nv_bfloat16* vpool,
                                                const __nv_bfloat16* knew, const __nv_bfloat16* vnew,
                                                float* norms, int64_t norm_ld, int* err) {
  static_assert(D == 64 || D == 128, "head dim");
  if ((unsigned)page >= (unsigned)num_pages) {
    if (lane == 0) latch_error(err, SFI_ERR_DEVICE_CHECK, kSiteAppend);
    return false;
  }
  constexpr int E = D / 32;
  const size_t src = (size_t)bg * D + lane * E;
  const size_t dst = ((size_t)(page * Hkv + h) * kPage + pos % kPage) * D + lane * E;
  uint32_t kx[E / 2], vx[E / 2];
  if constexpr (E == 4) {
    const uint2 k2 = *reinterpret_cast<const uint2*>(knew + src);
    const uint2 v2 = *reinterpret_cast<const uint2*>(vnew + src);
    *reinterpret_cast<uint2*>(kpool + dst) = k2;
    *reinterpret_cast<uint2*>(vpool + dst) = v2;
    kx[0] = k2.x;
    kx[1] = k2.y;
  } else {
    kx[0] = *reinterpret_cast<const uint32_t*>(knew + src);
    vx[0] = *reinterpret_cast<const uint32_t*>(vnew + src);
    *reinterpret_cast<uint32_t*>(kpool + dst) = kx[0];
    *reinterpret_cast<uint32_t*>(vpool + dst) = vx[0];
  }
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < E / 2; ++i) {
    const float2 f = unpack_bf16x2(kx[i]);
    ss += (double)f.x * f.x + (double)f.y * f.y;
  }
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, sh);
  if (lane == 0 && norms) norms[(size_t)bg * norm_ld + pos] = (float)sqrt(ss);
  fence_proxy_async_global();
  (void)vx;
  return true;
}

}  // namespace sfi
