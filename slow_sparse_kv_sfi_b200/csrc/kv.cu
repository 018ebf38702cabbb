// Paged KV cache maintenance: append the new token of every (sequence, KV
// head) and keep the key-norm statistic the Selector's prior reads
// ([ZH] "2.2" 先验分布 — Key 范数因子; [ES] "El Selector", Prioridad
// Estructural).  The norm of the stored bf16 key is accumulated in fp64 and
// rounded once to fp32.
#include "common.cuh"
#include "internal.h"

namespace sfi {

// One warp per (b, kv head).
template <int D>
__global__ void __launch_bounds__(128) append_kernel(int BH, int Hkv, int L, int max_pages, int num_pages,
                                                     const int32_t* __restrict__ pt, __nv_bfloat16* kpool,
                                                     __nv_bfloat16* vpool, const __nv_bfloat16* __restrict__ knew,
                                                     const __nv_bfloat16* __restrict__ vnew, float* norms,
                                                     int64_t norm_ld, int* err) {
  grid_dep_enter_writer();
  const int bg = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (bg >= BH) return;
  const int b = bg / Hkv, h = bg - b * Hkv;
  const int pos = L - 1;
  const int page = pt[(size_t)b * max_pages + pos / kPage];
  append_row_warp<D>(threadIdx.x & 31, bg, h, pos, page, Hkv, num_pages, kpool, vpool, knew, vnew, norms, norm_ld,
                     err);
}

// One warp per (b, kv head, position) in [lo, hi).
template <int D>
__global__ void key_norms_kernel(int Hkv, int lo, int hi, int max_pages, int num_pages,
                                 const int32_t* __restrict__ pt,
                                 const __nv_bfloat16* __restrict__ kpool, float* norms,
                                 int64_t norm_ld, int* err) {
  grid_dep_enter_writer();
  const int bg = blockIdx.y;
  const int b = bg / Hkv, h = bg - b * Hkv;
  const int lane = threadIdx.x & 31;
  const int pos = lo + blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (pos >= hi) return;
  const int page = pt[(size_t)b * max_pages + pos / kPage];
  if ((unsigned)page >= (unsigned)num_pages) {
    if (lane == 0) latch_error(err, SFI_ERR_DEVICE_CHECK, kSiteNorms);
    return;
  }
  const __nv_bfloat16* row = kpool + ((size_t)(page * Hkv + h) * kPage + pos % kPage) * D;
  double s = 0.0;
#pragma unroll
  for (int i = lane * 2; i < D; i += 64) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(row + i));
    s += (double)v.x * v.x + (double)v.y * v.y;
  }
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) s += __shfl_xor_sync(0xffffffffu, s, sh);
  if (lane == 0) norms[(size_t)bg * norm_ld + pos] = (float)sqrt(s);
}

sfi_status run_append(const sfi_shape& s, const sfi_paged_kv& kv, int L, const sfi_bf16* k_new,
                      const sfi_bf16* v_new, cudaStream_t st) {
  const int BH = s.B * s.Hkv;
  auto* kp = reinterpret_cast<__nv_bfloat16*>(kv.k_pool);
  auto* vp = reinterpret_cast<__nv_bfloat16*>(kv.v_pool);
  const auto* kn = reinterpret_cast<const __nv_bfloat16*>(k_new);
  const auto* vn = reinterpret_cast<const __nv_bfloat16*>(v_new);
  const int64_t ld = (int64_t)s.max_pages * kPage;
  const dim3 grid((BH + 3) / 4);
  if (s.D == 128)
    launch_k(append_kernel<128>, grid, dim3(128), 0, st, BH, s.Hkv, L, s.max_pages, s.num_pages, kv.page_table, kp, vp,
             kn, vn, kv.key_norms, ld, kv.err);
  else
    launch_k(append_kernel<64>, grid, dim3(128), 0, st, BH, s.Hkv, L, s.max_pages, s.num_pages, kv.page_table, kp, vp,
             kn, vn, kv.key_norms, ld, kv.err);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

sfi_status run_key_norms(const sfi_shape& s, const sfi_paged_kv& kv, int lo, int hi,
                         cudaStream_t st) {
  if (hi <= lo) return SFI_OK;
  dim3 grid((hi - lo + 7) / 8, s.B * s.Hkv);
  const auto* kp = reinterpret_cast<const __nv_bfloat16*>(kv.k_pool);
  const int64_t ld = (int64_t)s.max_pages * kPage;
  if (s.D == 128)
    launch_k(key_norms_kernel<128>, dim3(grid), dim3(256), 0, st, s.Hkv, lo, hi, s.max_pages, s.num_pages,
             kv.page_table, kp, kv.key_norms, ld, kv.err);
  else
    launch_k(key_norms_kernel<64>, dim3(grid), dim3(256), 0, st, s.Hkv, lo, hi, s.max_pages, s.num_pages,
             kv.page_table, kp, kv.key_norms, ld, kv.err);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace sfi
