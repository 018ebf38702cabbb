// Paged KV cache maintenance: append the new token of every (sequence, KV
// head) and keep the key-norm statistic the Selector's prior reads
// ([ZH] "2.2" 先验分布 — Key 范数因子; [ES] "El Selector", Prioridad
// Estructural).  The norm of the stored bf16 key is accumulated in fp64 and
// rounded once to fp32.
#include "common.cuh"
#include "internal.h"

namespace sfi {

// One CTA per (b, kv head), one thread per element of the row.
__global__ void append_kernel(int Hkv, int D, int L, int max_pages, int num_pages,
                              const int32_t* __restrict__ pt, __nv_bfloat16* kpool,
                              __nv_bfloat16* vpool, const __nv_bfloat16* __restrict__ knew,
                              const __nv_bfloat16* __restrict__ vnew, float* norms, int64_t norm_ld,
                              int* err) {
  __shared__ double wsum[4];
  const int bg = blockIdx.x;
  const int b = bg / Hkv, h = bg - b * Hkv;
  const int pos = L - 1;
  const int page = pt[(size_t)b * max_pages + pos / kPage];
  if ((unsigned)page >= (unsigned)num_pages) {
    if (threadIdx.x == 0) latch_error(err, SFI_ERR_DEVICE_CHECK, kSiteAppend);
    return;
  }
  const size_t row = ((size_t)(page * Hkv + h) * kPage + pos % kPage) * D;
  const int t = threadIdx.x;
  const __nv_bfloat16 k = knew[(size_t)bg * D + t];
  kpool[row + t] = k;
  vpool[row + t] = vnew[(size_t)bg * D + t];
  const double x = (double)__bfloat162float(k);
  double s = x * x;
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) s += __shfl_xor_sync(0xffffffffu, s, sh);
  if ((t & 31) == 0) wsum[t >> 5] = s;
  __syncthreads();
  if (t == 0) {
    double tot = 0.0;
    for (int w = 0; w < D / 32; ++w) tot += wsum[w];
    if (norms) norms[(size_t)bg * norm_ld + pos] = (float)sqrt(tot);
  }
}

// One warp per (b, kv head, position) in [lo, hi).
template <int D>
__global__ void key_norms_kernel(int Hkv, int lo, int hi, int max_pages, int num_pages,
                                 const int32_t* __restrict__ pt,
                                 const __nv_bfloat16* __restrict__ kpool, float* norms,
                                 int64_t norm_ld, int* err) {
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
  append_kernel<<<s.B * s.Hkv, s.D, 0, st>>>(
      s.Hkv, s.D, L, s.max_pages, s.num_pages, kv.page_table,
      reinterpret_cast<__nv_bfloat16*>(kv.k_pool), reinterpret_cast<__nv_bfloat16*>(kv.v_pool),
      reinterpret_cast<const __nv_bfloat16*>(k_new), reinterpret_cast<const __nv_bfloat16*>(v_new),
      kv.key_norms, (int64_t)s.max_pages * kPage, kv.err);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

sfi_status run_key_norms(const sfi_shape& s, const sfi_paged_kv& kv, int lo, int hi,
                         cudaStream_t st) {
  if (hi <= lo) return SFI_OK;
  dim3 grid((hi - lo + 7) / 8, s.B * s.Hkv);
  const auto* kp = reinterpret_cast<const __nv_bfloat16*>(kv.k_pool);
  const int64_t ld = (int64_t)s.max_pages * kPage;
  if (s.D == 128)
    key_norms_kernel<128><<<grid, 256, 0, st>>>(s.Hkv, lo, hi, s.max_pages, s.num_pages,
                                                kv.page_table, kp, kv.key_norms, ld, kv.err);
  else
    key_norms_kernel<64><<<grid, 256, 0, st>>>(s.Hkv, lo, hi, s.max_pages, s.num_pages,
                                               kv.page_table, kp, kv.key_norms, ld, kv.err);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // namespace sfi
