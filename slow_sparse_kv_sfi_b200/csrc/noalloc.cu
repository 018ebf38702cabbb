// Dense attention whose scratch lives in a static device array, for callers
// that cannot allocate device memory at the point of the call.
//
// sfi_dense_attn needs scratch (a work counter and the split-K partials) and
// takes it as a caller-allocated workspace.  Some callers have no way to
// provide one: serving runtimes whose memory pool hands the library only the
// input and output tensors, and plugin or embedded hosts that have no access
// to the CUDA allocator.  This entry point runs the same kernels with the scratch
// taken from g_noalloc_scratch, a file-scope device array of
// kNoAllocScratchBytes that every GPU which loads the library holds until the
// process exits.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace sfi {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB per device
constexpr size_t kCounterBytes = 256;                         // work counter, then partials

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_addr[64] = {nullptr};

// Device address of g_noalloc_scratch on the current device.  The first call
// on a device looks it up (host code only holds a stand-in for the symbol)
// and keeps it for the life of the process: this assumes the device's
// context is not reset (cudaDeviceReset) while the library is loaded.
sfi_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SFI_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SFI_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return SFI_OK;
}

__global__ void zero_counter_kernel(int* ctr) {
  grid_dep_enter();
  ctr[0] = 0;
}

}  // namespace
}  // namespace sfi

using namespace sfi;

extern "C" sfi_status sfi_dense_attn_noalloc(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L,
                                             const sfi_bf16* q, float* out, const sfi_dense_extras* extras,
                                             sfi_stream stream) {
  // the same argument checks as sfi_dense_attn
  const sfi_status v = check_dense_call(shape, kv, L, q, out, extras);
  if (v != SFI_OK) return v;
  const sfi_shape& s = *shape;
  const int G = s.Hq / s.Hkv;
  // partials this call needs, against the static capacity
  const int T = (L + kPage - 1) / kPage;
  const int ct = dense_chunk_tiles(s, L);
  const int n_items = s.B * s.Hkv * ((T + ct - 1) / ct);
  const size_t part_cap = kNoAllocScratchBytes - kCounterBytes;
  if (attn_part_bytes(n_items, G, s.D) > part_cap) return SFI_ERR_WORKSPACE;
  void* base = nullptr;
  const sfi_status r = scratch_address(&base);
  if (r != SFI_OK) return r;
  char* b = static_cast<char*>(base);
  int* ctr = reinterpret_cast<int*>(b);
  cudaStream_t st = (cudaStream_t)stream;
  // the area keeps whatever the last call left: the work counter must start at zero
  launch_k(zero_counter_kernel, dim3(1), dim3(1), 0, st, ctr);
  if (cudaPeekAtLastError() != cudaSuccess) return SFI_ERR_CUDA;
  return run_dense_attn(s, *kv, L, q, out, extras, ctr, reinterpret_cast<float*>(b + kCounterBytes), part_cap, st,
                        nullptr, nullptr);
}
