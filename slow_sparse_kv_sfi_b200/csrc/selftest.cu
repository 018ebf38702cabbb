// Failure detection of the device-side waits, exercised without a fault.
//
// Every wait of the library's kernels on an mbarrier is bounded: after the
// limit set by sfi_set_wait_limit (2 s by default, passed to each launch) it
// latches SFI_ERR_TIMEOUT with its site into the cache's error word, stops
// waiting and lets the kernel return, so the context stays usable and the
// host learns of it through sfi_poll_error.  sfi_selftest_wait runs that same
// wait on a barrier that nothing ever completes, so the expiry path can be
// checked on a healthy GPU.  The pages describe no failure handling.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace sfi {
namespace {

std::atomic<unsigned long long> g_wait_ns{kWaitLimitNs};

// One thread initialises a barrier that expects one arrival and waits for its
// first phase; no thread arrives, so the wait ends at its limit.
__global__ void wait_selftest_kernel(int* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err, kSiteSelfTest, limit_ns);
  __syncthreads();
}

}  // namespace

unsigned long long wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

}  // namespace sfi

using namespace sfi;

extern "C" {

sfi_status sfi_set_wait_limit(int64_t ns) {
  if (ns < 100000 || ns > 60000000000LL) return SFI_ERR_INVALID_ARG;
  g_wait_ns.store((unsigned long long)ns, std::memory_order_relaxed);
  return SFI_OK;
}

sfi_status sfi_get_wait_limit(int64_t* ns) {
  if (!ns) return SFI_ERR_INVALID_ARG;
  *ns = (int64_t)wait_limit_ns();
  return SFI_OK;
}

sfi_status sfi_selftest_wait(const sfi_paged_kv* kv, int64_t limit_ns, sfi_stream stream) {
  if (!kv || !kv->err) return SFI_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 60000000000LL) return SFI_ERR_INVALID_ARG;
  wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(kv->err, (unsigned long long)limit_ns);
  return cudaPeekAtLastError() == cudaSuccess ? SFI_OK : SFI_ERR_CUDA;
}

}  // extern "C"
