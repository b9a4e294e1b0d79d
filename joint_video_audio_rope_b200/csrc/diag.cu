// Self-test of the bounded device waits.  One warp waits on an mbarrier that
// nothing ever arrives at, through the same bounded-wait helper the attention
// kernels use, with a short limit; the wait gives up, records MMDIT_ETIMEOUT in
// the device error word and the kernel returns, leaving the context usable.
#include "internal.h"

namespace mmdit {
namespace {

__global__ void wait_timeout_kernel(int* err, uint64_t limit_ns, int* waited) {
  __shared__ __align__(8) uint64_t bar_storage;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);  // one arrival expected; none will come
    fence_mbar_init();
  }
  __syncwarp();
  const bool ok = mbar_wait_for(bar, 0, err, limit_ns);
  if (threadIdx.x == 0) *waited = ok ? 0 : 1;
}

}  // namespace
}  // namespace mmdit

using namespace mmdit;

extern "C" int mmdit_selftest_wait_timeout(int limit_ms, int* waited_out, mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_selftest_wait_timeout");
  if (limit_ms < 1 || limit_ms > 2000)
    return fail(MMDIT_EINVAL, "selftest: limit_ms must be in [1, 2000]");
  if (waited_out == nullptr || (reinterpret_cast<uintptr_t>(waited_out) & 3u) != 0)
    return fail(MMDIT_EINVAL, "selftest: waited_out must be an aligned device int");
  int* err = device_error_flag();
  if (err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");
  wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(err, (uint64_t)limit_ms * 1000000ull,
                                                          waited_out);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "selftest launch");
}
