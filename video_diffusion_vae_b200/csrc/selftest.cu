// Self-test of the bounded pipeline waits: a wait on an mbarrier phase that
// nothing completes must give up at its limit, record its bit in the device
// error word and let the kernel return (no trap, no hang).
#include "wvae.h"
#include "internal.h"
#include "ptx.cuh"

namespace wvae {

// Error-word bit of this deliberate timeout (the pipeline kernels use bits 0-3).
constexpr unsigned kDeverrTimeoutSelftest = 1u << 4;

__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns, unsigned* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(smem_u32(&bar), 1);
  abort_flag = 0;
  fence_mbar_init();
  // Nobody arrives: phase 0 never completes, so the wait runs out.
  mbar_wait_bounded(smem_u32(&bar), 0, &abort_flag, err, kDeverrTimeoutSelftest, limit_ns);
}

}  // namespace wvae

extern "C" wvae_status wvae_selftest_wait_timeout(unsigned int limit_us, wvae_stream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) return WVAE_ERR_INVALID_ARG;
  unsigned* err = wvae::device_error_word();
  if (err == nullptr) return WVAE_ERR_NO_DEVICE;
  wvae::wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      1000ull * limit_us, err);
  return cudaGetLastError() == cudaSuccess ? WVAE_OK : WVAE_ERR_CUDA;
}
