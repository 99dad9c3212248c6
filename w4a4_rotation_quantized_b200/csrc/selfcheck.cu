// selfcheck.cu -- failure-detection self-check: a kernel whose one bounded
// wait is meant to run out.  It exercises the same routine every library
// kernel waits with (mbar_wait_bounded): the limit passes, the code lands in
// the per-device status word, the kernel returns and the context stays usable.
#include "qr_device.cuh"
#include "qr_internal.h"

namespace qr {

namespace {

__global__ void wait_selfcheck_kernel(uint64_t limit_ns, int32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    // nothing ever arrives on `bar`, so this wait can only run out
    mbar_wait_bounded(&bar, 0, &abort_flag, status, kDevTimeoutSelfCheck, limit_ns);
  }
}

}  // namespace

qr_status launch_wait_selfcheck(uint64_t limit_ns, cudaStream_t stream) {
  int32_t* status = device_status_word();
  if (status == nullptr) return QR_ERR_CUDA;
  wait_selfcheck_kernel<<<1, 32, 0, stream>>>(limit_ns, status);
  return cudaGetLastError() == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

}  // namespace qr
