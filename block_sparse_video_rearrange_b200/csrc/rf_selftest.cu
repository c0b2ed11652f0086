// Device self-tests that are not part of the path.
//
// rf_expired_wait_selftest_kernel exercises the failure path every bounded
// wait of the attention kernel takes: one thread waits on an mbarrier that
// nothing arrives on, with the same helper and limit (mbar_wait, 1 s), and on
// expiry records it in the workspace status words the way an attention CTA
// does (set its abort flag, OR a bit into the expired-wait word; bit 31 here).
#include "rf_device.cuh"

namespace {

__global__ void rf_expired_wait_selftest_kernel(uint32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x != 0) return;
  mbar_init(rf_smem_u32(&bar), 1);
  abort = 0;
  fence_mbar_init();
  if (!mbar_wait(rf_smem_u32(&bar), 0, &abort)) {
    *reinterpret_cast<volatile int*>(&abort) = 1;
    atomicOr(status + RF_STATUS_TIMEOUT, 1u << 31);
  }
}

}  // namespace

rf_status_t rf_launch_expired_wait_selftest(const rf_plan* p, void* ws, cudaStream_t st) {
  uint32_t* status = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + p->off_status);
  rf_expired_wait_selftest_kernel<<<1, 32, 0, st>>>(status);
  return rf_check_launch("rf_expired_wait_selftest_kernel");
}
