// selftest.cuh - kernels that exercise the library's failure detection.
//
// Each waits, through the same bounded waits the pipelines use, on an
// mbarrier that nothing ever arrives at.  The wait gives up after the
// device's wait limit (dg_set_wait_limit_ns), records ERR_TIMEOUT in the
// error word and the kernel returns normally: nothing traps and nothing waits
// without bound, so the context stays usable and dg_check_device_errors()
// reports DG_ERR_TIMEOUT.
#pragma once

#include "dg_common.cuh"
#include "gemm.cuh"

namespace dg {

constexpr uint32_t kSiteSelfTest = 0x7F1;
constexpr uint32_t kSiteSelfTestPair = 0x7F2;

// One CTA: the single-CTA wait of the TMA / MMA pipelines.
__global__ void __launch_bounds__(32) wait_selftest_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, kSiteSelfTest);
  __syncthreads();
}

// A cluster of two CTAs: the CTA-pair wait, which on expiry also raises the
// peer's abort flag through distributed shared memory.  The cluster barriers
// make sure both flags exist before either CTA can write its peer's, and that
// neither CTA exits while its peer may still write.
__global__ void __launch_bounds__(32) wait_pair_selftest_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  gemm::cluster_sync();
  const uint32_t peer = gemm::cluster_rank() ^ 1u;
  const uint32_t peer_abort = gemm::map_to_rank(smem_u32(&abort_flag), peer);
  if (threadIdx.x == 0) mbar_wait_pair(&bar, 0, &abort_flag, peer_abort, kSiteSelfTestPair);
  gemm::cluster_sync();
}

}  // namespace dg
