// kda_selftest.cu -- kda_selftest_wait_timeout: drives the bounded-wait
// failure path of the kernels on purpose, so it can be tested without
// faulting or hanging a GPU.
//
// Every mbarrier wait in the library's kernels is bounded by %globaltimer;
// when a bound runs out the kernel records KDA_ERR_TIMEOUT (and a code naming
// the wait) in the device status word instead of trapping, and gives up its
// work. In normal operation no bound ever runs out, so that path is otherwise
// never executed. Here one thread waits, with the same helpers the kernels
// use, on an mbarrier that nothing ever arrives on: first with CTA-scope
// acquire, then with cluster-scope acquire (the wait the chunk kernel's ring
// uses), each for max_ns. Both must give up and record their codes.
#include "../../include/kda.h"
#include "kda_common.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace selftest {

constexpr int kCodeCtaWait = 90, kCodeClusterWait = 91;

__global__ void bounded_wait_kernel(uint64_t max_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t saddr = tc::smem_u32(&bar);
  tc::mbar_init(saddr, 1);   // expects one arrive, which never comes
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  if (!tc::mbar_wait_bounded(saddr, 0, max_ns)) report_timeout(kCodeCtaWait);
  if (!tc::mbar_wait_cluster_bounded(saddr, 0, max_ns)) {
    // the status word keeps the first code; count the second wait's timeout too
    atomicOr(&g_status.flags, kStatusTimeout);
    if (g_status.detail == kCodeCtaWait) g_status.detail = kCodeCtaWait * 100 + kCodeClusterWait;
  }
}

}  // namespace selftest
}  // namespace kda

extern "C" kda_status kda_selftest_wait_timeout(uint64_t max_ns, cudaStream_t stream) {
  if (max_ns < 1000ull || max_ns > 1000000000ull) return KDA_ERR_INVALID_ARG;
  kda::selftest::bounded_wait_kernel<<<1, 32, 0, stream>>>(max_ns);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
