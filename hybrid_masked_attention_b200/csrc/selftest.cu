// Self-test of the bounded-wait path that every tcgen05 kernel relies on: one
// CTA waits on an mbarrier that nothing arrives on, with the same bounded wait
// the kernels use (limit in SM clock cycles), gives up, and records the timeout
// bit in the metadata header exactly as an aborting kernel does.  No TMA, MMA or
// TMEM is involved, so nothing is left in flight; the context stays usable.
#include "mtfm_internal.cuh"
#include "sm100.cuh"

namespace mtfm {
namespace {

__global__ void wait_timeout_kernel(MetaHeader* hdr, long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_abort;
  if (threadIdx.x != 0) return;
  s_abort = 0;
  const uint32_t b = sm100::smem_addr(&bar);
  sm100::mbar_init(b, 1);
  sm100::fence_barrier_init();
  // phase 0 never completes: nothing arrives on this barrier
  if (!sm100::mbar_wait_limit(b, 0, &s_abort, limit)) atomicOr(&hdr->error, kErrTimeout);
}

}  // namespace

cudaError_t launch_wait_timeout(MetaHeader* hdr, long long limit, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(hdr, limit);
  return cudaGetLastError();
}

}  // namespace mtfm
