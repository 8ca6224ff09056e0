// Self-test of the bounded-wait path that every pipelined kernel relies on.
//
// A kernel whose wait on an mbarrier (or a peer's flag) runs past its limit
// does not trap: it records kStatusWaitTimeout in the device status word,
// releases what it holds and returns, so that the context stays usable and
// the host learns of it through gdn_get_device_status ("fail before unsafe or
// partial execution", DS4Server issue #95, implementation comment).  This
// kernel exercises exactly that path: it waits, with the same bounded wait
// the mixer kernels use, on an mbarrier that nothing will ever arrive on and
// that no copy targets, so the wait always runs out after `limit_ns`.
#include "../../include/gdn.h"
#include "internal.h"
#include "tc.cuh"

namespace gdn {
namespace {

__global__ void __launch_bounds__(32) wait_expiry_kernel(uint64_t limit_ns, int32_t* status) {
  __shared__ uint64_t mb;
  if (threadIdx.x == 0) {
    tc::mbar_init(&mb, 1);  // one arrival would complete phase 0; none is ever made
    tc::mbar_init_fence();
  }
  __syncwarp();
  // phase 0 of a fresh barrier is incomplete until an arrival, so this wait can only end by its limit
  const bool done = tc::mbar_wait(&mb, 0, limit_ns);
  if (!done && threadIdx.x == 0) set_status(status, kStatusWaitTimeout);
}

}  // namespace

cudaError_t launch_wait_expiry(uint64_t limit_ns, int32_t* status, cudaStream_t stream) {
  LaunchScope scope(GDN_K_DIAG, stream);
  wait_expiry_kernel<<<1, 32, 0, stream>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace gdn
