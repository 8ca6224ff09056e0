// 64-bit checksum of a state-blob payload: the sum (mod 2^64) over the
// payload's little-endian 64-bit words w_i of checksum_term(w_i, i).  Being a
// sum, it is computed in parallel on the device for device blobs and by the
// same term function on the host for host blobs.
#include "../../include/gdn.h"
#include "internal.h"

namespace gdn {
namespace {

constexpr int kSumThreads = 256;

__global__ void __launch_bounds__(kSumThreads) checksum_kernel(const uint64_t* __restrict__ words, size_t nwords,
                                                                 unsigned long long* __restrict__ out) {
  uint64_t acc = 0;
  for (size_t i = (size_t)blockIdx.x * kSumThreads + threadIdx.x; i < nwords; i += (size_t)gridDim.x * kSumThreads)
    acc += checksum_term(__ldg(words + i), i);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ uint64_t part[kSumThreads / 32];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t s = 0;
    for (int w = 0; w < kSumThreads / 32; ++w) s += part[w];
    atomicAdd(out, (unsigned long long)s);
  }
}

}  // namespace

// `out` must be zeroed on the stream before the launch.
cudaError_t launch_checksum(const void* payload, size_t bytes, unsigned long long* out, cudaStream_t stream) {
  const size_t nwords = bytes / 8;
  if (nwords == 0) return cudaSuccess;
  const unsigned grid = (unsigned)std::min<size_t>(148 * 4, (nwords + kSumThreads - 1) / kSumThreads);
  LaunchScope scope(GDN_K_STATE_CHECKSUM, stream);
  checksum_kernel<<<grid, kSumThreads, 0, stream>>>((const uint64_t*)payload, nwords, out);
  return cudaGetLastError();
}

uint64_t host_checksum(const void* payload, size_t bytes) {
  const uint64_t* w = (const uint64_t*)payload;
  uint64_t s = 0;
  for (size_t i = 0; i < bytes / 8; ++i) s += checksum_term(w[i], i);
  return s;
}

}  // namespace gdn
