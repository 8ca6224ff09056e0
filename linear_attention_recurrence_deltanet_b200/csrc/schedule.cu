// Varlen schedule of a packed prefill, built on the device from cu_seqlens.
//
// Outputs (in the caller's workspace):
//   order[N]          sequence ids by decreasing length (ties: lower id first),
//                     so the longest recurrences start first;
//   chunk_off[N+1]    exclusive prefix sum of ceil(len_n / chunk_size) in
//                     sequence-id order;
//   chunk_map[total]  one int4 per chunk {seq, first token, length, chunk index
//                     within the sequence}; chunks restart at every sequence
//                     start, so only a sequence's last chunk can be short.
// All integer work, bit-exact.  One CTA; O(N^2 / threads) for the ranking.
#include "../../include/gdn.h"
#include "internal.h"

namespace gdn {
namespace {

constexpr int kSchedThreads = 1024;

__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(const int32_t* __restrict__ cu, int32_t N,
                                                                   int32_t C, int32_t* __restrict__ order,
                                                                   int32_t* __restrict__ chunk_off,
                                                                   int4* __restrict__ chunk_map) {
  __shared__ int32_t warp_tot[kSchedThreads / 32];
  __shared__ int32_t carry;
  const int tid = threadIdx.x;
  // 1. rank sequences: rank(n) = #{m : len_m > len_n or (len_m == len_n and m < n)}
  for (int n = tid; n < N; n += kSchedThreads) {
    const int32_t ln = cu[n + 1] - cu[n];
    int32_t r = 0;
    for (int m = 0; m < N; ++m) {
      const int32_t lm = cu[m + 1] - cu[m];
      r += (lm > ln) || (lm == ln && m < n);
    }
    order[r] = n;
  }
  // 2. exclusive scan of chunk counts, in tiles of kSchedThreads sequences
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < N; base += kSchedThreads) {
    const int n = base + tid;
    const int32_t cnt = (n < N) ? (cu[n + 1] - cu[n] + C - 1) / C : 0;
    int32_t incl = cnt;  // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if ((tid & 31) >= o) incl += v;
    }
    if ((tid & 31) == 31) warp_tot[tid >> 5] = incl;
    __syncthreads();
    if (tid < 32) {
      int32_t w = warp_tot[tid];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, w, o);
        if (tid >= o) w += v;
      }
      warp_tot[tid] = w;  // inclusive over warps
    }
    __syncthreads();
    const int32_t excl = carry + incl - cnt + ((tid >> 5) ? warp_tot[(tid >> 5) - 1] : 0);
    if (n < N) {
      chunk_off[n] = excl;
      const int32_t start = cu[n], len = cu[n + 1] - cu[n];
      for (int32_t k = 0; k < cnt; ++k)
        chunk_map[excl + k] = make_int4(n, start + k * C, min(C, len - k * C), k);
    }
    __syncthreads();
    if (tid == kSchedThreads - 1) carry = excl + cnt;
    __syncthreads();
  }
  if (tid == 0) chunk_off[N] = carry;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

ScheduleLayout schedule_layout(int32_t num_seqs, int64_t total_chunks) {
  ScheduleLayout L;
  L.order_off = 0;
  L.chunk_off_off = align256((size_t)num_seqs * 4);
  L.chunk_map_off = L.chunk_off_off + align256((size_t)(num_seqs + 1) * 4);
  L.total_bytes = L.chunk_map_off + align256((size_t)total_chunks * 16);
  return L;
}

cudaError_t launch_schedule(const int32_t* cu, int32_t num_seqs, int32_t chunk_size, int64_t total_chunks,
                            void* workspace, cudaStream_t stream) {
  const ScheduleLayout L = schedule_layout(num_seqs, total_chunks);
  char* ws = (char*)workspace;
  LaunchScope scope(GDN_K_SCHEDULE, stream);
  schedule_kernel<<<1, kSchedThreads, 0, stream>>>(cu, num_seqs, chunk_size, (int32_t*)(ws + L.order_off),
                                                   (int32_t*)(ws + L.chunk_off_off), (int4*)(ws + L.chunk_map_off));
  return cudaGetLastError();
}

}  // namespace gdn
