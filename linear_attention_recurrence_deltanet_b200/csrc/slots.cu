// Slot-indexed state pools for continuous batching: row n of a prefill batch
// reads and writes slot state_indices[n] of the recurrent-state pool
// [num_slots, Hv, d_v, d_k] and of the conv-history pool [num_slots, W-1,
// C_conv] ("recurrent-state cache ownership", DS4Server issue #88, Scope; the
// serving gap on batching, Core AI model card, Limitations).
//
// The prefill kernels address their state and history by batch row, so an
// indexed prefill copies the batch's slots into contiguous buffers, runs the
// prefill on them and copies them back: one extra read and write of each
// sequence's state (3.1 MB at 48 value heads x 128 x 128), small next to the
// prefill's own traffic.  Decode indexes its slots in place (decode.cu).
#include <cuda_runtime.h>

#include "../../include/gdn.h"
#include "internal.h"

namespace gdn {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyVec = 4;  // 16-byte pieces per thread

// to_buffer: buffer row n <- pool slot (zeros for a padding row); else pool slot <- buffer row n (padding rows and
// out-of-pool slots are skipped).  blockIdx.y = row; the x blocks cover the row's 16-byte pieces.
__global__ void __launch_bounds__(kCopyThreads)
    slot_copy_kernel(Slots slots, int to_buffer, int64_t state_vecs, int64_t conv_vecs, uint4* __restrict__ pool_state,
                     uint4* __restrict__ pool_conv, uint4* __restrict__ buf_state, uint4* __restrict__ buf_conv,
                     int32_t* status) {
  const int n = blockIdx.y;
  const int sl = slot_of(slots, n, status);
  const int64_t row = state_vecs + conv_vecs;
  for (int64_t i0 = ((int64_t)blockIdx.x * kCopyThreads + threadIdx.x) * kCopyVec; i0 < row;
       i0 += (int64_t)gridDim.x * kCopyThreads * kCopyVec) {
#pragma unroll
    for (int v = 0; v < kCopyVec; ++v) {
      const int64_t i = i0 + v;
      if (i >= row) break;
      const bool st = i < state_vecs;
      const int64_t j = st ? i : i - state_vecs;
      uint4* pool = st ? pool_state + (int64_t)sl * state_vecs + j : pool_conv + (int64_t)sl * conv_vecs + j;
      uint4* buf = st ? buf_state + (int64_t)n * state_vecs + j : buf_conv + (int64_t)n * conv_vecs + j;
      if (to_buffer)
        *buf = sl >= 0 ? *pool : make_uint4(0u, 0u, 0u, 0u);
      else if (sl >= 0)
        *pool = *buf;
    }
  }
}

}  // namespace

cudaError_t launch_slot_copy(const Dims& d, bool bf16, Slots slots, int32_t num_seqs, bool to_buffer,
                             float* pool_state, void* pool_conv, float* buf_state, void* buf_conv, int32_t* status,
                             cudaStream_t stream) {
  if (num_seqs <= 0) return cudaSuccess;
  const int64_t state_vecs = (int64_t)d.Hv * d.dv * d.dk * 4 / 16;
  const int64_t conv_vecs = (int64_t)(d.W - 1) * d.C * (bf16 ? 2 : 4) / 16;
  const int64_t per_block = (int64_t)kCopyThreads * kCopyVec;
  const int64_t bx = (state_vecs + conv_vecs + per_block - 1) / per_block;
  LaunchScope scope(GDN_K_SLOT_COPY, stream);
  slot_copy_kernel<<<dim3((unsigned)(bx < 1024 ? bx : 1024), (unsigned)num_seqs), kCopyThreads, 0, stream>>>(
      slots, to_buffer ? 1 : 0, state_vecs, conv_vecs, (uint4*)pool_state, (uint4*)pool_conv, (uint4*)buf_state,
      (uint4*)buf_conv, status);
  return cudaGetLastError();
}

}  // namespace gdn
