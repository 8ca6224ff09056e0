// Host-side launchers of the GDN kernels.  Each returns cudaSuccess or the
// launch error; arguments are validated by the C-ABI layer (api.cu) first.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace gdn {

// Launch bracket used by every launcher: counts the launch and, when the
// profiler is on, records CUDA events around it on `stream`.
struct LaunchScope {
  LaunchScope(int kernel_id, cudaStream_t stream);
  ~LaunchScope();
  int id;
  cudaStream_t stream;
  void* token;
};

// conv.cu
cudaError_t launch_conv_prefill(const Dims& d, bool bf16, const void* x, const float* conv_w, const int32_t* cu,
                                int32_t num_seqs, int32_t max_len, const void* conv_state, void* y,
                                cudaStream_t stream);
cudaError_t launch_conv_history(const Dims& d, bool bf16, const void* x, const int32_t* cu, int32_t num_seqs,
                                bool zero_history, void* conv_state, cudaStream_t stream);
cudaError_t launch_conv_step(const Dims& d, bool bf16, const void* x, const float* conv_w, int32_t num_seqs,
                             void* conv_state, void* y, cudaStream_t stream);

// schedule.cu -- varlen schedule: longest-first sequence order and the chunk map.
struct ScheduleLayout {
  size_t order_off, chunk_off_off, chunk_map_off, total_bytes;
};
ScheduleLayout schedule_layout(int32_t num_seqs, int64_t total_chunks);
cudaError_t launch_schedule(const int32_t* cu, int32_t num_seqs, int32_t chunk_size, int64_t total_chunks,
                            void* workspace, cudaStream_t stream);

// decode.cu
cudaError_t launch_decode_step(const Dims& d, bool bf16, const float* conv_w, const float* A_log,
                               const float* dt_bias, const float* norm_w, const void* qkv, const void* z,
                               const void* a, const void* b, int32_t num_seqs, Slots slots, void* conv_state,
                               float* state, void* o, int32_t* status, cudaStream_t stream);

// multi-token decode (draft-and-verify), d = 128: verify (write_state 0) or commit
cudaError_t launch_decode_multi(const Dims& d, bool bf16, const float* conv_w, const float* A_log,
                                const float* dt_bias, const float* norm_w, const void* qkv, const void* z,
                                const void* a, const void* b, int32_t num_seqs, int32_t num_tokens,
                                const int32_t* accept, int write_state, Slots slots, void* conv_state, float* state,
                                void* o, int32_t* status, cudaStream_t stream);

// prefill_recurrent.cu
cudaError_t launch_prefill_recurrent(const Dims& d, bool bf16, const float* conv_w, const float* A_log,
                                     const float* dt_bias, const float* norm_w, const void* qkv, const void* z,
                                     const void* a, const void* b, const int32_t* cu, const int32_t* seq_order,
                                     int32_t num_seqs, bool zero_state, bool zero_conv, const void* conv_state,
                                     float* state, void* o, cudaStream_t stream);

// prefill_chunked.cu (tcgen05; bf16 io, d_k = d_v = 128, chunk 64)
bool prefill_chunked_supported(const Dims& d, bool bf16, int chunk_size);
cudaError_t launch_prefill_chunked(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                                   const float* norm_w, const void* qkv, const void* z, const void* a, const void* b,
                                   const int32_t* cu, const int32_t* order, int32_t N, int64_t total_tokens,
                                   bool zero_state, bool zero_conv, const void* conv_state, float* state, void* o,
                                   int32_t* status, cudaStream_t stream);

// cuTensorMapEncodeTiled, looked up once through the runtime (NULL if the driver lacks it)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// prefill_split.cu (tcgen05; bf16 io, d_k = d_v = 128, chunk 64): conv, per-chunk prep and
// state chain as three kernels over a workspace of intermediates (after the schedule)
struct SplitLayout {
  size_t qk_hi, qk_lo, records, total_bytes;
};
SplitLayout split_layout(const Dims& d, int64_t total_tokens, int64_t chunk_bound);
// the chunks go through conv, prep and chain in windows of at most this many chunks (65536 tokens), so the
// workspace holds the intermediates of one window: split_layout(d, min(T, window * 64), window)
constexpr int64_t kSplitWindowChunks = 1024;
int64_t split_window_chunks(int64_t total_chunks);
cudaError_t launch_prefill_split(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                                 const float* norm_w, const void* qkv, const void* z, const void* a, const void* b,
                                 const int32_t* cu, const int32_t* cu_host, const int32_t* order,
                                 const int32_t* chunk_off, const int4* chunk_map, int32_t N, int64_t total_tokens,
                                 int64_t total_chunks, bool zero_state, bool zero_conv, const void* conv_state,
                                 float* state, void* o, void* split_ws, int32_t* status, cudaStream_t stream);

// prefill_split.cu, sequence-parallel chain (one sequence, P chunk-aligned segments): segment count for a
// request (0 = from the SM count), workspace layout, launch
struct SeqparLayout {
  size_t cu1, cu_seg, coff, split, s1, s3, total_bytes;
};
int seqpar_segments(const Dims& d, int64_t total_tokens, int32_t requested, int32_t sms);
SeqparLayout seqpar_layout(const Dims& d, int64_t total_tokens, int32_t P);
cudaError_t launch_prefill_seqpar(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                                  const float* norm_w, const void* qkv, const void* z, const void* a, const void* b,
                                  int64_t total_tokens, int32_t P, bool zero_state, bool zero_conv,
                                  const void* conv_state, float* state, void* o, void* ws, int32_t* status,
                                  cudaStream_t stream);

// slots.cu: the batch's pool slots to contiguous buffers (to_buffer) or back
cudaError_t launch_slot_copy(const Dims& d, bool bf16, Slots slots, int32_t num_seqs, bool to_buffer,
                             float* pool_state, void* pool_conv, float* buf_state, void* buf_conv, int32_t* status,
                             cudaStream_t stream);

// gemm.cu: Y = X W^T in bf16 (fp32 accumulation), X [M, K] and W [N, K] row-major.
// Output column c goes to the output k with start[k] <= c < start[k + 1]:
// element (r, c) is ptr[k][r * ld[k] + c - start[k]].  start[0] = 0 and
// start[count] = N.  vec[k] says that ptr[k] is 16-byte aligned and ld[k],
// start[k] are multiples of 8, so whole 8-column groups may be stored at once.
constexpr int kGemmMaxOut = 4;
struct GemmOutputs {
  void* ptr[kGemmMaxOut];
  int64_t ld[kGemmMaxOut];
  int32_t start[kGemmMaxOut + 1];
  int32_t vec[kGemmMaxOut];
  int32_t count;
};
// kernel and tile width (a multiple of 32 up to 256 columns) a launch uses; tile_n 0 = chosen from M and N
struct GemmPlan {
  bool pair;   // CTA-pair kernel (256-row tiles) rather than one CTA per 128-row tile
  int tile_n;
};
GemmPlan gemm_plan(int32_t M, int32_t N, int32_t tile_n);
// up to 128 rows: tile width and K split of the cluster kernel (split 1 = not used); tile_n -1 = no split
struct SplitPlan {
  int tile_n;  // 0 when M > 128
  int split;
  int mp;      // rows of a partial tile kept for the reduction (M rounded up to 32)
};
SplitPlan gemm_split_plan(int32_t M, int32_t N, int32_t K, int32_t tile_n);
cudaError_t launch_gemm_bf16(const void* x, int32_t M, int32_t K, const void* w, int32_t N, int32_t tile_n,
                             const GemmOutputs& out, int32_t* status, cudaStream_t stream);

// api.cu: records a message for gdn_last_error() on the calling thread.
void set_error_message(const char* msg);
// api.cu: workspace bytes of gdn_prefill with GDN_PREFILL_FUSED (the schedule only)
size_t prefill_fused_ws_bytes(int64_t total_tokens, int32_t num_seqs, int32_t chunk_size);

// checksum.cu
cudaError_t launch_checksum(const void* payload, size_t bytes, unsigned long long* out, cudaStream_t stream);
uint64_t host_checksum(const void* payload, size_t bytes);

// prefill_wy.cu (tcgen05; bf16 io, d_k = d_v = 128, chunk 16/32/64): conv, per-tile operands of the
// affine chunk maps, and the state carry, over a workspace of intermediates (after the schedule, which
// is built for tiles of wy_tile(chunk) rows)
bool prefill_wy_supported(const Dims& d, bool bf16, int chunk_size);
int wy_tile(int chunk_size);
struct WyLayout {
  size_t qk_hi, qk_lo, vimg, gate, records, total_bytes;
};
WyLayout wy_layout(const Dims& d, int64_t total_tokens, int64_t tile_bound, int chunk_size);
// the tiles go through conv, prep and chain in windows of at most kWyWindowTokens / tile rows, so the
// workspace holds one window: wy_layout(d, min(T, window * tile), window, chunk)
constexpr int64_t kWyWindowTokens = 65536;
int64_t wy_window_tiles(int64_t total_tiles, int chunk_size);
cudaError_t launch_prefill_wy(const Dims& d, int chunk_size, const float* conv_w, const float* A_log,
                              const float* dt_bias, const float* norm_w, const void* qkv, const void* z,
                              const void* a, const void* b, const int32_t* cu, const int32_t* cu_host,
                              const int32_t* order,
                              const int32_t* tile_off, const int4* tile_map, int32_t N, int64_t total_tokens,
                              int64_t total_tiles, bool zero_state, bool zero_conv, const void* conv_state,
                              float* state, void* o, void* ws, int32_t* status, cudaStream_t stream);

// diag.cu: a kernel whose bounded wait always runs out (tests the status path)
cudaError_t launch_wait_expiry(uint64_t limit_ns, int32_t* status, cudaStream_t stream);

}  // namespace gdn
