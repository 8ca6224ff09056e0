/*
 * gdn.h -- C ABI of libgdn.so, the Gated DeltaNet (GDN) token mixer on
 * NVIDIA B200 (sm_100a).
 *
 * The mixer is the one the reference pages build for Qwen3.8's hybrid
 * 3-GDN + 1-attention layers: "causal depthwise Conv1D, Gated DeltaNet
 * recurrence, and recurrent-state cache", with "separately tuned GDN prefill
 * and single-step decode behind one semantic interface" (DS4Server issue
 * #88, "Add a performance-parity Qwen3.8-27B Q4 and Q8 text backend on
 * Metal", section Scope), in the "16-key/48-value-head GDN geometry,
 * convolution width 4, fp32 recurrent state, sigmoid output gate, and exact
 * L2-normalization epsilon placement" with "zero-centered norms" (DS4Server
 * issue #95, "Implement the Qwen3.8 Flash Next Rust and Metal text core",
 * section Implementation).
 *
 * Per token t and value head h (key head kh = h / (Hv/Hk)):
 *   u      = SiLU(causal depthwise conv, width W, over the raw q/k/v channels)
 *   q^     = q_scale * q / sqrt(sum q^2 + l2_eps),  k^ = k / sqrt(sum k^2 + l2_eps)
 *   g      = -exp(A_log[h]) * softplus(a + dt_bias[h]),  alpha = exp(g),  beta = sigmoid(b)
 *   S      = alpha*S + beta * k^ (v - alpha * S^T k^)^T      (S is d_k x d_v, fp32)
 *   o      = S^T q^
 *   out_j  = o_j / sqrt(mean(o^2) + norm_eps) * (1 + norm_w[j]) * sigmoid(z_j)
 *
 * Conventions shared by every entry point
 *   - Memory: every pointer is device memory owned by the caller unless a
 *     parameter says otherwise; the library never allocates device memory.
 *     Tensors are dense row-major and 16-byte aligned (a and b: aligned to
 *     their element size).
 *   - Streams: every call is asynchronous on the caller's stream and
 *     stream-ordered; nothing blocks the host except where stated.
 *   - Validation: every argument is checked on the host before anything is
 *     launched.  On any error no kernel runs and no buffer is written
 *     ("fail before unsafe or partial execution", issue #95 implementation
 *     comment); the message is available from gdn_last_error().
 *   - Layouts (N sequences, T_tot packed tokens, C_conv = 2*Hk*d_k + Hv*d_v):
 *       qkv        [T_tot, C_conv]   io dtype; channels q (Hk*d_k), k (Hk*d_k), v (Hv*d_v),
 *                                    each head's slice contiguous
 *       z          [T_tot, Hv*d_v]   io dtype
 *       a, b       [T_tot, Hv]       io dtype
 *       o          [T_tot, Hv*d_v]   io dtype (written)
 *       conv_state [N, W-1, C_conv]  io dtype; the last W-1 raw inputs, oldest first
 *       state      [N, Hv, d_v, d_k] fp32; element [n,h,j,i] = S[i][j] (S transposed)
 *       conv_w     [C_conv, W] fp32; tap W-1 multiplies the current token
 *       A_log, dt_bias [Hv] fp32;  norm_w [d_v] fp32 (applied as 1 + w)
 *   - Supported geometry: Hv % Hk == 0, d_k == d_v in {32, 64, 128}, W == 4,
 *     io dtype fp32 or bf16.  Anything else returns GDN_E_UNSUPPORTED.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_ABI_VERSION 1

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

typedef struct CUstream_st* gdn_stream_t; /* a cudaStream_t; NULL = the legacy default stream */

typedef enum {
  GDN_OK = 0,
  GDN_E_INVAL = -1,          /* bad pointer, size, alignment or cu_seqlens */
  GDN_E_UNSUPPORTED = -2,    /* geometry or dtype the library does not run */
  GDN_E_WORKSPACE = -3,      /* workspace missing or smaller than gdn_prefill_workspace_size() */
  GDN_E_CUDA = -4,           /* a CUDA runtime call failed; see gdn_last_error() */
  GDN_E_BLOB_FORMAT = -5,    /* state blob: bad magic, size or layout id */
  GDN_E_BLOB_VERSION = -6,   /* state blob: unknown format version */
  GDN_E_BLOB_GEOMETRY = -7,  /* state blob: saved under another geometry or dtype */
  GDN_E_BLOB_CHECKSUM = -8,  /* state blob: payload does not match its checksum */
  GDN_E_DEVICE = -9          /* no usable CUDA device, or not an sm_100 device */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

typedef struct {
  int32_t num_k_heads; /* Hk */
  int32_t num_v_heads; /* Hv; value heads G*kh .. G*kh+G-1 (G = Hv/Hk) share key head kh */
  int32_t head_k_dim;  /* d_k */
  int32_t head_v_dim;  /* d_v */
  int32_t conv_width;  /* W */
  float l2_eps;        /* inside the square root of the L2 norm's sum of squares */
  float norm_eps;      /* inside the square root of the output RMSNorm's mean square */
  float q_scale;       /* factor on the normalised query (1.0 for the plain rule) */
  int32_t io_dtype;    /* gdn_dtype of qkv, z, a, b, o and conv_state */
} gdn_config;

typedef struct {
  const float* conv_w;  /* [C_conv, W] */
  const float* A_log;   /* [Hv] */
  const float* dt_bias; /* [Hv] */
  const float* norm_w;  /* [d_v] */
} gdn_params;

/* flags of gdn_prefill */
#define GDN_ZERO_INIT_STATE 0x1u /* ignore the incoming recurrent state: start from S = 0 */
#define GDN_ZERO_INIT_CONV 0x2u  /* ignore the incoming conv history: treat it as zeros */
#define GDN_PREFILL_RECURRENT 0x4u /* run the token-recurrent fp32 kernel instead of the chunked one */
#define GDN_PREFILL_FUSED 0x8u     /* chunked path as one kernel per (sequence, value head): needs only the
                                      schedule as workspace (see gdn_prefill) */
#define GDN_PREFILL_FACTORED 0x10u /* chunk 64: the three-kernel chunked path in the factored form (W S,
                                      then K~^T Delta per chunk); the default at chunk 64 */
#define GDN_PREFILL_AFFINE 0x20u   /* bf16, d = 128: the three-kernel chunked path in the affine form (one
                                      M' S product per chunk on the carry); the default at 16, 32, 128 */

/* --------------------------------------------------------------------------
 * Causal depthwise Conv1D + SiLU over the q/k/v channels (issue #88, Scope:
 * "causal depthwise Conv1D"; width 4 per issue #95, Implementation).
 *
 * gdn_conv_prefill: y[t, c] = SiLU(sum_j conv_w[c, j] * x~[t - (W-1) + j, c])
 * where x~ is the sequence's inputs preceded by its conv_state.  cu_seqlens
 * [N+1] int32 gives the packed sequence boundaries (cu[0] = 0, non-decreasing,
 * cu[N] = T_tot); the device and host copies must hold the same values (the
 * host copy is validated and sizes the launch).  conv_state is read, then
 * replaced by the last W-1 raw inputs of each sequence (bit-exact copies).
 * y [T_tot, C_conv] in the io dtype.  Length-0 sequences are allowed.
 */
GDN_API gdn_status gdn_conv_prefill(const gdn_config* cfg, const void* x, const float* conv_w,
                            const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host, int32_t num_seqs,
                            void* conv_state, void* y, gdn_stream_t stream);

/* gdn_conv_step: the same for one token per sequence.  x and y are [N, C_conv]. */
GDN_API gdn_status gdn_conv_step(const gdn_config* cfg, const void* x, const float* conv_w, int32_t num_seqs,
                         void* conv_state, void* y, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * Chunked prefill over packed variable-length sequences ("separately tuned
 * GDN prefill", issue #88, Scope; "prefill/decode equivalence across chunk
 * sizes", issue #95, Verification).
 *
 * Workspace: caller-provided device scratch of at least the size that
 * gdn_prefill_workspace_size() returns for the same (cfg, total_tokens,
 * num_seqs, chunk_size); 256-byte aligned.  The size covers every path a flag
 * can select.  For the tensor-core paths (bf16, d_k = d_v = 128) it holds the
 * schedule (about 16 bytes per chunk) plus the chunked form's intermediates
 * for one window of at most 65536 tokens: the three kernels run window by
 * window, carrying each sequence's state between windows, so beyond the
 * schedule the size does not grow with total_tokens (at 16 key / 48 value
 * heads at most about 8.7 GB at chunk 64 and 14.4 GB at chunk 16, less for
 * shorter inputs).  With GDN_PREFILL_FUSED the schedule alone suffices.
 */
GDN_API gdn_status gdn_prefill_workspace_size(const gdn_config* cfg, int64_t total_tokens, int32_t num_seqs,
                                      int32_t chunk_size, size_t* bytes);

/* gdn_prefill: runs the whole mixer over every token of every sequence.
 *   chunk_size: 16, 32, 64 or 128 (tokens per chunk of the chunkwise form;
 *               chunks restart at each sequence start).
 *   flags:      GDN_ZERO_INIT_STATE / GDN_ZERO_INIT_CONV, and at most one of
 *               GDN_PREFILL_RECURRENT / GDN_PREFILL_FUSED / GDN_PREFILL_FACTORED /
 *               GDN_PREFILL_AFFINE (GDN_E_INVAL if more than one).
 *   conv_state and state are read and updated in place; o is written.
 * When io dtype is bf16 and d_k = d_v = 128 the chunked form runs on tensor
 * cores as three kernels (conv of every token; the state-independent operands
 * of every chunk; the state carry across chunks): at chunk 16, 32 and 128 in
 * the affine form (GDN_PREFILL_AFFINE), at chunk 64 by default in the
 * factored form (GDN_PREFILL_FACTORED), the affine form with
 * GDN_PREFILL_AFFINE, or one kernel per (sequence, value head) with
 * GDN_PREFILL_FUSED.  Paths and chunk sizes agree to fp32 rounding (not bit for
 * bit).  Every other supported case (and GDN_PREFILL_RECURRENT) runs the
 * token-recurrent fp32 kernel.  All compute in fp32 with an fp32 state. */
GDN_API gdn_status gdn_prefill(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                       const void* a, const void* b, const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                       int32_t num_seqs, int32_t chunk_size, uint32_t flags, void* conv_state, float* state,
                       void* o, void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/* gdn_prefill_noalloc: gdn_prefill for callers that cannot provide scratch
 * device memory -- for example a host runtime whose device memory is owned by
 * another allocator (a framework's caching allocator, a serving engine's
 * pre-reserved pool) with no way to borrow from it, or latency-critical code
 * that must not call cudaMalloc/cudaFree because they can synchronise the
 * device.  The reference pages have no counterpart to this entry point.
 *
 * Same arguments and results as gdn_prefill, minus the workspace: the scratch
 * is a fixed array of GDN_NOALLOC_SCRATCH_BYTES inside the library's device
 * memory, present on every GPU that loads the library until the process
 * exits.  The call allocates nothing.  It always runs gdn_prefill with
 * GDN_PREFILL_FUSED added to flags: the single-kernel chunked path where it
 * applies (bf16, d = 128, chunk 64), else the token-recurrent kernel; both
 * need only the varlen schedule as scratch, about 16 bytes per chunk plus 8
 * per sequence.  flags holding GDN_PREFILL_RECURRENT, GDN_PREFILL_FACTORED or
 * GDN_PREFILL_AFFINE are rejected with GDN_E_INVAL.  The limit is therefore the workspace gdn_prefill needs with
 * GDN_PREFILL_FUSED (not gdn_prefill_workspace_size, which reports the
 * default path's larger need): a problem whose schedule exceeds
 * GDN_NOALLOC_SCRATCH_BYTES, i.e. more than about 250,000 chunks plus
 * sequences, is rejected with GDN_E_WORKSPACE before anything runs.  The
 * schedule is sized for the chunk bound total_tokens / chunk_size + num_seqs
 * + 1 even for a single sequence, which launches no schedule, so one
 * sequence of more than about 16M tokens at chunk 64 (4M at chunk 16) is
 * rejected too.  The first call on a device looks up the array's device
 * address (with that device current) and caches it for the process; make
 * that first call before any stream capture.  The cached address does not
 * survive cudaDeviceReset: do not call this entry point on a device after
 * resetting it in the same process.
 * Every call on a device shares the one array, which keeps whatever the last
 * call left in it (nothing in it needs to start at zero: every kernel writes
 * the scratch it later reads), so calls whose executions overlap on the GPU --
 * for example on two streams -- race with each other and must be ordered by
 * the caller. */
#define GDN_NOALLOC_SCRATCH_BYTES (4u << 20)
GDN_API gdn_status gdn_prefill_noalloc(const gdn_config* cfg, const gdn_params* params, const void* qkv,
                                       const void* z, const void* a, const void* b, const int32_t* cu_seqlens_dev,
                                       const int32_t* cu_seqlens_host, int32_t num_seqs, int32_t chunk_size,
                                       uint32_t flags, void* conv_state, float* state, void* o,
                                       gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * Single-step decode ("single-step decode", issue #88, Scope): every one of
 * num_seqs sequences advances by one token.  qkv [N, C_conv], z [N, Hv*d_v],
 * a, b [N, Hv], o [N, Hv*d_v].  One fused kernel: conv step, L2 norms, gates,
 * rank-1 state update, readout, RMSNorm and output gate; each state is read
 * and written once.  conv_state and state are updated in place. */
GDN_API gdn_status gdn_decode_step(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                           const void* a, const void* b, int32_t num_seqs, void* conv_state, float* state, void* o,
                           gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * Multi-token decode for draft-and-verify rounds ("MTP candidate generation,
 * verification, cache updates, rollback, accepted tokens", issue #89,
 * Correctness gates; the K=2 draft-and-verify round of the Qwen3.8-27B FP8
 * Core AI model card, What is fused).  Each of num_seqs sequences takes
 * num_tokens (K, 1..GDN_MAX_DRAFT_TOKENS) consecutive tokens in one pass over
 * its state: qkv [N, K, C_conv], z [N, K, Hv*d_v], a, b [N, K, Hv],
 * o [N, K, Hv*d_v], token-major inside a sequence.  Token t is computed
 * exactly as the t-th of K gdn_decode_step calls would compute it -- the same
 * operations in the same order, so the results agree bit for bit.
 *
 *   commit == 0 (verify): o receives all K tokens' outputs; conv_state and
 *     state are read but not written, so a rejected draft needs no rollback.
 *     accept must be NULL.
 *   commit != 0: sequence n applies its first accept[n] tokens (accept is a
 *     device array of num_seqs counts, clamped to [0, K]; NULL means K) to
 *     conv_state and state, and writes o for those tokens only.  Committing
 *     a tokens equals a gdn_decode_step calls with those tokens.
 *
 * A verify followed by a commit of the accepted prefix reads each state twice
 * and writes it once; that is the rollback-free form of the round.  Only
 * d_k = d_v = 128 runs here; other geometries return GDN_E_UNSUPPORTED. */
#define GDN_MAX_DRAFT_TOKENS 4
GDN_API gdn_status gdn_decode_multi(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                                    const void* a, const void* b, int32_t num_seqs, int32_t num_tokens,
                                    int32_t commit, const int32_t* accept_dev, void* conv_state, float* state,
                                    void* o, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * Slot-indexed state pools for continuous batching ("recurrent-state cache
 * ownership", issue #88, Scope; batching listed as a gap, Core AI model card,
 * Limitations).  conv_state and state are pools of num_slots entries,
 * [num_slots, W-1, C_conv] (io dtype) and [num_slots, Hv, d_v, d_k] (fp32);
 * row n of the batch reads and writes entry state_indices[n], a device array
 * of num_seqs int32 (4-byte aligned).  Inputs and outputs stay indexed by
 * batch row.  Non-negative indices must be distinct.
 *   - A negative index marks a padding row: decode writes zeros to its o rows
 *     and touches nothing else; prefill runs it from a zero state and zero
 *     history and discards its final state and history (its o rows are
 *     written).
 *   - An index >= num_slots is an error found on the device: the row is
 *     treated as padding and gdn_get_device_status reports 3.
 * Host-side checks as for the unindexed calls, plus num_slots in
 * [1, 65535] and state_indices non-NULL.
 *
 * gdn_decode_step_indexed, gdn_decode_multi_indexed: the decode kernels read
 * and write the slots in place; results are bit-identical to the unindexed
 * calls on a pool whose first num_seqs entries are the batch's slots.
 *
 * gdn_prefill_indexed: copies the batch's slots into buffers in the
 * workspace, runs gdn_prefill on them (same flags, same path, bit-identical
 * results) and copies them back.  A batch that mixes prefill sequences with
 * decode steps (length-1 sequences) runs in one call.  Workspace:
 * gdn_prefill_indexed_workspace_size() bytes (gdn_prefill's plus the two
 * buffers, about 3.2 MB per sequence at 16 key / 48 value heads x 128). */
GDN_API gdn_status gdn_decode_step_indexed(const gdn_config* cfg, const gdn_params* params, const void* qkv,
                                           const void* z, const void* a, const void* b, int32_t num_seqs,
                                           const int32_t* state_indices, int32_t num_slots, void* conv_state,
                                           float* state, void* o, gdn_stream_t stream);
GDN_API gdn_status gdn_decode_multi_indexed(const gdn_config* cfg, const gdn_params* params, const void* qkv,
                                            const void* z, const void* a, const void* b, int32_t num_seqs,
                                            int32_t num_tokens, int32_t commit, const int32_t* accept_dev,
                                            const int32_t* state_indices, int32_t num_slots, void* conv_state,
                                            float* state, void* o, gdn_stream_t stream);
GDN_API gdn_status gdn_prefill_indexed_workspace_size(const gdn_config* cfg, int64_t total_tokens,
                                                      int32_t num_seqs, int32_t chunk_size, size_t* bytes);
GDN_API gdn_status gdn_prefill_indexed(const gdn_config* cfg, const gdn_params* params, const void* qkv,
                                       const void* z, const void* a, const void* b, const int32_t* cu_seqlens_dev,
                                       const int32_t* cu_seqlens_host, int32_t num_seqs,
                                       const int32_t* state_indices, int32_t num_slots, int32_t chunk_size,
                                       uint32_t flags, void* conv_state, float* state, void* o, void* workspace,
                                       size_t workspace_bytes, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * Sequence-parallel prefill of ONE long sequence (the long contexts, up to
 * 262K tokens, that issue #89 measures under Measurements and gates; the
 * state carry is the only step of the mixer that runs along the sequence).  The total_tokens tokens are cut into P chunk-aligned
 * segments.  Over one segment the state carry is affine in the state it
 * starts from, S -> A S + B: A depends only on keys and gates, B is linear
 * in the values.  So one chain pass computes every segment's A and B at
 * once, a short pass over the P segments composes them into each segment's
 * starting state, and a second chain pass writes the outputs.  Results match
 * gdn_prefill of the same sequence within floating-point rounding (the
 * composition reassociates the state products); same layouts, conv-history
 * update and flags (GDN_ZERO_INIT_STATE, GDN_ZERO_INIT_CONV) as gdn_prefill
 * with num_seqs = 1 and chunk 64.  bf16 io, d_k = d_v = 128 only.
 *
 * It pays when the GPU would otherwise sit idle during the carry: few value
 * heads on the GPU (as when heads are sharded across GPUs).  The carry of
 * gdn_prefill occupies 2 SMs per value head for the whole sequence; this
 * path runs 4 P per value head over segments P times shorter, at about three
 * times the carry's arithmetic (two output-free passes, then one with outputs).
 * segments: P, or 0 = as many as fill the SMs (SMs / (4 Hv)); the count used
 * (at most the number of 64-token chunks, every segment non-empty) is
 * written to *segments_used when that pointer is non-NULL.  With one segment
 * (e.g. 0 at 48 value heads on 148 SMs) it runs gdn_prefill's carry as is.
 * Workspace: gdn_prefill_seqpar_workspace_size() bytes for the same
 * (cfg, total_tokens, segments), 256-byte aligned: the chunked form's
 * intermediates plus 3 P fp32 states per value head. */
GDN_API gdn_status gdn_prefill_seqpar_workspace_size(const gdn_config* cfg, int64_t total_tokens,
                                                     int32_t segments, size_t* bytes);
GDN_API gdn_status gdn_prefill_seqpar(const gdn_config* cfg, const gdn_params* params, const void* qkv,
                                      const void* z, const void* a, const void* b, int64_t total_tokens,
                                      int32_t segments, uint32_t flags, void* conv_state, float* state, void* o,
                                      void* workspace, size_t workspace_bytes, int32_t* segments_used,
                                      gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * Dense projections either side of the mixer (the "GDN projection" primitive
 * of issue #95, Verification; its "BF16 projection kernels", implementation
 * comment).  All three are one bf16 GEMM on the tensor cores with fp32
 * accumulation and round-to-nearest bf16 output:
 *   Y[r, c] = sum_k X[r, k] * W[c, k]
 * X [M, K] and W [N, K] are row-major bf16 device arrays (W is a linear
 * layer's weight: output features x input features).  K must be a multiple
 * of 8 (16-byte row pitch) and X, W 16-byte aligned; M, N >= 0 (0 launches
 * nothing); M, N, K < 2^31.  No workspace.  tile_n picks the output tile
 * width: a multiple of 32 up to 256 columns, or 0 = chosen from M and N (a
 * power of two: the width that fills the SMs in the fewest, widest rounds).
 *
 * gdn_gemm_bf16: Y [M, N] row-major bf16 (2-byte aligned; rows 16-byte
 *   aligned give vector stores).
 * gdn_project_in: the input projection of one GDN layer.  W_in stacks the
 *   rows of the four outputs, [C_conv + Hv*d_v + 2*Hv, hidden]:
 *     rows [0, C_conv)               -> qkv [T, C_conv] (q, k, v channels)
 *     rows [C_conv, +Hv*d_v)          -> z   [T, Hv*d_v]
 *     next Hv rows                    -> a   [T, Hv]
 *     last Hv rows                    -> b   [T, Hv]
 *   with C_conv = 2*Hk*d_k + Hv*d_v; every output row-major, bf16.  The
 *   outputs are exactly what gdn_prefill / gdn_decode_step take as qkv, z, a,
 *   b, so a layer is project_in -> prefill or decode -> project_out.
 *   cfg->io_dtype must be GDN_BF16.
 * gdn_project_out: y [T, hidden] = o [T, Hv*d_v] W_out^T, W_out
 *   [hidden, Hv*d_v].
 * A bounded internal wait that runs out sets device status 1 (see
 * gdn_get_device_status). */
GDN_API gdn_status gdn_gemm_bf16(const void* x, int32_t M, int32_t K, const void* w, int32_t N, void* y,
                                 int32_t tile_n, gdn_stream_t stream);
GDN_API gdn_status gdn_project_in(const gdn_config* cfg, const void* x, int32_t num_tokens, int32_t hidden,
                                  const void* w_in, void* qkv, void* z, void* a, void* b, gdn_stream_t stream);
GDN_API gdn_status gdn_project_out(const gdn_config* cfg, const void* o, int32_t num_tokens, const void* w_out,
                                   int32_t hidden, void* y, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * Versioned state checkpoint of one sequence ("Persist every GDN convolution
 * and recurrent component in session checkpoints with versioned validation",
 * issue #95, Implementation; "identical ... BF16 convolution bytes, and fp32
 * recurrent bytes after checkpoint/resume", implementation comment).
 *
 * Blob = 128-byte header {magic "GDNSTATE", format version, geometry, io
 * dtype, state dtype, layout id, payload bytes, 64-bit checksum} followed by
 * the sequence's conv history bytes ([W-1, C_conv], io dtype) and recurrent
 * state bytes ([Hv, d_v, d_k], fp32), copied unchanged.
 *
 * blob may be host or device memory (detected).  With a host blob the call
 * synchronises the stream before returning (save) or before validating
 * (restore); with a device blob it synchronises once to read the header and
 * checksum.  Restore checks every header field and the checksum before it
 * writes anything; on a mismatch it returns the matching GDN_E_BLOB_* code and
 * leaves conv_state and state untouched.
 */
GDN_API gdn_status gdn_state_blob_size(const gdn_config* cfg, size_t* bytes);
GDN_API gdn_status gdn_state_save(const gdn_config* cfg, const void* conv_state, const float* state, int32_t seq,
                          void* blob, size_t blob_bytes, gdn_stream_t stream);
GDN_API gdn_status gdn_state_restore(const gdn_config* cfg, const void* blob, size_t blob_bytes, int32_t seq,
                             void* conv_state, float* state, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * Diagnostics and measurement.
 *
 * gdn_get_device_status: reads and clears the device status word, which a
 * kernel sets (never traps) when an internal wait reaches its time limit, or
 * a state slot index lies past its pool.  0 = clean.  The low byte is the
 * code (1 wait timeout, 3 slot past the pool); the bits above it, when set,
 * are the gdn_kernel_id of the kernel that reported it.  The first report
 * since the last read is kept.  Synchronises the stream.
 * gdn_last_error: message of the calling thread's last failed call.
 * gdn_launch_count: kernels this library has launched since load or reset.
 * gdn_profiler_*: when enabled, every launch is bracketed by CUDA events on
 * its own stream; gdn_profiler_read synchronises those events and returns the
 * launch count and summed device time of one kernel id (see gdn_kernel_name).
 */
GDN_API gdn_status gdn_get_device_status(int32_t* code, gdn_stream_t stream);

/* gdn_debug_wait_expiry: exercises the bounded-wait failure path on the
 * device.  Launches one small kernel that waits, with the same bounded
 * mbarrier wait the mixer kernels use, on an mbarrier that nothing arrives on
 * and that no copy targets; after limit_us microseconds (1 .. 1,000,000) the
 * wait gives up, the kernel records status 1 (wait timeout) in the device
 * status word and returns.  No trap, no hang: the context stays usable and
 * the next launch runs normally.  Asynchronous on `stream`; read the result
 * with gdn_get_device_status.  GDN_E_INVAL for a limit outside the range.
 * The pages' counterpart is the requirement to fail explicitly instead of
 * running unsafely (DS4Server issue #95, implementation comment). */
GDN_API gdn_status gdn_debug_wait_expiry(uint32_t limit_us, gdn_stream_t stream);
GDN_API const char* gdn_last_error(void);
GDN_API int32_t gdn_abi_version(void);
GDN_API int64_t gdn_launch_count(void);
GDN_API void gdn_launch_count_reset(void);

typedef enum {
  GDN_K_CONV_PREFILL = 0,
  GDN_K_CONV_STEP = 1,
  GDN_K_CONV_HISTORY = 2,
  GDN_K_SCHEDULE = 3,
  GDN_K_PREFILL_RECURRENT = 4,
  GDN_K_PREFILL_CHUNKED = 5,
  GDN_K_DECODE = 6,
  GDN_K_STATE_CHECKSUM = 7,
  GDN_K_SPLIT_CONV = 8,   /* chunked prefill, stage 1: conv + SiLU + L2 norm of every token */
  GDN_K_SPLIT_PREP = 9,   /* stage 2: per-(chunk, value head) operands of the state carry */
  GDN_K_SPLIT_CHAIN = 10, /* stage 3: the state carry across chunks and the output rows */
  GDN_K_SLOT_COPY = 11,   /* slot-indexed prefill: pool slots to and from the batch's buffers */
  GDN_K_GEMM = 12,        /* bf16 projection GEMM (gdn_gemm_bf16, gdn_project_in, gdn_project_out) */
  GDN_K_SEQPAR = 13,      /* sequence-parallel prefill: segment set-up and the combine across segments */
  GDN_K_DIAG = 14,        /* gdn_debug_wait_expiry */
  GDN_K_WY_CONV = 15,     /* chunked prefill (affine chunk maps), stage 1: conv + SiLU + L2 norm of every token */
  GDN_K_WY_PREP = 16,     /* stage 2: per-(tile, value head) operands: T by tensor-core doubling, M', Q', U, P, K~ */
  GDN_K_WY_CHAIN = 17,    /* stage 3: the state carry (one M' S product per chunk) and the output rows */
  GDN_K_COUNT = 18
} gdn_kernel_id;

GDN_API const char* gdn_kernel_name(int32_t kernel_id);
GDN_API gdn_status gdn_profiler_enable(int32_t enable);
GDN_API gdn_status gdn_profiler_reset(void);
GDN_API gdn_status gdn_profiler_read(int32_t kernel_id, int64_t* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
