// Chunked GDN prefill as three kernels (bf16 io, d_k = d_v = 128, chunk 64):
// the work that does not depend on the recurrent state runs over every chunk
// at once, and only the state carry walks the chunks in order.
//
// The chunkwise (WY/UT) form of the gated delta rule ("fp32 Gated DeltaNet
// recurrence", DS4Server issue #95, implementation comment).  Within a chunk
// of rows r with gamma_r = sum_{i<=r} g_i:
//   A_rj = beta_r e^{gamma_r - gamma_j} k_r.k_j (j < r),   T = (I + A)^-1
//   W = T diag(beta e^gamma) K,   U = T diag(beta) V
//   Delta = U - W S,   O = diag(e^gamma) Q S + (M o Q K^T) Delta
//   S <- e^{gamma_C} S + K~^T Delta,   K~ = diag(e^{gamma_C - gamma}) K.
//
//   conv_qkv_kernel   grid (chunk, head slot): causal conv + SiLU of q/k/v
//                     ("causal depthwise Conv1D", DS4Server issue #88, Scope),
//                     L2 norm of q and k with epsilon inside the square root;
//                     q^, k^ and v^ as fp16 hi + lo parts; and the output gate
//                     (1 + w) sigmoid(z) of every value head, fp16.
//   prep_kernel       grid (chunk, value head): gates, [K;Q]K^T in split
//                     precision on tcgen05, A and P, T = (I+A)^-1 by recursive
//                     doubling whose merges are tcgen05 MMAs, then W = T''K
//                     and U = T'v^ on tcgen05; writes one record per (chunk,
//                     value head) whose parts are byte images of the chain
//                     kernel's shared-memory operands.
//   chain_kernel      grid (sequence, value head, value-channel half), clusters
//                     of the two halves: per chunk, [-W;Qg] S on tcgen05 (S as
//                     fp16 hi + lo; Delta takes the hi products alone), Delta =
//                     U - W S, then K~^T Delta and [0;P] Delta, then the state
//                     update, each CTA for 64 of the 128 value channels (the
//                     columns of the state are independent); the output rows of
//                     chunk c (RMSNorm times the gate, the row sums of squares
//                     exchanged through distributed shared memory) are written
//                     by half of the warps while the other half carries chunk
//                     c+1 to its second MMA group.
//
// The three kernels run over windows of at most kSplitWindowChunks chunks, the
// chain carrying each sequence's state from window to window, so that the
// intermediates take a bounded workspace.
//
// Record of (chunk, value head), byte images of 128-byte-swizzled operands:
//   [     0,  32768) [-W ; Qg]  K-major 128 x 128   (Qg = diag(e^gamma) q^)
//   [ 32768,  65536) U = T' v^, fp32: channel half at 16384 half, row r at +256 r,
//                   16-byte piece j of the half row at (j ^ (r % 8)) * 16
//   [ 65536,  81920) v^ (from the conv)   MN-major K=64 x N=128, rows past the chunk zero
//   [ 81920,  90112) P                    K-major 64 x 64  (rows 64..127 of [0;P])
//   [ 90112, 106496) K~                   MN-major K=64 x M=128
//   [106496, 122880) output gate (1 + w) sigmoid(z) (from the conv), fp16: column half
//                   at 8192 half, row r at +128 r, 16-byte piece q at (q ^ (r % 8)) * 16
//   [122880, 122896) e^{gamma_C}, gamma_C (from the conv)
//   [122896, 123408) gamma_r, beta_r of the chunk's 64 rows (from the conv; 0 past the chunk's end)
//   [123520, 139904) v^ lo = v^ - fp16(v^) (from the conv), laid out as v^
// Operands are fp16 (all bounded: normalised keys and queries, decay factors
// <= 1), accumulation fp32, the state fp32.  U = T' v^ takes T' and v^ as hi +
// lo (T'hi v^hi + T'lo v^hi + T'hi v^lo) and is stored in fp32: the roundings
// of T' and of v^ feed Delta directly, and over thousands of tokens they would
// take the state past its tolerance.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/gdn.h"
#include "internal.h"
#include "tc.cuh"

namespace gdn {
namespace {

using namespace tc;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr uint64_t kWaitNs = 2000000000ull;

constexpr int kRec = 139904;  // a multiple of 128 bytes
constexpr int REC_A = 0, REC_U = 32768, REC_V = 65536, REC_P = 81920, REC_K = 90112, REC_G = 106496,
              REC_META = 122880, REC_GAM = 122896, REC_BETA = 123152, REC_VL = 123520;

// ------------------------------------------------------------------ conv_qkv_kernel
// Block = 8 warps = the 64 rows of one chunk for one 128-channel head slot
// (q heads, then k heads, then v heads, then the output gates of the v
// heads).  Warp w owns rows 8w .. 8w+7, lane l owns channels 4l .. 4l+3.
// A ninth warp computes the chunk's gates g, beta of the value head in the
// output-gate slots and exits in the others.
constexpr int kConvRows = 8;
constexpr int kConvGateWarp = 64 / kConvRows;

// Slots past the q/k/v heads compute the output gate of one value head,
// (1 + w_j) sigmoid(z_j), which depends on no other stage of the mixer.
__device__ __forceinline__ void gate_rows(const Dims& d, const float* __restrict__ norm_w,
                                          const __nv_bfloat16* __restrict__ z, unsigned char* __restrict__ grec,
                                          int64_t t0, int r0, int L, int hz, int lane) {
  const int64_t WV = (int64_t)d.Hv * kD;
  const int hcol = lane >> 4, q = (lane >> 1) & 7;  // channels 4 lane .. 4 lane + 3: column half, 16-byte piece
  const int64_t col = (int64_t)hz * kD + 4 * lane;
  const float4 w = __ldg(reinterpret_cast<const float4*>(norm_w + 4 * lane));
  const float nw[4] = {1.0f + w.x, 1.0f + w.y, 1.0f + w.z, 1.0f + w.w};
  uint2 u[kConvRows];
#pragma unroll
  for (int i = 0; i < kConvRows; ++i)
    u[i] = (r0 + i < L) ? __ldg(reinterpret_cast<const uint2*>(z + (t0 + r0 + i) * WV + col)) : make_uint2(0u, 0u);
#pragma unroll
  for (int i = 0; i < kConvRows; ++i) {
    if (r0 + i < L) {
      const float zz[4] = {__uint_as_float(u[i].x << 16), __uint_as_float(u[i].x & 0xffff0000u),
                           __uint_as_float(u[i].y << 16), __uint_as_float(u[i].y & 0xffff0000u)};
      float g[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) g[e] = nw[e] * __fdividef(1.0f, 1.0f + __expf(-zz[e]));
      const int r = r0 + i;
      st8(grec + hcol * 8192 + r * 128 + ((q ^ (r & 7)) << 4) + (lane & 1) * 8, g[0], g[1], g[2], g[3]);
    }
  }
}

// Gates of one chunk and value head ("fp32 Gated DeltaNet recurrence"):
// g_r = -exp(A_log) softplus(a_r + dt_bias), beta_r = sigmoid(b_r), the
// inclusive scan gamma_r of g within the chunk, into the record.  One warp:
// lane l owns rows 2l and 2l + 1.
__device__ __forceinline__ void chunk_gates(const Dims& d, const float* __restrict__ A_log,
                                            const float* __restrict__ dt_bias, const __nv_bfloat16* __restrict__ a,
                                            const __nv_bfloat16* __restrict__ b, int64_t t0, int L, int h, int lane,
                                            unsigned char* __restrict__ rec) {
  const float negA = -expf(A_log[h]);
  const float dtb = dt_bias[h];
  float g2[2], be2[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int r = 2 * lane + e;
    g2[e] = 0.f;
    be2[e] = 0.f;
    if (r < L) {
      g2[e] = negA * softplus_f(__bfloat162float(a[(t0 + r) * d.Hv + h]) + dtb);
      be2[e] = 1.0f / (1.0f + expf(-__bfloat162float(b[(t0 + r) * d.Hv + h])));
    }
  }
  float incl = g2[0] + g2[1];
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  const float gC = __shfl_sync(0xffffffffu, incl, 31);
  reinterpret_cast<float2*>(rec + REC_GAM)[lane] = make_float2(incl - g2[1], incl);
  reinterpret_cast<float2*>(rec + REC_BETA)[lane] = make_float2(be2[0], be2[1]);
  if (lane == 0) reinterpret_cast<float2*>(rec + REC_META)[0] = make_float2(expf(gC), gC);
}

constexpr int kConvThreads = 32 * (kConvGateWarp + 1);

// A window of the packed chunks handled by one conv + prep + chain pass: global chunks [g_base, g_base + the
// grid's chunk count), whose records start at record 0 of the window's buffer and whose q^/k^ rows start at
// row 0 of the window's hi and lo buffers (token t_base).
struct Window {
  int64_t g_base;
  int64_t t_base;
};

__global__ void __launch_bounds__(kConvThreads, 4)
    conv_qkv_kernel(Dims d, const float* __restrict__ conv_w, const __nv_bfloat16* __restrict__ qkv,
                    const __nv_bfloat16* __restrict__ hist, int zero_conv, const int4* __restrict__ chunk_map,
                    const float* __restrict__ norm_w, const __nv_bfloat16* __restrict__ z,
                    const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                    const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                    __half* __restrict__ qk_hi, __half* __restrict__ qk_lo, unsigned char* __restrict__ records,
                    int64_t single_len, Window win) {
  // chunks in reverse order: the first chunks' outputs are the freshest in L2 when the chain starts
  const int g = (int)(win.g_base + gridDim.x - 1 - blockIdx.x);
  const int64_t gw = g - win.g_base;  // the chunk's record in the window
  // {seq, first token, length, chunk index}; one sequence needs no map
  const int64_t rest = single_len - (int64_t)kC * g;
  const int4 cm = chunk_map ? chunk_map[g] : make_int4(0, kC * g, rest < kC ? (int)rest : kC, g);
  const int slot = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = kConvRows * warp;
  const int L = cm.z;
  const int nqk = 2 * d.Hk;
  if (slot >= nqk + d.Hv) {
    const int hz = slot - nqk - d.Hv;
    unsigned char* rec = records + (gw * d.Hv + hz) * kRec;
    if (warp == kConvGateWarp) chunk_gates(d, A_log, dt_bias, a, b, cm.y, L, hz, lane, rec);
    else if (r0 < L) gate_rows(d, norm_w, z, rec + REC_G, cm.y, r0, L, hz, lane);
    return;
  }
  if (warp == kConvGateWarp) return;
  // v^ goes straight into the record of (chunk, value head) as the chain kernel's operand image
  unsigned char* vrec = slot >= nqk ? records + (gw * d.Hv + (slot - nqk)) * kRec + REC_V : nullptr;
  if (vrec) {
#pragma unroll
    for (int i = 0; i < kConvRows; ++i)
      if (r0 + i >= L) {
        *reinterpret_cast<uint2*>(vrec + mnmaj(kC, r0 + i, 4 * lane)) = make_uint2(0u, 0u);
        *reinterpret_cast<uint2*>(vrec + (REC_VL - REC_V) + mnmaj(kC, r0 + i, 4 * lane)) = make_uint2(0u, 0u);
      }
  }
  if (r0 >= L) return;
  const int64_t C = d.C;
  const int64_t c = (int64_t)slot * kD + 4 * lane;  // q heads, k heads and v heads are consecutive in qkv
  float w[4][4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(conv_w + (c + e) * 4));
    w[e][0] = x.x; w[e][1] = x.y; w[e][2] = x.z; w[e][3] = x.w;
  }
  // raw rows r0-3 .. r0+15 of the chunk; rows before the sequence start come
  // from the conv history, rows past the chunk's end are never used
  uint2 xr[kConvRows + 3];  // raw bf16 pairs, unpacked where used
  const bool first = cm.w == 0;
#pragma unroll
  for (int i = 0; i < kConvRows + 3; ++i) {
    const int rr = r0 - 3 + i;
    xr[i] = make_uint2(0u, 0u);
    if (rr < L) {
      if (first && rr < 0) {
        if (!zero_conv) xr[i] = *reinterpret_cast<const uint2*>(hist + ((int64_t)cm.x * 3 + (3 + rr)) * C + c);
      } else {
        xr[i] = __ldg(reinterpret_cast<const uint2*>(qkv + ((int64_t)cm.y + rr) * C + c));
      }
    }
  }
  auto xf = [&](int i, int e) {
    const uint32_t u = (e < 2) ? xr[i].x : xr[i].y;
    return __uint_as_float((e & 1) ? (u & 0xffff0000u) : (u << 16));
  };
  float y[kConvRows][4];
#pragma unroll
  for (int i = 0; i < kConvRows; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float acc = 0.f;
#pragma unroll
      for (int tap = 0; tap < 4; ++tap) acc += w[e][tap] * xf(i + tap, e);
      y[i][e] = silu_fast(acc);
    }
  if (slot < nqk) {  // q or k: L2 norm over the head's 128 channels, then hi + lo fp16 parts
    float ss[kConvRows];
#pragma unroll
    for (int i = 0; i < kConvRows; ++i) ss[i] = y[i][0] * y[i][0] + y[i][1] * y[i][1] + y[i][2] * y[i][2] + y[i][3] * y[i][3];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int i = 0; i < kConvRows; ++i) ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], off);
    const float scale = slot < d.Hk ? d.q_scale : 1.0f;
    const int64_t W2 = (int64_t)nqk * kD;
#pragma unroll
    for (int i = 0; i < kConvRows; ++i) {
      if (r0 + i < L) {
        const float rs = scale * rsqrtf(ss[i] + d.l2_eps);
        float hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float v = y[i][e] * rs;
          hi[e] = __half2float(__float2half_rn(v));
          lo[e] = v - hi[e];
        }
        const int64_t off = ((int64_t)cm.y + r0 + i - win.t_base) * W2 + c;
        st8(reinterpret_cast<unsigned char*>(qk_hi + off), hi[0], hi[1], hi[2], hi[3]);
        st8(reinterpret_cast<unsigned char*>(qk_lo + off), lo[0], lo[1], lo[2], lo[3]);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < kConvRows; ++i)
      if (r0 + i < L) {
        float lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) lo[e] = y[i][e] - __half2float(__float2half_rn(y[i][e]));
        st8(vrec + mnmaj(kC, r0 + i, 4 * lane), y[i][0], y[i][1], y[i][2], y[i][3]);
        st8(vrec + (REC_VL - REC_V) + mnmaj(kC, r0 + i, 4 * lane), lo[0], lo[1], lo[2], lo[3]);
      }
  }
}

// ------------------------------------------------------------------ prep_kernel
// Three blocks per SM.  Shared memory (71 KB):
//   P_KQ   [k^ ; q^] hi parts, K-major 128 x 128.  Once [K;Q]K^T is done, v^
//          hi (MN-major, its two 64-channel blocks 16 KB apart) comes into the
//          q^ halves; once W = T''K is done, v^ lo into the k^ halves.
//   P_KQL  [k^ ; q^] lo parts.  After [K;Q]K^T: the solve's images A_off16,
//          A_off32, T and X (K-major 64 x 64 fp16 each; the fp32 16x16
//          diagonal blocks of A in X's place until X is first written); after
//          the solve T'' over A_off16, T' hi over A_off32 and T' lo over T.
//   P_TF   the 16x16 diagonal blocks of T in fp32.
// TMEM: 128 columns; [K;Q]K^T in columns 0..63, the solve's products in 0..63,
// then W and then U (M = 64 MMAs) in 0..127.
constexpr int kPrepThreads = 256;
constexpr int P_KQ = 0;
constexpr int P_KQL = 32768;
constexpr int P_MISC = 65536;
constexpr int P_GATES = P_MISC + 64 * 6 * 4;  // the record's e^{gamma_C}, gamma_C, gamma_r, beta_r (528 bytes)
constexpr int P_TF = P_GATES + 528;            // the 16x16 diagonal blocks of T in fp32 (4 KB)
constexpr int kPrepSmem = P_TF + 4096 + 1024;
// the solve's images in the lo tile once [K;Q]K^T is done (K-major 64 x 64 fp16 each)
constexpr int P_AOFF16 = P_KQL, P_AOFF32 = P_KQL + 8192, P_T = P_KQL + 16384, P_X = P_KQL + 24576;
constexpr int P_DIAG = P_X;  // the fp32 16x16 diagonal blocks of A (stride 17) until X is first written
constexpr uint32_t kPrepTmemCols = 128;

// The new conv history of sequence n: the last W-1 raw rows of [history ;
// inputs].  The prep block of the sequence's last chunk and value head h owns
// the v channels of h and, for the first value head of a key head, the q and
// k channels of that key head (nothing reads the old history after the conv
// kernel).  One thread per 16 bytes of channels reads its three rows before
// writing them.
__device__ __forceinline__ void write_history(const Dims& d, int h, int n, int64_t seq0, int len,
                                           const __nv_bfloat16* __restrict__ qkv, int zero_conv,
                                           __nv_bfloat16* __restrict__ hist) {
  const int G = d.G, kh = h / G;
  const int nvec = (h % G == 0 ? 3 : 1) * (kD / 8);
  for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
    const int part = i / (kD / 8), c8 = 8 * (i % (kD / 8));
    const int64_t ch = part == 0 ? 2LL * d.Hk * kD + (int64_t)h * kD + c8
                                 : (part == 1 ? (int64_t)kh * kD + c8 : (int64_t)d.Hk * kD + (int64_t)kh * kD + c8);
    uint4 v[3];
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      const int m = len + r - 3;
      v[r] = m >= 0 ? *reinterpret_cast<const uint4*>(qkv + (seq0 + m) * d.C + ch)
                    : (zero_conv ? make_uint4(0, 0, 0, 0)
                                 : *reinterpret_cast<const uint4*>(hist + ((int64_t)n * 3 + (m + 3)) * d.C + ch));
    }
#pragma unroll
    for (int r = 0; r < 3; ++r) *reinterpret_cast<uint4*>(hist + ((int64_t)n * 3 + r) * d.C + ch) = v[r];
  }
}

__global__ void __launch_bounds__(kPrepThreads, 3)
    prep_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo, Dims d,
                const int4* __restrict__ chunk_map, unsigned char* __restrict__ records, const int32_t* __restrict__ cu,
                const __nv_bfloat16* __restrict__ qkv, int zero_conv, __nv_bfloat16* __restrict__ hist,
                int64_t single_len, Window win, int32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t mb_tma, mb_mma, mb_v, mb_vl;
  __shared__ uint32_t tslot;
  bool bad = false;  // this thread saw a wait run out

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = blockIdx.x / d.Hv;  // chunks in reverse order, as in conv_qkv_kernel
  const int h = blockIdx.x - gr * d.Hv;
  const int g = (int)(win.g_base + gridDim.x / d.Hv - 1 - gr);
  const int kh = h / d.G;
  const int4 cm = chunk_map ? chunk_map[g] : make_int4(0, kC * g, 0, g);
  const int64_t t0 = cm.y;  // rows past the chunk's end carry beta = 0 (their gates are zero)
  {  // the block of a sequence's last chunk writes the sequence's new conv history for its channels
    const int64_t s0 = chunk_map ? cu[cm.x] : 0, s1 = chunk_map ? cu[cm.x + 1] : single_len;
    if (t0 + kC >= s1) write_history(d, h, cm.x, s0, (int)(s1 - s0), qkv, zero_conv, hist);
  }
  unsigned char* rec = records + ((g - win.g_base) * d.Hv + h) * kRec;
  const int trow = (int)(t0 - win.t_base);  // the chunk's first row in the window's q^/k^ buffers

  float* misc = reinterpret_cast<float*>(sm + P_MISC);
  float* s_gam = misc;
  float* s_beta = misc + 64;
  float* s_eg = misc + 128;
  float* s_ekd = misc + 192;
  float* s_tb = misc + 256;    // beta_j             (columns of T')
  float* s_tbg = misc + 320;   // beta_j e^{gamma_j} (columns of T'')

  if (tid == 0) {  // the copies go out before anything else
    mbar_init(&mb_tma, 1);
    mbar_init(&mb_mma, 1);
    mbar_init(&mb_v, 1);
    mbar_init(&mb_vl, 1);
    mbar_init_fence();
    mbar_expect_tx(&mb_tma, 8 * 8192 + 528);
    bulk_load(sm + P_GATES, rec + REC_META, 528, &mb_tma);
    const int qx = kh * kD, kx = d.Hk * kD + kh * kD;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      tma_load_2d(sm + P_KQ + j * 16384, &tm_hi, kx + 64 * j, trow, &mb_tma);
      tma_load_2d(sm + P_KQ + j * 16384 + 8192, &tm_hi, qx + 64 * j, trow, &mb_tma);
      tma_load_2d(sm + P_KQL + j * 16384, &tm_lo, kx + 64 * j, trow, &mb_tma);
      tma_load_2d(sm + P_KQL + j * 16384 + 8192, &tm_lo, qx + 64 * j, trow, &mb_tma);
    }
  }
  if (warp == 0) tmem_alloc(&tslot, kPrepTmemCols);
  sync_tc();
  const uint32_t tbase = tslot;
  if (!mbar_wait(&mb_tma, 0, kWaitNs)) bad = true;
  if (tid < 64) {  // the chunk's gates (computed by the conv kernel, copied in with the tiles) and exponentials
    const float* gr = reinterpret_cast<const float*>(sm + P_GATES);
    const float gam = gr[(REC_GAM - REC_META) / 4 + tid];
    const float be = gr[(REC_BETA - REC_META) / 4 + tid];
    const float gC = gr[1];
    const float eg = expf(gam);
    s_gam[tid] = gam;
    s_beta[tid] = be;
    s_eg[tid] = eg;
    s_ekd[tid] = expf(gC - gam);
    s_tb[tid] = be;
    s_tbg[tid] = be * eg;
  }
  if (sync_tc_any(bad)) {
    if (tid == 0) set_status(status, kStatusWaitTimeout);
    if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
    return;
  }

  // M1: [K;Q] K^T as hi.hi + hi.lo + lo.hi
  if (tid == 0) {
    const uint32_t kq = smem_u32(sm + P_KQ), kql = smem_u32(sm + P_KQL);
    constexpr uint32_t id = idesc_f16(128, 64, false, false);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase, desc_kmaj(kq, 128, s), desc_kmaj(kq, 128, s), id, s > 0);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase, desc_kmaj(kq, 128, s), desc_kmaj(kql, 128, s), id, 1);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase, desc_kmaj(kql, 128, s), desc_kmaj(kq, 128, s), id, 1);
    mma_commit(&mb_mma);
  }
  // meanwhile: Qg = diag(e^gamma) q^ -> rows 64..127 of the [-W;Qg] image, K~ = diag(e^{gC-gamma}) k^ -> its
  // image; q^ and k^ as hi + lo, so that each operand is rounded to fp16 once
  for (int e = tid; e < 64 * 16; e += kPrepThreads) {
    const int r = e >> 4, c8 = 8 * (e & 15);
    const uint32_t oq = kmaj_chunk(128, 64 + r, c8), ok = kmaj_chunk(128, r, c8);
    const uint4 uq = *reinterpret_cast<const uint4*>(sm + P_KQ + oq);
    const uint4 uk = *reinterpret_cast<const uint4*>(sm + P_KQ + ok);
    const uint4 lq = *reinterpret_cast<const uint4*>(sm + P_KQL + oq);
    const uint4 lk = *reinterpret_cast<const uint4*>(sm + P_KQL + ok);
    const float eg = s_eg[r], ek = s_ekd[r];
    const __half2* hq = reinterpret_cast<const __half2*>(&uq);
    const __half2* hk = reinterpret_cast<const __half2*>(&uk);
    const __half2* hql = reinterpret_cast<const __half2*>(&lq);
    const __half2* hkl = reinterpret_cast<const __half2*>(&lk);
    float fq[8], fk[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 a2 = __half22float2(hq[i]), b2 = __half22float2(hk[i]);
      const float2 a3 = __half22float2(hql[i]), b3 = __half22float2(hkl[i]);
      fq[2 * i] = (a2.x + a3.x) * eg;
      fq[2 * i + 1] = (a2.y + a3.y) * eg;
      fk[2 * i] = (b2.x + b3.x) * ek;
      fk[2 * i + 1] = (b2.y + b3.y) * ek;
    }
    *reinterpret_cast<uint4*>(rec + REC_A + kmaj_chunk(128, 64 + r, c8)) = pack8h(fq);
    *reinterpret_cast<uint4*>(rec + REC_K + mnmaj_chunk(64, r, c8)) = pack8h(fk);
  }
  if (!mbar_wait(&mb_mma, 0, kWaitNs)) bad = true;
  if (sync_tc_any(bad)) {  // also: the q^ rows are read, the lo tile is free
    if (tid == 0) set_status(status, kStatusWaitTimeout);
    if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
    return;
  }

  if (tid == 0) {  // the q^ rows of the hi tile are read: v^ comes into them while the solve runs
    fence_async_smem();
    mbar_expect_tx(&mb_v, 16384);
    bulk_load(sm + P_KQ + 8192, rec + REC_V, 8192, &mb_v);
    bulk_load(sm + P_KQ + 24576, rec + REC_V + 8192, 8192, &mb_v);
  }
  // A (rows 0..63) into the fp32 16x16 diagonal blocks and the two level images; P (rows 64..127, fp16)
  // into the record.  Element (r, j), j < r, of A belongs to the level b = 16, 32 whose blocks first put r
  // and j in different halves, or to a 16x16 diagonal block when r ^ j < 16.
  const int si = 32 * (warp & 3) + lane, hc = warp >> 2;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
  {
    float v[32];
    tmem_ld32(tbase + lane_base + 32 * hc, v);
    if (si < 64) {
      const float br = s_beta[si], gr = s_gam[si];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float a16[8], a32[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = 32 * hc + 8 * m + e;
          const float av = (j < si) ? br * __expf(gr - s_gam[j]) * v[8 * m + e] : 0.f;
          const int x = si ^ j;
          a16[e] = (x >= 16 && x < 32) ? av : 0.f;
          a32[e] = (x >= 32) ? av : 0.f;
          if (x < 16) reinterpret_cast<float*>(sm + P_DIAG)[(si >> 4) * 272 + (si & 15) * 17 + (j & 15)] = av;
        }
        *reinterpret_cast<uint4*>(sm + P_AOFF16 + kmaj_chunk(64, si, 32 * hc + 8 * m)) = pack8h(a16);
        *reinterpret_cast<uint4*>(sm + P_AOFF32 + kmaj_chunk(64, si, 32 * hc + 8 * m)) = pack8h(a32);
      }
    } else {
      const int r = si - 64;
      const float gr = s_gam[r];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = 32 * hc + 8 * m + e;
          p[e] = (j <= r) ? __expf(gr - s_gam[j]) * v[8 * m + e] : 0.f;
        }
        *reinterpret_cast<uint4*>(rec + REC_P + kmaj_chunk(64, r, 32 * hc + 8 * m)) = pack8h(p);
      }
    }
  }
  for (int i = tid; i < 8192 / 16; i += kPrepThreads) reinterpret_cast<uint4*>(sm + P_T)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  // T = (I + A)^-1 by recursive doubling.  Level 0: the 16x16 diagonal blocks by forward substitution, one
  // column of one block per thread, in fp32: kept in fp32 for T' and T'' (no later level changes them) and
  // as fp16 in the T image.  Levels b = 16, 32: T <- T - T (A_off,b T), every merge of two b-blocks at once,
  // both products on tcgen05 (M = N = K = 64, fp16 operands, fp32 accumulation).  T starts at zero, so
  // its upper blocks stay zero.
  if (tid < 64) {
    const int bb = tid >> 4, c = tid & 15, o = 16 * bb;
    const float* Ad = reinterpret_cast<const float*>(sm + P_DIAG) + bb * 272;
    float* Tf = reinterpret_cast<float*>(sm + P_TF) + bb * 256;
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = (i == c) ? 1.f : 0.f;
#pragma unroll
      for (int k = 0; k < i; ++k) acc -= Ad[i * 17 + k] * t[k];
      t[i] = (i < c) ? 0.f : acc;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      *reinterpret_cast<__half*>(sm + P_T + kmaj(64, o + i, o + c)) = __float2half_rn(t[i]);
      Tf[i * 16 + c] = t[i];
    }
  }
  fence_async_smem();
  sync_tc();
  const int r16 = 16 * (warp & 3) + lane;  // lanes 0..15 of each lane quarter hold rows 16 q .. 16 q + 15
  uint32_t mma_phase = 1;  // [K;Q]K^T completed phase 0
#pragma unroll 1
  for (int lv = 0; lv < 2; ++lv) {
    const uint32_t aoff = smem_u32(sm + (lv == 0 ? P_AOFF16 : P_AOFF32));
    const uint32_t ts = smem_u32(sm + P_T), xs = smem_u32(sm + P_X);
    constexpr uint32_t id = idesc_f16(64, 64, false, true);
    if (tid == 0) {  // X = A_off T
#pragma unroll
      for (int s = 0; s < 4; ++s) mma_f16(tbase, desc_kmaj(aoff, 64, s), desc_mnmaj(ts, 64, s), id, s > 0);
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, mma_phase, kWaitNs)) bad = true;
    mma_phase ^= 1;
    fence_after();
    {
      float v[32];
      tmem_ld32(tbase + lane_base + 32 * hc, v);
      if (lane < 16) {
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint4*>(sm + P_X + kmaj_chunk(64, r16, 32 * hc + 8 * m)) = pack8h(v + 8 * m);
      }
    }
    fence_async_smem();
    sync_tc();
    if (tid == 0) {  // Y = T X
#pragma unroll
      for (int s = 0; s < 4; ++s) mma_f16(tbase, desc_kmaj(ts, 64, s), desc_mnmaj(xs, 64, s), id, s > 0);
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, mma_phase, kWaitNs)) bad = true;
    mma_phase ^= 1;
    fence_after();
    {
      float v[32];
      tmem_ld32(tbase + lane_base + 32 * hc, v);
      if (lane < 16) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          unsigned char* pt = sm + P_T + kmaj_chunk(64, r16, 32 * hc + 8 * m);
          const uint4 tq = *reinterpret_cast<const uint4*>(pt);
          const __half2* t2 = reinterpret_cast<const __half2*>(&tq);
          float nt[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(t2[i]);
            nt[2 * i] = f.x - v[8 * m + 2 * i];
            nt[2 * i + 1] = f.y - v[8 * m + 2 * i + 1];
          }
          *reinterpret_cast<uint4*>(pt) = pack8h(nt);
        }
      }
    }
    fence_async_smem();
    if (sync_tc_any(bad)) break;
  }
  if (bad) {  // block-uniform after sync_tc_any
    if (tid == 0) {
      set_status(status, kStatusWaitTimeout);
      mbar_wait(&mb_v, 0, kWaitNs);  // the v^ copy is no longer in flight when the block leaves
    }
    if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
    return;
  }
  {  // T' = T diag(beta) as fp16 hi + lo and T'' = T diag(beta e^gamma), K-major 64 x 64 A operands of
     // U = T' v^ and W = T'' K: T'' over A_off16, T' hi over A_off32 and T' lo over T once every thread
     // has read its rows of T.  A thread's 16 columns are one 16-column block: the diagonal one comes from
     // the fp32 blocks.
    const int r = tid >> 2, j0 = 16 * (tid & 3);
    float tv[16], t1[16], t2[16];
    if ((tid & 3) == (r >> 4)) {
      const float4* tf = reinterpret_cast<const float4*>(sm + P_TF) + (r >> 4) * 64 + (r & 15) * 4;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 f = tf[m];
        tv[4 * m] = f.x; tv[4 * m + 1] = f.y; tv[4 * m + 2] = f.z; tv[4 * m + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const uint4 tq = *reinterpret_cast<const uint4*>(sm + P_T + kmaj_chunk(64, r, j0 + 8 * m));
        const __half2* h2 = reinterpret_cast<const __half2*>(&tq);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(h2[i]);
          tv[8 * m + 2 * i] = f.x;
          tv[8 * m + 2 * i + 1] = f.y;
        }
      }
    }
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      const float t = (j0 + jj <= r) ? tv[jj] : 0.f;
      t1[jj] = t * s_tb[j0 + jj];
      t2[jj] = t * s_tbg[j0 + jj];
    }
    __syncthreads();  // every thread has read its rows of T
    st16h(sm + P_KQL + kmaj_chunk(64, r, j0), t2);
    st16h(sm + P_KQL + kmaj_chunk(64, r, j0 + 8), t2 + 8);
    st16h(sm + P_KQL + 8192 + kmaj_chunk(64, r, j0), t1);
    st16h(sm + P_KQL + 8192 + kmaj_chunk(64, r, j0 + 8), t1 + 8);
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) t1[jj] -= __half2float(__float2half_rn(t1[jj]));
    st16h(sm + P_KQL + 16384 + kmaj_chunk(64, r, j0), t1);
    st16h(sm + P_KQL + 16384 + kmaj_chunk(64, r, j0 + 8), t1 + 8);
  }
  fence_async_smem();
  sync_tc();

  // M2: W = T'' K  (M = 64; B = the k^ rows of the hi tile read as MN-major: K = 64 rows, N = 128 channels).
  // An M = 64 accumulator puts row r in TMEM lane (r % 16) + 32 (r / 16).
  if (tid == 0) {
    const uint32_t ta = smem_u32(sm + P_KQL), kq = smem_u32(sm + P_KQ);
    constexpr uint32_t id = idesc_f16(64, 128, false, true);
#pragma unroll
    for (int s = 0; s < 4; ++s) mma_f16(tbase, desc_kmaj(ta, 64, s), sdesc(kq + s * 2048, 16384, 1024), id, s > 0);
    mma_commit(&mb_mma);
  }
  if (!mbar_wait(&mb_mma, 1, kWaitNs)) bad = true;
  fence_after();
  if (tid == 0) {  // the k^ rows of the hi tile are read: v^ lo comes into them while -W goes out
    fence_async_smem();
    mbar_expect_tx(&mb_vl, 16384);
    bulk_load(sm + P_KQ, rec + REC_VL, 8192, &mb_vl);
    bulk_load(sm + P_KQ + 16384, rec + REC_VL + 8192, 8192, &mb_vl);
  }
  {  // -W -> rows 0..63 of the [-W;Qg] image: its two 8 KB row blocks (64-column block hc at +16 KB hc of
     // the image) are staged over T'' (read by W) and X, and go out by bulk stores
    float v[32];
    unsigned char* stage = sm + P_KQL + 24576 * hc;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      tmem_ld32(tbase + lane_base + 64 * hc + 32 * hh, v);
      if (lane < 16) {
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) v[jj] = -v[jj];
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint4*>(stage + kmaj_chunk(64, r16, 32 * hh + 8 * m)) = pack8h(v + 8 * m);
      }
    }
  }
  fence_async_smem();
  if (tid == 0 && !mbar_wait(&mb_v, 0, kWaitNs)) bad = true;
  if (sync_tc_any(bad)) {  // also: W is read out, its columns take U
    if (tid == 0) {
      set_status(status, kStatusWaitTimeout);
      mbar_wait(&mb_vl, 0, kWaitNs);  // no copy is still in flight when the block leaves
    }
    if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
    return;
  }
  if (tid == 0) {
    bulk_store(rec + REC_A, sm + P_KQL, 8192);
    bulk_store(rec + REC_A + 16384, sm + P_KQL + 24576, 8192);
    bulk_commit();
  }
  // MU: U = T'hi v^hi + T'lo v^hi + T'hi v^lo  (M = 64, N = 128; v^ MN-major with its 64-channel blocks
  // 16 KB apart: hi in the q^ halves of the hi tile, lo in its k^ halves)
  if (tid == 0) {
    const uint32_t th = smem_u32(sm + P_KQL + 8192), tl = smem_u32(sm + P_KQL + 16384), vb = smem_u32(sm + P_KQ + 8192),
                   vlb = smem_u32(sm + P_KQ);
    constexpr uint32_t id = idesc_f16(64, 128, false, true);
#pragma unroll
    for (int s = 0; s < 4; ++s) mma_f16(tbase, desc_kmaj(th, 64, s), sdesc(vb + s * 2048, 16384, 1024), id, s > 0);
#pragma unroll
    for (int s = 0; s < 4; ++s) mma_f16(tbase, desc_kmaj(tl, 64, s), sdesc(vb + s * 2048, 16384, 1024), id, 1);
    if (!mbar_wait(&mb_vl, 0, kWaitNs)) bad = true;
    if (!bad) {
#pragma unroll
      for (int s = 0; s < 4; ++s) mma_f16(tbase, desc_kmaj(th, 64, s), sdesc(vlb + s * 2048, 16384, 1024), id, 1);
    }
    mma_commit(&mb_mma);
  }
  if (!mbar_wait(&mb_mma, 0, kWaitNs)) bad = true;
  if (tid == 0) bulk_wait_read<0>();  // the -W stores have read their staging (the U image goes over it)
  __syncthreads();
  fence_after();
  {  // U -> its record image staged over T'' .. X (all read by the U products): fp32, channel half c / 64
     // at 16384 (c / 64), row r at 256 r, 16-byte piece j of the half row at (j ^ (r % 8)) * 16
    float v[32];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      tmem_ld32(tbase + lane_base + 64 * hc + 32 * hh, v);
      if (lane < 16) {
        unsigned char* urow = sm + P_KQL + 16384 * hc + 256 * r16;
#pragma unroll
        for (int m = 0; m < 8; ++m)
          *reinterpret_cast<float4*>(urow + (((8 * hh + m) ^ (r16 & 7)) << 4)) =
              make_float4(v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]);
      }
    }
  }
  fence_async_smem();
  const bool fail = sync_tc_any(bad);
  if (tid == 0) {
    if (fail) set_status(status, kStatusWaitTimeout);
    bulk_store(rec + REC_U, sm + P_KQL, 32768);
    bulk_commit();
    bulk_wait<0>();  // every record image has left shared memory
  }
  if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
}

// ------------------------------------------------------------------ chain_kernel
// One cluster of two CTAs per (sequence, value head); CTA `vh` of the pair
// carries value channels [64 vh, 64 vh + 64), i.e. 64 columns of the state,
// which evolve independently of the other 64.  Both read the chunk's shared
// operands ([-W;Qg], P, K~; the second read hits L2) and their own half of U
// and of the gate rows.  Every operand buffer is doubled, so that each copy
// goes out two chunks ahead.
constexpr int kChainThreads = 320;  // eight compute warps, the MMA-issuing warp, the copy-issuing warp
struct ChainScan {
  int32_t nseg;         // > 0: segmented use (see chain_kernel)
  int32_t zero_u_from;  // first cluster-pair index whose U is taken as zero
  int32_t win_lo = 0;   // the window of global chunks [win_lo, win_hi) whose records `records` holds,
  int32_t win_hi = 0x7fffffff;  // record 0 being chunk win_lo's
};
constexpr int C_A = 0;          // [-W ; Qg]   K-major 128 x 128; buffer cc % 2 at +32768 (cc % 2)
constexpr int C_P = 65536;      // [0 ; P]     K-major 128 x 64 (8 KB of zero rows, then P); buffer at +16384 (cc % 2)
constexpr int C_U = 98304;      // U half      fp32 64 x 64, the record's image; buffer at +16384 (cc % 2)
constexpr int C_KT = 131072;    // K~          MN-major K=64 x M=128; buffer at +16384 (cc % 2)
constexpr int C_DB = 163840;    // Delta half  MN-major K=64 x N=64
constexpr int C_SB = 172032;    // S half as fp16 hi (+0) and lo (+16384), MN-major K=128 x N=64 each
constexpr int C_G = 204800;     // output gate rows of this half; buffer at +8192 (cc % 2)
constexpr int C_O = 221184;     // output staging, 32 rows x 64 bytes per output warp (16-byte pieces swizzled)
constexpr int C_MISC = 229376;  // row sums of squares: this CTA's [2][64], the peer's [2 buffers][64]
constexpr int kChainSmem = C_MISC + 256 * 4 + 1024;
// accumulators of chunk cc at COL_U0 + 128 (cc % 2): [-W;Qg] S hi in its first 64 columns, [-W;Qg] S lo in
// the next 64 (the output warps sum the two; Delta takes the hi block alone); K~^T Delta at COL_Y
constexpr uint32_t COL_U0 = 0, COL_Y = 256, kChainTmemCols = 512;

// Roles: warps 0, 1, 4, 5 ("delta warps", TMEM lanes 0..63) form Delta = U -
// W S and store it to shared memory; warps 2, 3, 6, 7 ("output warps", lanes
// 64..127) write the previous chunk's output rows meanwhile; all eight carry
// the state, thread (row i, warp w) columns 32 (w / 4) .. + 31 of row i in
// registers.  Warp 8 issues the MMAs, warp 9 the bulk copies (each as soon as
// the MMAs that read its buffer are done), so that neither waits for the other.
//
// Segmented use (the sequence-parallel prefill): with scan.nseg > 0 the grid
// runs cluster pair oi over segment oi % nseg of the schedule (cu, chunk_off)
// with its own state slot oi; pairs oi >= scan.zero_u_from treat U as zero
// (the homogeneous part of the chunk maps).  o == nullptr skips the output rows.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kChainThreads, 1)
    chain_kernel(Dims d, const unsigned char* __restrict__ records, const int32_t* __restrict__ chunk_off,
                 const int32_t* __restrict__ order, const int32_t* __restrict__ cu, int zero_state, ChainScan scan,
                 float* __restrict__ state, __nv_bfloat16* __restrict__ o, int32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t mb_a[2], mb_u[2], mb_ld1[2], mb_g[2];  // copies into buffer cc % 2, one phase per use
  __shared__ uint64_t mb_m3, mb_m5;  // completions of [-WS;QgS] and K~^T Delta, one phase per chunk
  __shared__ uint64_t mb_m3a;        // completion of [-W;Qg] S lo, the last reader of the chunk's A buffer
  __shared__ uint64_t mb_m4[2];      // completion of [0;P] Delta (O of chunk cc complete), cc % 2, one phase per use
  __shared__ uint64_t mb_x[2];       // the peer's row sums of chunk cc arrived, cc % 2, one phase per use
  __shared__ uint32_t tslot;
  bool bad = false;  // this thread saw a wait run out

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vh = (int)cluster_ctarank();  // value-channel half
  const int pair = blockIdx.x >> 1;
  const int h = pair % d.Hv;
  const int oi = pair / d.Hv;
  const int n = scan.nseg > 0 ? oi % scan.nseg : (order ? order[oi] : oi);
  const int slot = scan.nseg > 0 ? oi : n;       // state slot read at the start and written at the end
  const bool zero_u = oi >= scan.zero_u_from;    // cluster-uniform
  const bool write_o = o != nullptr;
  const int64_t seq0 = cu[n];
  const int len = cu[n + 1] - cu[n];
  if (len <= 0) return;  // both CTAs of the cluster, before any cluster barrier
  // the sequence's chunks inside the window: local chunks cc0 .. cc0 + nchunks - 1; the state carries in from
  // the previous window (or from zero at the sequence's first chunk) and out to the next
  const int64_t gfirst = chunk_off ? chunk_off[n] : 0;
  const int64_t ga = max(gfirst, (int64_t)scan.win_lo), gb = min(gfirst + (len + kC - 1) / kC, (int64_t)scan.win_hi);
  if (ga >= gb) return;  // both CTAs of the cluster, before any cluster barrier
  const int cc0 = (int)(ga - gfirst);
  const int nchunks = (int)(gb - ga);
  const int64_t g0 = ga - scan.win_lo;  // record of the window's first chunk of this sequence
  const bool zero_here = zero_state && cc0 == 0;
  const int64_t HvD = (int64_t)d.Hv * kD;
  float* s_rms = reinterpret_cast<float*>(sm + C_MISC);         // [2][64], this CTA's column quarters
  float* s_peer = reinterpret_cast<float*>(sm + C_MISC) + 128;  // [2][64], written by the peer
  const bool compute = warp < 8, mma_warp = warp == 8, copy_warp = warp == 9;
  const bool out_warp = compute && (warp & 3) >= 2;
  // compute warps: thread owns row si of S (d_k index) / of the accumulators, local columns [32 hc, 32 hc + 32)
  const int si = 32 * (warp & 3) + lane, hc = (warp >> 2) & 1;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
  const int c0 = 64 * vh + 32 * hc;  // first value channel of this thread's columns
  float* gst = state + ((int64_t)slot * d.Hv + h) * kD * kD;  // stored [j][i]

  if (tid == 0) {
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      mbar_init(&mb_a[b], 1);
      mbar_init(&mb_u[b], 1);
      mbar_init(&mb_ld1[b], 1);
      mbar_init(&mb_g[b], 1);
      mbar_init(&mb_m4[b], 1);
      mbar_init(&mb_x[b], 1);  // one local arrival with the expected bytes; the peer's stores complete them
    }
    mbar_init(&mb_m3, 1);
    mbar_init(&mb_m3a, 1);
    mbar_init(&mb_m5, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(&tslot, kChainTmemCols);
  for (int i = tid; i < 512; i += kChainThreads) {  // the zero rows of both [0;P] buffers
    reinterpret_cast<uint4*>(sm + C_P)[i] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4*>(sm + C_P + 16384)[i] = make_uint4(0, 0, 0, 0);
  }

  auto rec_of = [&](int cc) { return records + ((g0 + cc) * d.Hv + h) * (int64_t)kRec; };
  auto issue_a = [&](int cc) {
    mbar_expect_tx(&mb_a[cc & 1], 32768);
    bulk_load(sm + C_A + 32768 * (cc & 1), rec_of(cc) + REC_A, 32768, &mb_a[cc & 1]);
  };
  auto issue_u = [&](int cc) {
    mbar_expect_tx(&mb_u[cc & 1], 16384);
    bulk_load(sm + C_U + 16384 * (cc & 1), rec_of(cc) + REC_U + 16384 * vh, 16384, &mb_u[cc & 1]);
  };
  auto issue_ld1 = [&](int cc) {  // P and K~
    uint64_t* mb = &mb_ld1[cc & 1];
    const unsigned char* r = rec_of(cc);
    mbar_expect_tx(mb, 8192 + 16384);
    bulk_load(sm + C_P + 16384 * (cc & 1) + 8192, r + REC_P, 8192, mb);
    bulk_load(sm + C_KT + 16384 * (cc & 1), r + REC_K, 16384, mb);
  };
  auto issue_gate = [&](int cc) {
    mbar_expect_tx(&mb_g[cc & 1], 8192);
    bulk_load(sm + C_G + (cc & 1) * 8192, rec_of(cc) + REC_G + 8192 * vh, 8192, &mb_g[cc & 1]);
  };
  auto prefetch = [&](int cc) {  // the parts this kernel reads, into L2 (one CTA of the pair)
    bulk_prefetch_l2(rec_of(cc), REC_V);
    bulk_prefetch_l2(rec_of(cc) + REC_P, REC_META + 16 - REC_P);
  };
  float S[32];  // this thread's part of the state, fp32
  // its fp16 hi and lo parts: the output Qg S + P Delta can cancel to far below |Qg||S| when q is nearly
  // orthogonal to the state's columns, so the state's fp16 rounding alone would cost o up to about 2e-3 of
  // its largest value; [-W;Qg] S lo goes out behind the critical [-W;Qg] S hi, and only the output reads it
  auto store_s = [&]() {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float lo[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) lo[e] = S[8 * m + e] - __half2float(__float2half_rn(S[8 * m + e]));
      st16h(sm + C_SB + mnmaj_chunk(kD, si, 32 * hc + 8 * m), S + 8 * m);
      st16h(sm + C_SB + 16384 + mnmaj_chunk(kD, si, 32 * hc + 8 * m), lo);
    }
  };
  if (compute) {
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) S[jj] = zero_here ? 0.f : gst[(int64_t)(c0 + jj) * kD + si];
    store_s();
  }
  fence_async_smem();
  sync_tc();
  const uint32_t tbase = tslot;
  // the first copies go out only after the block barrier that publishes the mbarriers' initialisation
  if (copy_warp && lane == 0) {
    issue_a(0);
    if (!zero_u) issue_u(0);
    issue_ld1(0);
    if (write_o) issue_gate(0);
    if (nchunks > 1) {
      issue_a(1);
      if (!zero_u) issue_u(1);
      issue_ld1(1);
    }
    if (nchunks > 2 && vh == 0) prefetch(2);
  }
  cluster_sync();  // the peer's mbarriers are initialised before any arrival on them
  const uint32_t peer = (uint32_t)(vh ^ 1);
  const uint32_t peer_x0 = mapa_shared(smem_u32(&mb_x[0]), peer), peer_x1 = mapa_shared(smem_u32(&mb_x[1]), peer);
  const uint32_t peer_sums = mapa_shared(smem_u32(s_peer), peer);

  // Output rows of chunk cc (O in lanes 64..127 of its accumulator): zero-centred
  // RMSNorm over all d_v channels times the precomputed gate (1 + w) sigmoid(z),
  // bf16 out.  Each CTA holds half of a row: the two 32-column sums of squares
  // meet at named barrier 1 (the output warps), their total goes to the peer's
  // buffer cc % 2 by asynchronous stores that complete the transaction bytes of
  // the peer's mbarrier, and the peer's total comes back the same way.  A buffer
  // is rewritten only two chunks later, after the peer has sent the chunk in
  // between, which it does after reading it.
  auto epilogue = [&](int cc) {
    const int r = si - 64;
    const int Lc = min(kC, len - (cc0 + cc) * kC);
    if (!mbar_wait(&mb_m4[cc & 1], (cc >> 1) & 1, kWaitNs)) bad = true;
    fence_after();
    float v[32], vl[32];
    tmem_ld32(tbase + lane_base + COL_U0 + 128 * (cc & 1) + 32 * hc, v);
    tmem_ld32(tbase + lane_base + COL_U0 + 128 * (cc & 1) + 64 + 32 * hc, vl);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] += vl[j];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) ss += v[j] * v[j];
    s_rms[64 * hc + r] = ss;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const float part = s_rms[r] + s_rms[64 + r];
    if (hc == 0) {
      st_async_f32(peer_sums + 4 * (64 * (cc & 1) + r), part, (cc & 1) ? peer_x1 : peer_x0);
      if (r == 0) mbar_expect_tx(&mb_x[cc & 1], 64 * 4);  // the local arrival of this phase
    }
    if (!mbar_wait_cluster(&mb_x[cc & 1], (cc >> 1) & 1, kWaitNs)) bad = true;
    const float rinv = rsqrtf((part + s_peer[64 * (cc & 1) + r]) * (1.0f / kD) + d.norm_eps);
    const unsigned char* grow = sm + C_G + (cc & 1) * 8192 + r * 128;
    unsigned char* stage = sm + C_O + (2 * hc + (warp & 1)) * 2048;  // this warp's 32 rows x 64 bytes
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int q = 4 * hc + m;  // 16-byte piece of the gate row half
      const uint4 gq = *reinterpret_cast<const uint4*>(grow + ((q ^ (r & 7)) << 4));
      const __half2* g2 = reinterpret_cast<const __half2*>(&gq);
      uint32_t ow[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 gf = __half22float2(g2[e]);
        __nv_bfloat162 pr = __floats2bfloat162_rn(v[8 * m + 2 * e] * rinv * gf.x, v[8 * m + 2 * e + 1] * rinv * gf.y);
        ow[e] = *reinterpret_cast<uint32_t*>(&pr);
      }
      *reinterpret_cast<uint4*>(stage + lane * 64 + ((m ^ ((lane >> 1) & 3)) << 4)) =
          make_uint4(ow[0], ow[1], ow[2], ow[3]);
    }
    __syncwarp();
    // four lanes per row: each store instruction writes eight whole 64-byte row pieces
    const int rbase = 32 * (warp & 1);
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int rr = 8 * it + (lane >> 2), q = lane & 3;
      if (rbase + rr < Lc) {
        const uint4 val = *reinterpret_cast<const uint4*>(stage + rr * 64 + ((q ^ ((rr >> 1) & 3)) << 4));
        *reinterpret_cast<uint4*>(o + (seq0 + (int64_t)(cc0 + cc) * kC + rbase + rr) * HvD + (int64_t)h * kD + c0 + 8 * q) =
            val;
      }
    }
    __syncwarp();
  };

  for (int c = 0; c < nchunks; ++c) {
    const uint32_t colU = COL_U0 + 128 * (c & 1);
    const uint32_t par = (c >> 1) & 1;  // phase parity of the buffers of chunk c
    if (mma_warp) {
      if (lane == 0) {  // [-W;Qg] S -> [-WS ; QgS]
        if (!mbar_wait(&mb_a[c & 1], par, kWaitNs)) bad = true;
        if (!bad) {
          const uint32_t aa = smem_u32(sm + C_A + 32768 * (c & 1)), sb = smem_u32(sm + C_SB);
          constexpr uint32_t id = idesc_f16(128, 64, false, true);
#pragma unroll
          for (int s = 0; s < 8; ++s) mma_f16(tbase + colU, desc_kmaj(aa, 128, s), desc_mnmaj(sb, kD, s), id, s > 0);
          mma_commit(&mb_m3);
#pragma unroll
          for (int s = 0; s < 8; ++s)
            mma_f16(tbase + colU + 64, desc_kmaj(aa, 128, s), desc_mnmaj(sb + 16384, kD, s), id, s > 0);
          mma_commit(&mb_m3a);
        }
        if (!mbar_wait(&mb_ld1[c & 1], par, kWaitNs)) bad = true;  // P and K~, long in place
      }
      __syncwarp();
      fence_before();
      asm volatile("bar.sync 2, 160;" ::: "memory");  // Delta is in shared memory
      fence_after();
      if (lane == 0) {  // Y = K~^T Delta first (the state update waits for it), then O += [0;P] Delta
        if (!bad) {
          const uint32_t pa = smem_u32(sm + C_P + 16384 * (c & 1)), db = smem_u32(sm + C_DB),
                         kt = smem_u32(sm + C_KT + 16384 * (c & 1));
          constexpr uint32_t id4 = idesc_f16(128, 64, false, true);
          constexpr uint32_t id5 = idesc_f16(128, 64, true, true);
#pragma unroll
          for (int s = 0; s < 4; ++s) mma_f16(tbase + COL_Y, desc_mnmaj(kt, kC, s), desc_mnmaj(db, kC, s), id5, s > 0);
          mma_commit(&mb_m5);
#pragma unroll
          for (int s = 0; s < 4; ++s) mma_f16(tbase + colU, desc_kmaj(pa, 128, s), desc_mnmaj(db, kC, s), id4, 1);
          mma_commit(&mb_m4[c & 1]);
        }
      }
    } else if (copy_warp) {
      if (lane == 0) {  // each buffer takes the chunk two ahead once its last reader is done
        if (c > 0) {  // [0;P] Delta of chunk c-1 was the last reader of its P and K~ buffers
          if (!mbar_wait(&mb_m4[(c - 1) & 1], ((c - 1) >> 1) & 1, kWaitNs)) bad = true;
          if (c + 1 < nchunks) issue_ld1(c + 1);
          if (c + 2 < nchunks && vh == 0) prefetch(c + 2);  // behind the copies in the queue
        }
        if (!mbar_wait(&mb_m3a, c & 1, kWaitNs)) bad = true;  // the lo products still read the A buffer after M3
        if (c + 2 < nchunks) issue_a(c + 2);
        if (!mbar_wait(&mb_m5, c & 1, kWaitNs)) bad = true;  // M5 follows the delta warps' reads of U
        if (c + 2 < nchunks && !zero_u) issue_u(c + 2);
      }
    } else {
      const float egC = __ldg(reinterpret_cast<const float*>(rec_of(c) + REC_META));  // used by the state update
      if (out_warp) {
        if (c > 0 && write_o) {
          if (!mbar_wait(&mb_g[(c - 1) & 1], ((c - 1) >> 1) & 1, kWaitNs)) bad = true;
          epilogue(c - 1);
        }
      } else {  // Delta = U + (-W S) -> shared (MN-major B operand)
        float u[32];
        if (zero_u) {
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] = 0.f;
        } else {
          if (!mbar_wait(&mb_u[c & 1], par, kWaitNs)) bad = true;
          const unsigned char* urow = sm + C_U + 16384 * (c & 1) + 256 * si;
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float4 f = *reinterpret_cast<const float4*>(urow + (((8 * hc + m) ^ (si & 7)) << 4));
            u[4 * m] = f.x; u[4 * m + 1] = f.y; u[4 * m + 2] = f.z; u[4 * m + 3] = f.w;
          }
        }
        if (!mbar_wait(&mb_m3, c & 1, kWaitNs)) bad = true;
        fence_after();
        float v[32];
        tmem_ld32(tbase + lane_base + colU + 32 * hc, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += u[j];
#pragma unroll
        for (int m = 0; m < 4; ++m) st16h(sm + C_DB + mnmaj_chunk(kC, si, 32 * hc + 8 * m), v + 8 * m);
        fence_async_smem();
        fence_before();
        asm volatile("bar.sync 2, 160;" ::: "memory");
        fence_after();
      }
      // no MMA barrier can run a phase ahead: the next chunk's MMAs follow the block barrier below
      if (!mbar_wait(&mb_m5, c & 1, kWaitNs)) bad = true;
      fence_after();
      // S = e^{gamma_C} S + K~^T Delta, and its fp16 copy for the next chunk
      float y[32];
      tmem_ld32(tbase + lane_base + COL_Y + 32 * hc, y);
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) S[jj] = egC * S[jj] + y[jj];
      store_s();
    }
    fence_async_smem();
    if (sync_tc_any(bad)) break;
    // the output of chunk c-1 is written: its gate buffer takes chunk c+1's rows
    if (copy_warp && lane == 0 && c + 1 < nchunks && write_o) issue_gate(c + 1);
  }
  // block-uniform: either every output warp reaches the epilogue's named barrier or none does
  if (!sync_tc_any(bad) && out_warp && write_o) {
    const int cl = nchunks - 1;
    if (!mbar_wait(&mb_g[cl & 1], (cl >> 1) & 1, kWaitNs)) bad = true;
    epilogue(cl);
  }
  if (sync_tc_any(bad)) {
    if (tid == 0) set_status(status, kStatusWaitTimeout);
  } else if (compute) {
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) gst[(int64_t)(c0 + jj) * kD + si] = S[jj];
  }
  sync_tc();
  if (warp == 0) tmem_dealloc(tbase, kChainTmemCols);
  cluster_sync();  // no CTA leaves while its peer may still write its row sums
}

bool encode_2d(EncodeTiledFn enc, CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t cols,
               uint64_t rows) {
  const cuuint64_t dim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t stride[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  return enc(tm, dt, 2, const_cast<void*>(base), dim, stride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

SplitLayout split_layout(const Dims& d, int64_t total_tokens, int64_t chunk_bound) {
  SplitLayout S;
  const size_t qkw = (size_t)2 * d.Hk * kD;
  S.qk_hi = 0;
  S.qk_lo = al256(S.qk_hi + (size_t)total_tokens * qkw * 2);
  S.records = al256(S.qk_lo + (size_t)total_tokens * qkw * 2);
  S.total_bytes = al256(S.records + (size_t)chunk_bound * d.Hv * kRec);
  return S;
}

namespace {

// conv + prep over the packed tokens: the per-token parts and the record of every (chunk, value head)
// conv + prep over one window of the packed chunks (see Window): the per-token parts and the record of every
// (chunk, value head) of the window, in the buffers of layout S (sized for the largest window)
cudaError_t launch_stages12(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                            const float* norm_w, const void* qkv, const void* z, const void* a, const void* b,
                            const int32_t* cu, const int4* chunk_map, int64_t total_tokens, Window win,
                            int64_t win_chunks, int64_t win_tokens, const SplitLayout& S, bool zero_conv,
                            const void* conv_state, void* split_ws, int32_t* status, cudaStream_t stream) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  unsigned char* ws = (unsigned char*)split_ws;
  __half* qk_hi = (__half*)(ws + S.qk_hi);
  __half* qk_lo = (__half*)(ws + S.qk_lo);
  unsigned char* records = ws + S.records;
  CUtensorMap tm_hi, tm_lo;
  const uint64_t qkw = (uint64_t)2 * d.Hk * kD;
  if (!encode_2d(enc, &tm_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, qk_hi, qkw, win_tokens) ||
      !encode_2d(enc, &tm_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, qk_lo, qkw, win_tokens))
    return cudaErrorInvalidValue;
  cudaError_t e;
  {
    LaunchScope scope(GDN_K_SPLIT_CONV, stream);
    conv_qkv_kernel<<<dim3((unsigned)win_chunks, (unsigned)(2 * d.Hk + 2 * d.Hv)), kConvThreads, 0, stream>>>(
        d, conv_w, (const __nv_bfloat16*)qkv, (const __nv_bfloat16*)conv_state, zero_conv ? 1 : 0, chunk_map, norm_w,
        (const __nv_bfloat16*)z, A_log, dt_bias, (const __nv_bfloat16*)a, (const __nv_bfloat16*)b, qk_hi, qk_lo,
        records, total_tokens, win);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPrepSmem)) != cudaSuccess)
    return e;
  LaunchScope scope(GDN_K_SPLIT_PREP, stream);
  prep_kernel<<<(unsigned)(win_chunks * d.Hv), kPrepThreads, kPrepSmem, stream>>>(
      tm_hi, tm_lo, d, chunk_map, records, cu, (const __nv_bfloat16*)qkv, zero_conv ? 1 : 0,
      (__nv_bfloat16*)const_cast<void*>(conv_state), total_tokens, win, status);
  return cudaGetLastError();
}

cudaError_t launch_chain(const Dims& d, const unsigned char* records, const int32_t* chunk_off, const int32_t* order,
                         const int32_t* cu, int64_t pairs, bool zero_state, ChainScan scan, float* state, void* o,
                         int32_t* status, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kChainSmem);
  if (e != cudaSuccess) return e;
  LaunchScope scope(GDN_K_SPLIT_CHAIN, stream);
  chain_kernel<<<(unsigned)(pairs * 2), kChainThreads, kChainSmem, stream>>>(
      d, records, chunk_off, order, cu, zero_state ? 1 : 0, scan, state, (__nv_bfloat16*)o, status);
  return cudaGetLastError();
}

}  // namespace

int64_t split_window_chunks(int64_t total_chunks) { return total_chunks < kSplitWindowChunks ? total_chunks
                                                                                            : kSplitWindowChunks; }

cudaError_t launch_prefill_split(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                                 const float* norm_w, const void* qkv, const void* z, const void* a, const void* b,
                                 const int32_t* cu, const int32_t* cu_host, const int32_t* order,
                                 const int32_t* chunk_off, const int4* chunk_map, int32_t N, int64_t total_tokens,
                                 int64_t total_chunks, bool zero_state, bool zero_conv, const void* conv_state,
                                 float* state, void* o, void* split_ws, int32_t* status, cudaStream_t stream) {
  if (N <= 0 || total_tokens <= 0 || total_chunks <= 0) return cudaSuccess;
  // The chunks go through conv, prep and the chain one window at a time, so that the intermediates take a
  // bounded workspace whatever the length; the chain carries each sequence's state from window to window
  // through `state` (a sequence starts from zero only in the window that holds its first chunk).
  const int64_t W = split_window_chunks(total_chunks);
  const SplitLayout S = split_layout(d, std::min<int64_t>(total_tokens, W * kC), W);
  const unsigned char* records = (unsigned char*)split_ws + S.records;
  // first token of chunk g (chunks are numbered sequence by sequence in id order)
  int32_t n = 0;
  int64_t n_first_chunk = 0;
  auto chunk_token = [&](int64_t g) -> int64_t {
    if (N == 1 || !cu_host) return kC * g;
    while (n < N) {
      const int64_t nch = (cu_host[n + 1] - cu_host[n] + kC - 1) / kC;
      if (g < n_first_chunk + nch) return cu_host[n] + kC * (g - n_first_chunk);
      n_first_chunk += nch;
      ++n;
    }
    return total_tokens;
  };
  cudaError_t e = cudaSuccess;
  for (int64_t g0 = 0; g0 < total_chunks && e == cudaSuccess; g0 += W) {
    const int64_t g1 = std::min<int64_t>(g0 + W, total_chunks);
    const int64_t t0 = chunk_token(g0), t1 = g1 < total_chunks ? chunk_token(g1) : total_tokens;
    e = launch_stages12(d, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, cu, chunk_map, total_tokens,
                        Window{g0, t0}, g1 - g0, t1 - t0, S, zero_conv, conv_state, split_ws, status, stream);
    if (e != cudaSuccess) break;
    ChainScan scan{0, 0x7fffffff};
    scan.win_lo = (int32_t)g0;
    scan.win_hi = (int32_t)g1;
    e = launch_chain(d, records, chunk_off, order, cu, (int64_t)N * d.Hv, zero_state, scan, state, o, status,
                     stream);
  }
  return e;
}

// ------------------------------------------------------------------ sequence-parallel chain
// One sequence cut into P chunk-aligned segments.  Over segment j the state
// carry is affine in the state it starts from, S -> A_j S + B_j (A_j acts on
// the key index and depends only on the keys and gates; B_j is linear in the
// values), so
//   B_j = the segment's final state from S = 0,
//   A_j = its final state from S = I with every U taken as zero (d_k = d_v),
// both from one chain launch over all segments at once.  A sequential pass over
// the P segments then gives every segment's true starting state, and a second
// chain launch writes the outputs.  The per-chunk records come from one conv +
// prep pass over the whole sequence: they do not depend on the state.
// States are stored transposed (stored = S^T), so the update is
//   T_{j+1} = T_j stored(A_j) + stored(B_j)   (row-major products).
namespace {

constexpr int kCombRows = 16;  // rows of T per combine block

// cu1 = {0, T}; segment table; phase-1 state slots: zeros (B runs), identities (A runs)
__global__ void __launch_bounds__(256)
    seqpar_init_kernel(int32_t T, int32_t P, int32_t seg_chunks, int32_t Hv, int32_t* cu1, int32_t* cu_seg,
                       int32_t* coff, float* s1) {
  const int64_t D2 = (int64_t)kD * kD;
  if (blockIdx.x == gridDim.x - 1) {
    if (threadIdx.x == 0) {
      cu1[0] = 0;
      cu1[1] = T;
    }
    for (int j = threadIdx.x; j <= P; j += blockDim.x) {
      const int64_t t = (int64_t)j * seg_chunks * kC;
      cu_seg[j] = (int32_t)(t < T ? t : T);
      if (j < P) coff[j] = j * seg_chunks;
    }
    return;
  }
  const int slot = blockIdx.x / Hv;  // blockIdx.x = slot * Hv + h
  float* dst = s1 + (int64_t)blockIdx.x * D2;
  const bool ident = slot >= P;
  for (int i = threadIdx.x; i < D2; i += blockDim.x) dst[i] = (ident && (i / kD) == (i % kD)) ? 1.0f : 0.0f;
}

// T_0 = the sequence's starting state (or zero); s3[j] = T_j, T_{j+1} = T_j A'_j + B'_j
// with A'_j = s1[P + j], B'_j = s1[j] (stored forms).  Block = (value head, 16 rows of T); thread = column.
__global__ void __launch_bounds__(kD)
    seqpar_combine_kernel(int32_t P, int32_t Hv, const float* __restrict__ s1, const float* __restrict__ s_init,
                          float* __restrict__ s3) {
  extern __shared__ float smc[];
  float* As = smc;                 // [kD][kD] stored A'_j
  float* Ts = smc + kD * kD;       // [kCombRows][kD] rows of T_j
  const int64_t D2 = (int64_t)kD * kD;
  const int groups = kD / kCombRows;
  const int h = blockIdx.x / groups, r0 = (blockIdx.x % groups) * kCombRows, k = threadIdx.x;
  float t[kCombRows];
#pragma unroll
  for (int r = 0; r < kCombRows; ++r) t[r] = s_init ? s_init[h * D2 + (int64_t)(r0 + r) * kD + k] : 0.0f;
  for (int j = 0; j < P; ++j) {
#pragma unroll
    for (int r = 0; r < kCombRows; ++r) s3[((int64_t)j * Hv + h) * D2 + (int64_t)(r0 + r) * kD + k] = t[r];
    if (j == P - 1) break;
    const float* A = s1 + ((int64_t)(P + j) * Hv + h) * D2;
    const float* B = s1 + ((int64_t)j * Hv + h) * D2;
    __syncthreads();  // the previous step's reads of As and Ts are done
    for (int i = k; i < D2 / 4; i += kD) reinterpret_cast<float4*>(As)[i] = reinterpret_cast<const float4*>(A)[i];
#pragma unroll
    for (int r = 0; r < kCombRows; ++r) Ts[r * kD + k] = t[r];
    __syncthreads();
    float acc[kCombRows];
#pragma unroll
    for (int r = 0; r < kCombRows; ++r) acc[r] = B[(int64_t)(r0 + r) * kD + k];
#pragma unroll 4
    for (int l = 0; l < kD; ++l) {
      const float a = As[l * kD + k];
#pragma unroll
      for (int r = 0; r < kCombRows; ++r) acc[r] = fmaf(Ts[r * kD + l], a, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < kCombRows; ++r) t[r] = acc[r];
  }
}

constexpr int kCombSmem = (kD * kD + kCombRows * kD) * 4;

}  // namespace

int seqpar_segments(const Dims& d, int64_t total_tokens, int32_t requested, int32_t sms) {
  const int64_t nchunks = (total_tokens + kC - 1) / kC;
  if (nchunks <= 0) return 1;
  int64_t P = requested > 0 ? requested : (int64_t)sms / (4 * d.Hv);  // phase 1 runs 2 P Hv clusters of two CTAs
  P = P < 1 ? 1 : (P > nchunks ? nchunks : P);
  const int64_t seg_chunks = (nchunks + P - 1) / P;
  return (int)((nchunks + seg_chunks - 1) / seg_chunks);  // every segment non-empty
}

SeqparLayout seqpar_layout(const Dims& d, int64_t total_tokens, int32_t P) {
  SeqparLayout S;
  const int64_t nchunks = (total_tokens + kC - 1) / kC;
  const size_t st = (size_t)d.Hv * kD * kD * 4;
  S.cu1 = 0;
  S.cu_seg = 256;
  S.coff = al256(S.cu_seg + 4 * (size_t)(P + 1));
  S.split = al256(S.coff + 4 * (size_t)P);
  S.s1 = al256(S.split + split_layout(d, total_tokens, nchunks).total_bytes);
  S.s3 = al256(S.s1 + 2 * (size_t)P * st);
  S.total_bytes = al256(S.s3 + (size_t)P * st);
  return S;
}

cudaError_t launch_prefill_seqpar(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                                  const float* norm_w, const void* qkv, const void* z, const void* a, const void* b,
                                  int64_t total_tokens, int32_t P, bool zero_state, bool zero_conv,
                                  const void* conv_state, float* state, void* o, void* ws, int32_t* status,
                                  cudaStream_t stream) {
  if (total_tokens <= 0) return cudaSuccess;
  const int64_t nchunks = (total_tokens + kC - 1) / kC;
  const int32_t seg_chunks = (int32_t)((nchunks + P - 1) / P);
  const SeqparLayout L = seqpar_layout(d, total_tokens, P);
  unsigned char* w = (unsigned char*)ws;
  int32_t* cu1 = (int32_t*)(w + L.cu1);
  int32_t* cu_seg = (int32_t*)(w + L.cu_seg);
  int32_t* coff = (int32_t*)(w + L.coff);
  float* s1 = (float*)(w + L.s1);
  float* s3 = (float*)(w + L.s3);
  const size_t st = (size_t)d.Hv * kD * kD;
  cudaError_t e;
  {  // one segment needs only cu1 (the last block's tables), not the phase-1 slots
    LaunchScope scope(GDN_K_SEQPAR, stream);
    seqpar_init_kernel<<<(unsigned)((P > 1 ? 2 * P * d.Hv : 0) + 1), 256, 0, stream>>>(
        (int32_t)total_tokens, P, seg_chunks, d.Hv, cu1, cu_seg, coff, s1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = launch_stages12(d, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, cu1, nullptr, total_tokens, Window{0, 0},
                           nchunks, total_tokens, split_layout(d, total_tokens, nchunks), zero_conv, conv_state,
                           w + L.split, status, stream)) != cudaSuccess)
    return e;
  const unsigned char* records = w + L.split + split_layout(d, total_tokens, nchunks).records;
  if (P == 1)  // the ordinary carry over the whole sequence
    return launch_chain(d, records, nullptr, nullptr, cu1, d.Hv, zero_state, ChainScan{0, 0x7fffffff}, state, o,
                        status, stream);
  // every segment's B (pairs 0 .. P-1) and A (pairs P .. 2P-1), no output
  if ((e = launch_chain(d, records, coff, nullptr, cu_seg, 2LL * P * d.Hv, false, ChainScan{P, P}, s1, nullptr,
                        status, stream)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(seqpar_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCombSmem)) !=
      cudaSuccess)
    return e;
  {
    LaunchScope scope(GDN_K_SEQPAR, stream);
    seqpar_combine_kernel<<<(unsigned)(d.Hv * (kD / kCombRows)), kD, kCombSmem, stream>>>(
        P, d.Hv, s1, zero_state ? nullptr : state, s3);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // the outputs, every segment from its true starting state; slot P-1 ends with the sequence's final state
  if ((e = launch_chain(d, records, coff, nullptr, cu_seg, (int64_t)P * d.Hv, false, ChainScan{P, 0x7fffffff}, s3,
                        o, status, stream)) != cudaSuccess)
    return e;
  return cudaMemcpyAsync(state, s3 + (size_t)(P - 1) * st, st * sizeof(float), cudaMemcpyDeviceToDevice, stream);
}
}  // namespace gdn
