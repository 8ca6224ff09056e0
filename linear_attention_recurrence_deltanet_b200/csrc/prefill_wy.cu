// Chunked GDN prefill in the affine (transition-matrix) form, for chunk sizes
// 16, 32, 64 and 128 (bf16 io, d_k = d_v = 128), as three kernels: the conv
// of every token, the state-independent operands of every chunk, and the
// state carry across chunks.
//
// The chunkwise (WY/UT) form of the gated delta rule ("fp32 Gated DeltaNet
// recurrence", DS4Server issue #95, implementation comment).  Within a chunk
// of rows r with gamma_r = sum_{i<=r} g_i (the sum restarts at every chunk):
//   A_rj = beta_r e^{gamma_r - gamma_j} k_r.k_j (j < r),   T = (I + A)^-1
//   W = T diag(beta e^gamma) K,   U = T diag(beta) V
//   S' = e^{gamma_C} S + K~^T (U - W S),     K~ = diag(e^{gamma_C - gamma}) K
//   O  = diag(e^gamma) Q S + P (U - W S),    P = M o Q K^T, M_rj = e^{gamma_r - gamma_j} (j <= r)
// Collecting the terms that multiply the state gives an affine map per chunk,
//   S' = e^{gamma_C} S + M' S + K~^T U,   M' = -K~^T W        (d_k x d_k)
//   O  = Q' S + P U,                      Q' = diag(e^gamma) Q - P W
// so the only step that waits for the previous chunk is one product M' S
// (plus Q' S for the outputs, which nothing waits for).
//
//   wy_conv_kernel   grid (tile part, head slot): causal conv + SiLU
//                    ("causal depthwise Conv1D", DS4Server issue #88, Scope),
//                    L2 norms of q and k with epsilon inside the square root;
//                    q^, k^ as fp16 hi + lo parts (row-major) and v^ as fp16
//                    hi + lo operand images per (tile, value head); and the
//                    output gate (1 + w) sigmoid(z) of every value head, fp16.
//   wy_prep_kernel   grid (tile, value head): gates and their per-chunk scan,
//                    [K;Q]K^T in split precision, A and P, T = (I+A)^-1 by
//                    recursive doubling whose merges are tcgen05 MMAs, W and
//                    U, then M' = -K~^T W per chunk and Q' = diag(e^gamma)Q -
//                    P W, all written as byte images of the chain kernel's
//                    shared-memory operands.
//   wy_chain_kernel  grid (sequence, value head, value-channel half), clusters
//                    of the two halves: per chunk Y = K~^T U + M' S and O =
//                    P U + Q' S on tcgen05, S = e^{gamma_C} S + Y in fp32
//                    registers, and the output rows (RMSNorm over d_v times
//                    the gate) by separate warps.
//
// Tiles: the prep and chain kernels work on tiles of 64 rows (chunk sizes 16,
// 32 and 64: a tile holds 64 / C chunks, and every intra-chunk matrix is block
// diagonal within the tile) or of 128 rows (chunk size 128).  Tiles restart at
// every sequence start, so chunk boundaries align with tile boundaries.  The
// three kernels run over windows of at most kWyWindowTokens tokens' tiles, the
// chain carrying each sequence's state from window to window, so that the
// intermediates take a bounded workspace.
//
// Precision: operands are fp16 with fp32 accumulation; where a rounding would
// show in the output or the state the operand is carried as hi + lo parts:
// [K;Q]K^T (hi.hi + hi.lo + lo.hi), T' and v^ in U, U itself, the state in
// the output products (Q'S loses digits to cancellation when q is nearly
// orthogonal to the state's columns) and, at chunk 16, Q'.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/gdn.h"
#include "internal.h"
#include "tc.cuh"

namespace gdn {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr uint64_t kWaitNs = 2000000000ull;
// a wait that runs out is reported as the code in the low byte and the reporting kernel's id above it
constexpr int32_t kTimeoutPrep = kStatusWaitTimeout | (GDN_K_WY_PREP << 8);
constexpr int32_t kTimeoutChain = kStatusWaitTimeout | (GDN_K_WY_CHAIN << 8);

// ------------------------------------------------------------------ record of one (tile, value head)
// Byte images of the chain kernel's operands (fp16, 128-byte swizzle):
//   [0, NCH * 32768)   M'_s of each chunk s of the tile, K-major 128 x 128 (row = output key index)
//   REC_Q              Q', K-major TILE x 128; at chunk 16 followed by its fp16 low part (the
//                      output's error from Q' alone otherwise reaches 2e-3 of o on long sequences)
//   REC_KT             K~, MN-major K=TILE x M=128
//   REC_U              U = T diag(beta) V per value-channel half: [half][hi, lo], MN-major K=TILE x N=64
//   REC_P              P, K-major TILE x TILE
//   REC_META           e^{gamma_C} of each chunk (fp32)
template <int TILE, int C>
struct Rec {
  static constexpr int NCH = TILE / C;
  static constexpr int M = 0;
  static constexpr bool QLO = C == 16;
  static constexpr int Q = NCH * 32768;
  static constexpr int QBYTES = (QLO ? 2 : 1) * TILE * 256;
  static constexpr int KT = Q + QBYTES;
  static constexpr int U = KT + TILE * 256;
  static constexpr int UH = TILE * 128;  // one hi or lo image of one half
  static constexpr int P = U + 4 * UH;
  static constexpr int META = P + TILE * TILE * 2;
  static constexpr int BYTES = META + 256;
};

// A window of the packed tiles handled by one conv + prep + chain pass: global tiles [win_lo, win_hi), whose
// records and v^ images start at entry 0 of the window's buffers and whose per-token parts (q^/k^ rows, gate
// rows) start at row 0 of theirs (token t_base).
struct WyWin {
  int64_t win_lo, win_hi;
  int64_t t_base;
};

// v^ image of one (tile, value head): hi then lo, each MN-major K=TILE x N=128
template <int TILE>
constexpr int kVImg = TILE * 512;

// ------------------------------------------------------------------ wy_conv_kernel
// Block = 8 warps = 64 rows of one tile for one 128-channel head slot (q heads,
// then k heads, then v heads).  Warp w owns rows 8w .. 8w+7 of its 64-row part,
// lane l owns channels 4l .. 4l+3.
constexpr int kConvRows = 8;

template <int TILE>
__global__ void __launch_bounds__(256)
    wy_conv_kernel(Dims d, const float* __restrict__ conv_w, const __nv_bfloat16* __restrict__ qkv,
                   const __nv_bfloat16* __restrict__ hist, int zero_conv, const int4* __restrict__ tile_map,
                   int64_t single_len, __half* __restrict__ qk_hi, __half* __restrict__ qk_lo,
                   unsigned char* __restrict__ vimg, const float* __restrict__ norm_w,
                   const __nv_bfloat16* __restrict__ z, __half* __restrict__ gate, WyWin win) {
  constexpr int SUB = TILE / 64;
  const int part = blockIdx.x % SUB;
  const int gt = (int)(win.win_lo + blockIdx.x / SUB);
  const int64_t rest = single_len - (int64_t)TILE * gt;
  const int4 cm = tile_map ? tile_map[gt] : make_int4(0, TILE * gt, rest < TILE ? (int)rest : TILE, gt);
  const int slot = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = 64 * part + kConvRows * warp;  // first row of this warp within the tile
  const int L = cm.z;
  const int nqk = 2 * d.Hk;
  if (slot >= nqk + d.Hv) {  // the output gate (1 + w_j) sigmoid(z_j) of one value head, fp16
    const int64_t HvD = (int64_t)d.Hv * kD;
    const int64_t col = (int64_t)(slot - nqk - d.Hv) * kD + 4 * lane;
    const float4 w = __ldg(reinterpret_cast<const float4*>(norm_w + 4 * lane));
    const float nw[4] = {1.0f + w.x, 1.0f + w.y, 1.0f + w.z, 1.0f + w.w};
    uint2 u[kConvRows];
#pragma unroll
    for (int i = 0; i < kConvRows; ++i)
      u[i] = (r0 + i < L) ? __ldg(reinterpret_cast<const uint2*>(z + (cm.y + r0 + i) * HvD + col)) : make_uint2(0u, 0u);
#pragma unroll
    for (int i = 0; i < kConvRows; ++i) {
      if (r0 + i < L) {
        const float zz[4] = {__uint_as_float(u[i].x << 16), __uint_as_float(u[i].x & 0xffff0000u),
                             __uint_as_float(u[i].y << 16), __uint_as_float(u[i].y & 0xffff0000u)};
        float g[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) g[e] = nw[e] * __fdividef(1.0f, 1.0f + __expf(-zz[e]));
        st8(reinterpret_cast<unsigned char*>(gate + (cm.y + r0 + i - win.t_base) * HvD + col), g[0], g[1], g[2], g[3]);
      }
    }
    return;
  }
  unsigned char* vrec = slot >= nqk ? vimg + ((gt - win.win_lo) * d.Hv + (slot - nqk)) * kVImg<TILE> : nullptr;
  if (vrec) {  // rows past the tile's end are zero in both parts
#pragma unroll
    for (int i = 0; i < kConvRows; ++i)
      if (r0 + i >= L) {
        *reinterpret_cast<uint2*>(vrec + mnmaj(TILE, r0 + i, 4 * lane)) = make_uint2(0u, 0u);
        *reinterpret_cast<uint2*>(vrec + TILE * 256 + mnmaj(TILE, r0 + i, 4 * lane)) = make_uint2(0u, 0u);
      }
  }
  if (r0 >= L) return;
  const int64_t Cc = d.C;
  const int64_t c = (int64_t)slot * kD + 4 * lane;  // q heads, k heads and v heads are consecutive in qkv
  float w[4][4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(conv_w + (c + e) * 4));
    w[e][0] = x.x; w[e][1] = x.y; w[e][2] = x.z; w[e][3] = x.w;
  }
  // raw rows r0-3 .. r0+7; rows before the sequence start come from the conv history
  uint2 xr[kConvRows + 3];
  const bool first = cm.w == 0;
#pragma unroll
  for (int i = 0; i < kConvRows + 3; ++i) {
    const int rr = r0 - 3 + i;
    xr[i] = make_uint2(0u, 0u);
    if (rr < L) {
      if (first && rr < 0) {
        if (!zero_conv) xr[i] = *reinterpret_cast<const uint2*>(hist + ((int64_t)cm.x * 3 + (3 + rr)) * Cc + c);
      } else {
        xr[i] = __ldg(reinterpret_cast<const uint2*>(qkv + ((int64_t)cm.y + rr) * Cc + c));
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
    for (int i = 0; i < kConvRows; ++i)
      ss[i] = y[i][0] * y[i][0] + y[i][1] * y[i][1] + y[i][2] * y[i][2] + y[i][3] * y[i][3];
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
  } else {  // v: hi and lo images (U is formed from both)
#pragma unroll
    for (int i = 0; i < kConvRows; ++i) {
      if (r0 + i < L) {
        float hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = __half2float(__float2half_rn(y[i][e]));
          lo[e] = y[i][e] - hi[e];
        }
        st8(vrec + mnmaj(TILE, r0 + i, 4 * lane), hi[0], hi[1], hi[2], hi[3]);
        st8(vrec + TILE * 256 + mnmaj(TILE, r0 + i, 4 * lane), lo[0], lo[1], lo[2], lo[3]);
      }
    }
  }
}

// The new conv history of sequence n: the last W-1 raw rows of [history ;
// inputs].  The prep block of the sequence's last tile and value head h owns
// the v channels of h and, for the first value head of a key head, the q and
// k channels of that key head (nothing reads the old history after the conv
// kernel).  One thread per 16 bytes of channels reads its three rows before
// writing them.
__device__ __forceinline__ void write_history(const Dims& d, int h, int n, int64_t seq0, int len,
                                              const __nv_bfloat16* __restrict__ qkv, int zero_conv,
                                              __nv_bfloat16* __restrict__ hist, int tid, int nthreads) {
  const int G = d.G, kh = h / G;
  const int nvec = (h % G == 0 ? 3 : 1) * (kD / 8);
  for (int i = tid; i < nvec; i += nthreads) {
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

// ------------------------------------------------------------------ wy_prep_kernel (64-row tiles)
// One block per (tile, value head), two blocks per SM (111 KB shared memory,
// 256 TMEM columns).  Shared memory:
//   KQH  [K;Q] hi, K-major 128 x 128 (K rows 0..63, Q rows 64..127).  Its K
//        halves, read as MN-major K=64 x N=128 (LBO 16 KB), are the B operand
//        of W = T''K; its Q halves receive v^ lo (MN-major, LBO 16 KB) as soon
//        as [K;Q]K^T is done, so that copy overlaps the solve.
//   KQL  [K;Q] lo.  After [K;Q]K^T: Aoff16 (+0), Aoff32 (+8192), T (+16384),
//        X (+24576), K-major 64 x 64 each, the fp32 16x16 diagonal blocks of
//        A in X's place until X is first written; after the solve T'hi (+0),
//        T'lo (+8192), T'' (+24576); after W, -W as MN-major K=64 x N=128
//        (+16384, LBO 8 KB).
//   V    v^ hi, MN-major K=64 x N=128 (LBO 8 KB).
//   KT   K~, MN-major K=64 x M=128 (LBO 8 KB).
//   PS   P, K-major 64 x 64.
//   TF   the 16x16 diagonal blocks of T in fp32 (T' and T'' take them from here).
// TMEM (256 columns): [K;Q]K^T in 0..63, the solve's products in 64..127,
// diag(e^gamma) Q and then Q' in 128..255 (M = 64 layout), W, U and M' in turn
// in 0..127.
// A 64-row 64 x 64 tile is stored in the same bytes whether it is read as a
// K-major A operand (rows = M) or an MN-major B operand (rows = K), so T and X
// serve both roles of the solve's products without a copy.
constexpr int kPrepThreads = 256;
constexpr int WP_KQH = 0;
constexpr int WP_KQL = 32768;
constexpr int WP_V = 65536;
constexpr int WP_KT = 81920;
constexpr int WP_P = 98304;
constexpr int WP_MISC = WP_P + 8192;
constexpr int WP_VLO = WP_KQH + 8192;
constexpr int WP_DIAG = WP_KQL + 24576;
constexpr int WP_AOFF16 = WP_KQL;
constexpr int WP_AOFF32 = WP_KQL + 8192;
constexpr int WP_T = WP_KQL + 16384;
constexpr int WP_X = WP_KQL + 24576;
constexpr int WP_TPH = WP_KQL;
constexpr int WP_TPL = WP_KQL + 8192;
constexpr int WP_TPP = WP_KQL + 24576;
constexpr int WP_NW = WP_KQL + 16384;
constexpr int WP_TF = WP_MISC + 7 * 64 * 4;  // the 16x16 diagonal blocks of T in fp32 (4 KB)
constexpr int kPrepSmem = WP_TF + 4096 + 1024;
constexpr uint32_t kPrepTmemCols = 256;
constexpr uint32_t TP_M1 = 0, TP_SOLVE = 64, TP_Q = 128, TP_BIG = 0;

// 16x16 block and 2b x 2b block structure of the doubling: element (r, j), j < r,
// of a chunk's A belongs to the level b = 16, 32, 64 whose blocks first put
// r and j in different halves, or to a 16x16 diagonal block when r ^ j < 16.

template <int C>
__global__ void __launch_bounds__(kPrepThreads, 2)
    wy_prep_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo, Dims d,
                   const int4* __restrict__ tile_map, const unsigned char* __restrict__ vimg,
                   unsigned char* __restrict__ records, const int32_t* __restrict__ cu,
                   const __nv_bfloat16* __restrict__ qkv, int zero_conv, __nv_bfloat16* __restrict__ hist,
                   const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                   const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b, int64_t single_len,
                   WyWin win, int32_t* status) {
  constexpr int TILE = 64;
  using R = Rec<TILE, C>;
  constexpr int NCH = R::NCH;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t mb_tma, mb_mma, mb_vlo;
  __shared__ uint32_t tslot;
  bool bad = false;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = blockIdx.x / d.Hv;  // tiles in reverse order: the first tiles are the freshest in L2 for the chain
  const int h = blockIdx.x - gr * d.Hv;
  const int g = (int)(win.win_lo + gridDim.x / d.Hv - 1 - gr);
  const int kh = h / d.G;
  const int64_t rest = single_len - (int64_t)TILE * g;
  const int4 cm = tile_map ? tile_map[g] : make_int4(0, TILE * g, rest < TILE ? (int)rest : TILE, g);
  const int64_t t0 = cm.y;
  const int trow = (int)(t0 - win.t_base);  // the tile's first row in the window's q^/k^ buffers
  const int L = cm.z;
  const int64_t gw = g - win.win_lo;  // the tile's entry in the window's buffers
  unsigned char* rec = records + (gw * d.Hv + h) * R::BYTES;

  float* misc = reinterpret_cast<float*>(sm + WP_MISC);
  float* s_g = misc;            // g_r, then gamma_r (in-chunk inclusive sum)
  float* s_beta = misc + 64;    // beta_r (0 past the tile's end)
  float* s_eg = misc + 128;     // e^{gamma_r}
  float* s_ekd = misc + 192;    // e^{gamma_C - gamma_r} (0 past the tile's end)
  float* s_tbg = misc + 256;    // beta_r e^{gamma_r}
  float* s_gam = misc + 320;    // gamma_r

  if (tid == 0) {
    mbar_init(&mb_tma, 1);
    mbar_init(&mb_mma, 1);
    mbar_init(&mb_vlo, 1);
    mbar_init_fence();
    mbar_expect_tx(&mb_tma, 8 * 8192 + 16384);
    const int qx = kh * kD, kx = d.Hk * kD + kh * kD;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      tma_load_2d(sm + WP_KQH + j * 16384, &tm_hi, kx + 64 * j, trow, &mb_tma);
      tma_load_2d(sm + WP_KQH + j * 16384 + 8192, &tm_hi, qx + 64 * j, trow, &mb_tma);
      tma_load_2d(sm + WP_KQL + j * 16384, &tm_lo, kx + 64 * j, trow, &mb_tma);
      tma_load_2d(sm + WP_KQL + j * 16384 + 8192, &tm_lo, qx + 64 * j, trow, &mb_tma);
    }
    bulk_load(sm + WP_V, vimg + (gw * d.Hv + h) * kVImg<TILE>, 16384, &mb_tma);
  }
  if (warp == 0) tmem_alloc(&tslot, kPrepTmemCols);
  {  // the block of a sequence's last tile writes the sequence's new conv history for its channels
    const int64_t s0 = tile_map ? cu[cm.x] : 0, s1 = tile_map ? cu[cm.x + 1] : single_len;
    if (t0 + TILE >= s1) write_history(d, h, cm.x, s0, (int)(s1 - s0), qkv, zero_conv, hist, tid, kPrepThreads);
  }
  // gates of the tile's rows, and their inclusive sum within each chunk
  if (tid < TILE) {
    float gg = 0.f, be = 0.f;
    if (tid < L) {
      gg = -expf(A_log[h]) * softplus_f(__bfloat162float(a[(t0 + tid) * d.Hv + h]) + dt_bias[h]);
      be = 1.0f / (1.0f + expf(-__bfloat162float(b[(t0 + tid) * d.Hv + h])));
    }
    s_g[tid] = gg;
    s_beta[tid] = be;
  }
  __syncthreads();
  float gam = 0.f, gC = 0.f;
  if (tid < TILE) {
    const int c0 = tid - tid % C;
    for (int i = c0; i < c0 + C; ++i) {
      const float gi = s_g[i];
      if (i <= tid) gam += gi;
      gC += gi;  // g = 0 past the tile's end: the chunk's total decay is over its valid rows
    }
  }
  __syncthreads();
  if (tid < TILE) {
    const bool ok = tid < L;
    s_gam[tid] = gam;
    s_eg[tid] = expf(gam);
    s_ekd[tid] = ok ? expf(gC - gam) : 0.f;
    s_tbg[tid] = s_beta[tid] * expf(gam);
    if (tid % C == C - 1) reinterpret_cast<float*>(rec + R::META)[tid / C] = expf(gC);
  }
  sync_tc();
  const uint32_t tbase = tslot;
  if (!mbar_wait(&mb_tma, 0, kWaitNs)) bad = true;
  if (sync_tc_any(bad)) {
    if (tid == 0) {
      set_status(status, kTimeoutPrep);
      bulk_wait<0>();  // no record image is still being read from shared memory
    }
    if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
    return;
  }

  // M1: [K;Q] K^T as hi.hi + hi.lo + lo.hi
  uint32_t mma_phase = 0;
  if (tid == 0) {
    const uint32_t kq = smem_u32(sm + WP_KQH), kql = smem_u32(sm + WP_KQL);
    constexpr uint32_t id = idesc_f16(128, 64, false, false);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase + TP_M1, desc_kmaj(kq, 128, s), desc_kmaj(kq, 128, s), id, s > 0);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase + TP_M1, desc_kmaj(kq, 128, s), desc_kmaj(kql, 128, s), id, 1);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase + TP_M1, desc_kmaj(kql, 128, s), desc_kmaj(kq, 128, s), id, 1);
    mma_commit(&mb_mma);
  }
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
  const int hc = warp >> 2;
  // meanwhile: K~ = e^{gamma_C - gamma} (k^ hi + lo) -> shared (MN-major) and the record;
  // Qg = e^gamma (q^ hi + lo) -> TMEM columns 128..255 in the M = 64 layout
  for (int e = tid; e < 64 * 16; e += kPrepThreads) {
    const int r = e >> 4, c8 = 8 * (e & 15);
    const uint32_t ok = kmaj_chunk(128, r, c8);
    const uint4 uk = *reinterpret_cast<const uint4*>(sm + WP_KQH + ok);
    const uint4 lk = *reinterpret_cast<const uint4*>(sm + WP_KQL + ok);
    const float ek = s_ekd[r];
    const __half2* hk = reinterpret_cast<const __half2*>(&uk);
    const __half2* hkl = reinterpret_cast<const __half2*>(&lk);
    float fk[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 b2 = __half22float2(hk[i]), b3 = __half22float2(hkl[i]);
      fk[2 * i] = (b2.x + b3.x) * ek;
      fk[2 * i + 1] = (b2.y + b3.y) * ek;
    }
    *reinterpret_cast<uint4*>(sm + WP_KT + mnmaj_chunk(64, r, c8)) = pack8h(fk);
  }
  fence_async_smem();  // K~ is read by the bulk store below and by the M' products
  {
    const int r16 = 16 * (warp & 3) + (lane & 15);  // M = 64 layout: row r16 in lane (r16 % 16) + 32 (r16 / 16)
    float v[32];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cb = 64 * hc + 32 * hh;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint32_t oq = kmaj_chunk(128, 64 + r16, cb + 8 * m);
        const uint4 uq = *reinterpret_cast<const uint4*>(sm + WP_KQH + oq);
        const uint4 lq = *reinterpret_cast<const uint4*>(sm + WP_KQL + oq);
        const __half2* hq = reinterpret_cast<const __half2*>(&uq);
        const __half2* hql = reinterpret_cast<const __half2*>(&lq);
        const float eg = s_eg[r16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 a2 = __half22float2(hq[i]), a3 = __half22float2(hql[i]);
          v[8 * m + 2 * i] = (a2.x + a3.x) * eg;
          v[8 * m + 2 * i + 1] = (a2.y + a3.y) * eg;
        }
      }
      if (lane >= 16) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      tmem_st32(tbase + lane_base + TP_Q + cb, v);
    }
  }
  if (!mbar_wait(&mb_mma, mma_phase, kWaitNs)) bad = true;
  mma_phase ^= 1;
  if (sync_tc_any(bad)) {  // also: the tiles are read; KQL and the Q halves of KQH are free
    if (tid == 0) {
      set_status(status, kTimeoutPrep);
      bulk_wait<0>();  // no record image is still being read from shared memory
    }
    if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
    return;
  }
  if (tid == 0) {  // v^ lo into the Q halves of KQH (MN-major, LBO 16 KB), behind the generic reads of q^
    fence_async_smem();
    mbar_expect_tx(&mb_vlo, 16384);
    const unsigned char* vl = vimg + (gw * d.Hv + h) * kVImg<TILE> + TILE * 256;
    bulk_load(sm + WP_VLO, vl, 8192, &mb_vlo);
    bulk_load(sm + WP_VLO + 16384, vl + 8192, 8192, &mb_vlo);
    bulk_store(rec + R::KT, sm + WP_KT, 16384);  // the K~ image goes to the record as it is
    bulk_commit();
  }

  // A (rows 0..63 of M1) into the diagonal fp32 blocks and the two level images;
  // P (rows 64..127) into shared memory and the record
  {
    const int si = 32 * (warp & 3) + lane;
    float v[32];
    tmem_ld32(tbase + lane_base + TP_M1 + 32 * hc, v);
    if (si < 64) {
      const int r = si;
      const float br = s_beta[r], gr = s_gam[r];
      float a16[8], a32[8];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = 32 * hc + 8 * m + e;
          const bool same = (j / C) == (r / C);
          const float av = (j < r && same) ? br * __expf(gr - s_gam[j]) * v[8 * m + e] : 0.f;
          const int x = r ^ j;
          a16[e] = (x >= 16 && x < 32) ? av : 0.f;
          a32[e] = (x >= 32) ? av : 0.f;
          if (x < 16) reinterpret_cast<float*>(sm + WP_DIAG)[(r >> 4) * 272 + (r & 15) * 17 + (j & 15)] = av;
        }
        *reinterpret_cast<uint4*>(sm + WP_AOFF16 + kmaj_chunk(64, r, 32 * hc + 8 * m)) = pack8h(a16);
        *reinterpret_cast<uint4*>(sm + WP_AOFF32 + kmaj_chunk(64, r, 32 * hc + 8 * m)) = pack8h(a32);
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
          const bool same = (j / C) == (r / C);
          p[e] = (j <= r && same) ? __expf(gr - s_gam[j]) * v[8 * m + e] : 0.f;
        }
        *reinterpret_cast<uint4*>(sm + WP_P + kmaj_chunk(64, r, 32 * hc + 8 * m)) = pack8h(p);
      }
    }
  }
  for (int i = tid; i < 8192 / 16; i += kPrepThreads)
    reinterpret_cast<uint4*>(sm + WP_T)[i] = make_uint4(0, 0, 0, 0);
  fence_async_smem();
  __syncthreads();
  if (tid == 0) {  // the P image goes to the record as it is
    bulk_store(rec + R::P, sm + WP_P, 8192);
    bulk_commit();
  }
  // T = (I + A)^-1, level 0: the 16x16 diagonal blocks by forward substitution,
  // one column of one block per thread, in fp32: kept in fp32 for T' and T''
  // (the doubling levels never change these blocks) and as fp16 in the T image
  if (tid < 64) {
    const int bb = tid >> 4, c = tid & 15, o = 16 * bb;
    const float* Ad = reinterpret_cast<const float*>(sm + WP_DIAG) + bb * 272;
    float* Tf = reinterpret_cast<float*>(sm + WP_TF) + bb * 256;
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
      *reinterpret_cast<__half*>(sm + WP_T + kmaj(64, o + i, o + c)) = __float2half_rn(t[i]);
      Tf[i * 16 + c] = t[i];
    }
  }
  fence_async_smem();
  sync_tc();
  // levels b = 16 (C >= 32) and b = 32 (C = 64): T <- T - T (Aoff_b T), every
  // merge of two b-blocks at once; the products on tcgen05 (M = N = K = 64)
  const int r16 = 16 * (warp & 3) + (lane & 15);
  bool abort = false;  // block-uniform
#pragma unroll
  for (int lv = 0; lv < 2; ++lv) {
    if ((lv == 0 && C < 32) || (lv == 1 && C < 64)) continue;
    const uint32_t aoff = smem_u32(sm + (lv == 0 ? WP_AOFF16 : WP_AOFF32));
    const uint32_t ts = smem_u32(sm + WP_T), xs = smem_u32(sm + WP_X);
    constexpr uint32_t id = idesc_f16(64, 64, false, true);
    if (tid == 0) {  // X = Aoff T
#pragma unroll
      for (int s = 0; s < 4; ++s) mma_f16(tbase + TP_SOLVE, desc_kmaj(aoff, 64, s), desc_mnmaj(ts, 64, s), id, s > 0);
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, mma_phase, kWaitNs)) bad = true;
    mma_phase ^= 1;
    fence_after();
    {
      float v[32];
      tmem_ld32(tbase + lane_base + TP_SOLVE + 32 * hc, v);
      if (lane < 16) {
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint4*>(sm + WP_X + kmaj_chunk(64, r16, 32 * hc + 8 * m)) = pack8h(v + 8 * m);
      }
    }
    fence_async_smem();
    sync_tc();
    if (tid == 0) {  // Y = T X
#pragma unroll
      for (int s = 0; s < 4; ++s) mma_f16(tbase + TP_SOLVE, desc_kmaj(ts, 64, s), desc_mnmaj(xs, 64, s), id, s > 0);
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, mma_phase, kWaitNs)) bad = true;
    mma_phase ^= 1;
    fence_after();
    {
      float v[32];
      tmem_ld32(tbase + lane_base + TP_SOLVE + 32 * hc, v);
      if (lane < 16) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          unsigned char* p = sm + WP_T + kmaj_chunk(64, r16, 32 * hc + 8 * m);
          const uint4 tq = *reinterpret_cast<const uint4*>(p);
          const __half2* t2 = reinterpret_cast<const __half2*>(&tq);
          float nt[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(t2[i]);
            nt[2 * i] = f.x - v[8 * m + 2 * i];
            nt[2 * i + 1] = f.y - v[8 * m + 2 * i + 1];
          }
          *reinterpret_cast<uint4*>(p) = pack8h(nt);
        }
      }
    }
    fence_async_smem();
    if (sync_tc_any(bad)) {
      abort = true;
      break;
    }
  }
  if (abort) {
    if (tid == 0) {
      set_status(status, kTimeoutPrep);
      bulk_wait<0>();  // no record image is still being read from shared memory
    }
    if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
    return;
  }
  {  // T' = T diag(beta) as fp16 hi + lo, T'' = T diag(beta e^gamma), K-major 64 x 64; a thread's 16
     // columns are one 16-column block: the diagonal one comes from the fp32 blocks
    const int r = tid >> 2, j0 = 16 * (tid & 3);
    float t1[16], t2[16], tl[16], tv[16];
    if ((tid & 3) == (r >> 4)) {
      const float4* tf = reinterpret_cast<const float4*>(sm + WP_TF) + (r >> 4) * 64 + (r & 15) * 4;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 f = tf[m];
        tv[4 * m] = f.x; tv[4 * m + 1] = f.y; tv[4 * m + 2] = f.z; tv[4 * m + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const uint4 tq = *reinterpret_cast<const uint4*>(sm + WP_T + kmaj_chunk(64, r, j0 + 8 * m));
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
      t1[jj] = tv[jj] * s_beta[j0 + jj];
      t2[jj] = tv[jj] * s_tbg[j0 + jj];
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) tl[i] = t1[i] - __half2float(__float2half_rn(t1[i]));
    __syncthreads();  // every thread has read its rows of T (T' hi lands over Aoff16, T'' over X)
    st16h(sm + WP_TPH + kmaj_chunk(64, r, j0), t1);
    st16h(sm + WP_TPH + kmaj_chunk(64, r, j0 + 8), t1 + 8);
    st16h(sm + WP_TPL + kmaj_chunk(64, r, j0), tl);
    st16h(sm + WP_TPL + kmaj_chunk(64, r, j0 + 8), tl + 8);
    st16h(sm + WP_TPP + kmaj_chunk(64, r, j0), t2);
    st16h(sm + WP_TPP + kmaj_chunk(64, r, j0 + 8), t2 + 8);
  }
  fence_async_smem();
  sync_tc();
  // W = T'' K  (M = 64, N = 128; B = the k^ hi rows of KQH read as MN-major, LBO 16 KB)
  if (tid == 0) {
    const uint32_t ta = smem_u32(sm + WP_TPP), kq = smem_u32(sm + WP_KQH);
    constexpr uint32_t id = idesc_f16(64, 128, false, true);
#pragma unroll
    for (int s = 0; s < 4; ++s) mma_f16(tbase + TP_BIG, desc_kmaj(ta, 64, s), sdesc(kq + s * 2048, 16384, 1024), id, s > 0);
    mma_commit(&mb_mma);
  }
  if (!mbar_wait(&mb_mma, mma_phase, kWaitNs)) bad = true;
  mma_phase ^= 1;
  fence_after();
  {  // -W -> MN-major K=64 x N=128 (LBO 8 KB)
    float v[32];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      tmem_ld32(tbase + lane_base + TP_BIG + 64 * hc + 32 * hh, v);
      if (lane < 16) {
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) v[jj] = -v[jj];
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint4*>(sm + WP_NW + mnmaj_chunk(64, r16, 64 * hc + 32 * hh + 8 * m)) = pack8h(v + 8 * m);
      }
    }
  }
  fence_async_smem();
  if (sync_tc_any(bad)) {
    if (tid == 0) {
      set_status(status, kTimeoutPrep);
      bulk_wait<0>();  // no record image is still being read from shared memory
    }
    if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
    return;
  }
  // U = T'hi V hi + T'lo V hi + T'hi V lo (columns 0..127), Q' = Qg + P (-W) (columns 128..255)
  if (tid == 0) {
    const uint32_t th = smem_u32(sm + WP_TPH), tl = smem_u32(sm + WP_TPL), vb = smem_u32(sm + WP_V),
                   vlb = smem_u32(sm + WP_VLO), pa = smem_u32(sm + WP_P), nw = smem_u32(sm + WP_NW);
    constexpr uint32_t id = idesc_f16(64, 128, false, true);
#pragma unroll
    for (int s = 0; s < 4; ++s) mma_f16(tbase + TP_Q, desc_kmaj(pa, 64, s), sdesc(nw + s * 2048, 8192, 1024), id, 1);
#pragma unroll
    for (int s = 0; s < 4; ++s) mma_f16(tbase + TP_BIG, desc_kmaj(th, 64, s), sdesc(vb + s * 2048, 8192, 1024), id, s > 0);
#pragma unroll
    for (int s = 0; s < 4; ++s) mma_f16(tbase + TP_BIG, desc_kmaj(tl, 64, s), sdesc(vb + s * 2048, 8192, 1024), id, 1);
    if (!mbar_wait(&mb_vlo, 0, kWaitNs)) bad = true;
    if (!bad) {
#pragma unroll
      for (int s = 0; s < 4; ++s)
        mma_f16(tbase + TP_BIG, desc_kmaj(th, 64, s), sdesc(vlb + s * 2048, 16384, 1024), id, 1);
    }
    mma_commit(&mb_mma);
  }
  if (!mbar_wait(&mb_mma, mma_phase, kWaitNs)) bad = true;
  mma_phase ^= 1;
  fence_after();
  {  // U -> its record image (hi + lo per value-channel half) staged in KQH; Q' -> its image staged in V
    float v[32];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cb = 64 * hc + 32 * hh;  // value channels cb .. cb + 31, all in half hc
      tmem_ld32(tbase + lane_base + TP_BIG + cb, v);
      if (lane < 16) {
        unsigned char* uh = sm + WP_KQH + hc * 2 * R::UH;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float hi[8], lo[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            hi[e] = __half2float(__float2half_rn(v[8 * m + e]));
            lo[e] = v[8 * m + e] - hi[e];
          }
          const uint32_t off = mnmaj_chunk(TILE, r16, 32 * hh + 8 * m);
          *reinterpret_cast<uint4*>(uh + off) = pack8h(hi);
          *reinterpret_cast<uint4*>(uh + R::UH + off) = pack8h(lo);
        }
      }
      tmem_ld32(tbase + lane_base + TP_Q + cb, v);
      if (lane < 16) {
        const bool ok = r16 < L;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float q8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) q8[e] = ok ? v[8 * m + e] : 0.f;
          *reinterpret_cast<uint4*>(sm + WP_V + kmaj_chunk(TILE, r16, cb + 8 * m)) = pack8h(q8);
          if (R::QLO) {  // the low part goes over T' (read by the products just completed)
#pragma unroll
            for (int e = 0; e < 8; ++e) q8[e] -= __half2float(__float2half_rn(q8[e]));
            *reinterpret_cast<uint4*>(sm + WP_KQL + kmaj_chunk(TILE, r16, cb + 8 * m)) = pack8h(q8);
          }
        }
      }
    }
  }
  fence_async_smem();
  if (sync_tc_any(bad)) {  // also: columns 0..127 are read out
    if (tid == 0) {
      set_status(status, kTimeoutPrep);
      bulk_wait<0>();  // no record image is still being read from shared memory
    }
    if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
    return;
  }
  if (tid == 0) {
    bulk_store(rec + R::U, sm + WP_KQH, 4 * R::UH);
    bulk_store(rec + R::Q, sm + WP_V, TILE * 256);
    if (R::QLO) bulk_store(rec + R::Q + TILE * 256, sm + WP_KQL, TILE * 256);
    bulk_commit();
  }
  // M'_s = K~_s^T (-W_s) for each chunk s of the tile (M = N = 128, K = the chunk's rows)
  const int si = 32 * (warp & 3) + lane;
#pragma unroll 1
  for (int s = 0; s < NCH; ++s) {
    if (s * C >= L) break;  // chunks past the tile's end are never read
    if (tid == 0) {
      const uint32_t kt = smem_u32(sm + WP_KT), nw = smem_u32(sm + WP_NW);
      constexpr uint32_t id = idesc_f16(128, 128, true, true);
#pragma unroll
      for (int k = 0; k < C / 16; ++k) {
        const int st = s * (C / 16) + k;
        mma_f16(tbase + TP_BIG, sdesc(kt + st * 2048, 8192, 1024), sdesc(nw + st * 2048, 8192, 1024), id, k > 0);
      }
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, mma_phase, kWaitNs)) bad = true;
    mma_phase ^= 1;
    if (tid == 0) bulk_wait_read<0>();  // the staging area (KQH) has been read by the previous bulk store
    __syncthreads();
    fence_after();
    {  // M'_s -> its record image staged in KQH
      float v[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        tmem_ld32(tbase + lane_base + TP_BIG + 64 * hc + 32 * hh, v);
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint4*>(sm + WP_KQH + kmaj_chunk(128, si, 64 * hc + 32 * hh + 8 * m)) = pack8h(v + 8 * m);
      }
    }
    fence_async_smem();
    if (sync_tc_any(bad)) {
      abort = true;
      break;
    }
    if (tid == 0) {
      bulk_store(rec + R::M + s * 32768, sm + WP_KQH, 32768);
      bulk_commit();
    }
  }
  if (tid == 0) {
    if (abort) set_status(status, kTimeoutPrep);
    bulk_wait<0>();  // every record image has left shared memory
  }
  if (warp == 0) tmem_dealloc(tbase, kPrepTmemCols);
}

// ------------------------------------------------------------------ wy_prep128_kernel (chunk 128)
// One block per (128-row tile, value head); one block per SM (205 KB shared
// memory, all 512 TMEM columns).  The same steps as the 64-row kernel on
// 128 x 128 matrices, with one more doubling level (b = 64).  Shared memory:
//   KH   k^ hi, K-major 128 x 128 (rows = tokens); read as MN-major (LBO 16 KB)
//        it is the B operand of W = T''K; after W it receives v^ hi.
//   KL   k^ lo; after [K;Q]K^T: T; after T' and T'': -W (MN-major, LBO 16 KB).
//   QH   q^ hi; after [K;Q]K^T: A (fp16, strictly lower); after the solve T'hi;
//        after U: P, copied back from the record for P(-W).
//   QL   q^ lo; after [K;Q]K^T: the level image Aoff_b; after the solve T'lo.
//   X    the solve's product X (the fp32 16x16 diagonal blocks of A until X is
//        first written); after the solve T''; after W, v^ lo.
//   KT   K~, MN-major K=128 x M=128 (LBO 16 KB).
// TMEM: K K^T then W in 0..127, Q K^T then U in 128..255, the solve's
// products then M' in 256..383, diag(e^gamma) Q then Q' in 384..511.
constexpr int W8_KH = 0, W8_KL = 32768, W8_QH = 65536, W8_QL = 98304, W8_X = 131072, W8_KT = 163840,
              W8_MISC = 196608;
constexpr int W8_TF = W8_MISC + 7 * 128 * 4;  // the 16x16 diagonal blocks of T in fp32 (8 KB)
constexpr int kPrep128Smem = W8_TF + 8192 + 1024;
constexpr uint32_t T8_KK = 0, T8_QK = 128, T8_SOLVE = 256, T8_Q = 384;

__global__ void __launch_bounds__(kPrepThreads, 1)
    wy_prep128_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo, Dims d,
                      const int4* __restrict__ tile_map, const unsigned char* __restrict__ vimg,
                      unsigned char* __restrict__ records, const int32_t* __restrict__ cu,
                      const __nv_bfloat16* __restrict__ qkv, int zero_conv, __nv_bfloat16* __restrict__ hist,
                      const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                      const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b, int64_t single_len,
                      WyWin win, int32_t* status) {
  constexpr int TILE = 128;
  using R = Rec<128, 128>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t mb_tma, mb_mma, mb_v, mb_p;
  __shared__ uint32_t tslot;
  bool bad = false, abort = false;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = blockIdx.x / d.Hv;
  const int h = blockIdx.x - gr * d.Hv;
  const int g = (int)(win.win_lo + gridDim.x / d.Hv - 1 - gr);
  const int kh = h / d.G;
  const int64_t rest = single_len - (int64_t)TILE * g;
  const int4 cm = tile_map ? tile_map[g] : make_int4(0, TILE * g, rest < TILE ? (int)rest : TILE, g);
  const int64_t t0 = cm.y;
  const int trow = (int)(t0 - win.t_base);  // the tile's first row in the window's q^/k^ buffers
  const int L = cm.z;
  const int64_t gw = g - win.win_lo;  // the tile's entry in the window's buffers
  unsigned char* rec = records + (gw * d.Hv + h) * R::BYTES;
  const unsigned char* vsrc = vimg + (gw * d.Hv + h) * kVImg<TILE>;

  float* misc = reinterpret_cast<float*>(sm + W8_MISC);
  float* s_g = misc;
  float* s_beta = misc + 128;
  float* s_eg = misc + 256;
  float* s_ekd = misc + 384;
  float* s_tbg = misc + 512;
  float* s_gam = misc + 640;

  if (tid == 0) {
    mbar_init(&mb_tma, 1);
    mbar_init(&mb_mma, 1);
    mbar_init(&mb_v, 1);
    mbar_init(&mb_p, 1);
    mbar_init_fence();
    mbar_expect_tx(&mb_tma, 16 * 8192);
    const int qx = kh * kD, kx = d.Hk * kD + kh * kD;
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int rh = 0; rh < 2; ++rh) {  // 64-column block j, 64-row half rh
        const int y = trow + 64 * rh, o = j * 16384 + rh * 8192;
        tma_load_2d(sm + W8_KH + o, &tm_hi, kx + 64 * j, y, &mb_tma);
        tma_load_2d(sm + W8_KL + o, &tm_lo, kx + 64 * j, y, &mb_tma);
        tma_load_2d(sm + W8_QH + o, &tm_hi, qx + 64 * j, y, &mb_tma);
        tma_load_2d(sm + W8_QL + o, &tm_lo, qx + 64 * j, y, &mb_tma);
      }
  }
  if (warp == 0) tmem_alloc(&tslot, 512);
  {
    const int64_t s0 = tile_map ? cu[cm.x] : 0, s1 = tile_map ? cu[cm.x + 1] : single_len;
    if (t0 + TILE >= s1) write_history(d, h, cm.x, s0, (int)(s1 - s0), qkv, zero_conv, hist, tid, kPrepThreads);
  }
  if (tid < TILE) {
    float gg = 0.f, be = 0.f;
    if (tid < L) {
      gg = -expf(A_log[h]) * softplus_f(__bfloat162float(a[(t0 + tid) * d.Hv + h]) + dt_bias[h]);
      be = 1.0f / (1.0f + expf(-__bfloat162float(b[(t0 + tid) * d.Hv + h])));
    }
    s_g[tid] = gg;
    s_beta[tid] = be;
  }
  __syncthreads();
  float gam = 0.f, gC = 0.f;
  if (tid < TILE) {
    for (int i = 0; i < TILE; ++i) {
      const float gi = s_g[i];
      if (i <= tid) gam += gi;
      gC += gi;
    }
  }
  __syncthreads();
  if (tid < TILE) {
    const bool ok = tid < L;
    s_gam[tid] = gam;
    s_eg[tid] = expf(gam);
    s_ekd[tid] = ok ? expf(gC - gam) : 0.f;
    s_tbg[tid] = s_beta[tid] * expf(gam);
    if (tid == TILE - 1) reinterpret_cast<float*>(rec + R::META)[0] = expf(gC);
  }
  sync_tc();
  const uint32_t tbase = tslot;
  if (!mbar_wait(&mb_tma, 0, kWaitNs)) bad = true;
  if (sync_tc_any(bad)) {
    if (tid == 0) set_status(status, kTimeoutPrep);
    if (warp == 0) tmem_dealloc(tbase, 512);
    return;
  }
  uint32_t ph = 0;
  // M1: K K^T and Q K^T, each as hi.hi + hi.lo + lo.hi (M = N = 128)
  if (tid == 0) {
    const uint32_t khs = smem_u32(sm + W8_KH), kls = smem_u32(sm + W8_KL), qhs = smem_u32(sm + W8_QH),
                   qls = smem_u32(sm + W8_QL);
    constexpr uint32_t id = idesc_f16(128, 128, false, false);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase + T8_KK, desc_kmaj(khs, 128, s), desc_kmaj(khs, 128, s), id, s > 0);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase + T8_KK, desc_kmaj(khs, 128, s), desc_kmaj(kls, 128, s), id, 1);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase + T8_KK, desc_kmaj(kls, 128, s), desc_kmaj(khs, 128, s), id, 1);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase + T8_QK, desc_kmaj(qhs, 128, s), desc_kmaj(khs, 128, s), id, s > 0);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase + T8_QK, desc_kmaj(qhs, 128, s), desc_kmaj(kls, 128, s), id, 1);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_f16(tbase + T8_QK, desc_kmaj(qls, 128, s), desc_kmaj(khs, 128, s), id, 1);
    mma_commit(&mb_mma);
  }
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
  const int hc = warp >> 2;
  const int si = 32 * (warp & 3) + lane;  // M = 128 layout: row si in lane si
  // meanwhile K~ -> shared (MN-major) and the record; Qg -> TMEM 384..511
  for (int e = tid; e < 128 * 16; e += kPrepThreads) {
    const int r = e >> 4, c8 = 8 * (e & 15);
    const uint32_t ok = kmaj_chunk(128, r, c8);
    const uint4 uk = *reinterpret_cast<const uint4*>(sm + W8_KH + ok);
    const uint4 lk = *reinterpret_cast<const uint4*>(sm + W8_KL + ok);
    const float ek = s_ekd[r];
    const __half2* hk = reinterpret_cast<const __half2*>(&uk);
    const __half2* hkl = reinterpret_cast<const __half2*>(&lk);
    float fk[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 b2 = __half22float2(hk[i]), b3 = __half22float2(hkl[i]);
      fk[2 * i] = (b2.x + b3.x) * ek;
      fk[2 * i + 1] = (b2.y + b3.y) * ek;
    }
    const uint4 pk = pack8h(fk);
    *reinterpret_cast<uint4*>(sm + W8_KT + mnmaj_chunk(128, r, c8)) = pk;
    *reinterpret_cast<uint4*>(rec + R::KT + mnmaj_chunk(128, r, c8)) = pk;
  }
  {
    float v[32];
    const float eg = s_eg[si];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cb = 64 * hc + 32 * hh;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint32_t oq = kmaj_chunk(128, si, cb + 8 * m);
        const uint4 uq = *reinterpret_cast<const uint4*>(sm + W8_QH + oq);
        const uint4 lq = *reinterpret_cast<const uint4*>(sm + W8_QL + oq);
        const __half2* hq = reinterpret_cast<const __half2*>(&uq);
        const __half2* hql = reinterpret_cast<const __half2*>(&lq);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 a2 = __half22float2(hq[i]), a3 = __half22float2(hql[i]);
          v[8 * m + 2 * i] = (a2.x + a3.x) * eg;
          v[8 * m + 2 * i + 1] = (a2.y + a3.y) * eg;
        }
      }
      tmem_st32(tbase + lane_base + T8_Q + cb, v);
    }
  }
  if (!mbar_wait(&mb_mma, ph, kWaitNs)) bad = true;
  ph ^= 1;
  if (sync_tc_any(bad)) {
    if (tid == 0) set_status(status, kTimeoutPrep);
    if (warp == 0) tmem_dealloc(tbase, 512);
    return;
  }
  // A -> fp16 image in QH (strictly lower) and fp32 16x16 diagonal blocks in X; P -> the record
  {
    const float br = s_beta[si], gr = s_gam[si];
    float v[32];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cb = 64 * hc + 32 * hh;
      tmem_ld32(tbase + lane_base + T8_KK + cb, v);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float a8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = cb + 8 * m + e;
          const float av = (j < si) ? br * __expf(gr - s_gam[j]) * v[8 * m + e] : 0.f;
          a8[e] = av;
          if ((si ^ j) < 16) reinterpret_cast<float*>(sm + W8_X)[(si >> 4) * 256 + (si & 15) * 16 + (j & 15)] = av;
        }
        *reinterpret_cast<uint4*>(sm + W8_QH + kmaj_chunk(128, si, cb + 8 * m)) = pack8h(a8);
      }
      tmem_ld32(tbase + lane_base + T8_QK + cb, v);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float p8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = cb + 8 * m + e;
          p8[e] = (j <= si) ? __expf(gr - s_gam[j]) * v[8 * m + e] : 0.f;
        }
        *reinterpret_cast<uint4*>(rec + R::P + kmaj_chunk(128, si, cb + 8 * m)) = pack8h(p8);
      }
    }
  }
  for (int i = tid; i < 32768 / 16; i += kPrepThreads) reinterpret_cast<uint4*>(sm + W8_KL)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (tid < 128) {  // level 0: the eight 16x16 diagonal blocks of T, one column per thread
    const int bb = tid >> 4, c = tid & 15, o = 16 * bb;
    const float* Ad = reinterpret_cast<const float*>(sm + W8_X) + bb * 256;
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = (i == c) ? 1.f : 0.f;
#pragma unroll
      for (int k = 0; k < i; ++k) acc -= Ad[i * 16 + k] * t[k];
      t[i] = (i < c) ? 0.f : acc;
    }
    float* Tf = reinterpret_cast<float*>(sm + W8_TF) + bb * 256;  // kept in fp32 for T' and T''
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      *reinterpret_cast<__half*>(sm + W8_KL + kmaj(128, o + i, o + c)) = __float2half_rn(t[i]);
      Tf[i * 16 + c] = t[i];
    }
  }
  fence_async_smem();
  sync_tc();
  // levels b = 16, 32, 64: T <- T - T (Aoff_b T), Aoff_b masked out of A into QL first
#pragma unroll 1
  for (int bl = 16; bl <= 64; bl <<= 1) {
    for (int e = tid; e < 128 * 16; e += kPrepThreads) {
      const int r = e >> 4, c8 = 8 * (e & 15);
      const uint32_t off = kmaj_chunk(128, r, c8);
      uint4 u = *reinterpret_cast<const uint4*>(sm + W8_QH + off);
      __half* hv = reinterpret_cast<__half*>(&u);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int x = r ^ (c8 + i);
        if (!(x >= bl && x < 2 * bl)) hv[i] = __float2half_rn(0.f);
      }
      *reinterpret_cast<uint4*>(sm + W8_QL + off) = u;
    }
    fence_async_smem();
    sync_tc();
    const uint32_t aoff = smem_u32(sm + W8_QL), ts = smem_u32(sm + W8_KL), xs = smem_u32(sm + W8_X);
    constexpr uint32_t id = idesc_f16(128, 128, false, true);
    if (tid == 0) {
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_f16(tbase + T8_SOLVE, desc_kmaj(aoff, 128, s), sdesc(ts + s * 2048, 16384, 1024), id, s > 0);
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, ph, kWaitNs)) bad = true;
    ph ^= 1;
    fence_after();
    {
      float v[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int cb = 64 * hc + 32 * hh;
        tmem_ld32(tbase + lane_base + T8_SOLVE + cb, v);
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint4*>(sm + W8_X + kmaj_chunk(128, si, cb + 8 * m)) = pack8h(v + 8 * m);
      }
    }
    fence_async_smem();
    sync_tc();
    if (tid == 0) {
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_f16(tbase + T8_SOLVE, desc_kmaj(ts, 128, s), sdesc(xs + s * 2048, 16384, 1024), id, s > 0);
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, ph, kWaitNs)) bad = true;
    ph ^= 1;
    fence_after();
    {
      float v[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int cb = 64 * hc + 32 * hh;
        tmem_ld32(tbase + lane_base + T8_SOLVE + cb, v);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          unsigned char* p = sm + W8_KL + kmaj_chunk(128, si, cb + 8 * m);
          const uint4 tq = *reinterpret_cast<const uint4*>(p);
          const __half2* t2 = reinterpret_cast<const __half2*>(&tq);
          float nt[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(t2[i]);
            nt[2 * i] = f.x - v[8 * m + 2 * i];
            nt[2 * i + 1] = f.y - v[8 * m + 2 * i + 1];
          }
          *reinterpret_cast<uint4*>(p) = pack8h(nt);
        }
      }
    }
    fence_async_smem();
    if (sync_tc_any(bad)) {
      abort = true;
      break;
    }
  }
  if (abort) {
    if (tid == 0) set_status(status, kTimeoutPrep);
    if (warp == 0) tmem_dealloc(tbase, 512);
    return;
  }
  {  // T' = T diag(beta) hi -> QH, lo -> QL; T'' = T diag(beta e^gamma) -> X
    const int r = tid >> 1, j0 = 64 * (tid & 1);
#pragma unroll 1
    for (int q = 0; q < 8; ++q) {
      const int jb = j0 + 8 * q;
      float tv[8], t1[8], t2[8], tl[8];
      if ((jb >> 4) == (r >> 4)) {  // the diagonal 16x16 block: its fp32 values (the levels never change it)
        const float4* tf = reinterpret_cast<const float4*>(sm + W8_TF) + (r >> 4) * 64 + (r & 15) * 4 + ((jb & 15) >> 2);
        const float4 f0 = tf[0], f1 = tf[1];
        tv[0] = f0.x; tv[1] = f0.y; tv[2] = f0.z; tv[3] = f0.w;
        tv[4] = f1.x; tv[5] = f1.y; tv[6] = f1.z; tv[7] = f1.w;
      } else {
        const uint4 tq = *reinterpret_cast<const uint4*>(sm + W8_KL + kmaj_chunk(128, r, jb));
        const __half2* h2 = reinterpret_cast<const __half2*>(&tq);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(h2[i]);
          tv[2 * i] = f.x;
          tv[2 * i + 1] = f.y;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        t1[i] = tv[i] * s_beta[jb + i];
        t2[i] = tv[i] * s_tbg[jb + i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) tl[i] = t1[i] - __half2float(__float2half_rn(t1[i]));
      const uint32_t off = kmaj_chunk(128, r, jb);
      *reinterpret_cast<uint4*>(sm + W8_QH + off) = pack8h(t1);
      *reinterpret_cast<uint4*>(sm + W8_QL + off) = pack8h(tl);
      *reinterpret_cast<uint4*>(sm + W8_X + off) = pack8h(t2);
    }
  }
  fence_async_smem();
  sync_tc();
  // W = T'' K (M = N = K = 128)
  if (tid == 0) {
    const uint32_t ta = smem_u32(sm + W8_X), khs = smem_u32(sm + W8_KH);
    constexpr uint32_t id = idesc_f16(128, 128, false, true);
#pragma unroll
    for (int s = 0; s < 8; ++s)
      mma_f16(tbase + T8_KK, desc_kmaj(ta, 128, s), sdesc(khs + s * 2048, 16384, 1024), id, s > 0);
    mma_commit(&mb_mma);
  }
  if (!mbar_wait(&mb_mma, ph, kWaitNs)) bad = true;
  ph ^= 1;
  fence_after();
  if (tid == 0 && !bad) {  // k^ hi and T'' are read: v^ hi and lo take their places (MN-major, LBO 16 KB)
    fence_async_smem();
    mbar_expect_tx(&mb_v, 65536);
    bulk_load(sm + W8_KH, vsrc, 32768, &mb_v);
    bulk_load(sm + W8_X, vsrc + TILE * 256, 32768, &mb_v);
  }
  {  // -W -> KL, MN-major K=128 x N=128 (LBO 16 KB)
    float v[32];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cb = 64 * hc + 32 * hh;
      tmem_ld32(tbase + lane_base + T8_KK + cb, v);
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) v[jj] = -v[jj];
#pragma unroll
      for (int m = 0; m < 4; ++m)
        *reinterpret_cast<uint4*>(sm + W8_KL + mnmaj_chunk(128, si, cb + 8 * m)) = pack8h(v + 8 * m);
    }
  }
  fence_async_smem();
  if (sync_tc_any(bad)) {
    if (tid == 0) set_status(status, kTimeoutPrep);
    if (warp == 0) tmem_dealloc(tbase, 512);
    return;
  }
  // M' = K~^T (-W) (columns 256..383); U = T'hi V hi + T'lo V hi + T'hi V lo (columns 128..255)
  if (tid == 0) {
    const uint32_t kt = smem_u32(sm + W8_KT), nw = smem_u32(sm + W8_KL), th = smem_u32(sm + W8_QH),
                   tl = smem_u32(sm + W8_QL), vh = smem_u32(sm + W8_KH), vl = smem_u32(sm + W8_X);
    constexpr uint32_t idm = idesc_f16(128, 128, true, true), idu = idesc_f16(128, 128, false, true);
#pragma unroll
    for (int s = 0; s < 8; ++s)
      mma_f16(tbase + T8_SOLVE, sdesc(kt + s * 2048, 16384, 1024), sdesc(nw + s * 2048, 16384, 1024), idm, s > 0);
    if (!mbar_wait(&mb_v, 0, kWaitNs)) bad = true;
    if (!bad) {
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_f16(tbase + T8_QK, desc_kmaj(th, 128, s), sdesc(vh + s * 2048, 16384, 1024), idu, s > 0);
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_f16(tbase + T8_QK, desc_kmaj(tl, 128, s), sdesc(vh + s * 2048, 16384, 1024), idu, 1);
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_f16(tbase + T8_QK, desc_kmaj(th, 128, s), sdesc(vl + s * 2048, 16384, 1024), idu, 1);
    }
    mma_commit(&mb_mma);
  }
  if (!mbar_wait(&mb_mma, ph, kWaitNs)) bad = true;
  ph ^= 1;
  fence_after();
  if (tid == 0 && !bad) {  // T' is read: P comes back from the record into QH for P (-W)
    fence_async_all();  // this block's generic writes of P (before the block barriers above) -> the bulk copy
    mbar_expect_tx(&mb_p, 32768);
    bulk_load(sm + W8_QH, rec + R::P, 32768, &mb_p);
  }
  {  // M' (K-major 128 x 128) staged in KT and U (hi + lo per value-channel half) in KH (half 0) and X
     // (half 1), all read by the products just completed; they go to the record by bulk stores
    float v[32];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cb = 64 * hc + 32 * hh;
      tmem_ld32(tbase + lane_base + T8_SOLVE + cb, v);
#pragma unroll
      for (int m = 0; m < 4; ++m)
        *reinterpret_cast<uint4*>(sm + W8_KT + kmaj_chunk(128, si, cb + 8 * m)) = pack8h(v + 8 * m);
      tmem_ld32(tbase + lane_base + T8_QK + cb, v);
      unsigned char* uh = sm + (hc == 0 ? W8_KH : W8_X);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          hi[e] = __half2float(__float2half_rn(v[8 * m + e]));
          lo[e] = v[8 * m + e] - hi[e];
        }
        const uint32_t off = mnmaj_chunk(TILE, si, 32 * hh + 8 * m);
        *reinterpret_cast<uint4*>(uh + off) = pack8h(hi);
        *reinterpret_cast<uint4*>(uh + R::UH + off) = pack8h(lo);
      }
    }
  }
  fence_async_smem();
  __syncthreads();
  if (tid == 0) {
    bulk_store(rec + R::M, sm + W8_KT, 32768);
    bulk_store(rec + R::U, sm + W8_KH, 2 * R::UH);
    bulk_store(rec + R::U + 2 * R::UH, sm + W8_X, 2 * R::UH);
    bulk_commit();
  }
  // Q' = Qg + P (-W) (columns 384..511)
  if (tid == 0) {
    if (!mbar_wait(&mb_p, 0, kWaitNs)) bad = true;
    if (!bad) {
      const uint32_t pa = smem_u32(sm + W8_QH), nw = smem_u32(sm + W8_KL);
      constexpr uint32_t id = idesc_f16(128, 128, false, true);
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_f16(tbase + T8_Q, desc_kmaj(pa, 128, s), sdesc(nw + s * 2048, 16384, 1024), id, 1);
    }
    mma_commit(&mb_mma);
  }
  if (!mbar_wait(&mb_mma, ph, kWaitNs)) bad = true;
  ph ^= 1;
  fence_after();
  {  // Q' staged in QL (T' lo, read by U) and written by a bulk store
    float v[32];
    const bool ok = si < L;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cb = 64 * hc + 32 * hh;
      tmem_ld32(tbase + lane_base + T8_Q + cb, v);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float q8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) q8[e] = ok ? v[8 * m + e] : 0.f;
        *reinterpret_cast<uint4*>(sm + W8_QL + kmaj_chunk(TILE, si, cb + 8 * m)) = pack8h(q8);
      }
    }
  }
  fence_async_smem();
  const bool fail = sync_tc_any(bad);
  if (tid == 0) {
    if (fail) set_status(status, kTimeoutPrep);
    bulk_store(rec + R::Q, sm + W8_QL, TILE * 256);
    bulk_commit();
    bulk_wait<0>();  // every record image has left shared memory
  }
  if (warp == 0) tmem_dealloc(tbase, 512);
}

// ------------------------------------------------------------------ wy_chain_kernel
// One cluster of two CTAs per (sequence, value head); CTA `vh` of the pair
// carries value channels [64 vh, 64 vh + 64), i.e. 64 columns of the state,
// which evolve independently of the other 64.  Per chunk c (chunk s of its
// tile):
//   Y_c = K~_s^T U_s,  O_c = P_s U_s   (nothing from the state: issued a chunk ahead)
//   Y_c += M'_c S_c                    (the one product on the carry's path)
//   S_{c+1} = e^{gamma_C} S_c + Y_c    (fp32 registers; its fp16 copy is the next operand)
//   O_c += Q' S_c                      (rows of chunk s; nothing waits for it)
// then RMSNorm over all d_v (row sums exchanged with the peer CTA) times the
// output gate, bf16 out.  The output products carry the state as fp16 hi + lo
// parts (Q'S loses up to half of o's digits to cancellation when q is nearly
// orthogonal to the state's columns): B = [S hi | S lo] and [U hi | U lo] as
// N = 128 operands, the two column blocks of O summed by the output warps.
// Warps 0..7 carry the state (thread: key row 32 (w % 4) + lane, columns
// 32 (w / 4) .. + 31 of this half); warps 8..11 write the output rows; warp 12
// issues the products with the state (Y += M'S, O += Q'S), warp 14 the
// state-free ones (issuing a tcgen05.mma takes its thread tens of cycles, so
// the two streams of MMAs go out in parallel), warp 13 the bulk copies.
// Every wait is bounded.
template <int TILE, int C>
struct ChainCfg {
  static constexpr int NCH = TILE / C;
  static constexpr int NM = TILE == 64 ? 2 : 1;    // M' buffers
  static constexpr int NB = TILE == 64 && C != 16 ? 2 : 1;  // K~, U, P buffers (Q' has one)
  static constexpr int MB = 0;                                  // M' K-major 128 x 128, 32 KB each
  static constexpr int SB = MB + NM * 32768;                    // S copies (2): hi, lo MN-major K=128 x N=64
  static constexpr int QB = SB + 2 * 32768;                     // Q' (hi, and lo at chunk 16) K-major TILE x 128
  static constexpr int KTB = QB + Rec<TILE, C>::QBYTES;         // K~ MN-major K=TILE x M=128
  static constexpr int UB = KTB + NB * TILE * 256;              // U of this half: hi, lo MN-major K=TILE x N=64
  static constexpr int PB = UB + NB * TILE * 256;               // P K-major TILE x TILE
  static constexpr int MISC = PB + NB * TILE * TILE * 2;
  static constexpr int MS_PEER = 0;               // the peer's row sums [2][TILE]
  static constexpr int MISC_BYTES = 2 * TILE * 4;
  static constexpr int SMEM = MISC + MISC_BYTES + 1024;
};
constexpr int kChainThreads = 480;
constexpr int kEaSlots = 8;  // commits of the state-free products, slot c % 8
// TMEM: Y_c in columns 64 (c % 2), O_c in 128 + 128 (c % 3) (the hi and lo column blocks)
constexpr uint32_t CY0 = 0, CO0 = 128, kChainTmemCols = 512;
constexpr int kOBufs = 3;

template <int TILE, int C>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kChainThreads, 1)
    wy_chain_kernel(Dims d, const unsigned char* __restrict__ records,
                    const int32_t* __restrict__ tile_off, const int32_t* __restrict__ order,
                    const int32_t* __restrict__ cu, int zero_state, const __half* __restrict__ gate, WyWin win,
                    float* __restrict__ state, __nv_bfloat16* __restrict__ o, int32_t* status) {
  using R = Rec<TILE, C>;
  using F = ChainCfg<TILE, C>;
  constexpr int NCH = F::NCH, NM = F::NM, NB = F::NB;
  constexpr int OM = TILE == 64 ? 64 : 128;  // M of the output products
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t mb_m[NM], mb_ta[NB], mb_tq;      // copies: M', tile operands (K~, U, P), Q'
  __shared__ uint64_t mb_s;                            // S_c is in shared memory (8 state warps)
  __shared__ uint64_t mb_ea[kEaSlots];                 // commit of chunk c's state-free products (warp 14)
  __shared__ uint64_t mb_yf[2];                        // the state warps have read Y_c, slot c % 2 (8 warps)
  __shared__ uint64_t mb_y[2];                         // commit of Y_c (and every earlier MMA), slot c % 2
  __shared__ uint64_t mb_o[kOBufs];                    // commit of O_c (and every earlier MMA), slot c % 3
  __shared__ uint64_t mb_e[kOBufs];                    // output warps done reading O_c (4 warps), slot c % 3
  __shared__ uint64_t mb_x[2];                         // the peer's row sums of chunk c arrived
  __shared__ uint32_t tslot;
  bool bad = false;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vh = (int)cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int h = pair % d.Hv;
  const int n = order ? order[pair / d.Hv] : pair / d.Hv;
  const int len_all = cu[n + 1] - cu[n];
  if (len_all <= 0) return;  // both CTAs of the cluster, before any cluster barrier
  // the sequence's tiles inside the window; the state carries in from the previous window (or from zero at
  // the sequence's first tile) and out to the next
  const int64_t gfirst = tile_off ? tile_off[n] : 0, win_lo = win.win_lo, t_base = win.t_base;
  const int64_t ga = max(gfirst, win_lo), gb = min(gfirst + (len_all + TILE - 1) / TILE, (int64_t)win.win_hi);
  if (ga >= gb) return;  // both CTAs of the cluster, before any cluster barrier
  const int tile0 = (int)(ga - gfirst);
  const int64_t seq0 = cu[n] + (int64_t)tile0 * TILE;                   // this window's first token of the sequence
  const int len = min(len_all - tile0 * TILE, (int)(gb - ga) * TILE);   // and its number of tokens here
  const int ntiles = (len + TILE - 1) / TILE;
  const int nsteps = (len + C - 1) / C;
  const int64_t g0 = ga - win_lo;
  // with several windows a zero start is written into `state` before the first one, so zero_state is only
  // set when the whole sequence is in this window
  const bool zero_here = zero_state;
  const int64_t HvD = (int64_t)d.Hv * kD;
  const bool state_warp = warp < 8, out_warp = warp >= 8 && warp < 12, mma_warp = warp == 12,
             copy_warp = warp == 13, early_warp = warp == 14;
  float* s_peer = reinterpret_cast<float*>(sm + F::MISC + F::MS_PEER);
  float* gst = state + ((int64_t)n * d.Hv + h) * kD * kD;  // stored [j][i]

  if (tid == 0) {
    for (int i = 0; i < NM; ++i) mbar_init(&mb_m[i], 1);
    for (int i = 0; i < NB; ++i) {
      mbar_init(&mb_ta[i], 1);

    }
    mbar_init(&mb_tq, 1);
    mbar_init(&mb_s, 8);
    for (int i = 0; i < kEaSlots; ++i) mbar_init(&mb_ea[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&mb_yf[i], 8);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&mb_y[i], 1);
      mbar_init(&mb_x[i], 1);  // one local arrival with the expected bytes; the peer's stores complete them
    }
    for (int i = 0; i < kOBufs; ++i) {
      mbar_init(&mb_o[i], 1);
      mbar_init(&mb_e[i], 4);
    }
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(&tslot, kChainTmemCols);

  auto rec_of = [&](int t) { return records + ((g0 + t) * d.Hv + h) * (int64_t)R::BYTES; };
  auto issue_ops = [&](int t) {  // K~, U of this half, P
    const int b = t % NB;
    const unsigned char* r = rec_of(t);
    mbar_expect_tx(&mb_ta[b], TILE * 256 + TILE * 256 + TILE * TILE * 2);
    bulk_load(sm + F::KTB + b * TILE * 256, r + R::KT, TILE * 256, &mb_ta[b]);
    bulk_load(sm + F::UB + b * TILE * 256, r + R::U + vh * 2 * R::UH, 2 * R::UH, &mb_ta[b]);
    bulk_load(sm + F::PB + b * TILE * TILE * 2, r + R::P, TILE * TILE * 2, &mb_ta[b]);
  };
  auto issue_q = [&](int t) {
    mbar_expect_tx(&mb_tq, R::QBYTES);
    bulk_load(sm + F::QB, rec_of(t) + R::Q, R::QBYTES, &mb_tq);
  };
  auto issue_m = [&](int c) {
    const int b = c % NM;
    mbar_expect_tx(&mb_m[b], 32768);
    bulk_load(sm + F::MB + b * 32768, rec_of(c / NCH) + R::M + (c % NCH) * 32768, 32768, &mb_m[b]);
  };
  float S[32];
  const int si = 32 * (warp & 3) + lane, hc = (warp >> 2) & 1;
  const int c0 = 64 * vh + 32 * hc;  // first value channel of a state thread's columns
  if (state_warp) {
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) S[jj] = zero_here ? 0.f : gst[(int64_t)(c0 + jj) * kD + si];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float lo[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) lo[e] = S[8 * m + e] - __half2float(__float2half_rn(S[8 * m + e]));
      st16h(sm + F::SB + mnmaj_chunk(kD, si, 32 * hc + 8 * m), S + 8 * m);
      st16h(sm + F::SB + 16384 + mnmaj_chunk(kD, si, 32 * hc + 8 * m), lo);
    }
  }
  fence_async_smem();
  sync_tc();
  const uint32_t tbase = tslot;
  // the first copies go out only after the block barrier that publishes the mbarriers' initialisation
  if (copy_warp && lane == 0) {
    for (int t = 0; t < NB && t < ntiles; ++t) issue_ops(t);
    issue_q(0);
    for (int c = 0; c < NM && c < nsteps; ++c) issue_m(c);
  }
  cluster_sync();  // the peer's mbarriers are initialised before any arrival on them
  const uint32_t peer = (uint32_t)(vh ^ 1);
  const uint32_t peer_x0 = mapa_shared(smem_u32(&mb_x[0]), peer), peer_x1 = mapa_shared(smem_u32(&mb_x[1]), peer);
  const uint32_t peer_sums = mapa_shared(smem_u32(s_peer), peer);
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;

  if (early_warp) {
    if (lane == 0) {
      const uint32_t id_y = idesc_f16(128, 64, true, true);  // K~^T U: A MN-major
      const uint32_t id_o = idesc_f16(OM, 128, false, true);  // P [U hi | U lo]
      // Y_c = K~_s^T U_s and O_c = P_s U_s need nothing from the state: they go out ahead of the carry, and
      // their commit tells warp 12 that Y_c and O_c may take the state's products, and the copy warp when
      // the tile's operand buffer is free again
      for (int c = 0; c < nsteps && !bad; ++c) {
        const int t = c / NCH, s = c % NCH, b = t % NB;
        if (s == 0 && !mbar_wait(&mb_ta[b], (t / NB) & 1, kWaitNs)) bad = true;
        // Y buffer c % 2 is free once the state warps have read Y_{c-2}; O buffer c % 3 once the output
        // warps have read O_{c-3}
        if (c >= 2 && !mbar_wait(&mb_yf[c & 1], ((c - 2) >> 1) & 1, kWaitNs)) bad = true;
        if (c >= kOBufs && !mbar_wait(&mb_e[c % kOBufs], ((c - kOBufs) / kOBufs) & 1, kWaitNs)) bad = true;
        tc::fence_after();
        if (bad) break;
        const uint32_t kt = smem_u32(sm + F::KTB + b * TILE * 256), ub = smem_u32(sm + F::UB + b * TILE * 256),
                       pb = smem_u32(sm + F::PB + b * TILE * TILE * 2);
        const uint32_t y = tbase + CY0 + 64 * (c & 1), od = tbase + CO0 + 128 * (c % kOBufs);
#pragma unroll
        for (int k = 0; k < C / 16; ++k) {
          const int st = s * (C / 16) + k;
          mma_f16(y, sdesc(kt + st * 2048, TILE * 128, 1024), sdesc(ub + st * 2048, TILE * 128, 1024), id_y, k > 0);
          mma_f16(y, sdesc(kt + st * 2048, TILE * 128, 1024), sdesc(ub + TILE * 128 + st * 2048, TILE * 128, 1024),
                  id_y, 1);
        }
#pragma unroll
        for (int k = 0; k < C / 16; ++k) {
          const int st = s * (C / 16) + k;
          mma_f16(od, desc_kmaj(pb, TILE, st), sdesc(ub + st * 2048, TILE * 128, 1024), id_o, k > 0);
        }
        mma_commit(&mb_ea[c % kEaSlots]);
      }
    }
  } else if (mma_warp) {
    if (lane == 0) {
      const uint32_t id_ys = idesc_f16(128, 64, false, true);  // M' S
      const uint32_t id_o = idesc_f16(OM, 128, false, true);   // Q' [S hi | S lo]
      for (int c = 0; c < nsteps && !bad; ++c) {
        const int t = c / NCH, s = c % NCH;
        if (!mbar_wait(&mb_m[c % NM], (c / NM) & 1, kWaitNs)) bad = true;
        // S_c in shared memory (S_0 was written before the block barrier; S_c, c >= 1, completes phase c - 1)
        if (c > 0 && !mbar_wait(&mb_s, (c - 1) & 1, kWaitNs)) bad = true;
        // the state-free parts of Y_c and O_c are in place (issued by warp 14)
        if (!mbar_wait(&mb_ea[c % kEaSlots], (c / kEaSlots) & 1, kWaitNs)) bad = true;
        tc::fence_after();
        if (bad) break;
        const uint32_t ma = smem_u32(sm + F::MB + (c % NM) * 32768), sb = smem_u32(sm + F::SB + (c & 1) * 32768);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_f16(tbase + CY0 + 64 * (c & 1), desc_kmaj(ma, 128, k), desc_mnmaj(sb, kD, k), id_ys, 1);
        mma_commit(&mb_y[c & 1]);
        if (s == 0 && !mbar_wait(&mb_tq, t & 1, kWaitNs)) bad = true;
        if (bad) break;
        const uint32_t qb = smem_u32(sm + F::QB), od = tbase + CO0 + 128 * (c % kOBufs);
#pragma unroll
        for (int k = 0; k < 8; ++k) mma_f16(od, desc_kmaj(qb, TILE, k), desc_mnmaj(sb, kD, k), id_o, 1);
        if (R::QLO) {
#pragma unroll
          for (int k = 0; k < 8; ++k) mma_f16(od, desc_kmaj(qb + TILE * 256, TILE, k), desc_mnmaj(sb, kD, k), id_o, 1);
        }
        mma_commit(&mb_o[c % kOBufs]);
      }
    }
  } else if (copy_warp) {
    if (lane == 0) {
      for (int c = 0; c < nsteps && !bad; ++c) {
        const int t = c / NCH;
        const bool tile_end = c % NCH == NCH - 1 || c == nsteps - 1;
        // the tile's K~, U, P are free once the state-free products of its last chunk are done
        if (!mbar_wait(&mb_ea[c % kEaSlots], (c / kEaSlots) & 1, kWaitNs)) bad = true;
        if (bad) break;
        if (tile_end && t + NB < ntiles) issue_ops(t + NB);
        // M'_c and the tile's Q' are free once O_c is done (its commit covers every earlier MMA)
        if (!mbar_wait(&mb_y[c & 1], (c >> 1) & 1, kWaitNs)) bad = true;
        if (!mbar_wait(&mb_o[c % kOBufs], (c / kOBufs) & 1, kWaitNs)) bad = true;
        if (bad) break;
        if (c + NM < nsteps) issue_m(c + NM);
        if (tile_end && t + 1 < ntiles) issue_q(t + 1);
      }
    }
  } else if (state_warp) {
    // e^{gamma_C} of chunk c, read from the record two chunks ahead (it is not on the tile buffers' path)
    auto eg_of = [&](int c) {
      return c < nsteps ? __ldg(reinterpret_cast<const float*>(rec_of(c / NCH) + R::META) + c % NCH) : 0.f;
    };
    float egA = eg_of(0), egB = eg_of(1);
    for (int c = 0; c < nsteps; ++c) {
      if (!mbar_wait(&mb_y[c & 1], (c >> 1) & 1, kWaitNs)) bad = true;
      tc::fence_after();
      if (bad) break;
      float y[32];
      tmem_ld32(tbase + lane_base + CY0 + 64 * (c & 1) + 32 * hc, y);
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&mb_yf[c & 1]);  // Y buffer c % 2 may take Y_{c+2}'s state-free part
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) S[jj] = egA * S[jj] + y[jj];
      if (c + 1 < nsteps) {
        unsigned char* sbn = sm + F::SB + ((c + 1) & 1) * 32768;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float lo[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) lo[e] = S[8 * m + e] - __half2float(__float2half_rn(S[8 * m + e]));
          st16h(sbn + mnmaj_chunk(kD, si, 32 * hc + 8 * m), S + 8 * m);
          st16h(sbn + 16384 + mnmaj_chunk(kD, si, 32 * hc + 8 * m), lo);
        }
        fence_async_smem();
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&mb_s);
      }
      egA = egB;
      egB = eg_of(c + 2);
    }
  } else if (out_warp) {
    const int q = warp - 8;
    const int r = TILE == 64 ? 16 * q + (lane & 15) : 32 * q + lane;  // this thread's row of the tile
    const bool has_row = TILE == 64 ? lane < 16 : true;
    // the gate row (128 bytes) of this thread's row of chunk c: prefetched into L2 a few chunks ahead
    // (a plain per-row prefetch: nothing asynchronous outlives the block), loaded one chunk ahead
    constexpr int kGAhead = 3;
    const __half* gate_r = gate + (seq0 - t_base + r) * HvD + (int64_t)h * kD + 64 * vh;  // row r of tile 0
    auto gate_row = [&](int c) -> const __half* {
      const int t = c / NCH, s = c % NCH;
      if (c < nsteps && has_row && (r / C) == s && (t * TILE + r) < len) return gate_r + (int64_t)t * TILE * HvD;
      return nullptr;
    };
    uint4 gr[8];
    auto load_gate = [&](int c) {
      if (const __half* p = gate_row(c)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) gr[i] = __ldg(reinterpret_cast<const uint4*>(p) + i);
      }
    };
    for (int c = 0; c < kGAhead; ++c)
      if (const __half* p = gate_row(c)) asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
    load_gate(0);
    for (int c = 0; c < nsteps; ++c) {
      const int t = c / NCH, s = c % NCH;
      const bool mine = has_row && (r / C) == s;
      const int64_t tok = seq0 + (int64_t)t * TILE + r;
      const bool valid = mine && (t * TILE + r) < len;
      if (!mbar_wait(&mb_o[c % kOBufs], (c / kOBufs) & 1, kWaitNs)) bad = true;
      tc::fence_after();
      // O = its hi column block + its lo block, read 16 columns at a time (warp-collective: every lane)
      float v[16], vl[16], ss = 0.f;
      const uint32_t ob = tbase + lane_base + CO0 + 128 * (c % kOBufs);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        tmem_ld16(ob + 16 * q, v);
        tmem_ld16(ob + 64 + 16 * q, vl);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          v[j] += vl[j];
          ss += v[j] * v[j];
        }
      }
      if (mine) st_async_f32(peer_sums + 4 * (TILE * (c & 1) + r), ss, (c & 1) ? peer_x1 : peer_x0);
      if (warp == 8 && lane == 0) mbar_expect_tx(&mb_x[c & 1], C * 4);  // the local arrival of this phase
      if (!mbar_wait_cluster(&mb_x[c & 1], (c >> 1) & 1, kWaitNs)) bad = true;
      const float rinv = valid ? rsqrtf((ss + s_peer[TILE * (c & 1) + r]) * (1.0f / kD) + d.norm_eps) : 0.f;
      __nv_bfloat16* orow = o + tok * HvD + (int64_t)h * kD + 64 * vh;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        tmem_ld16(ob + 16 * q, v);
        tmem_ld16(ob + 64 + 16 * q, vl);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] += vl[j];
        if (q == 3) {  // the products of chunk c are read: the buffer takes chunk c+3's
          tc::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&mb_e[c % kOBufs]);
        }
        if (valid) {
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const uint4 gq = gr[2 * q + m];
            const __half2* g2 = reinterpret_cast<const __half2*>(&gq);
            uint32_t ow[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 gf = __half22float2(g2[e]);
              __nv_bfloat162 pr = __floats2bfloat162_rn(v[8 * m + 2 * e] * rinv * gf.x, v[8 * m + 2 * e + 1] * rinv * gf.y);
              ow[e] = *reinterpret_cast<uint32_t*>(&pr);
            }
            *reinterpret_cast<uint4*>(orow + 16 * q + 8 * m) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
          }
        }
      }
      if (const __half* p = gate_row(c + kGAhead)) asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
      if (c + 1 < nsteps) load_gate(c + 1);
      if (bad) break;
    }
  }
  if (sync_tc_any(bad)) {
    if (tid == 0) set_status(status, kTimeoutChain);
  } else if (state_warp) {
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) gst[(int64_t)(c0 + jj) * kD + si] = S[jj];
  }
  sync_tc();
  if (warp == 0) tmem_dealloc(tbase, kChainTmemCols);
  cluster_sync();  // no CTA leaves while its peer may still write its row sums
}

bool encode_2d(EncodeTiledFn enc, CUtensorMap* tm, const void* base, uint64_t cols, uint64_t rows) {
  const cuuint64_t dim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t stride[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dim, stride, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t rec_bytes(int chunk) {
  switch (chunk) {
    case 16: return Rec<64, 16>::BYTES;
    case 32: return Rec<64, 32>::BYTES;
    case 64: return Rec<64, 64>::BYTES;
    default: return Rec<128, 128>::BYTES;
  }
}

template <int TILE, int C>
cudaError_t launch_wy(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                      const float* norm_w, const void* qkv, const void* z, const void* a, const void* b,
                      const int32_t* cu, const int32_t* cu_host, const int32_t* order, const int32_t* tile_off,
                      const int4* tile_map, int32_t N, int64_t total_tokens, int64_t total_tiles, bool zero_state,
                      bool zero_conv, const void* conv_state, float* state, void* o, void* ws, int32_t* status,
                      cudaStream_t stream) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  // The tiles go through conv, prep and the chain one window at a time, so that the intermediates take a
  // bounded workspace whatever the length; the chain carries each sequence's state from window to window
  // through `state`.
  const int64_t W = wy_window_tiles(total_tiles, C);
  const WyLayout Lw = wy_layout(d, std::min<int64_t>(total_tokens, W * TILE), W, C);
  unsigned char* w = (unsigned char*)ws;
  __half* qk_hi = (__half*)(w + Lw.qk_hi);
  __half* qk_lo = (__half*)(w + Lw.qk_lo);
  unsigned char* vimg = w + Lw.vimg;
  __half* gate = (__half*)(w + Lw.gate);
  unsigned char* records = w + Lw.records;
  const uint64_t qkw = (uint64_t)2 * d.Hk * kD;
  using F = ChainCfg<TILE, C>;
  cudaError_t e;
  if constexpr (TILE == 64) {
    if ((e = cudaFuncSetAttribute(wy_prep_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPrepSmem)) !=
        cudaSuccess)
      return e;
  } else {
    if ((e = cudaFuncSetAttribute(wy_prep128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kPrep128Smem)) != cudaSuccess)
      return e;
  }
  if ((e = cudaFuncSetAttribute(wy_chain_kernel<TILE, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM)) !=
      cudaSuccess)
    return e;
  // first token of tile g (tiles are numbered sequence by sequence in id order)
  int32_t n = 0;
  int64_t n_first = 0;
  auto tile_token = [&](int64_t g) -> int64_t {
    if (N == 1 || !cu_host) return TILE * g;
    while (n < N) {
      const int64_t nt = (cu_host[n + 1] - cu_host[n] + TILE - 1) / TILE;
      if (g < n_first + nt) return cu_host[n] + TILE * (g - n_first);
      n_first += nt;
      ++n;
    }
    return total_tokens;
  };
  if (zero_state && W < total_tiles) {  // a sequence may start in a later window: its zero state comes from here
    if ((e = cudaMemsetAsync(state, 0, (size_t)N * d.Hv * kD * kD * sizeof(float), stream)) != cudaSuccess) return e;
    zero_state = false;
  }
  for (int64_t g0 = 0; g0 < total_tiles; g0 += W) {
    const int64_t g1 = std::min<int64_t>(g0 + W, total_tiles);
    const int64_t t0 = tile_token(g0), t1 = g1 < total_tiles ? tile_token(g1) : total_tokens;
    const WyWin win{g0, g1, t0};
    CUtensorMap tm_hi, tm_lo;
    if (!encode_2d(enc, &tm_hi, qk_hi, qkw, t1 - t0) || !encode_2d(enc, &tm_lo, qk_lo, qkw, t1 - t0))
      return cudaErrorInvalidValue;
    {
      LaunchScope scope(GDN_K_WY_CONV, stream);
      wy_conv_kernel<TILE><<<dim3((unsigned)((g1 - g0) * (TILE / 64)), (unsigned)(2 * d.Hk + 2 * d.Hv)), 256, 0,
                             stream>>>(d, conv_w, (const __nv_bfloat16*)qkv, (const __nv_bfloat16*)conv_state,
                                       zero_conv ? 1 : 0, tile_map, total_tokens, qk_hi, qk_lo, vimg, norm_w,
                                       (const __nv_bfloat16*)z, gate, win);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if constexpr (TILE == 64) {
      LaunchScope scope(GDN_K_WY_PREP, stream);
      wy_prep_kernel<C><<<(unsigned)((g1 - g0) * d.Hv), kPrepThreads, kPrepSmem, stream>>>(
          tm_hi, tm_lo, d, tile_map, vimg, records, cu, (const __nv_bfloat16*)qkv, zero_conv ? 1 : 0,
          (__nv_bfloat16*)const_cast<void*>(conv_state), A_log, dt_bias, (const __nv_bfloat16*)a,
          (const __nv_bfloat16*)b, total_tokens, win, status);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else {
      LaunchScope scope(GDN_K_WY_PREP, stream);
      wy_prep128_kernel<<<(unsigned)((g1 - g0) * d.Hv), kPrepThreads, kPrep128Smem, stream>>>(
          tm_hi, tm_lo, d, tile_map, vimg, records, cu, (const __nv_bfloat16*)qkv, zero_conv ? 1 : 0,
          (__nv_bfloat16*)const_cast<void*>(conv_state), A_log, dt_bias, (const __nv_bfloat16*)a,
          (const __nv_bfloat16*)b, total_tokens, win, status);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    LaunchScope scope(GDN_K_WY_CHAIN, stream);
    wy_chain_kernel<TILE, C><<<(unsigned)((int64_t)N * d.Hv * 2), kChainThreads, F::SMEM, stream>>>(
        d, records, tile_off, order, cu, zero_state ? 1 : 0, gate, win, state, (__nv_bfloat16*)o, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

bool prefill_wy_supported(const Dims& d, bool bf16, int chunk_size) {
  return bf16 && d.dk == 128 && d.dv == 128 &&
         (chunk_size == 16 || chunk_size == 32 || chunk_size == 64 || chunk_size == 128);
}

int wy_tile(int chunk_size) { return chunk_size == 128 ? 128 : 64; }

int64_t wy_window_tiles(int64_t total_tiles, int chunk_size) {
  const int64_t cap = kWyWindowTokens / wy_tile(chunk_size);
  return total_tiles < cap ? total_tiles : cap;
}

WyLayout wy_layout(const Dims& d, int64_t total_tokens, int64_t tile_bound, int chunk_size) {
  WyLayout S;
  const size_t qkw = (size_t)2 * d.Hk * kD;
  const int tile = wy_tile(chunk_size);
  S.qk_hi = 0;
  S.qk_lo = al256(S.qk_hi + (size_t)total_tokens * qkw * 2);
  S.vimg = al256(S.qk_lo + (size_t)total_tokens * qkw * 2);
  S.gate = al256(S.vimg + (size_t)tile_bound * d.Hv * (tile * 512));
  S.records = al256(S.gate + (size_t)total_tokens * d.Hv * kD * 2);
  S.total_bytes = al256(S.records + (size_t)tile_bound * d.Hv * rec_bytes(chunk_size));
  return S;
}

cudaError_t launch_prefill_wy(const Dims& d, int chunk_size, const float* conv_w, const float* A_log,
                              const float* dt_bias, const float* norm_w, const void* qkv, const void* z,
                              const void* a, const void* b, const int32_t* cu, const int32_t* cu_host,
                              const int32_t* order,
                              const int32_t* tile_off, const int4* tile_map, int32_t N, int64_t total_tokens,
                              int64_t total_tiles, bool zero_state, bool zero_conv, const void* conv_state,
                              float* state, void* o, void* ws, int32_t* status, cudaStream_t stream) {
  if (N <= 0 || total_tokens <= 0 || total_tiles <= 0) return cudaSuccess;
#define GDN_WY_ARGS                                                                                               \
  d, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, cu, cu_host, order, tile_off, tile_map, N, total_tokens,      \
      total_tiles,                                                                                                \
      zero_state, zero_conv, conv_state, state, o, ws, status, stream
  switch (chunk_size) {
    case 16: return launch_wy<64, 16>(GDN_WY_ARGS);
    case 32: return launch_wy<64, 32>(GDN_WY_ARGS);
    case 64: return launch_wy<64, 64>(GDN_WY_ARGS);
    case 128: return launch_wy<128, 128>(GDN_WY_ARGS);
    default: return cudaErrorNotSupported;
  }
#undef GDN_WY_ARGS
}

}  // namespace gdn
