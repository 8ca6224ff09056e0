// Chunked GDN prefill on tcgen05 tensor cores (bf16 io, d_k = d_v = 128,
// chunk 64).
//
// The gated delta rule ("fp32 Gated DeltaNet recurrence", DS4Server issue #95,
// implementation comment) in its chunkwise WY/UT form.  Within a chunk of
// rows r (cumulative log decay gamma_r = sum_{i<=r} g_i):
//   A_rj = beta_r e^{gamma_r - gamma_j} k_r.k_j  (j < r),   T = (I + A)^-1
//   W = T diag(beta e^gamma) K,   U = T diag(beta) V
//   Delta = U - W S,   O = diag(e^gamma) Q S + (M o Q K^T) Delta,
//   S <- e^{gamma_C} S + K~^T Delta,   K~ = diag(e^{gamma_C - gamma}) K,
// with M_rj = e^{gamma_r - gamma_j} for j <= r.  Every decay factor is an
// exponential of a non-positive number, so nothing overflows.
//
// One CTA per (sequence, value head); 8 warps; chunks in order.  Per chunk:
//   P0  TMA loads the raw q/k/v channels of rows t0-3 .. t0+63 (128-byte
//       swizzle), the gates come from a/b; conv + SiLU + L2 norm on CUDA
//       cores write the fp16 MMA operands;
//   M1  [K;Q] K^T                          (M=128, N=64,  K=128), in split
//       precision: each of q^, k^ is hi + lo (two fp16 parts) and the product
//       takes hi.hi + hi.lo + lo.hi, because O = Qg S + P Delta partly cancels
//       and P must carry q^.k^ to fp32 accuracy
//   P1  A and P = M o QK^T from the accumulator; T = (I+A)^-1 by blocked
//       forward substitution in fp32 on CUDA cores
//   M2  [T;0] [beta e^g K | beta V]         (M=128, N=256, K=64)  -> W | U
//   P2  -W and diag(e^gamma) Q into one A operand
//   M3  U += [-W;Qg] S                      (M=128, N=128, K=128) -> [Delta; QgS]
//   P3  Delta to shared memory
//   M4  += [0;P] Delta   -> O in rows 64..127;  M5  K~^T Delta (M=128, N=128, K=64)
//   P4  S = e^{gamma_C} S + K~^T Delta (fp32 in registers, fp16 copy for M3);
//       O rows: zero-centred RMSNorm over d_v times sigmoid(z), bf16 out.
// Operands are fp16 (inputs to every MMA are bounded: normalised keys and
// queries, decay factors <= 1), accumulation fp32, the state fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "../../include/gdn.h"
#include "internal.h"
#include "tc.cuh"

namespace gdn {
namespace {

using namespace tc;

constexpr int kC = 64;     // chunk rows
constexpr int kD = 128;    // head dim
constexpr int kThreads = 256;
constexpr int kHalo = 3;   // conv width - 1
constexpr int kRawRows = kC + kHalo;
constexpr int kRawBoxBytes = 64 * kRawRows * 2;  // 64 channels x 67 rows bf16 = 8576
constexpr int kRawBox = 9216;                      // box slot, 1024-aligned

constexpr int OFF_RAW = 0;                     // 6 boxes: q[0:64], q[64:128], k.., k.., v.., v..
constexpr int OFF_KQ = 6 * kRawBox;            // [k^ ; q^] 128x128 K-major, later [-W ; Qg]
constexpr int OFF_X = OFF_KQ + 32768;          // [beta e^g k^ | beta v]  MN-major K=64 x N=256
constexpr int OFF_KD = OFF_X + 32768;          // e^{gC-g} k^             MN-major K=64 x M=128
constexpr int OFF_TA = OFF_KD + 16384;         // [T ; 0]                 K-major 128 x 64
constexpr int OFF_PA = OFF_TA + 16384;         // [0 ; P]                 K-major 128 x 64
constexpr int OFF_KQL = OFF_TA;                // [k^ lo ; q^ lo] 128x128 K-major, until M1 is done (spans TA and PA)
constexpr int OFF_DB = OFF_PA + 16384;         // Delta                   MN-major K=64 x N=128
constexpr int OFF_SB = OFF_DB + 16384;         // S (fp16)                MN-major K=128 x N=128
constexpr int OFF_MISC = OFF_SB + 32768;
constexpr int kMiscFloats = 64 * 6 + 8 + 128;  // gates, row sums, gamma_C, norm weights
constexpr int kSmemBytes = OFF_MISC + kMiscFloats * 4 + 1024;  // + base alignment slack
constexpr int LDS = 68;                         // fp32 solve scratch row stride (aliases RAW; 16-byte rows)

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t COL_D1 = 0;     // [K;Q]K^T           64 columns
constexpr uint32_t COL_S = 128;    // the fp32 state S   128 columns (row i = d_k index, column j)
constexpr uint32_t COL_W = 256;    // W (M2), later K~^T Delta (M5)
constexpr uint32_t COL_U = 384;    // U -> [Delta ; O]
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait, then report and stop

__device__ __forceinline__ void ld4bf(const unsigned char* p, float* f) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  f[0] = __uint_as_float(u.x << 16);
  f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xffff0000u);
}
// raw element offset: 64-channel box, 128-byte rows, 128-byte swizzle
__device__ __forceinline__ int raw_off(int row, int cc) {
  return row * 128 + ((((cc >> 3) ^ (row & 7))) << 4) + (cc & 7) * 2;
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_chunked_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_z, Dims d, const float* __restrict__ conv_w,
                           const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                           const float* __restrict__ norm_w, const __nv_bfloat16* __restrict__ z,
                           const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                           const int32_t* __restrict__ cu, const int32_t* __restrict__ order, int zero_state,
                           int zero_conv, const __nv_bfloat16* __restrict__ hist, float* __restrict__ state,
                           __nv_bfloat16* __restrict__ o, int32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t mb_tma, mb_mma, mb_z;
  __shared__ uint32_t tslot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x % d.Hv;
  const int oi = blockIdx.x / d.Hv;
  const int n = order ? order[oi] : oi;
  const int kh = h / d.G;
  const int64_t seq0 = cu[n];
  const int len = cu[n + 1] - cu[n];
  if (len <= 0) return;
  const int64_t C = d.C;
  const int64_t HvD = (int64_t)d.Hv * kD;

  float* misc = reinterpret_cast<float*>(sm + OFF_MISC);
  float* s_gam = misc;         // gamma_r
  float* s_beta = misc + 64;   // beta_r (0 beyond the sequence end)
  float* s_eg = misc + 128;    // e^{gamma_r}
  float* s_ekd = misc + 192;   // e^{gamma_C - gamma_r}
  float* s_rms = misc + 256;   // [2][64] partial sums of squares of the O rows
  float* s_gC = misc + 384;    // gamma_C
  float* s_nw = misc + 392;    // 1 + norm_w
  float* Am = reinterpret_cast<float*>(sm + OFF_RAW);   // solve scratch, aliases the raw tiles
  float* Tm = Am + 64 * LDS;
  float* Ym = Tm + 64 * LDS;

  if (tid == 0) {
    mbar_init(&mb_tma, 1);
    mbar_init(&mb_mma, 1);
    mbar_init(&mb_z, 1);
    mbar_init_fence();
    abort_flag = 0;
  }
  if (warp == 0) tmem_alloc(&tslot, kTmemCols);

  if (tid < kD) s_nw[tid] = 1.0f + norm_w[tid];
  // recurrent state (fp32, in TMEM): thread owns row si of S (d_k index), columns [64 hc, 64 hc + 64)
  const int si = 32 * (warp & 3) + lane, hc = warp >> 2;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
  float* gst = state + ((int64_t)n * d.Hv + h) * kD * kD;  // stored [j][i]
  sync_tc();
  const uint32_t tbase = tslot;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float S[32];
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) S[jj] = zero_state ? 0.f : gst[(int64_t)(64 * hc + 32 * hh + jj) * kD + si];
    tmem_st32(tbase + lane_base + COL_S + 64 * hc + 32 * hh, S);
#pragma unroll
    for (int m = 0; m < 4; ++m) st16h(sm + OFF_SB + mnmaj_chunk(kD, si, 64 * hc + 32 * hh + 8 * m), S + 8 * m);
  }
  fence_async_smem();
  sync_tc();

  const float negA = -expf(A_log[h]);
  const float dtb = dt_bias[h];
  const int nchunks = (len + kC - 1) / kC;
  uint32_t ph_tma = 0, ph_mma = 0, ph_z = 0;
  const int64_t q_col = (int64_t)kh * kD, k_col = (int64_t)d.Hk * kD + q_col, v_col = 2LL * d.Hk * kD + (int64_t)h * kD;

  // The raw tiles and the a/b gate inputs of chunk c+1 are requested while
  // chunk c is still in its MMA phases (the raw-tile space is idle by then).
  auto issue_raw = [&](int cc) {
    const int64_t tt = seq0 + (int64_t)cc * kC;
    mbar_expect_tx(&mb_tma, 6 * kRawBoxBytes);
#pragma unroll
    for (int bx = 0; bx < 6; ++bx) {
      const int64_t col = (bx < 2 ? q_col : bx < 4 ? k_col : v_col) + (bx & 1) * 64;
      tma_load_2d(sm + OFF_RAW + bx * kRawBox, &tm_qkv, (int)col, (int)(tt - kHalo), &mb_tma);
    }
  };
  // gate inputs of the next chunk (warp 0), kept as raw bf16 bits so that the
  // loads are not waited for until the chunk that uses them
  unsigned short pa[2] = {0, 0}, pb[2] = {0, 0};
  const unsigned short* a16 = reinterpret_cast<const unsigned short*>(a);
  const unsigned short* b16 = reinterpret_cast<const unsigned short*>(b);
  auto load_gates = [&](int cc) {
    const int64_t tt = seq0 + (int64_t)cc * kC;
    const int LL = min(kC, len - cc * kC);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = 2 * lane + e;
      if (r < LL) {
        pa[e] = __ldg(a16 + (tt + r) * d.Hv + h);
        pb[e] = __ldg(b16 + (tt + r) * d.Hv + h);
      }
    }
  };
  if (tid == 0) issue_raw(0);
  if (warp == 0) load_gates(0);

  for (int c = 0; c < nchunks; ++c) {
    const int64_t t0 = seq0 + (int64_t)c * kC;
    const int L = min(kC, len - c * kC);

    // ------------------------------------------------------------ P0: raw tiles, gates
    if (warp == 0) {  // gates of rows 2*lane, 2*lane+1; inclusive scan of g
      float g2[2], be2[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = 2 * lane + e;
        g2[e] = 0.f;
        be2[e] = 0.f;
        if (r < L) {
          g2[e] = negA * softplus_f(__uint_as_float((uint32_t)pa[e] << 16) + dtb);
          be2[e] = 1.0f / (1.0f + expf(-__uint_as_float((uint32_t)pb[e] << 16)));
        }
      }
      float incl = g2[0] + g2[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const float gam1 = incl, gam0 = incl - g2[1];
      const float gC = __shfl_sync(0xffffffffu, incl, 31);
      s_gam[2 * lane] = gam0;
      s_gam[2 * lane + 1] = gam1;
      s_beta[2 * lane] = be2[0];
      s_beta[2 * lane + 1] = be2[1];
      s_eg[2 * lane] = expf(gam0);
      s_eg[2 * lane + 1] = expf(gam1);
      s_ekd[2 * lane] = expf(gC - gam0);
      s_ekd[2 * lane + 1] = expf(gC - gam1);
      if (lane == 0) *s_gC = gC;
    }
    // conv weights of this lane's 12 channels, requested before waiting for the raw tiles
    float wq[4][4], wk[4][4], wv[4][4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(conv_w + (q_col + 4 * lane + e) * 4));
      const float4 y = __ldg(reinterpret_cast<const float4*>(conv_w + (k_col + 4 * lane + e) * 4));
      const float4 zz = __ldg(reinterpret_cast<const float4*>(conv_w + (v_col + 4 * lane + e) * 4));
      wq[e][0] = x.x; wq[e][1] = x.y; wq[e][2] = x.z; wq[e][3] = x.w;
      wk[e][0] = y.x; wk[e][1] = y.y; wk[e][2] = y.z; wk[e][3] = y.w;
      wv[e][0] = zz.x; wv[e][1] = zz.y; wv[e][2] = zz.z; wv[e][3] = zz.w;
    }
    if (!mbar_wait(&mb_tma, ph_tma, kWaitNs)) abort_flag = 1;
    ph_tma ^= 1;
    if (c == 0) {  // rows before the sequence start come from the conv history
      for (int idx = tid; idx < 3 * 384; idx += kThreads) {
        const int row = idx / 384, ch = idx % 384;
        const int64_t gch = (ch < 128 ? q_col + ch : ch < 256 ? k_col + (ch - 128) : v_col + (ch - 256));
        const __nv_bfloat16 val = zero_conv ? __float2bfloat16(0.f) : hist[((int64_t)n * 3 + row) * C + gch];
        *reinterpret_cast<__nv_bfloat16*>(sm + OFF_RAW + (ch >> 6) * kRawBox + raw_off(row, ch & 63)) = val;
      }
    }
    __syncthreads();
    if (abort_flag) break;

    // ------------------------------------------------------------ P0c: conv + SiLU + L2 norm -> operands
    {
      const int cc = (4 * lane) & 63;  // channel inside the lane's 64-channel box
      const int half = lane >> 4;
      const unsigned char* rq = sm + OFF_RAW + (0 + half) * kRawBox;
      const unsigned char* rk = sm + OFF_RAW + (2 + half) * kRawBox;
      const unsigned char* rv = sm + OFF_RAW + (4 + half) * kRawBox;
#pragma unroll 1
      for (int rp = 0; rp < 2; ++rp) {  // four rows per pass for instruction-level parallelism
        const int r0 = 8 * warp + 4 * rp;
        float yq[4][4], yk[4][4], yv[4][4];
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int e = 0; e < 4; ++e) yq[x][e] = yk[x][e] = yv[x][e] = 0.f;
#pragma unroll
        for (int rowi = 0; rowi < 7; ++rowi) {  // raw rows r0 .. r0+6 feed the taps of the four rows
          float xq[4], xk[4], xv[4];
          const int off = raw_off(r0 + rowi, cc);
          ld4bf(rq + off, xq);
          ld4bf(rk + off, xk);
          ld4bf(rv + off, xv);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int tap = rowi - x;
            if (tap >= 0 && tap < 4) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                yq[x][e] += wq[e][tap] * xq[e];
                yk[x][e] += wk[e][tap] * xk[e];
                yv[x][e] += wv[e][tap] * xv[e];
              }
            }
          }
        }
        float sq[4] = {0.f, 0.f, 0.f, 0.f}, sk[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            yq[x][e] = silu_fast(yq[x][e]);
            yk[x][e] = silu_fast(yk[x][e]);
            yv[x][e] = silu_fast(yv[x][e]);
            sq[x] += yq[x][e] * yq[x][e];
            sk[x] += yk[x][e] * yk[x][e];
          }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            sq[x] += __shfl_xor_sync(0xffffffffu, sq[x], off);
            sk[x] += __shfl_xor_sync(0xffffffffu, sk[x], off);
          }
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int r = r0 + x;
          const bool valid = r < L;
          const float rqs = d.q_scale * rsqrtf(sq[x] + d.l2_eps);
          const float rks = valid ? rsqrtf(sk[x] + d.l2_eps) : 0.f;
          const float be = s_beta[r], eg = s_eg[r], ekd = s_ekd[r];
          float qh[4], kk[4], vv[4], kl[4], ql[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            qh[e] = yq[x][e] * rqs;
            kk[e] = yk[x][e] * rks;
            vv[e] = valid ? yv[x][e] : 0.f;
            kl[e] = kk[e] - __half2float(__float2half_rn(kk[e]));
            ql[e] = qh[e] - __half2float(__float2half_rn(qh[e]));
          }
          const int k4 = 4 * lane;
          st8(sm + OFF_KQ + kmaj(128, r, k4), kk[0], kk[1], kk[2], kk[3]);
          st8(sm + OFF_KQ + kmaj(128, 64 + r, k4), qh[0], qh[1], qh[2], qh[3]);
          st8(sm + OFF_KQL + kmaj(128, r, k4), kl[0], kl[1], kl[2], kl[3]);
          st8(sm + OFF_KQL + kmaj(128, 64 + r, k4), ql[0], ql[1], ql[2], ql[3]);
          const float bg = be * eg;
          st8(sm + OFF_X + mnmaj(kC, r, k4), bg * kk[0], bg * kk[1], bg * kk[2], bg * kk[3]);
          st8(sm + OFF_X + mnmaj(kC, r, 128 + k4), be * vv[0], be * vv[1], be * vv[2], be * vv[3]);
          st8(sm + OFF_KD + mnmaj(kC, r, k4), ekd * kk[0], ekd * kk[1], ekd * kk[2], ekd * kk[3]);
        }
      }
    }
    fence_async_smem();
    sync_tc();

    // ------------------------------------------------------------ M1: [K;Q] K^T
    if (tid == 0) {
      const uint32_t kq = smem_u32(sm + OFF_KQ);
      constexpr uint32_t id = idesc_f16(128, 64, false, false);
      const uint32_t kql = smem_u32(sm + OFF_KQL);
#pragma unroll
      for (int s = 0; s < 8; ++s) mma_f16(tbase + COL_D1, desc_kmaj(kq, 128, s), desc_kmaj(kq, 128, s), id, s > 0);
#pragma unroll
      for (int s = 0; s < 8; ++s) mma_f16(tbase + COL_D1, desc_kmaj(kq, 128, s), desc_kmaj(kql, 128, s), id, 1);
#pragma unroll
      for (int s = 0; s < 8; ++s) mma_f16(tbase + COL_D1, desc_kmaj(kql, 128, s), desc_kmaj(kq, 128, s), id, 1);
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, ph_mma, kWaitNs)) abort_flag = 1;
    ph_mma ^= 1;
    fence_after();

    // ------------------------------------------------------------ P1: A, P, T = (I + A)^-1
    for (int i = tid; i < 512; i += kThreads) {  // constant zero halves of [T;0] and [0;P]
      reinterpret_cast<uint4*>(sm + OFF_TA + 8192)[i] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(sm + OFF_PA)[i] = make_uint4(0, 0, 0, 0);
    }
    {
      float v[32];
      tmem_ld32(tbase + lane_base + COL_D1 + 32 * hc, v);
      const int row = si;
      if (row < 64) {  // A_rj = beta_r e^{gamma_r - gamma_j} (k_r . k_j), j < r
        const float br = s_beta[row], gr = s_gam[row];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          float a4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 32 * hc + 4 * m + e;
            a4[e] = (j < row) ? br * __expf(gr - s_gam[j]) * v[4 * m + e] : 0.f;
          }
          *reinterpret_cast<float4*>(Am + row * LDS + 32 * hc + 4 * m) = make_float4(a4[0], a4[1], a4[2], a4[3]);
        }
      } else {  // P_rj = e^{gamma_r - gamma_j} (q_r . k_j), j <= r
        const int r = row - 64;
        const float gr = s_gam[r];
        float p[8];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = 32 * hc + 8 * m + e;
            p[e] = (j <= r) ? __expf(gr - s_gam[j]) * v[8 * m + e] : 0.f;
          }
          st16h(sm + OFF_PA + kmaj_chunk(128, row, 32 * hc + 8 * m), p);
        }
      }
    }
    __syncthreads();
    // T = (I + A)^-1 in 16x16 blocks.  Diagonal blocks T_bb = (I + A_bb)^-1 by
    // right-looking forward substitution (one column per thread: each new
    // entry updates the running sums of the rows below it, so the dependent
    // chain is one FMA per row).
    if (tid < 64) {
      const int bb = tid >> 4, c16 = tid & 15;
      const float* Ab = Am + (16 * bb) * LDS + 16 * bb;
      float acc[16], t[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        t[k] = (k < c16) ? 0.f : (k == c16 ? 1.f : -acc[k]);
#pragma unroll
        for (int i = k + 1; i < 16; ++i) acc[i] += Ab[i * LDS + k] * t[k];
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) Tm[(16 * bb + i) * LDS + 16 * bb + c16] = t[i];
    }
    __syncthreads();
    // At_ij = T_ii A_ij for the six blocks below the diagonal (into Ym); each work
    // item is one row p and four columns q..q+3 of one block (float4 along q)
    for (int e = tid; e < 6 * 64; e += kThreads) {
      const int pr = e >> 6, p = (e >> 2) & 15, q = 4 * (e & 3);
      // pairs pr = 0..5: (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
      const int bi = pr == 0 ? 1 : (pr < 3 ? 2 : 3), bj = pr == 0 ? 0 : (pr < 3 ? pr - 1 : pr - 3);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        const float t = Tm[(16 * bi + p) * LDS + 16 * bi + kk];
        const float4 a4 = *reinterpret_cast<const float4*>(Am + (16 * bi + kk) * LDS + 16 * bj + q);
        acc.x += t * a4.x; acc.y += t * a4.y; acc.z += t * a4.z; acc.w += t * a4.w;
      }
      *reinterpret_cast<float4*>(Ym + (16 * bi + p) * LDS + 16 * bj + q) = acc;
    }
    __syncthreads();
    // off-diagonal blocks by distance: T_ij = -sum_{k=j}^{i-1} At_ik T_kj
    for (int dl = 1; dl < 4; ++dl) {
      for (int e = tid; e < (4 - dl) * 64; e += kThreads) {
        const int bj = e >> 6, bi = bj + dl, p = (e >> 2) & 15, q = 4 * (e & 3);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int bk = bj; bk < bi; ++bk) {
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            const float y = Ym[(16 * bi + p) * LDS + 16 * bk + kk];
            const float4 t4 = *reinterpret_cast<const float4*>(Tm + (16 * bk + kk) * LDS + 16 * bj + q);
            acc.x += y * t4.x; acc.y += y * t4.y; acc.z += y * t4.z; acc.w += y * t4.w;
          }
        }
        *reinterpret_cast<float4*>(Tm + (16 * bi + p) * LDS + 16 * bj + q) = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
      }
      __syncthreads();
    }
    {  // T (lower triangular, unit diagonal) -> fp16 rows 0..63 of [T;0]
      const int r = tid >> 2, j0 = 16 * (tid & 3);
      float tv[16];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 t4 = *reinterpret_cast<const float4*>(Tm + r * LDS + j0 + 4 * m);
        tv[4 * m] = t4.x; tv[4 * m + 1] = t4.y; tv[4 * m + 2] = t4.z; tv[4 * m + 3] = t4.w;
      }
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) tv[jj] = (j0 + jj <= r) ? tv[jj] : 0.f;
      st16h(sm + OFF_TA + kmaj_chunk(128, r, j0), tv);
      st16h(sm + OFF_TA + kmaj_chunk(128, r, j0 + 8), tv + 8);
    }
    fence_async_smem();
    sync_tc();

    // ------------------------------------------------------------ M2: [T;0] [beta e^g K | beta V]
    if (c + 1 < nchunks) {  // the raw-tile space is idle from here on: fetch the next chunk
      if (tid == 0) issue_raw(c + 1);
      if (warp == 0) load_gates(c + 1);
    }
    if (tid == 0) {
      const uint32_t ta = smem_u32(sm + OFF_TA), x = smem_u32(sm + OFF_X);
      constexpr uint32_t id = idesc_f16(128, 256, false, true);
#pragma unroll
      for (int s = 0; s < 4; ++s) mma_f16(tbase + COL_W, desc_kmaj(ta, 128, s), desc_mnmaj(x, kC, s), id, s > 0);
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, ph_mma, kWaitNs)) abort_flag = 1;
    ph_mma ^= 1;
    fence_after();

    // ------------------------------------------------------------ P2: [-W ; diag(e^gamma) Q]
    if (tid == 0) {  // z rows of this chunk, for the output gate (into the X tile, idle after M2)
      mbar_expect_tx(&mb_z, 2 * 64 * 64 * 2);
      tma_load_2d(sm + OFF_X, &tm_z, h * kD, (int)t0, &mb_z);
      tma_load_2d(sm + OFF_X + 8192, &tm_z, h * kD + 64, (int)t0, &mb_z);
    }
    if (si < 64) {
      float v[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        tmem_ld32(tbase + lane_base + COL_W + 64 * hc + 32 * hh, v);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) v[jj] = -v[jj];
#pragma unroll
        for (int m = 0; m < 4; ++m) st16h(sm + OFF_KQ + kmaj_chunk(128, si, 64 * hc + 32 * hh + 8 * m), v + 8 * m);
      }
    } else {
      const float eg = s_eg[si - 64];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        uint4* p = reinterpret_cast<uint4*>(sm + OFF_KQ + kmaj_chunk(128, si, 64 * hc + 8 * m));
        uint4 u = *p;
        __half2* hp = reinterpret_cast<__half2*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hp[e]);
          hp[e] = __floats2half2_rn(f.x * eg, f.y * eg);
        }
        *p = u;
      }
    }
    fence_async_smem();
    sync_tc();

    // ------------------------------------------------------------ M3: U += [-W;Qg] S  -> [Delta ; Qg S]
    if (tid == 0) {
      const uint32_t kq = smem_u32(sm + OFF_KQ), sb = smem_u32(sm + OFF_SB);
      constexpr uint32_t id = idesc_f16(128, 128, false, true);
#pragma unroll
      for (int s = 0; s < 8; ++s) mma_f16(tbase + COL_U, desc_kmaj(kq, 128, s), desc_mnmaj(sb, kD, s), id, 1);
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, ph_mma, kWaitNs)) abort_flag = 1;
    ph_mma ^= 1;
    fence_after();

    // ------------------------------------------------------------ P3: Delta -> shared (MN-major B)
    if (si < 64) {
      float v[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        tmem_ld32(tbase + lane_base + COL_U + 64 * hc + 32 * hh, v);
#pragma unroll
        for (int m = 0; m < 4; ++m) st16h(sm + OFF_DB + mnmaj_chunk(kC, si, 64 * hc + 32 * hh + 8 * m), v + 8 * m);
      }
    }
    fence_async_smem();
    sync_tc();

    // ------------------------------------------------------------ M4: O += [0;P] Delta ;  M5: K~^T Delta
    if (tid == 0) {
      const uint32_t pa = smem_u32(sm + OFF_PA), db = smem_u32(sm + OFF_DB), kd = smem_u32(sm + OFF_KD);
      constexpr uint32_t id4 = idesc_f16(128, 128, false, true);
      constexpr uint32_t id5 = idesc_f16(128, 128, true, true);
#pragma unroll
      for (int s = 0; s < 4; ++s) mma_f16(tbase + COL_U, desc_kmaj(pa, 128, s), desc_mnmaj(db, kC, s), id4, 1);
#pragma unroll
      for (int s = 0; s < 4; ++s) mma_f16(tbase + COL_W, desc_mnmaj(kd, kC, s), desc_mnmaj(db, kC, s), id5, s > 0);
      mma_commit(&mb_mma);
    }
    if (!mbar_wait(&mb_mma, ph_mma, kWaitNs)) abort_flag = 1;
    ph_mma ^= 1;
    fence_after();

    // ------------------------------------------------------------ P4: state update, output rows
    {
      const float egC = expf(*s_gC);
      float v[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float S[32];
        tmem_ld32(tbase + lane_base + COL_W + 64 * hc + 32 * hh, v);
        tmem_ld32(tbase + lane_base + COL_S + 64 * hc + 32 * hh, S);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) S[jj] = egC * S[jj] + v[jj];
        tmem_st32(tbase + lane_base + COL_S + 64 * hc + 32 * hh, S);
#pragma unroll
        for (int m = 0; m < 4; ++m) st16h(sm + OFF_SB + mnmaj_chunk(kD, si, 64 * hc + 32 * hh + 8 * m), S + 8 * m);
      }
      if (si >= 64) {  // O rows: fp32 into the [-W;Qg] tile (idle after M3), row sums of squares
        const int r = si - 64;
        float* orow = reinterpret_cast<float*>(sm + OFF_KQ) + r * kD;
        float ss = 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tmem_ld32(tbase + lane_base + COL_U + 64 * hc + 32 * hh, v);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) ss += v[jj] * v[jj];
#pragma unroll
          for (int m = 0; m < 8; ++m) {  // float4 slot c4 stored at c4 ^ (r % 8): conflict-free rows
            const int c4 = 16 * hc + 8 * hh + m;
            *reinterpret_cast<float4*>(orow + 4 * (c4 ^ (r & 7))) =
                make_float4(v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]);
          }
        }
        s_rms[64 * hc + r] = ss;
      }
    }
    if (!mbar_wait(&mb_z, ph_z, kWaitNs)) abort_flag = 1;
    ph_z ^= 1;
    __syncthreads();
    {  // zero-centred RMSNorm over d_v, times sigmoid(z): row r = tid / 4, columns [32 q4, 32 q4 + 32)
      const int r = tid >> 2, q4 = tid & 3;
      if (r < L) {
        const float rinv = rsqrtf((s_rms[r] + s_rms[64 + r]) * (1.0f / kD) + d.norm_eps);
        const float* orow = reinterpret_cast<const float*>(sm + OFF_KQ) + r * kD;
        const unsigned char* zbox = sm + OFF_X + (q4 >> 1) * 8192;
        const int64_t off = (t0 + r) * HvD + (int64_t)h * kD + 32 * q4;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int zc = 32 * (q4 & 1) + 8 * m;  // column inside the 64-column z box
          const uint4 zr = *reinterpret_cast<const uint4*>(zbox + r * 128 + ((((zc >> 3) ^ (r & 7))) << 4));
          const int c4 = 8 * q4 + 2 * m;
          const float4 oa = *reinterpret_cast<const float4*>(orow + 4 * (c4 ^ (r & 7)));
          const float4 ob = *reinterpret_cast<const float4*>(orow + 4 * ((c4 + 1) ^ (r & 7)));
          const float ov[8] = {oa.x, oa.y, oa.z, oa.w, ob.x, ob.y, ob.z, ob.w};
          const uint32_t zw[4] = {zr.x, zr.y, zr.z, zr.w};
          uint32_t ow[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 32 * q4 + 8 * m + 2 * e;
            const float z0 = __uint_as_float(zw[e] << 16), z1 = __uint_as_float(zw[e] & 0xffff0000u);
            const float o0 = ov[2 * e] * rinv * s_nw[j] * __fdividef(1.0f, 1.0f + __expf(-z0));
            const float o1 = ov[2 * e + 1] * rinv * s_nw[j + 1] * __fdividef(1.0f, 1.0f + __expf(-z1));
            __nv_bfloat162 pr = __floats2bfloat162_rn(o0, o1);
            ow[e] = *reinterpret_cast<uint32_t*>(&pr);
          }
          *reinterpret_cast<uint4*>(o + off + 8 * m) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        }
      }
    }
    fence_async_smem();
    sync_tc();
  }

  if (abort_flag) {
    if (tid == 0) set_status(status, kStatusWaitTimeout);
  } else {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float S[32];
      tmem_ld32(tbase + lane_base + COL_S + 64 * hc + 32 * hh, S);
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) gst[(int64_t)(64 * hc + 32 * hh + jj) * kD + si] = S[jj];
    }
  }
  sync_tc();
  if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

// ---------------------------------------------------------------- host side

}  // namespace

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
    else
      cudaGetLastError();
  });
  return fn;
}

bool prefill_chunked_supported(const Dims& d, bool bf16, int chunk_size) {
  return bf16 && d.dk == kD && d.dv == kD && chunk_size == kC;
}

cudaError_t launch_prefill_chunked(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                                   const float* norm_w, const void* qkv, const void* z, const void* a, const void* b,
                                   const int32_t* cu, const int32_t* order, int32_t N, int64_t total_tokens,
                                   bool zero_state, bool zero_conv, const void* conv_state, float* state, void* o,
                                   int32_t* status, cudaStream_t stream) {
  if (N <= 0 || total_tokens <= 0) return cudaSuccess;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tm, tmz;
  const cuuint64_t zdim[2] = {(cuuint64_t)d.Hv * kD, (cuuint64_t)total_tokens};
  const cuuint64_t zstride[1] = {(cuuint64_t)d.Hv * kD * 2};
  const cuuint32_t zbox[2] = {64, 64};
  const cuuint64_t gdim[2] = {(cuuint64_t)d.C, (cuuint64_t)total_tokens};
  const cuuint64_t gstride[1] = {(cuuint64_t)d.C * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kRawRows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(qkv), gdim, gstride, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
      enc(&tmz, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(z), zdim, zstride, zbox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(prefill_chunked_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  LaunchScope scope(GDN_K_PREFILL_CHUNKED, stream);
  prefill_chunked_kernel<<<(unsigned)((int64_t)N * d.Hv), kThreads, kSmemBytes, stream>>>(
      tm, tmz, d, conv_w, A_log, dt_bias, norm_w, (const __nv_bfloat16*)z, (const __nv_bfloat16*)a,
      (const __nv_bfloat16*)b, cu, order, zero_state, zero_conv, (const __nv_bfloat16*)conv_state, state,
      (__nv_bfloat16*)o, status);
  return cudaGetLastError();
}

}  // namespace gdn
