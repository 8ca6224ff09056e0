// Single-step GDN decode: one fused, HBM-bound kernel ("single-step decode",
// DS4Server issue #88, section Scope; fp32 recurrent state, sigmoid output
// gate, exact L2 epsilon placement: issue #95, section Implementation).
//
// One CTA per (sequence n, key head kh).  It owns the conv channels of q and k
// of key head kh and of v for the G value heads that share it, so the rolling
// conv history is read and rewritten by exactly one CTA (no race on the
// shared q/k channels).  Per value head the state is stored transposed,
// state[n,h,j,:] = column j of S (d_k contiguous floats), and the rank-1
// update decomposes into independent rows:
//   kappa_j = k^ . r_j,  rho_j = q^ . r_j              (r_j = old row j)
//   delta_j = beta * (v_j - alpha * kappa_j)
//   r_j'    = alpha * r_j + delta_j * k^               (written back once)
//   o_j     = q^ . r_j' = alpha * rho_j + delta_j * (q^ . k^)
// so every state byte crosses HBM exactly once in each direction.  Eight
// lanes share a row (16-byte loads, 3 shuffle steps for the two dots); each
// warp keeps two row groups of loads in flight.
#include "../../include/gdn.h"
#include "internal.h"
#include "tc.cuh"

namespace gdn {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kUnroll = 2;

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_kernel(Dims d, const float* __restrict__ conv_w, const float* __restrict__ A_log,
                  const float* __restrict__ dt_bias, const float* __restrict__ norm_w, const T* __restrict__ qkv,
                  const T* __restrict__ z, const T* __restrict__ a, const T* __restrict__ b, Slots slots,
                  T* __restrict__ hist, float* __restrict__ state, T* __restrict__ o, int32_t* status) {
  constexpr int F4 = D / 32;  // float4s of a row held by one lane (8 lanes per row)
  extern __shared__ float smem[];
  const int G = d.G;
  const int nch = (2 + G) * D;
  float* u = smem;                 // [q (D) | k (D) | v of the G heads (G*D)] after conv + SiLU
  float* osm = u + nch;            // [G*D] o before the output norm
  float* gate = osm + G * D;       // alpha[G], beta[G]
  __shared__ float red[3];         // q scale, k scale, q^.k^

  const int n = blockIdx.x / d.Hk;
  const int kh = blockIdx.x - n * d.Hk;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t C = d.C;
  const int h0 = G * kh;  // first value head of this key head
  const int sl = slot_of(slots, n, status);  // state and history slot of batch row n
  if (sl < 0) {  // padding row: zero output, nothing else touched
    for (int i = tid; i < G * D; i += kDecThreads) o[((int64_t)n * d.Hv + h0) * D + i] = from_f<T>(0.f);
    return;
  }

  // ---- conv step + SiLU for the owned channels; rotate the history
  for (int idx = tid; idx < nch; idx += kDecThreads) {
    const int64_t c = idx < D ? (int64_t)kh * D + idx
                              : (idx < 2 * D ? (int64_t)d.Hk * D + (int64_t)kh * D + (idx - D)
                                             : 2LL * d.Hk * D + (int64_t)h0 * D + (idx - 2 * D));
    T* hp = hist + (int64_t)sl * 3 * C + c;
    const T h0v = hp[0], h1v = hp[C], h2v = hp[2 * C];
    const T xv = qkv[(int64_t)n * C + c];
    const float4 w = __ldg(reinterpret_cast<const float4*>(conv_w + c * 4));
    const float y = w.x * to_f(h0v) + w.y * to_f(h1v) + w.z * to_f(h2v) + w.w * to_f(xv);
    u[idx] = silu_f(y);
    hp[0] = h1v;
    hp[C] = h2v;
    hp[2 * C] = xv;
  }
  if (tid < G) {
    const int h = h0 + tid;
    float g, al, be;
    gates_f(ldg_f(a + (int64_t)n * d.Hv + h), dt_bias[h], A_log[h], ldg_f(b + (int64_t)n * d.Hv + h), g, al, be);
    gate[tid] = al;
    gate[G + tid] = be;
  }
  __syncthreads();

  // ---- L2 norms of q and k (epsilon inside the square root of the sum)
  if (warp == 0) {
    float sq = 0.f, sk = 0.f, sqk = 0.f;
    for (int i = lane; i < D; i += 32) {
      const float qv = u[i], kv = u[D + i];
      sq += qv * qv;
      sk += kv * kv;
      sqk += qv * kv;
    }
    sq = warp_sum(sq);
    sk = warp_sum(sk);
    sqk = warp_sum(sqk);
    if (lane == 0) {
      const float rq = d.q_scale * rsqrtf(sq + d.l2_eps), rk = rsqrtf(sk + d.l2_eps);
      red[0] = rq;
      red[1] = rk;
      red[2] = rq * rk * sqk;
    }
  }
  __syncthreads();

  // ---- stream the G states of this key head, row by row
  const int l8 = lane & 7, grp = lane >> 3;
  float kq[F4][4], qq[F4][4];
  {
    const float rq = red[0], rk = red[1];
#pragma unroll
    for (int m = 0; m < F4; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qq[m][e] = u[4 * (l8 + 8 * m) + e] * rq;
        kq[m][e] = u[D + 4 * (l8 + 8 * m) + e] * rk;
      }
  }
  const float qk = red[2];
  const int rows = G * D;
  const int groups = rows / 4;
  float* st = state + ((int64_t)sl * d.Hv + h0) * D * D;  // the G heads' rows are contiguous
  for (int base = warp; base < groups; base += kDecWarps * kUnroll) {
    float4 r[kUnroll][F4];
#pragma unroll
    for (int x = 0; x < kUnroll; ++x) {
      const int g4 = base + x * kDecWarps;
      if (g4 < groups) {
        const float4* p = reinterpret_cast<const float4*>(st + (int64_t)(g4 * 4 + grp) * D);
#pragma unroll
        for (int m = 0; m < F4; ++m) r[x][m] = __ldcs(p + l8 + 8 * m);
      }
    }
#pragma unroll
    for (int x = 0; x < kUnroll; ++x) {
      const int g4 = base + x * kDecWarps;
      if (g4 < groups) {  // warp-uniform
        const int row = g4 * 4 + grp;
        float kap = 0.f, rho = 0.f;
#pragma unroll
        for (int m = 0; m < F4; ++m) {
          kap += kq[m][0] * r[x][m].x + kq[m][1] * r[x][m].y + kq[m][2] * r[x][m].z + kq[m][3] * r[x][m].w;
          rho += qq[m][0] * r[x][m].x + qq[m][1] * r[x][m].y + qq[m][2] * r[x][m].z + qq[m][3] * r[x][m].w;
        }
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
          kap += __shfl_xor_sync(0xffffffffu, kap, off);
          rho += __shfl_xor_sync(0xffffffffu, rho, off);
        }
        const int hh = row / D;
        const float al = gate[hh], be = gate[G + hh];
        const float delta = be * (u[2 * D + row] - al * kap);
        float4* p = reinterpret_cast<float4*>(st + (int64_t)row * D);
#pragma unroll
        for (int m = 0; m < F4; ++m) {
          float4 w4;
          w4.x = al * r[x][m].x + delta * kq[m][0];
          w4.y = al * r[x][m].y + delta * kq[m][1];
          w4.z = al * r[x][m].z + delta * kq[m][2];
          w4.w = al * r[x][m].w + delta * kq[m][3];
          __stcs(p + l8 + 8 * m, w4);
        }
        if (l8 == 0) osm[row] = al * rho + delta * qk;
      }
    }
  }
  __syncthreads();

  // ---- zero-centred RMSNorm over d_v, times sigmoid(z); one rounding to io dtype
  for (int hh = warp; hh < G; hh += kDecWarps) {
    float ss = 0.f;
    for (int j = lane; j < D; j += 32) ss += osm[hh * D + j] * osm[hh * D + j];
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / D + d.norm_eps);
    const int64_t off = ((int64_t)n * d.Hv + h0 + hh) * D;
    for (int j = lane; j < D; j += 32) {
      const float zz = ldg_f(z + off + j);
      o[off + j] = from_f<T>(osm[hh * D + j] * r * (1.0f + norm_w[j]) * sigmoid_f(zz));
    }
  }
}

// d_k = d_v = 128: the state rows stream through a 4-stage shared-memory ring
// fed by 1D bulk copies (cp.async.bulk), so the bytes in flight no longer
// depend on registers.  128 threads and ~21 KB of shared memory per CTA let 8
// CTAs share an SM, so the whole B=64 grid (1024 CTAs) is resident in one
// wave; the first stages are requested before the conv/norm prologue runs.
constexpr int kBulkThreads = 128;
constexpr int kBulkRows = 8;     // state rows per stage (4 KB)
constexpr int kBulkStages = 4;
constexpr uint64_t kBulkWaitNs = 2000000000ull;

// One sequence advances by up to K tokens in one pass over its state (K = 1 is
// the single-step decode).  Token t sees the history [h0, h1, h2, x_0 ..
// x_{K-1}] and the state after tokens 0..t-1; every row of the state is
// updated K times in registers between one read and one write.  With
// write_state == 0 (verify) nothing but o is written; otherwise sequence n
// applies its first accept[n] tokens (all K when accept is NULL) to the state
// and the history.  All per-token arithmetic uses explicit fused/unfused
// operations, so a K-token commit of a tokens rounds exactly like a one-token
// steps.
__device__ __forceinline__ float conv4(const float4& w, float x0, float x1, float x2, float x3) {
  return __fmaf_rn(w.w, x3, __fmaf_rn(w.z, x2, __fmaf_rn(w.y, x1, __fmul_rn(w.x, x0))));
}
__device__ __forceinline__ float dot4(const float4& a, const float4& b, float acc) {
  return __fmaf_rn(a.w, b.w, __fmaf_rn(a.z, b.z, __fmaf_rn(a.y, b.y, __fmaf_rn(a.x, b.x, acc))));
}

template <typename T, int K>
__global__ void __launch_bounds__(kBulkThreads, K <= 2 ? 8 : 4)
    decode_bulk_kernel(Dims d, const float* __restrict__ conv_w, const float* __restrict__ A_log,
                       const float* __restrict__ dt_bias, const float* __restrict__ norm_w,
                       const T* __restrict__ qkv, const T* __restrict__ z, const T* __restrict__ a,
                       const T* __restrict__ b, const int32_t* __restrict__ accept, int write_state, Slots slots,
                       T* __restrict__ hist, float* __restrict__ state, T* __restrict__ o, int32_t* status) {
  constexpr int D = 128;
  constexpr int kStageFloats = kBulkRows * D;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* ring = reinterpret_cast<float*>(smem_raw);          // kBulkStages x 8 rows x 128
  const int G = d.G;
  const int nch = (2 + G) * D;
  float* u = ring + kBulkStages * kStageFloats;               // [K][q (D) | k (D) | v of G heads]
  float* osm = u + K * nch;                                   // [K][G*D]
  float* gate = osm + K * G * D;                              // [K][alpha[G], beta[G]]
  __shared__ uint64_t full[kBulkStages], empty[kBulkStages];
  __shared__ float red[K][3];
  __shared__ int abort_flag;

  const int n = blockIdx.x / d.Hk;
  const int kh = blockIdx.x - n * d.Hk;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t C = d.C;
  const int h0 = G * kh;
  const int nst = G * D / kBulkRows;
  const int sl = slot_of(slots, n, status);  // state and history slot of batch row n
  if (sl < 0) {  // padding row: zero output for every token, nothing else touched
    for (int i = tid; i < K * G * D; i += kBulkThreads) {
      const int t = i / (G * D);
      o[(((int64_t)n * K + t) * d.Hv + h0) * D + (i - t * G * D)] = from_f<T>(0.f);
    }
    return;
  }
  float* st = state + ((int64_t)sl * d.Hv + h0) * D * D;  // the G heads' rows are contiguous
  // tokens applied to the state and history (and outputs written)
  int nk = K;
  if (write_state && accept) nk = min(max(accept[n], 0), K);
  const int nout = write_state ? nk : K;

  if (tid == 0) {
    for (int s = 0; s < kBulkStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kBulkThreads / 32);
    }
    tc::mbar_init_fence();
    abort_flag = 0;
  }
  __syncthreads();
  if (tid == 0) {
    for (int s = 0; s < kBulkStages && s < nst; ++s) {
      tc::mbar_expect_tx(&full[s], kStageFloats * 4);
      tc::bulk_load(ring + s * kStageFloats, st + (int64_t)s * kStageFloats, kStageFloats * 4, &full[s]);
    }
  }

  // ---- conv + SiLU of the owned channels for every token; shift the history by nk
  for (int idx = tid; idx < nch; idx += kBulkThreads) {
    const int64_t c = idx < D ? (int64_t)kh * D + idx
                              : (idx < 2 * D ? (int64_t)d.Hk * D + (int64_t)kh * D + (idx - D)
                                             : 2LL * d.Hk * D + (int64_t)h0 * D + (idx - 2 * D));
    T* hp = hist + (int64_t)sl * 3 * C + c;
    T xs[3 + K];  // raw inputs, oldest first
    xs[0] = hp[0];
    xs[1] = hp[C];
    xs[2] = hp[2 * C];
#pragma unroll
    for (int t = 0; t < K; ++t) xs[3 + t] = qkv[((int64_t)n * K + t) * C + c];
    const float4 w = __ldg(reinterpret_cast<const float4*>(conv_w + c * 4));
#pragma unroll
    for (int t = 0; t < K; ++t)
      u[t * nch + idx] = silu_f(conv4(w, to_f(xs[t]), to_f(xs[t + 1]), to_f(xs[t + 2]), to_f(xs[t + 3])));
    if (write_state && nk > 0) {  // new history: the last 3 of [h0, h1, h2, x_0 .. x_{nk-1}]
      T n0 = xs[1], n1 = xs[2], n2 = xs[3];
#pragma unroll
      for (int m = 2; m <= K; ++m)
        if (nk == m) {
          n0 = xs[m];
          n1 = xs[m + 1];
          n2 = xs[m + 2];
        }
      hp[0] = n0;
      hp[C] = n1;
      hp[2 * C] = n2;
    }
  }
  for (int e = tid; e < K * G; e += kBulkThreads) {
    const int t = e / G, hh = e - t * G, h = h0 + hh;
    float g, al, be;
    gates_f(ldg_f(a + ((int64_t)n * K + t) * d.Hv + h), dt_bias[h], A_log[h], ldg_f(b + ((int64_t)n * K + t) * d.Hv + h),
            g, al, be);
    gate[t * 2 * G + hh] = al;
    gate[t * 2 * G + G + hh] = be;
  }
  __syncthreads();
  for (int t = warp; t < K; t += kBulkThreads / 32) {  // L2 norms of q and k per token
    const float* ut = u + t * nch;
    float sq = 0.f, sk = 0.f, sqk = 0.f;
    for (int i = lane; i < D; i += 32) {
      const float qv = ut[i], kv = ut[D + i];
      sq = __fmaf_rn(qv, qv, sq);
      sk = __fmaf_rn(kv, kv, sk);
      sqk = __fmaf_rn(qv, kv, sqk);
    }
    sq = warp_sum(sq);
    sk = warp_sum(sk);
    sqk = warp_sum(sqk);
    if (lane == 0) {
      const float rq = __fmul_rn(d.q_scale, rsqrtf(sq + d.l2_eps)), rk = rsqrtf(sk + d.l2_eps);
      red[t][0] = rq;
      red[t][1] = rk;
      red[t][2] = __fmul_rn(__fmul_rn(rq, rk), sqk);
    }
  }
  __syncthreads();

  // ---- stream the rows: 16 lanes per row, 2 rows per warp, 8 rows per stage
  const int l16 = lane & 15, hr = lane >> 4;
  float4 kq[K][2], qq[K][2];
#pragma unroll
  for (int t = 0; t < K; ++t) {
    const float rq = red[t][0], rk = red[t][1];
    const float* ut = u + t * nch;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int i0 = 4 * l16 + 64 * m;
      qq[t][m] = make_float4(__fmul_rn(ut[i0], rq), __fmul_rn(ut[i0 + 1], rq), __fmul_rn(ut[i0 + 2], rq),
                             __fmul_rn(ut[i0 + 3], rq));
      kq[t][m] = make_float4(__fmul_rn(ut[D + i0], rk), __fmul_rn(ut[D + i0 + 1], rk), __fmul_rn(ut[D + i0 + 2], rk),
                             __fmul_rn(ut[D + i0 + 3], rk));
    }
  }
  for (int s = 0; s < nst; ++s) {
    const int slot = s % kBulkStages;
    const uint32_t par = (uint32_t)(s / kBulkStages) & 1u;
    if (!tc::mbar_wait(&full[slot], par, kBulkWaitNs)) abort_flag = 1;
    if (!abort_flag) {
      const int lrow = 2 * warp + hr;
      const int row = s * kBulkRows + lrow;
      const float* src = ring + slot * kStageFloats + lrow * D;
      float4 r[2];
      r[0] = *reinterpret_cast<const float4*>(src + 4 * l16);
      r[1] = *reinterpret_cast<const float4*>(src + 64 + 4 * l16);
      const int hh = row / D;
#pragma unroll
      for (int t = 0; t < K; ++t) {
        if (t < nout) {
          float kap = dot4(kq[t][1], r[1], dot4(kq[t][0], r[0], 0.f));
          float rho = dot4(qq[t][1], r[1], dot4(qq[t][0], r[0], 0.f));
#pragma unroll
          for (int off = 1; off < 16; off <<= 1) {
            kap += __shfl_xor_sync(0xffffffffu, kap, off);
            rho += __shfl_xor_sync(0xffffffffu, rho, off);
          }
          const float al = gate[t * 2 * G + hh], be = gate[t * 2 * G + G + hh];
          const float delta = __fmul_rn(be, __fsub_rn(u[t * nch + 2 * D + row], __fmul_rn(al, kap)));
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            r[m].x = __fmaf_rn(delta, kq[t][m].x, __fmul_rn(al, r[m].x));
            r[m].y = __fmaf_rn(delta, kq[t][m].y, __fmul_rn(al, r[m].y));
            r[m].z = __fmaf_rn(delta, kq[t][m].z, __fmul_rn(al, r[m].z));
            r[m].w = __fmaf_rn(delta, kq[t][m].w, __fmul_rn(al, r[m].w));
          }
          if (l16 == 0) osm[t * G * D + row] = __fmaf_rn(delta, red[t][2], __fmul_rn(al, rho));
          if (t + 1 == nk && write_state) {
            float4* dst = reinterpret_cast<float4*>(st + (int64_t)row * D);
            __stcs(dst + l16, r[0]);
            __stcs(dst + l16 + 16, r[1]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&empty[slot]);
    if (tid == 0 && s + kBulkStages < nst) {  // refill this slot once every warp has read it
      if (!tc::mbar_wait(&empty[slot], par, kBulkWaitNs)) abort_flag = 1;
      tc::fence_async_smem();
      tc::mbar_expect_tx(&full[slot], kStageFloats * 4);
      tc::bulk_load(ring + slot * kStageFloats, st + (int64_t)(s + kBulkStages) * kStageFloats, kStageFloats * 4,
                    &full[slot]);
    }
  }
  __syncthreads();
  if (abort_flag) {
    if (tid == 0) set_status(status, kStatusWaitTimeout);
    return;
  }

  // ---- zero-centred RMSNorm over d_v, times sigmoid(z); one rounding to io dtype
  for (int e = warp; e < nout * G; e += kBulkThreads / 32) {
    const int t = e / G, hh = e - t * G;
    const float* ot = osm + t * G * D + hh * D;
    float ss = 0.f;
    for (int j = lane; j < D; j += 32) ss = __fmaf_rn(ot[j], ot[j], ss);
    ss = warp_sum(ss);
    const float rr = rsqrtf(ss / D + d.norm_eps);
    const int64_t off = (((int64_t)n * K + t) * d.Hv + h0 + hh) * D;
    for (int j = lane; j < D; j += 32) {
      const float zz = ldg_f(z + off + j);
      o[off + j] = from_f<T>(__fmul_rn(__fmul_rn(__fmul_rn(ot[j], rr), 1.0f + norm_w[j]), sigmoid_f(zz)));
    }
  }
}

template <typename T, int K>
cudaError_t launch_bulk(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                        const float* norm_w, const void* qkv, const void* z, const void* a, const void* b, int32_t N,
                        const int32_t* accept, int write_state, Slots slots, void* hist, float* state, void* o,
                        int32_t* status, cudaStream_t stream) {
  const size_t smem =
      (size_t)(kBulkStages * kBulkRows * 128 + K * (2 + d.G) * 128 + K * d.G * 128 + K * 2 * d.G) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(decode_bulk_kernel<T, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  LaunchScope scope(GDN_K_DECODE, stream);
  decode_bulk_kernel<T, K><<<(unsigned)((int64_t)N * d.Hk), kBulkThreads, smem, stream>>>(
      d, conv_w, A_log, dt_bias, norm_w, (const T*)qkv, (const T*)z, (const T*)a, (const T*)b, accept, write_state,
      slots, (T*)hist, state, (T*)o, status);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_multi_t(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                           const float* norm_w, const void* qkv, const void* z, const void* a, const void* b, int32_t N,
                           int32_t K, const int32_t* accept, int write_state, Slots slots, void* hist, float* state,
                           void* o, int32_t* status, cudaStream_t stream) {
#define GDN_MULTI(KK)                                                                                                 \
  return launch_bulk<T, KK>(d, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, N, accept, write_state, slots, hist, \
                            state, o, status, stream)
  switch (K) {
    case 1: GDN_MULTI(1);
    case 2: GDN_MULTI(2);
    case 3: GDN_MULTI(3);
    default: GDN_MULTI(4);
  }
#undef GDN_MULTI
}

template <typename T, int D>
cudaError_t launch_t(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                     const float* norm_w, const void* qkv, const void* z, const void* a, const void* b, int32_t N,
                     Slots slots, void* hist, float* state, void* o, int32_t* status, cudaStream_t stream) {
  const size_t smem = (size_t)((2 + d.G) * D + d.G * D + 2 * d.G) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  LaunchScope scope(GDN_K_DECODE, stream);
  decode_kernel<T, D><<<(unsigned)((int64_t)N * d.Hk), kDecThreads, smem, stream>>>(
      d, conv_w, A_log, dt_bias, norm_w, (const T*)qkv, (const T*)z, (const T*)a, (const T*)b, slots, (T*)hist, state,
      (T*)o, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_step(const Dims& d, bool bf16, const float* conv_w, const float* A_log,
                               const float* dt_bias, const float* norm_w, const void* qkv, const void* z,
                               const void* a, const void* b, int32_t N, Slots slots, void* conv_state, float* state,
                               void* o, int32_t* status, cudaStream_t stream) {
  if (N <= 0) return cudaSuccess;
  if (d.dk == 128) {
    return bf16 ? launch_bulk<__nv_bfloat16, 1>(d, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, N, nullptr, 1, slots,
                                                conv_state, state, o, status, stream)
                : launch_bulk<float, 1>(d, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, N, nullptr, 1, slots,
                                        conv_state, state, o, status, stream);
  }
#define GDN_DEC(T, D) \
  return launch_t<T, D>(d, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, N, slots, conv_state, state, o, status, stream)
  if (bf16) {
    switch (d.dk) {
      case 32: GDN_DEC(__nv_bfloat16, 32);
      case 64: GDN_DEC(__nv_bfloat16, 64);
      default: GDN_DEC(__nv_bfloat16, 128);
    }
  } else {
    switch (d.dk) {
      case 32: GDN_DEC(float, 32);
      case 64: GDN_DEC(float, 64);
      default: GDN_DEC(float, 128);
    }
  }
#undef GDN_DEC
}

cudaError_t launch_decode_multi(const Dims& d, bool bf16, const float* conv_w, const float* A_log,
                                const float* dt_bias, const float* norm_w, const void* qkv, const void* z,
                                const void* a, const void* b, int32_t N, int32_t K, const int32_t* accept,
                                int write_state, Slots slots, void* conv_state, float* state, void* o,
                                int32_t* status, cudaStream_t stream) {
  if (N <= 0) return cudaSuccess;
  return bf16 ? launch_multi_t<__nv_bfloat16>(d, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, N, K, accept,
                                              write_state, slots, conv_state, state, o, status, stream)
              : launch_multi_t<float>(d, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, N, K, accept, write_state,
                                      slots, conv_state, state, o, status, stream);
}

}  // namespace gdn
