// Token-recurrent GDN prefill on CUDA cores, fp32 throughout.
//
// This is the fp32-input path (and an independent twin of the chunked
// tensor-core prefill): it runs the gated delta rule one token at a time,
// exactly in the form the recurrence is defined ("fp32 Gated DeltaNet
// recurrence", DS4Server issue #95, implementation comment), so its only
// deviation from float64 is fp32 rounding.
//
// One CTA per (sequence, value head); 4*D threads.  Thread (j, rg) keeps rows
// [rg*D/4, (rg+1)*D/4) of column j of the fp32 state S (d_k x d_v) in
// registers for the whole sequence.  Tokens are staged 32 at a time:
//   A  conv + SiLU of the head's q/k/v channels (one thread per channel, the
//      3-input window carried in registers) and the gates;
//   B  L2 norms of q and k (one warp per token);
//   C  the recurrence, token by token: two dots over d_k (local FMAs + 2
//      shuffles), delta_j, the rank-1 update, and o_j = alpha*rho + delta*q^.k^;
//   D  RMSNorm over d_v times sigmoid(z), one rounding to the io dtype.
// The conv history is not written here (other value heads of the same key
// head still read it); the history kernel runs afterwards.
#include "../../include/gdn.h"
#include "internal.h"

namespace gdn {
namespace {

constexpr int kCT = 32;  // tokens staged per pass

template <int D> struct RecLayout {
  static constexpr int NT = 4 * D;       // threads
  static constexpr int RPT = D / 4;      // state rows per thread
  static constexpr int SEG = D / 4 + 4;  // padded row-group segment of q^/k^ (bank spread)
  static constexpr int QK = 4 * SEG;     // padded q^/k^ vector
  static constexpr size_t smem_floats = (size_t)kCT * (2 * QK + 2 * D) + 3 * kCT;
};

template <typename T, int D>
__global__ void __launch_bounds__(4 * D, 1)
    prefill_recurrent_kernel(Dims d, const float* __restrict__ conv_w, const float* __restrict__ A_log,
                             const float* __restrict__ dt_bias, const float* __restrict__ norm_w,
                             const T* __restrict__ qkv, const T* __restrict__ z, const T* __restrict__ a,
                             const T* __restrict__ b, const int32_t* __restrict__ cu,
                             const int32_t* __restrict__ order, int zero_state, int zero_conv,
                             const T* __restrict__ hist, float* __restrict__ state, T* __restrict__ o) {
  using L = RecLayout<D>;
  constexpr int NW = L::NT / 32;
  extern __shared__ float smem[];
  float* Uq = smem;                  // [kCT][QK]
  float* Uk = Uq + kCT * L::QK;      // [kCT][QK]
  float* Uv = Uk + kCT * L::QK;      // [kCT][D]
  float* Os = Uv + kCT * D;          // [kCT][D]
  float* Ga = Os + kCT * D;          // alpha
  float* Gb = Ga + kCT;              // beta
  float* Gqk = Gb + kCT;             // q^.k^

  const int h = blockIdx.x % d.Hv;
  const int oi = blockIdx.x / d.Hv;
  const int n = order ? order[oi] : oi;
  const int kh = h / d.G;
  const int64_t t0 = cu[n];
  const int64_t len = cu[n + 1] - t0;
  if (len <= 0) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t C = d.C;
  const int64_t HvD = (int64_t)d.Hv * D;

  // state column j, row group rg
  const int j = tid >> 2, rg = tid & 3;
  float S[L::RPT];
  float* st = state + (((int64_t)n * d.Hv + h) * D + j) * D + rg * L::RPT;
  if (zero_state) {
#pragma unroll
    for (int m = 0; m < L::RPT; ++m) S[m] = 0.f;
  } else {
#pragma unroll
    for (int m = 0; m < L::RPT; m += 4) {
      const float4 v = *reinterpret_cast<const float4*>(st + m);
      S[m] = v.x; S[m + 1] = v.y; S[m + 2] = v.z; S[m + 3] = v.w;
    }
  }

  // conv channel owned by this thread (threads < 3D) and its smem slot
  const bool conv_thread = tid < 3 * D;
  int64_t c = 0;
  float* dst = nullptr;
  int dst_stride = 0;
  float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, x0 = 0.f, x1 = 0.f, x2 = 0.f;
  if (conv_thread) {
    if (tid < D) {
      c = (int64_t)kh * D + tid;
      dst = Uq + (tid / L::RPT) * L::SEG + tid % L::RPT;
      dst_stride = L::QK;
    } else if (tid < 2 * D) {
      c = (int64_t)d.Hk * D + (int64_t)kh * D + (tid - D);
      dst = Uk + ((tid - D) / L::RPT) * L::SEG + (tid - D) % L::RPT;
      dst_stride = L::QK;
    } else {
      c = 2LL * d.Hk * D + (int64_t)h * D + (tid - 2 * D);
      dst = Uv + (tid - 2 * D);
      dst_stride = D;
    }
    const float4 w = __ldg(reinterpret_cast<const float4*>(conv_w + c * 4));
    w0 = w.x; w1 = w.y; w2 = w.z; w3 = w.w;
    if (!zero_conv) {
      const T* hp = hist + (int64_t)n * 3 * C + c;
      x0 = to_f(hp[0]); x1 = to_f(hp[C]); x2 = to_f(hp[2 * C]);
    }
  }
  const float Alog = A_log[h], dtb = dt_bias[h];

  for (int64_t p0 = 0; p0 < len; p0 += kCT) {
    const int nt = (int)min((int64_t)kCT, len - p0);
    const T* xrow = qkv + (t0 + p0) * C;
    // ---- A: conv + SiLU, gates
    if (conv_thread) {
      for (int tok = 0; tok < nt; tok += 8) {
        float xv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) xv[e] = (tok + e < nt) ? ldg_f(xrow + (int64_t)(tok + e) * C + c) : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (tok + e < nt) {
            const float y = w0 * x0 + w1 * x1 + w2 * x2 + w3 * xv[e];
            dst[(tok + e) * dst_stride] = silu_f(y);
            x0 = x1; x1 = x2; x2 = xv[e];
          }
        }
      }
    } else if (tid - 3 * D < nt) {
      const int tok = tid - 3 * D;
      const int64_t t = t0 + p0 + tok;
      float g, al, be;
      gates_f(ldg_f(a + t * d.Hv + h), dtb, Alog, ldg_f(b + t * d.Hv + h), g, al, be);
      Ga[tok] = al;
      Gb[tok] = be;
    }
    __syncthreads();
    // ---- B: L2 norms of q and k, and q^.k^
    for (int tok = warp; tok < nt; tok += NW) {
      float* q = Uq + tok * L::QK;
      float* k = Uk + tok * L::QK;
      float sq = 0.f, sk = 0.f, sqk = 0.f;
      for (int i = lane; i < D; i += 32) {
        const int s = (i / L::RPT) * L::SEG + i % L::RPT;
        sq += q[s] * q[s];
        sk += k[s] * k[s];
        sqk += q[s] * k[s];
      }
      sq = warp_sum(sq);
      sk = warp_sum(sk);
      sqk = warp_sum(sqk);
      const float rq = d.q_scale * rsqrtf(sq + d.l2_eps), rk = rsqrtf(sk + d.l2_eps);
      for (int i = lane; i < D; i += 32) {
        const int s = (i / L::RPT) * L::SEG + i % L::RPT;
        q[s] *= rq;
        k[s] *= rk;
      }
      if (lane == 0) Gqk[tok] = rq * rk * sqk;
    }
    __syncthreads();
    // ---- C: the recurrence, token by token
    for (int tok = 0; tok < nt; ++tok) {
      const float4* k4 = reinterpret_cast<const float4*>(Uk + tok * L::QK + rg * L::SEG);
      const float4* q4 = reinterpret_cast<const float4*>(Uq + tok * L::QK + rg * L::SEG);
      float kap = 0.f, rho = 0.f;
#pragma unroll
      for (int m = 0; m < L::RPT / 4; ++m) {
        const float4 kk = k4[m], qq = q4[m];
        kap += kk.x * S[4 * m] + kk.y * S[4 * m + 1] + kk.z * S[4 * m + 2] + kk.w * S[4 * m + 3];
        rho += qq.x * S[4 * m] + qq.y * S[4 * m + 1] + qq.z * S[4 * m + 2] + qq.w * S[4 * m + 3];
      }
      kap += __shfl_xor_sync(0xffffffffu, kap, 1);
      rho += __shfl_xor_sync(0xffffffffu, rho, 1);
      kap += __shfl_xor_sync(0xffffffffu, kap, 2);
      rho += __shfl_xor_sync(0xffffffffu, rho, 2);
      const float al = Ga[tok], be = Gb[tok];
      const float delta = be * (Uv[tok * D + j] - al * kap);
#pragma unroll
      for (int m = 0; m < L::RPT / 4; ++m) {
        const float4 kk = k4[m];
        S[4 * m] = al * S[4 * m] + delta * kk.x;
        S[4 * m + 1] = al * S[4 * m + 1] + delta * kk.y;
        S[4 * m + 2] = al * S[4 * m + 2] + delta * kk.z;
        S[4 * m + 3] = al * S[4 * m + 3] + delta * kk.w;
      }
      if (rg == 0) Os[tok * D + j] = al * rho + delta * Gqk[tok];
    }
    __syncthreads();
    // ---- D: RMSNorm over d_v, times sigmoid(z)
    for (int tok = warp; tok < nt; tok += NW) {
      const float* os = Os + tok * D;
      float ss = 0.f;
      for (int i = lane; i < D; i += 32) ss += os[i] * os[i];
      ss = warp_sum(ss);
      const float r = rsqrtf(ss / D + d.norm_eps);
      const int64_t off = (t0 + p0 + tok) * HvD + (int64_t)h * D;
      for (int i = lane; i < D; i += 32)
        o[off + i] = from_f<T>(os[i] * r * (1.0f + norm_w[i]) * sigmoid_f(ldg_f(z + off + i)));
    }
    // stage A of the next pass writes Uq/Uk/Uv/Ga/Gb only, which D does not read
  }
#pragma unroll
  for (int m = 0; m < L::RPT; m += 4) *reinterpret_cast<float4*>(st + m) = make_float4(S[m], S[m + 1], S[m + 2], S[m + 3]);
}

template <typename T, int D>
cudaError_t launch_t(const Dims& d, const float* conv_w, const float* A_log, const float* dt_bias,
                     const float* norm_w, const void* qkv, const void* z, const void* a, const void* b,
                     const int32_t* cu, const int32_t* order, int32_t N, bool zero_state, bool zero_conv,
                     const void* hist, float* state, void* o, cudaStream_t stream) {
  const size_t smem = RecLayout<D>::smem_floats * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(prefill_recurrent_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  LaunchScope scope(GDN_K_PREFILL_RECURRENT, stream);
  prefill_recurrent_kernel<T, D><<<(unsigned)((int64_t)N * d.Hv), RecLayout<D>::NT, smem, stream>>>(
      d, conv_w, A_log, dt_bias, norm_w, (const T*)qkv, (const T*)z, (const T*)a, (const T*)b, cu, order,
      zero_state, zero_conv, (const T*)hist, state, (T*)o);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_recurrent(const Dims& d, bool bf16, const float* conv_w, const float* A_log,
                                     const float* dt_bias, const float* norm_w, const void* qkv, const void* z,
                                     const void* a, const void* b, const int32_t* cu, const int32_t* order,
                                     int32_t N, bool zero_state, bool zero_conv, const void* conv_state,
                                     float* state, void* o, cudaStream_t stream) {
  if (N <= 0) return cudaSuccess;
#define GDN_REC(T, D)                                                                                         \
  return launch_t<T, D>(d, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, cu, order, N, zero_state, zero_conv, \
                        conv_state, state, o, stream)
  if (bf16) {
    switch (d.dk) {
      case 32: GDN_REC(__nv_bfloat16, 32);
      case 64: GDN_REC(__nv_bfloat16, 64);
      default: GDN_REC(__nv_bfloat16, 128);
    }
  } else {
    switch (d.dk) {
      case 32: GDN_REC(float, 32);
      case 64: GDN_REC(float, 64);
      default: GDN_REC(float, 128);
    }
  }
#undef GDN_REC
}

}  // namespace gdn
