// Causal depthwise Conv1D (width 4) + SiLU over the q/k/v channels, and the
// rolling conv-history cache ("causal depthwise Conv1D ... and
// recurrent-state cache": DS4Server issue #88, section Scope; "BF16 width-4
// convolution history": issue #95, implementation comment).
//
// y[t, c] = SiLU(sum_{j<4} w[c, j] * x~[t - 3 + j, c]), x~ = history ++ inputs;
// the history holds the last 3 raw inputs of a sequence in the io dtype and is
// carried as raw bytes (bit-exact).  All three kernels are HBM-bound
// elementwise passes: each thread owns 16 bytes of channels (8 bf16 or 4 fp32)
// so every global access is a 16-byte vector and a warp touches 512
// contiguous bytes per row.
#include "../../include/gdn.h"
#include "internal.h"
#include "vec.cuh"

namespace gdn {
namespace {

constexpr int kW = 4;                 // conv width (validated by the ABI layer)
constexpr int kConvThreads = 128;
constexpr int kTokensPerCta = 32;     // conv prefill: tokens walked by one thread

template <typename T>
__device__ __forceinline__ void load_w(const float* conv_w, int64_t c0, float (*w)[kW]) {
  constexpr int V = Vec16<T>::N;
#pragma unroll
  for (int v = 0; v < V; ++v) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(conv_w + (c0 + v) * kW));
    w[v][0] = t.x; w[v][1] = t.y; w[v][2] = t.z; w[v][3] = t.w;
  }
}

template <typename T>
__global__ void __launch_bounds__(kConvThreads) conv_prefill_kernel(Dims d, const T* __restrict__ x,
                                                                      const float* __restrict__ conv_w,
                                                                      const int32_t* __restrict__ cu,
                                                                      const T* __restrict__ hist, T* __restrict__ y) {
  constexpr int V = Vec16<T>::N;
  const int n = blockIdx.z;
  const int64_t t0 = cu[n];
  const int64_t len = cu[n + 1] - t0;
  const int64_t p0 = (int64_t)blockIdx.y * kTokensPerCta;
  const int64_t c0 = ((int64_t)blockIdx.x * kConvThreads + threadIdx.x) * V;
  if (p0 >= len || c0 >= d.C) return;
  float w[V][kW];
  load_w<T>(conv_w, c0, w);
  float win[kW - 1][V];  // raw inputs at positions p-3, p-2, p-1
#pragma unroll
  for (int i = 0; i < kW - 1; ++i) {
    const int64_t m = p0 - (kW - 1) + i;
    const T* src = (m < 0) ? hist + ((int64_t)n * (kW - 1) + (m + kW - 1)) * d.C + c0 : x + (t0 + m) * d.C + c0;
    Vec16<T>::unpack(ld16(src), win[i]);
  }
  const int64_t pend = min(len, p0 + kTokensPerCta);
  for (int64_t p = p0; p < pend; ++p) {
    float cur[V], out[V];
    Vec16<T>::unpack(ld16(x + (t0 + p) * d.C + c0), cur);
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const float yv = w[v][0] * win[0][v] + w[v][1] * win[1][v] + w[v][2] * win[2][v] + w[v][3] * cur[v];
      out[v] = silu_f(yv);
      win[0][v] = win[1][v];
      win[1][v] = win[2][v];
      win[2][v] = cur[v];
    }
    st16(y + (t0 + p) * d.C + c0, Vec16<T>::pack(out));
  }
}

// New history of every sequence: the last 3 raw entries of history ++ inputs.
// Runs after every kernel that reads the old history (stream order).
template <typename T>
__global__ void __launch_bounds__(kConvThreads) conv_history_kernel(Dims d, const T* __restrict__ x,
                                                                      const int32_t* __restrict__ cu, int zero_hist,
                                                                      T* __restrict__ hist) {
  constexpr int V = Vec16<T>::N;
  const int n = blockIdx.y;
  const int64_t c0 = ((int64_t)blockIdx.x * kConvThreads + threadIdx.x) * V;
  if (c0 >= d.C) return;
  const int64_t t0 = cu[n];
  const int64_t len = cu[n + 1] - t0;
  T* h = hist + (int64_t)n * (kW - 1) * d.C + c0;
  uint4 v[kW - 1];
#pragma unroll
  for (int i = 0; i < kW - 1; ++i) {
    const int64_t m = len + i - (kW - 1);
    if (m >= 0)
      v[i] = ld16(x + (t0 + m) * d.C + c0);
    else
      v[i] = zero_hist ? make_uint4(0, 0, 0, 0) : ld16_rw(h + (m + kW - 1) * d.C);
  }
#pragma unroll
  for (int i = 0; i < kW - 1; ++i) st16(h + i * d.C, v[i]);
}

template <typename T>
__global__ void __launch_bounds__(kConvThreads) conv_step_kernel(Dims d, const T* __restrict__ x,
                                                                   const float* __restrict__ conv_w,
                                                                   T* __restrict__ hist, T* __restrict__ y) {
  constexpr int V = Vec16<T>::N;
  const int n = blockIdx.y;
  const int64_t c0 = ((int64_t)blockIdx.x * kConvThreads + threadIdx.x) * V;
  if (c0 >= d.C) return;
  float w[V][kW];
  load_w<T>(conv_w, c0, w);
  T* h = hist + (int64_t)n * (kW - 1) * d.C + c0;
  const uint4 r0 = ld16_rw(h), r1 = ld16_rw(h + d.C), r2 = ld16_rw(h + 2 * d.C);
  const uint4 rx = ld16(x + (int64_t)n * d.C + c0);
  float h0[V], h1[V], h2[V], cur[V], out[V];
  Vec16<T>::unpack(r0, h0); Vec16<T>::unpack(r1, h1); Vec16<T>::unpack(r2, h2); Vec16<T>::unpack(rx, cur);
#pragma unroll
  for (int v = 0; v < V; ++v)
    out[v] = silu_f(w[v][0] * h0[v] + w[v][1] * h1[v] + w[v][2] * h2[v] + w[v][3] * cur[v]);
  st16(y + (int64_t)n * d.C + c0, Vec16<T>::pack(out));
  st16(h, r1);
  st16(h + d.C, r2);
  st16(h + 2 * d.C, rx);
}

template <typename T> dim3 channel_grid(const Dims& d, int y, int z = 1) {
  const int64_t per_cta = (int64_t)kConvThreads * Vec16<T>::N;
  return dim3((unsigned)((d.C + per_cta - 1) / per_cta), y, z);
}

}  // namespace

cudaError_t launch_conv_prefill(const Dims& d, bool bf16, const void* x, const float* conv_w, const int32_t* cu,
                                int32_t num_seqs, int32_t max_len, const void* conv_state, void* y,
                                cudaStream_t stream) {
  if (max_len <= 0 || num_seqs <= 0) return cudaSuccess;
  const int ytiles = (max_len + kTokensPerCta - 1) / kTokensPerCta;
  LaunchScope scope(GDN_K_CONV_PREFILL, stream);
  if (bf16) {
    using T = __nv_bfloat16;
    conv_prefill_kernel<T><<<channel_grid<T>(d, ytiles, num_seqs), kConvThreads, 0, stream>>>(
        d, (const T*)x, conv_w, cu, (const T*)conv_state, (T*)y);
  } else {
    conv_prefill_kernel<float><<<channel_grid<float>(d, ytiles, num_seqs), kConvThreads, 0, stream>>>(
        d, (const float*)x, conv_w, cu, (const float*)conv_state, (float*)y);
  }
  return cudaGetLastError();
}

cudaError_t launch_conv_history(const Dims& d, bool bf16, const void* x, const int32_t* cu, int32_t num_seqs,
                                bool zero_history, void* conv_state, cudaStream_t stream) {
  if (num_seqs <= 0) return cudaSuccess;
  LaunchScope scope(GDN_K_CONV_HISTORY, stream);
  if (bf16) {
    using T = __nv_bfloat16;
    conv_history_kernel<T><<<channel_grid<T>(d, num_seqs), kConvThreads, 0, stream>>>(d, (const T*)x, cu,
                                                                                     zero_history, (T*)conv_state);
  } else {
    conv_history_kernel<float><<<channel_grid<float>(d, num_seqs), kConvThreads, 0, stream>>>(
        d, (const float*)x, cu, zero_history, (float*)conv_state);
  }
  return cudaGetLastError();
}

cudaError_t launch_conv_step(const Dims& d, bool bf16, const void* x, const float* conv_w, int32_t num_seqs,
                             void* conv_state, void* y, cudaStream_t stream) {
  if (num_seqs <= 0) return cudaSuccess;
  LaunchScope scope(GDN_K_CONV_STEP, stream);
  if (bf16) {
    using T = __nv_bfloat16;
    conv_step_kernel<T><<<channel_grid<T>(d, num_seqs), kConvThreads, 0, stream>>>(d, (const T*)x, conv_w,
                                                                                  (T*)conv_state, (T*)y);
  } else {
    conv_step_kernel<float><<<channel_grid<float>(d, num_seqs), kConvThreads, 0, stream>>>(
        d, (const float*)x, conv_w, (float*)conv_state, (float*)y);
  }
  return cudaGetLastError();
}

}  // namespace gdn
