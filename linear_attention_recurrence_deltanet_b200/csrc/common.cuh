// Device helpers shared by the GDN kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// Geometry as the kernels see it (validated on the host).
struct Dims {
  int32_t Hk, Hv, dk, dv, W, G;  // G = Hv / Hk value heads per key head
  int64_t C;                      // conv channels = 2*Hk*dk + Hv*dv
  float l2_eps, norm_eps, q_scale;
};

// Device status word codes (read and cleared by gdn_get_device_status).
enum : int32_t {
  kStatusOk = 0,
  kStatusWaitTimeout = 1,   // a bounded wait gave up
  kStatusBadSlot = 3,       // a state slot index past the end of the pool (the row was skipped)
};

__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// State slots of a batch: row n of the batch reads and writes slot idx[n] of
// the state and conv-history pools (slot n when idx is NULL).  A negative slot
// marks a padding row; a slot at or past `count` is reported and treated as
// padding.
struct Slots {
  const int32_t* idx;
  int32_t count;
};
__device__ __forceinline__ int slot_of(const Slots& s, int n, int32_t* status) {
  if (!s.idx) return n;
  const int v = s.idx[n];
  if (v >= s.count) {
    set_status(status, kStatusBadSlot);
    return -1;
  }
  return v;
}

// io element access: fp32 or bf16 storage, fp32 arithmetic.
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Read-only, streaming load of one io element.
template <typename T> __device__ __forceinline__ float ldg_f(const T* p) { return to_f(__ldg(p)); }

__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + __expf(-x)); }
// SiLU(y) = y * sigmoid(y), written as y / (1 + e^-y).
__device__ __forceinline__ float silu_f(float y) { return y / (1.0f + __expf(-y)); }
// softplus in the overflow-free form max(x,0) + log1p(exp(-|x|)).
__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.0f) + log1pf(__expf(-fabsf(x))); }

// Gates of one token and value head: g = -exp(A_log) * softplus(a + dt_bias),
// alpha = exp(g), beta = sigmoid(b).
__device__ __forceinline__ void gates_f(float a, float dt_bias, float A_log, float b, float& g, float& alpha,
                                        float& beta) {
  g = -expf(A_log) * softplus_f(a + dt_bias);
  alpha = expf(g);
  beta = 1.0f / (1.0f + expf(-b));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 64-bit finaliser of SplitMix64 (Steele, Lea, Flood, "Fast splittable
// pseudorandom number generators", OOPSLA 2014), used as the word mixer of the
// state-blob checksum.
__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}
// Checksum term of 64-bit word `w` at word index `i` (terms are summed mod 2^64).
__host__ __device__ __forceinline__ uint64_t checksum_term(uint64_t w, uint64_t i) {
  return mix64(w + (i + 1) * 0x9e3779b97f4a7c15ULL);
}

}  // namespace gdn
