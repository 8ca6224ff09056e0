// bf16 GEMM on tcgen05 for the dense projections either side of the mixer
// (the "GDN projection" primitive and the BF16 projection kernels of DS4Server
// issue #95, sections Verification and implementation comment):
//   Y[M, N] = X[M, K] W[N, K]^T
// with W stored as a linear layer's weight (output features x input
// features), both operands K-major, fp32 accumulation in TMEM, bf16 out.
//
// Persistent: one CTA per SM walks the 128 x BN output tiles (m fastest, so
// the CTAs running together share the same few weight panels in L2).  K
// advances 64 columns per stage through a ring of TMA loads (128-byte
// swizzle).  Warp 0 issues the loads, warp 1 the MMAs (M = 128, N = BN,
// K = 16; each stage's commit frees its slot), warps 2..5 drain the
// accumulator.  TMEM holds two accumulators, so the epilogue of one tile
// overlaps the main loop of the next.  The epilogue routes every 8-column
// group to one of up to four outputs: the input projection writes the
// mixer's qkv, z, a and b from one GEMM.
#include <cuda.h>
#include <cuda_bf16.h>

#include "../../include/gdn.h"
#include "internal.h"
#include "tc.cuh"

namespace gdn {
namespace {

using namespace tc;

constexpr int GM = 128, GK = 64, kMaxStages = 8;
constexpr int kStageA = GM * GK * 2;  // 16 KB
constexpr int kRing = 196608;         // 192 KB of stages
constexpr int kGemmSmem = kRing + 1024;
constexpr int kGemmThreads = 192;
constexpr uint32_t kTmemCols = 512;  // two accumulators of up to 256 columns
constexpr uint64_t kWaitNs = 2000000000ull;

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw, int32_t M, int32_t N,
                int32_t K, int32_t BN, const __grid_constant__ GemmOutputs out, int32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tslot;
  bool bad = false;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int stage_bytes = kStageA + BN * GK * 2;
  const int stages = min(kMaxStages, kRing / stage_bytes);
  const int mt = (M + GM - 1) / GM, nt = (N + BN - 1) / BN, tiles = mt * nt;
  const int nk = (K + GK - 1) / GK;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(&drain, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(&tslot, kTmemCols);
  sync_tc();
  const uint32_t tbase = tslot;

  if (warp == 0) {
    if (lane == 0) {  // loads: ring slot i % stages, once the MMAs of load i - stages are done with it
      int i = 0;
      int last[kMaxStages];
      for (int s = 0; s < kMaxStages; ++s) last[s] = -1;
      for (int t = blockIdx.x; t < tiles && !bad; t += gridDim.x) {
        const int m0 = (t % mt) * GM, n0 = (t / mt) * BN;
        for (int kb = 0; kb < nk; ++kb, ++i) {
          const int s = i % stages;
          if (i >= stages && !mbar_wait(&empty[s], ((i / stages) & 1) ^ 1, kWaitNs)) {
            bad = true;
            break;
          }
          unsigned char* a = sm + s * stage_bytes;
          mbar_expect_tx(&full[s], stage_bytes);
          tma_load_2d(a, &tx, GK * kb, m0, &full[s]);
          tma_load_2d(a + kStageA, &tw, GK * kb, n0, &full[s]);
          last[s] = i;
        }
      }
      if (bad)  // let the copies already issued land before the block exits
        for (int s = 0; s < stages; ++s)
          if (last[s] >= 0) mbar_wait(&full[s], (last[s] / stages) & 1, kWaitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_f16(GM, BN, false, false) | (1u << 7) | (1u << 10);  // bf16 A and B
      int i = 0, j = 0;
      for (int t = blockIdx.x; t < tiles && !bad; t += gridDim.x, ++j) {
        const int ab = j & 1;
        if (j >= 2 && !mbar_wait(&acc_empty[ab], ((j >> 1) & 1) ^ 1, kWaitNs)) {
          bad = true;
          break;
        }
        fence_after();
        const uint32_t d = tbase + 256 * ab;
        for (int kb = 0; kb < nk; ++kb, ++i) {
          const int s = i % stages;
          if (!mbar_wait(&full[s], (i / stages) & 1, kWaitNs)) {
            bad = true;
            break;
          }
          fence_after();
          const uint32_t a = smem_u32(sm + s * stage_bytes), b = a + kStageA;
#pragma unroll
          for (int kk = 0; kk < GK / 16; ++kk)
            mma_f16(d, desc_kmaj(a, GM, kk), desc_kmaj(b, BN, kk), id, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (!bad) mma_commit(&acc_full[ab]);
      }
      // every MMA issued has finished before TMEM is released
      mma_commit(&drain);
      mbar_wait(&drain, 0, kWaitNs);
    }
  } else {  // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31, i.e. tile rows 32 q + lane
    const int q = warp & 3;
    int j = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
      const int ab = j & 1;
      const bool ok = mbar_wait(&acc_full[ab], (j >> 1) & 1, kWaitNs);
      if (__any_sync(0xffffffffu, !ok)) {  // the whole warp leaves together (the TMEM loads are warp-wide)
        bad = true;
        break;
      }
      fence_after();
      const int m0 = (t % mt) * GM, n0 = (t / mt) * BN;
      const int row = m0 + 32 * q + lane;
      const uint32_t src = tbase + 256 * ab + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        float v[32];
        tmem_ld32(src + 32 * cb, v);
        if (row >= M) continue;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = n0 + 32 * cb + 8 * g;
          if (col >= N) break;
          int k = 0;
#pragma unroll
          for (int u = 1; u < kGemmMaxOut; ++u)
            if (u < out.count && col >= out.start[u]) k = u;
          if (out.vec[k] && col + 8 <= out.start[k + 1]) {  // the 8 columns land in one output: one 16-byte store
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 p = __floats2bfloat162_rn(v[8 * g + 2 * e], v[8 * g + 2 * e + 1]);
              w4[e] = *reinterpret_cast<uint32_t*>(&p);
            }
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out.ptr[k]) + (int64_t)row * out.ld[k] +
                                 (col - out.start[k]);
            *reinterpret_cast<uint4*>(dst) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          } else {  // the group crosses an output boundary or the end, or its output is not 16-byte alignable
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int c = col + e;
              if (c >= N) break;
              while (k + 1 < out.count && c >= out.start[k + 1]) ++k;
              reinterpret_cast<__nv_bfloat16*>(out.ptr[k])[(int64_t)row * out.ld[k] + (c - out.start[k])] =
                  __float2bfloat16_rn(v[8 * g + e]);
            }
          }
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }
  if (sync_tc_any(bad) && tid == 0) set_status(status, kStatusWaitTimeout);
  if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

bool encode_bf16_2d(EncodeTiledFn enc, CUtensorMap* tm, const void* base, uint64_t cols, uint64_t rows,
                    uint32_t box_rows) {
  const cuuint64_t dim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t stride[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)GK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dim, stride, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

int gemm_tile_n(int32_t M, int32_t N, int32_t tile_n) {
  if (tile_n == 64 || tile_n == 128 || tile_n == 256) return tile_n;
  // fewest (rounds of tiles over the SMs) x (cost of one tile), a tile costing
  // its width plus a fixed 64 columns' worth of prologue and epilogue
  const int64_t mt = (M + GM - 1) / GM, sms = num_sms();
  int best = 256;
  int64_t best_cost = -1;
  for (int bn = 256; bn >= 64; bn >>= 1) {
    const int64_t rounds = (mt * ((N + bn - 1) / bn) + sms - 1) / sms;
    const int64_t cost = rounds * (bn + 64);
    if (best_cost < 0 || cost < best_cost) best = bn, best_cost = cost;
  }
  return best;
}

cudaError_t launch_gemm_bf16(const void* x, int32_t M, int32_t K, const void* w, int32_t N, int32_t tile_n,
                             const GemmOutputs& out, int32_t* status, cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  const int bn = gemm_tile_n(M, N, tile_n);
  CUtensorMap tx, tw;
  if (!encode_bf16_2d(enc, &tx, x, (uint64_t)K, (uint64_t)M, GM) ||
      !encode_bf16_2d(enc, &tw, w, (uint64_t)K, (uint64_t)N, (uint32_t)bn))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (int64_t)((M + GM - 1) / GM) * ((N + bn - 1) / bn);
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
  LaunchScope scope(GDN_K_GEMM, stream);
  gemm_kernel<<<grid, kGemmThreads, kGemmSmem, stream>>>(tx, tw, M, N, K, bn, out, status);
  return cudaGetLastError();
}

}  // namespace gdn
