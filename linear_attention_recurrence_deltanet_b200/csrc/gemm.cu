// bf16 GEMM on tcgen05 for the dense projections either side of the mixer
// (the "GDN projection" primitive and the BF16 projection kernels of DS4Server
// issue #95, sections Verification and implementation comment):
//   Y[M, N] = X[M, K] W[N, K]^T
// with W stored as a linear layer's weight (output features x input
// features), both operands K-major, fp32 accumulation in TMEM, bf16 out.
//
// K advances 64 columns per TMA box (128-byte swizzle); a ring stage holds one
// or two boxes of each operand.  Warp 0 issues the loads, warp 1 the MMAs
// (each stage's commit frees its slot), warps 2..5 drain the accumulator.
//   gemm_kernel         persistent, one CTA per 128 x BN tile (m fastest, so
//                       the CTAs running together share the same few weight
//                       panels in L2); two TMEM accumulators, so the epilogue
//                       of one tile overlaps the main loop of the next
//   gemm_pair_kernel    the same with a CTA pair per 256 x BN tile, MMAs of
//                       M = 256 issued by the even CTA over both CTAs' shared
//                       memory: each CTA loads only half of the weight panel,
//                       which cuts the operand bytes each SM moves per MMA by
//                       a third at BN = 256
//   gemm_splitk_kernel  up to 128 rows: a cluster of CTAs per tile, each on a
//                       slice of K, partial rows reduced through DSMEM
// BN is any multiple of 32 up to 256 (64 up for pairs); the host picks a
// power-of-two width from the number of tiles per wave.
// The epilogue routes every 8-column group to one of up to four outputs: the
// input projection writes the mixer's qkv, z, a and b from one GEMM.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>

#include "../../include/gdn.h"
#include "internal.h"
#include "tc.cuh"

namespace gdn {
namespace {

using namespace tc;

constexpr int GM = 128, GK = 64, kMaxStages = 8;
constexpr int kStageA = GM * GK * 2;  // 16 KB: 128 rows of X
constexpr int kRing = 229376;         // 224 KB of stages (seven of a pair CTA's 32 KB at BN = 256)
constexpr int kGemmSmem = kRing + 1024;  // + alignment slack: 225 KB of the 227 KB a block may have
constexpr int kGemmThreads = 192;
constexpr uint32_t kTmemCols = 512;  // two accumulators of up to 256 columns
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kIdescBf16 = (1u << 7) | (1u << 10);  // A and B bf16 (kind::f16)

// Store columns [col0, col0 + 32) of output row `row` (fp32 in v) as bf16.
__device__ __forceinline__ void store_block(const GemmOutputs& out, int row, int col0, int N, const float* v) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int col = col0 + 8 * g;
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
      __nv_bfloat16* dst =
          reinterpret_cast<__nv_bfloat16*>(out.ptr[k]) + (int64_t)row * out.ld[k] + (col - out.start[k]);
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

// ------------------------------------------------------------------ one CTA per tile
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw, int32_t M, int32_t N,
                int32_t K, int32_t BN, int32_t ksub, const __grid_constant__ GemmOutputs out, int32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tslot;
  bool bad = false;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int blk_b = BN * GK * 2;
  const int stage_bytes = ksub * (kStageA + blk_b);  // ksub 64-wide K blocks per stage
  const int stages = min(kMaxStages, kRing / stage_bytes);
  const int mt = (M + GM - 1) / GM, nt = (N + BN - 1) / BN, tiles = mt * nt;
  const int nk = (K + GK * ksub - 1) / (GK * ksub);

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
          for (int u = 0; u < ksub; ++u) {
            tma_load_2d(a + u * kStageA, &tx, GK * (kb * ksub + u), m0, &full[s]);
            tma_load_2d(a + ksub * kStageA + u * blk_b, &tw, GK * (kb * ksub + u), n0, &full[s]);
          }
          last[s] = i;
        }
      }
      if (bad)  // let the copies already issued land before the block exits
        for (int s = 0; s < stages; ++s)
          if (last[s] >= 0) mbar_wait(&full[s], (last[s] / stages) & 1, kWaitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_f16(GM, BN, false, false) | kIdescBf16;
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
          const uint32_t a = smem_u32(sm + s * stage_bytes), b = a + ksub * kStageA;
          for (int u = 0; u < ksub; ++u)
#pragma unroll
            for (int kk = 0; kk < GK / 16; ++kk)
              mma_f16(d, desc_kmaj(a + u * kStageA, GM, kk), desc_kmaj(b + u * blk_b, BN, kk), id,
                      (kb > 0 || u > 0 || kk > 0) ? 1u : 0u);
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
        if (row < M) store_block(out, row, n0 + 32 * cb, N, v);
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }
  if (sync_tc_any(bad) && tid == 0) set_status(status, kStatusWaitTimeout);
  if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------ split-K over a cluster (M <= 128)
// A cluster of S CTAs per 128 x BN output tile (only one row tile: M <= 128),
// CTA `rank` accumulating K blocks [kb0, kb1) in its own TMEM.  When M is
// small the weight stream is the limit and few tiles leave SMs idle; slicing
// K puts S CTAs on each tile.  After a cluster barrier (every MMA of the
// cluster is done, the leader's ring is free) the other CTAs store their fp32
// partial rows into the leader's ring through distributed shared memory;
// after a second barrier the leader adds them to its own and writes the tile.
__device__ __forceinline__ void st_cluster_v4(uint32_t caddr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(caddr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_splitk_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw, int32_t M,
                       int32_t N, int32_t K, int32_t BN, int32_t S, int32_t Mp, uint32_t tcols,
                       const __grid_constant__ GemmOutputs out, int32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages], acc_full;
  __shared__ uint32_t tslot;
  bool bad = false;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = (int)cluster_ctarank(), tile = blockIdx.x / S;
  const int n0 = tile * BN;
  const int blk_b = BN * GK * 2, stage_bytes = kStageA + blk_b;
  const int stages = min(kMaxStages, kRing / stage_bytes);
  const int nkb = (K + GK - 1) / GK;
  const int kb0 = (int)((int64_t)nkb * rank / S), kb1 = (int)((int64_t)nkb * (rank + 1) / S);
  const int nk = kb1 - kb0;  // >= 1: the host keeps S <= nkb

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(&tslot, tcols);
  sync_tc();
  const uint32_t tbase = tslot;

  if (warp == 0) {
    if (lane == 0) {
      int last[kMaxStages];
      for (int s = 0; s < kMaxStages; ++s) last[s] = -1;
      for (int i = 0; i < nk; ++i) {
        const int s = i % stages;
        if (i >= stages && !mbar_wait(&empty[s], ((i / stages) & 1) ^ 1, kWaitNs)) {
          bad = true;
          break;
        }
        unsigned char* a = sm + s * stage_bytes;
        mbar_expect_tx(&full[s], stage_bytes);
        tma_load_2d(a, &tx, GK * (kb0 + i), 0, &full[s]);
        tma_load_2d(a + kStageA, &tw, GK * (kb0 + i), n0, &full[s]);
        last[s] = i;
      }
      if (bad)
        for (int s = 0; s < stages; ++s)
          if (last[s] >= 0) mbar_wait(&full[s], (last[s] / stages) & 1, kWaitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_f16(GM, BN, false, false) | kIdescBf16;
      for (int i = 0; i < nk; ++i) {
        const int s = i % stages;
        if (!mbar_wait(&full[s], (i / stages) & 1, kWaitNs)) {
          bad = true;
          break;
        }
        fence_after();
        const uint32_t a = smem_u32(sm + s * stage_bytes), b = a + kStageA;
#pragma unroll
        for (int kk = 0; kk < GK / 16; ++kk)
          mma_f16(tbase, desc_kmaj(a, GM, kk), desc_kmaj(b, BN, kk), id, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      mma_commit(&acc_full);  // also when a wait ran out: every MMA issued has finished once it arrives
    }
  } else {
    const bool ok = mbar_wait(&acc_full, 0, kWaitNs);
    if (__any_sync(0xffffffffu, !ok)) bad = true;
    fence_after();
  }
  // every MMA of the cluster is done: the leader's ring takes the partial rows
  fence_before();
  __syncwarp();
  cluster_sync();
  fence_after();
  const int q = warp & 3, row = 32 * q + lane;
  const bool epi = warp >= 2;
  if (epi && rank > 0 && !bad) {
    const uint32_t slot = mapa_shared(smem_u32(sm), 0) + (uint32_t)((rank - 1) * Mp + row) * (uint32_t)(BN * 4);
#pragma unroll 1
    for (int cb = 0; cb < BN / 32; ++cb) {
      float v[32];
      tmem_ld32(tbase + ((uint32_t)(32 * q) << 16) + 32 * cb, v);
      if (row < Mp)
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // 16-byte piece c of the 32 columns, rotated by row against bank conflicts
          const int pc = (c + row) & 7;
          st_cluster_v4(slot + 128 * cb + 16 * pc, v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        }
    }
  }
  fence_before();
  __syncwarp();
  cluster_sync();  // the partial rows are in the leader's shared memory
  fence_after();
  if (epi && rank == 0 && !bad) {
#pragma unroll 1
    for (int cb = 0; cb < BN / 32; ++cb) {
      float v[32];
      tmem_ld32(tbase + ((uint32_t)(32 * q) << 16) + 32 * cb, v);
      if (row < M) {
        for (int r = 1; r < S; ++r) {
          const float* p = reinterpret_cast<const float*>(sm + ((size_t)(r - 1) * Mp + row) * BN * 4 + 128 * cb);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 f = *reinterpret_cast<const float4*>(p + 4 * ((c + row) & 7));
            v[4 * c] += f.x;
            v[4 * c + 1] += f.y;
            v[4 * c + 2] += f.z;
            v[4 * c + 3] += f.w;
          }
        }
        store_block(out, row, n0 + 32 * cb, N, v);
      }
    }
  }
  if (sync_tc_any(bad) && tid == 0) set_status(status, kStatusWaitTimeout);
  if (warp == 0) tmem_dealloc(tbase, tcols);
}

// ------------------------------------------------------------------ a CTA pair per tile
// cta_group::2 forms.  The pair's TMEM columns are allocated by one warp of
// each CTA together; an MMA issued by the even CTA reads A rows 0..127 and B
// rows 0..BN/2-1 from its own shared memory and A rows 128..255, B rows
// BN/2..BN-1 from the same offsets in the odd CTA's, and writes accumulator
// rows 0..127 to the even CTA's TMEM, rows 128..255 to the odd CTA's.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
// one arrival on the mbarrier at this shared offset in both CTAs once this thread's MMAs are done
__device__ __forceinline__ void commit_pair_both(uint64_t* m) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(m)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void commit_pair(uint64_t* m) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(m))
               : "memory");
}
// 2D tiled load into this CTA's shared memory whose bytes complete on an
// mbarrier of either CTA of the pair (`mbar` is a shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int x, int y, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.cta_group::2 [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t mbar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(mbar) : "memory");
}

constexpr int kPairRows = 256;  // output rows per pair tile; each CTA holds 128 of them

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw, int32_t M,
                     int32_t N, int32_t K, int32_t BN, int32_t ksub, const __grid_constant__ GemmOutputs out,
                     int32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  // full[s] and acc_empty[b] are used in the even CTA only (both CTAs complete them);
  // empty[s], acc_full[b] in both (the even CTA's MMA commits arrive on both)
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tslot;
  bool bad = false;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int half = BN / 2;
  const int blk_b = half * GK * 2;
  const int stage_bytes = ksub * (kStageA + blk_b);  // this CTA's share of one stage: ksub 64-wide K blocks
  const int stages = min(kMaxStages, kRing / stage_bytes);
  const int mt = (M + kPairRows - 1) / kPairRows, nt = (N + BN - 1) / BN, tiles = mt * nt;
  const int nk = (K + GK * ksub - 1) / (GK * ksub);
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);   // the even CTA's expect_tx arrival; both CTAs' loads complete its bytes
      mbar_init(&empty[s], 1);  // the MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(&drain, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc_pair(&tslot, kTmemCols);
  fence_before();
  cluster_sync();  // both CTAs' barriers initialised and the pair's TMEM allocated
  fence_after();
  const uint32_t tbase = tslot;
  const uint32_t full_lead = mapa_shared(smem_u32(&full[0]), 0);
  const uint32_t acc_empty_lead = mapa_shared(smem_u32(&acc_empty[0]), 0);

  if (warp == 0) {
    if (lane == 0) {  // loads of this CTA's halves: A rows 128 rank .., B rows half * rank ..
      int i = 0;
      int last[kMaxStages];
      for (int s = 0; s < kMaxStages; ++s) last[s] = -1;
      for (int t = pair; t < tiles && !bad; t += npairs) {
        const int m0 = (t % mt) * kPairRows + GM * (int)rank, n0 = (t / mt) * BN + half * (int)rank;
        for (int kb = 0; kb < nk; ++kb, ++i) {
          const int s = i % stages;
          if (i >= stages && !mbar_wait_cluster(&empty[s], ((i / stages) & 1) ^ 1, kWaitNs)) {
            bad = true;
            break;
          }
          unsigned char* a = sm + s * stage_bytes;
          if (leader) mbar_expect_tx(&full[s], 2 * stage_bytes);
          for (int u = 0; u < ksub; ++u) {
            tma_load_2d_pair(a + u * kStageA, &tx, GK * (kb * ksub + u), m0, full_lead + 8 * s);
            tma_load_2d_pair(a + ksub * kStageA + u * blk_b, &tw, GK * (kb * ksub + u), n0, full_lead + 8 * s);
          }
          last[s] = i;
        }
      }
      if (bad) {  // let the copies already issued land before the block exits
        if (leader) {
          for (int s = 0; s < stages; ++s)
            if (last[s] >= 0) mbar_wait(&full[s], (last[s] / stages) & 1, kWaitNs);
        } else {  // their completions go to the other CTA: give them a fixed grace period
          const uint64_t t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 200000ull) __nanosleep(1000);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t id = idesc_f16(kPairRows, BN, false, false) | kIdescBf16;
      int i = 0, j = 0;
      for (int t = pair; t < tiles && !bad; t += npairs, ++j) {
        const int ab = j & 1;
        if (j >= 2 && !mbar_wait_cluster(&acc_empty[ab], ((j >> 1) & 1) ^ 1, kWaitNs)) {
          bad = true;
          break;
        }
        fence_after();
        const uint32_t d = tbase + 256 * ab;
        for (int kb = 0; kb < nk; ++kb, ++i) {
          const int s = i % stages;
          if (!mbar_wait_cluster(&full[s], (i / stages) & 1, kWaitNs)) {
            bad = true;
            break;
          }
          fence_after();
          const uint32_t a = smem_u32(sm + s * stage_bytes), b = a + ksub * kStageA;
          for (int u = 0; u < ksub; ++u)
#pragma unroll
            for (int kk = 0; kk < GK / 16; ++kk)
              mma_pair(d, desc_kmaj(a + u * kStageA, GM, kk), desc_kmaj(b + u * blk_b, half, kk), id,
                       (kb > 0 || u > 0 || kk > 0) ? 1u : 0u);
          commit_pair_both(&empty[s]);
        }
        if (!bad) commit_pair_both(&acc_full[ab]);
      }
      commit_pair(&drain);  // every MMA issued has finished before the pair's TMEM is released
      mbar_wait(&drain, 0, kWaitNs);
    }
  } else {  // epilogue: this CTA's 128 rows of the tile, warp w on TMEM lanes 32 (w % 4) ..
    const int q = warp & 3;
    int j = 0;
    for (int t = pair; t < tiles; t += npairs, ++j) {
      const int ab = j & 1;
      const bool ok = mbar_wait_cluster(&acc_full[ab], (j >> 1) & 1, kWaitNs);
      if (__any_sync(0xffffffffu, !ok)) {
        bad = true;
        break;
      }
      fence_after();
      const int m0 = (t % mt) * kPairRows + GM * (int)rank, n0 = (t / mt) * BN;
      const int row = m0 + 32 * q + lane;
      const uint32_t src = tbase + 256 * ab + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        float v[32];
        tmem_ld32(src + 32 * cb, v);
        if (row < M) store_block(out, row, n0 + 32 * cb, N, v);
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty_lead + 8 * ab);
    }
  }
  if (sync_tc_any(bad) && tid == 0) set_status(status, kStatusWaitTimeout);
  __syncwarp();
  cluster_sync();  // the even CTA's MMAs no longer read this CTA's shared memory or write its TMEM
  fence_after();
  if (warp == 0) tmem_dealloc_pair(tbase, kTmemCols);
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

// SMs of the current device, looked up once (thread-safe; a failed query
// leaves no CUDA error behind for the next launch to report)
int num_sms() {
  static const int n = [] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      v = 148;
    }
    return v;
  }();
  return n;
}

// CTA pairs of gemm_pair_kernel that fit on the device at once, looked up once
int max_pairs() {
  static const int n = [] {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * num_sms());
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = kGemmSmem;
    int c = 0;
    if (cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem) ==
            cudaSuccess &&
        cudaOccupancyMaxActiveClusters(&c, gemm_pair_kernel, &cfg) == cudaSuccess && c > 0)
      return c;
    cudaGetLastError();
    return num_sms() / 2;
  }();
  return n;
}

// rounds of `tiles` over `slots` concurrent tiles, times the tile width plus a
// fixed 64 columns' worth of per-tile cost (narrower MMAs and the per-tile
// handshakes make a narrow tile cost more than its width)
int64_t tile_cost(int64_t tiles, int64_t slots, int bn) { return (tiles + slots - 1) / slots * (bn + 64); }

// K blocks per ring stage: two wherever that still leaves three stages.  Every
// stage costs a fixed handshake (full barrier, commit, refill), so fewer,
// larger stages keep the tensor pipe busier; measured on the Qwen-shaped
// projections, two blocks per stage raise the pair kernel from about 1.1 to
// 1.5 PFLOP/s.
int ksub(int kblock_bytes) { return kRing / (2 * kblock_bytes) >= 3 ? 2 : 1; }

}  // namespace

GemmPlan gemm_plan(int32_t M, int32_t N, int32_t tile_n) {
  const int64_t sms = num_sms(), pairs = max_pairs();
  GemmPlan best{false, 256};
  int64_t best_cost = -1;
  for (int pair = 0; pair < 2; ++pair)
    for (int bn = 256; bn >= 32; bn -= 32) {
      // widths other than powers of two only on request: measured, 224 or 192
      // columns never beat 256 even where they fill the last wave better
      if (tile_n != 0 ? bn != tile_n : (bn & (bn - 1)) != 0) continue;
      if (pair && (bn < 64 || M < kPairRows)) continue;  // pairs only where both CTAs have rows to compute
      const int64_t rows = pair ? kPairRows : GM;
      const int64_t tiles = (M + rows - 1) / rows * ((N + bn - 1) / bn);
      // a pair tile is two SMs' work: its cost is that of a 128-row tile on each
      const int64_t cost = tile_cost(tiles, pair ? pairs : sms, bn);
      if (best_cost < 0 || cost < best_cost || (cost == best_cost && pair && !best.pair))
        best = GemmPlan{pair != 0, bn}, best_cost = cost;
    }
  return best;
}

SplitPlan gemm_split_plan(int32_t M, int32_t N, int32_t K, int32_t tile_n) {
  SplitPlan best{0, 1, 0};
  if (M > GM) return best;
  // Up to 128 rows the weight stream bounds the time.  Measured per CTA (one
  // per SM): about 46, 27 and 18 GB/s of weights at 256-, 128- and 64-column
  // tiles, and about 4.2 TB/s for the whole device.  A split tile pays about
  // 6 us more (pipeline fill, two cluster barriers, the partial rows through
  // DSMEM), and at 256 columns its reduction outweighs the split: measured,
  // 64 x 6144 x 5120 took 28.7 us split 3 ways at 128 columns, 38.9 us split
  // 4 ways at 256 and 36.9 us unsplit at 64.
  const int64_t sms = num_sms(), nkb = (K + GK - 1) / GK;
  const int Mp = (M + 31) / 32 * 32;
  double best_t = -1.0;
  for (int bn = 256; bn >= 64; bn >>= 1) {
    if (tile_n != 0 && bn != tile_n) continue;
    const double rate = bn == 256 ? 46e9 : (bn == 128 ? 27e9 : 18e9);
    const int64_t ntiles = (N + bn - 1) / bn;
    for (int S = 1; S <= 8 && S <= nkb; ++S) {
      if (S > 1 && (bn > 128 || ntiles * S > sms || (int64_t)(S - 1) * Mp * bn * 4 > kRing)) break;
      const double per_cta = (double)bn * 128.0 * (double)((nkb + S - 1) / S);  // weight bytes of one CTA's tile
      const double rounds = S > 1 ? 1.0 : (double)((ntiles + sms - 1) / sms);
      const double t = std::max(rounds * per_cta / rate + (S > 1 ? 6e-6 : 0.0), (double)N * K * 2.0 / 4.2e12);
      if (best_t < 0 || t < best_t * 0.97) best = SplitPlan{bn, S, Mp}, best_t = t;
    }
  }
  return best;
}

cudaError_t launch_gemm_bf16(const void* x, int32_t M, int32_t K, const void* w, int32_t N, int32_t tile_n,
                             const GemmOutputs& out, int32_t* status, cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  const SplitPlan sp = gemm_split_plan(M, N, K, tile_n == 0 || tile_n == 64 || tile_n == 128 || tile_n == 256
                                                    ? tile_n : -1);
  if (sp.split > 1) {  // a cluster of sp.split CTAs per tile, each on a slice of K
    CUtensorMap tx, tw;
    if (!encode_bf16_2d(enc, &tx, x, (uint64_t)K, (uint64_t)M, GM) ||
        !encode_bf16_2d(enc, &tw, w, (uint64_t)K, (uint64_t)N, (uint32_t)sp.tile_n))
      return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(gemm_splitk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
    if (e != cudaSuccess) return e;
    const int ntiles = (N + sp.tile_n - 1) / sp.tile_n;
    uint32_t tcols = 32;
    while ((int)tcols < sp.tile_n) tcols <<= 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ntiles * sp.split));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = kGemmSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)sp.split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LaunchScope scope(GDN_K_GEMM, stream);
    e = cudaLaunchKernelEx(&cfg, gemm_splitk_kernel, tx, tw, M, N, K, (int32_t)sp.tile_n, (int32_t)sp.split,
                           (int32_t)sp.mp, tcols, out, status);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  const GemmPlan plan = gemm_plan(M, N, sp.tile_n ? sp.tile_n : tile_n);
  const int bn = plan.tile_n;
  CUtensorMap tx, tw;
  if (!encode_bf16_2d(enc, &tx, x, (uint64_t)K, (uint64_t)M, GM) ||
      !encode_bf16_2d(enc, &tw, w, (uint64_t)K, (uint64_t)N, (uint32_t)(plan.pair ? bn / 2 : bn)))
    return cudaErrorInvalidValue;
  const void* fn = plan.pair ? (const void*)gemm_pair_kernel : (const void*)gemm_kernel;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  LaunchScope scope(GDN_K_GEMM, stream);
  if (plan.pair) {
    const int64_t tiles = (int64_t)((M + kPairRows - 1) / kPairRows) * ((N + bn - 1) / bn);
    const int pairs = (int)(tiles < max_pairs() ? tiles : max_pairs());
    gemm_pair_kernel<<<2 * pairs, kGemmThreads, kGemmSmem, stream>>>(tx, tw, M, N, K, bn, ksub(kStageA + bn * GK),
                                                                      out, status);
  } else {
    const int64_t tiles = (int64_t)((M + GM - 1) / GM) * ((N + bn - 1) / bn);
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
    gemm_kernel<<<grid, kGemmThreads, kGemmSmem, stream>>>(tx, tw, M, N, K, bn, ksub(kStageA + bn * GK * 2), out,
                                                          status);
  }
  return cudaGetLastError();
}

}  // namespace gdn
